"""Host-side helpers of bench.py that need no GPU."""
import bench


def test_comment_stripping_keeps_code_and_literals():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x//y/*z*/";\nchar c = \'"\';  float b;'
    assert bench.strip_c_comments(src) == 'int a = 1; const char* s = "x//y/*z*/"; char c = \'"\'; float b;'


def test_kernel_hash_ignores_comments_but_not_code():
    base = {rel: "int f() { return 1; }\n" for rel in bench.KERNEL_SOURCES}
    commented = {rel: "// header\nint f() { /* one */ return 1; }   \n" for rel in bench.KERNEL_SOURCES}
    changed = {rel: "int f() { return 2; }\n" for rel in bench.KERNEL_SOURCES}
    h = bench.kernel_source_hash(base.__getitem__)
    assert h == bench.kernel_source_hash(commented.__getitem__)
    assert h != bench.kernel_source_hash(changed.__getitem__)
