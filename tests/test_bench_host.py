"""Host-side helpers of bench.py, on CPU: the comment-insensitive kernel hash that
decides whether the committed DRAM-traffic record still describes the kernel, the
reader of that record, and the compact `targets` summary."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_strip_c_comments_drops_comments_and_keeps_literals():
    b = _bench()
    src = 'int a = 1; // one\n/* block\n comment */ int b = 2;\nconst char* s = "// not a comment";\n'
    out = b.strip_c_comments(src)
    assert "one" not in out and "block" not in out
    assert '"// not a comment"' in out
    assert out == 'int a = 1; int b = 2; const char* s = "// not a comment";'


def test_strip_c_comments_keeps_escaped_quotes_in_literals():
    b = _bench()
    src = 'const char* s = "a \\" // still inside"; int x; // gone'
    assert b.strip_c_comments(src) == 'const char* s = "a \\" // still inside"; int x;'


def test_comment_stripping_keeps_code_and_literals():
    b = _bench()
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x//y/*z*/";\nchar c = \'"\';  float b;'
    assert b.strip_c_comments(src) == 'int a = 1; const char* s = "x//y/*z*/"; char c = \'"\'; float b;'


def test_kernel_hash_ignores_comments_but_not_code():
    b = _bench()
    base = {rel: "int f() { return 1; }\n" for rel in b.KERNEL_SOURCES}
    commented = {rel: "// header\nint f() { /* one */ return 1; }   \n" for rel in b.KERNEL_SOURCES}
    changed = {rel: "int f() { return 2; }\n" for rel in b.KERNEL_SOURCES}
    h = b.kernel_source_hash(base.__getitem__)
    assert h == b.kernel_source_hash(commented.__getitem__)
    assert h != b.kernel_source_hash(changed.__getitem__)


def _hash_with(b, edit):
    texts = {}
    for rel in b.KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            texts[rel] = f.read()
    texts = edit(texts)
    return b.kernel_source_hash(read=lambda rel: texts[rel])


def test_kernel_hash_ignores_comment_and_whitespace_edits():
    b = _bench()
    base = _hash_with(b, lambda t: t)
    first = b.KERNEL_SOURCES[0]

    def comment_edit(t):
        t = dict(t)
        t[first] = "// a new leading comment\n/* and a block */\n" + t[first].replace("\n", "\n\n", 3)
        return t

    assert _hash_with(b, comment_edit) == base


def test_kernel_hash_changes_with_code():
    b = _bench()
    base = _hash_with(b, lambda t: t)
    first = b.KERNEL_SOURCES[0]

    def code_edit(t):
        t = dict(t)
        t[first] = t[first] + "\nstatic const int kNotInTheKernel = 1;\n"
        return t

    assert _hash_with(b, code_edit) != base


def test_load_traffic_follows_the_hash(tmp_path, monkeypatch):
    b = _bench()
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = prof / "swattn_fwd_pair_kernel_wan720p_traffic.txt"
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "kernel_source_hash", lambda read=None: "abc123")
    rec.write_text("# comment line\nkernel = swattn_fwd_pair_kernel\n"
                   "dram_bytes_per_launch = 2991771520.0\nkernel_source_hash = abc123\n")
    assert b.load_traffic() == {"dram_bytes_per_launch": 2991771520.0}
    rec.write_text("dram_bytes_per_launch = 2991771520.0\nkernel_source_hash = 0000\n")
    assert b.load_traffic() is None          # taken on other kernel sources: not reported
    rec.unlink()
    assert b.load_traffic() is None          # no record


def _row(name, ms_w, frac_w, ms_full, full_frac, flops_w, speedup, theo):
    return {"workload": name, "flops_window": flops_w,
            "window": [{"ms": m, "frac_of_peak": f} for m, f in zip(ms_w, frac_w)],
            "ms_window_mean": sum(ms_w) / len(ms_w), "ms_full": ms_full, "full_frac_of_peak": full_frac,
            "speedup_vs_full": speedup, "speedup_frac_of_theoretical": speedup / theo}


def test_targets_of_summarises_the_two_target_workloads():
    b = _bench()
    per_wl = [
        _row("tiny-2d-16x16-w8", [0.01, 0.01], [0.0, 0.0], 0.02, 0.0, 8.4e6, 1.3, 4),
        _row(b.TARGET_WORKLOADS["flux4096"], [0.8, 0.9], [0.6, 0.5], 50.0, 0.6, 8.25e11, 58.0, 64),
        _row(b.TARGET_WORKLOADS["wan720p"], [3.3, 3.3], [0.47, 0.47], 107.0, 0.65, 2.6e12, 32.0, 45),
    ]
    t = b.targets_of(per_wl)
    assert set(t) == {"flux4096", "wan720p"}
    f = t["flux4096"]
    assert f["ms_window"] == [0.8, 0.9]
    assert f["frac_of_peak"] == pytest.approx(0.55)
    assert f["tflops"] == pytest.approx(8.25e11 / 0.85 / 1e9, rel=1e-3)
    assert f["speedup_frac_of_theoretical"] == pytest.approx(58.0 / 64, abs=1e-4)
    assert t["wan720p"]["ms_full"] == 107.0


def test_targets_of_skips_missing_workloads():
    b = _bench()
    assert b.targets_of([]) == {}
