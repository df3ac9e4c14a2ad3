/*
 * basa_swattn.h -- C ABI of the B200 (sm_100a) shifted-window attention library
 * (libbasa_swattn.so).
 *
 * Operation: the shifted local-window self-attention of "Backend-Agnostic
 * Sparse Attention for Fast High-Resolution Visual Generation" (BASA),
 * §3.1 "Shifted Window Sparse Attention": the visual token grid is cyclically
 * shifted by -Delta, cut into non-overlapping windows, standard scaled
 * dot-product softmax attention runs inside each window with the unchanged
 * Q/K/V, and the outputs are merged and shifted back by +Delta.  Appendix A.1
 * ("Regular execution with standard attention backends") describes the
 * windows as dense attention problems folded into the batch; here the roll,
 * the window gather, the attention and the inverse roll are one kernel.
 *
 * Conventions shared by every entry point
 *   - Tensors Q, K, V and out are bf16, row-major [B, T*H*W, heads, d]; tokens
 *     in raster order (t, h, w); d contiguous.  All four are DEVICE pointers,
 *     16-byte aligned, owned by the caller; the library keeps no reference
 *     after the call returns.
 *   - win[3] and shift[3] are ordered (t, h, w).  1 <= win[a] <= extent[a].
 *     A window that the grid does not divide is truncated at the grid edge
 *     (the last window along that axis holds extent mod win tokens).
 *   - shift[a] is any integer Delta_a; it is reduced modulo the extent.  The
 *     grid is rolled by -Delta, so window m starts at original coordinate
 *     (m_a * win[a] + Delta_a) mod extent[a] along each axis.
 *   - Full attention is win = {T, H, W} with shift = {0, 0, 0}: one window.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Launches are asynchronous; nothing is synchronised and nothing is
 *     allocated per call.
 *   - Errors are returned as BASA_* codes.  Argument errors are detected on
 *     the host before anything is launched.  The library never prints, exits
 *     or throws across this boundary.
 */
#ifndef BASA_SWATTN_H
#define BASA_SWATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BASA_OK 0
#define BASA_ERR_INVALID_ARG (-1)  /* null pointer, bad extent, window or size */
#define BASA_ERR_UNSUPPORTED (-2)  /* head dim other than 64/128, too many rows, not sm_100 */
#define BASA_ERR_ALIGNMENT (-3)    /* a tensor pointer is not 16-byte aligned */
#define BASA_ERR_CUDA (-4)         /* a CUDA runtime or driver call failed */
#define BASA_ERR_DEVICE (-5)       /* a bounded device-side wait expired in a launch */
#define BASA_ERR_ALIAS (-6)        /* out overlaps q, k or v */
#define BASA_ERR_SCRATCH_LIMIT (-7) /* larger than the fixed device scratch of basa_route_noalloc */

/*
 * Shifted-window attention forward (§3.1 "Shifted Window Sparse Attention").
 *
 *   q, k, v  in : device bf16 [B, T*H*W, heads, d]
 *   out      out: device bf16 [B, T*H*W, heads, d]; must not overlap q, k or v
 *   d        64 or 128
 *   scale    softmax scale applied to Q K^T (1/sqrt(d) for standard attention);
 *            finite and >= 0 (a negative scale returns BASA_ERR_UNSUPPORTED)
 *
 * out[b, p, h, :] = sum_j softmax_j(scale * <q_p, k_j>) v_j over the tokens j
 * that share the (shifted) window of token p.  Accumulation is fp32; P is
 * rounded to bf16 before the P V product; the result is rounded to bf16.
 * B * T*H*W * heads must be below 2^31.
 */
int basa_swattn_fwd(const void* q, const void* k, const void* v, void* out, int B, int heads,
                    int T, int H, int W, int d, const int win[3], const int shift[3],
                    float scale, void* stream);

/*
 * The index map of the shifted partition, computed on the device by the same
 * device function the attention kernel uses for its gathers and scatters.
 *
 *   d_token_of_slot out: device int32 [n_windows, win[0]*win[1]*win[2]], the
 *                        raster token index held by (window, slot); -1 in the
 *                        slots a truncated window does not fill.
 * Windows are numbered in raster order over (m_t, m_h, m_w) and slots in raster
 * order over (s_t, s_h, s_w) of the rolled grid; n_windows is the product of
 * ceil(extent[a] / win[a]).
 */
int basa_swattn_index_map(int T, int H, int W, const int win[3], const int shift[3],
                          int32_t* d_token_of_slot, void* stream);

/* The same index map computed on the host (same source function as the kernel's). */
int basa_swattn_index_map_host(int T, int H, int W, const int win[3], const int shift[3],
                               int32_t* token_of_slot);

/*
 * Algorithmic FLOPs of one forward (the O(N n_w d) cost of §3.1 "Attention
 * complexity"): the sum over windows of 4 * n_m^2 * d, times B * heads, where
 * n_m is the token count of window m.  Written to *flops.
 */
int basa_swattn_flops(int B, int heads, int T, int H, int W, int d, const int win[3],
                      double* flops);

/*
 * The forward with an extra key/value segment (§3.2 "K/V-Pooled Global
 * Memory": each window's keys and values become [K_W; K_bar], [V_W; V_bar]).
 * kx, vx: device bf16 [B, E, heads, d], contiguous, 16-byte aligned: E extra
 * tokens per (batch item, head), appended to the keys and values of every
 * window of that (batch item, head) -- the pooled memory from basa_kv_pool,
 * any other shared tokens (e.g. text), or both concatenated.  Queries and the
 * output are unchanged: out[b, token, head, :] is the softmax attention of the
 * query over its window's tokens and the E extra tokens.  E = 0 (kx, vx may
 * then be null) is exactly basa_swattn_fwd.  Other arguments, errors and
 * ownership as basa_swattn_fwd; out must not overlap kx or vx either.
 */
int basa_swattn_fwd_mem(const void* q, const void* k, const void* v, const void* kx,
                        const void* vx, int E, void* out, int B, int heads, int T, int H, int W,
                        int d, const int win[3], const int shift[3], float scale, void* stream);

/*
 * Pooled global memory (§3.2): kbar[b, g, head, :] and vbar[b, g, head, :]
 * are the means of k and v over patch g of the unshifted grid.  The grid is cut
 * into patches of pool[0] x pool[1] x pool[2] tokens (t, h, w), the last patch
 * along an axis holding what is left; patches are numbered in raster order over
 * (g_t, g_h, g_w), G = prod ceil(n_a / pool[a]) (basa_kv_pool_tokens).
 * k, v: device bf16 [B, T*H*W, heads, d]; kbar, vbar: device bf16
 * [B, G, heads, d] (fp32 sums, rounded to nearest even); all 16-byte aligned,
 * outputs overlapping neither the inputs nor each other (BASA_ERR_ALIAS).
 * d must be 64 or 128.  Asynchronous on `stream`.
 */
int basa_kv_pool(const void* k, const void* v, void* kbar, void* vbar, int B, int heads, int T,
                 int H, int W, int d, const int pool[3], void* stream);

/* Pooled tokens G = prod ceil(n_a / pool[a]) of a T x H x W grid, written to *G. */
int basa_kv_pool_tokens(int T, int H, int W, const int pool[3], int* G);

/*
 * The per-layer window offsets of the interleaved shift schedule
 * (§3.1 "Interleaved shift schedule"), per axis a with window w = win[a]:
 *   delta = max(1, floor(w / L)),  a_i = (i * delta) mod w  for i = 0..L-1,
 *   b = (a_0, a_K, a_1, a_{K+1}, ...)  with K = ceil(L / 2)  (the first and
 *        second halves of a interleaved; for odd L the first half has the
 *        extra element, which comes last),
 *   shift[l][a] = (b_l + step_offset[a]) mod w.
 * step_offset is the denoising-step term c_s of the schedule (the pages leave
 * its values open; pass zeros for a step-independent schedule).
 * shifts: host array of L * 3 ints, written as [l][t, h, w]; each entry is a
 * value for basa_swattn_fwd's `shift` argument.  An axis whose window spans
 * the whole grid may be given any shift: it does not change the result.
 * Returns BASA_ERR_INVALID_ARG for L < 1, a window < 1 or null pointers.
 */
int basa_shift_schedule(int L, const int win[3], const int step_offset[3], int* shifts);

/*
 * Bytes of device workspace basa_route needs: two fp32 arrays of
 * B * heads * n_windows * d (the window descriptors).  Written to *bytes.
 * The workspace does not depend on the shift.
 */
int basa_route_workspace_bytes(int B, int heads, int T, int H, int W, int d, const int win[3],
                               size_t* bytes);

/*
 * Content-adaptive true-window routing (§3.3 "Content-Adaptive True-Window
 * Routing"), top-1: for every window i of the shifted partition and every
 * (batch item, head), the window descriptors q_i and k_i are the means of Q
 * and K over the window's tokens, and routed[b, head, i] is the candidate j
 * with the largest s_ij = q_i k_j^T / sqrt(d).  Routing is spatial (as for
 * video in the same section): the candidates of i are the other windows with
 * the same temporal window index whose (m_h, m_w) lie within Chebyshev
 * distance `radius` of i's, without wrap-around.  Ties go to the lower window
 * index; a window with no candidate (radius 0, or one spatial window) gets -1.
 * A radius larger than the window grid is treated as the grid's extent.
 *
 *   q, k       device bf16 [B, T*H*W, heads, d], 16-byte aligned (as basa_swattn_fwd)
 *   workspace  device, >= basa_route_workspace_bytes(...) bytes, 16-byte
 *              aligned; overwritten (fp32 descriptors)
 *   routed     out: device int32 [B, heads, n_windows], 4-byte aligned
 * Descriptors and scores are fp32 and summed in a fixed order, so the result
 * is the same on every run; where two candidates' scores differ by less than
 * the fp32 rounding of the sums, either may be chosen.  Two launches on
 * `stream`.  Errors: BASA_ERR_INVALID_ARG (null pointer, radius < 0, workspace
 * too small, bad geometry), BASA_ERR_UNSUPPORTED (d not 64/128, sizes past
 * 2^31 rows), BASA_ERR_ALIGNMENT, BASA_ERR_ALIAS (routed or the workspace
 * overlapping q, k or each other), BASA_ERR_CUDA.
 */
int basa_route(const void* q, const void* k, int B, int heads, int T, int H, int W, int d,
               const int win[3], const int shift[3], int radius, void* workspace,
               size_t workspace_bytes, int32_t* routed, void* stream);

/*
 * Bytes of device scratch basa_route_noalloc has: a fixed array inside the
 * library, 4 MiB.
 */
#define BASA_ROUTE_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * basa_route without a workspace argument, for callers that cannot allocate
 * device memory at the point where they route: code running inside another
 * framework's execution step (a plugin's enqueue callback, a serving loop that
 * owns a fixed memory budget) where cudaMalloc is forbidden or would stall the
 * device.  The paper has no counterpart; this is a deployment variant of the
 * routing above.
 *
 * Same arguments, results, errors and ownership as basa_route, minus the
 * workspace: the window descriptors (2 * B * heads * n_windows * d * 4 bytes)
 * are kept in a fixed array of BASA_ROUTE_NOALLOC_SCRATCH_BYTES bytes inside
 * the library, which every GPU that loads the library holds until the process
 * exits.  A problem whose descriptors do not fit returns
 * BASA_ERR_SCRATCH_LIMIT before anything is launched (B * heads * n_windows *
 * d up to 524,288: e.g. 4,096 window-heads at d = 128).  The call allocates
 * nothing and calls no allocating routine.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on a device share the one array:
 * calls whose work can overlap on the GPU (on different streams, or from
 * different host threads without ordering) race on it and must not be made.
 * Each call overwrites every descriptor it reads, so no clearing is needed.
 */
int basa_route_noalloc(const void* q, const void* k, int B, int heads, int T, int H, int W, int d,
                       const int win[3], const int shift[3], int radius, int32_t* routed, void* stream);

/*
 * The forward over the key/value source S_i = W_i u R_i u G of §3.3: the
 * queries of window i attend to the tokens of window i, then to the tokens of
 * window routed[b, head, i] (its own token order; any entry outside
 * [0, n_windows), -1 by convention, routes nothing), then to the E extra
 * tokens kx, vx (G, e.g. the pooled memory; E = 0 allowed, kx, vx may then be
 * null), all in one softmax.  routed: device int32 [B, heads, n_windows],
 * 4-byte aligned, not null (from basa_route or the caller's own choice).  With
 * every entry -1 the result is basa_swattn_fwd_mem's.  Other arguments,
 * errors and ownership as basa_swattn_fwd_mem; out must not overlap routed.
 */
int basa_swattn_fwd_route(const void* q, const void* k, const void* v, const int32_t* routed,
                          const void* kx, const void* vx, int E, void* out, int B, int heads,
                          int T, int H, int W, int d, const int win[3], const int shift[3],
                          float scale, void* stream);

/*
 * Synchronises `stream`, then returns BASA_ERR_DEVICE if any launch since the
 * previous call gave up on a bounded wait (BASA_OK otherwise), and clears the
 * record.  Also returns BASA_ERR_CUDA if the synchronisation itself fails.
 */
int basa_swattn_last_device_error(void* stream);

/*
 * Upper bound, in nanoseconds, on every wait inside the kernels (default one
 * second), process-wide: launches from every host thread read it.  A launch
 * whose wait runs out stops its work, drains what it has in flight, releases
 * its tensor memory, and records BASA_ERR_DEVICE.
 */
int basa_swattn_set_wait_timeout_ns(unsigned long long ns);

/*
 * Test hook for the bounded-wait error path (not part of the method): while
 * `on` is non-zero, every launch's MMA issuer first waits on a barrier that
 * nothing arrives on, so the launch times out after the wait limit, stops,
 * drains and reports BASA_ERR_DEVICE.  Off by default.  The setting (like the
 * wait limit above) is process-wide: it applies to launches made from every
 * host thread while it is on.
 */
int basa_swattn_set_test_stall(int on);

/* Static, human-readable text for a BASA_* code. */
const char* basa_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* BASA_SWATTN_H */
