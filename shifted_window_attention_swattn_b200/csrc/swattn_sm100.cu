// swattn_sm100.cu -- shifted local-window self-attention forward for B200 (sm_100a).
//
// Method: "Backend-Agnostic Sparse Attention for Fast High-Resolution Visual
// Generation" (BASA), §3.1 "Shifted Window Sparse Attention": roll the token
// grid by -Delta, cut it into non-overlapping windows, run softmax attention
// inside each window, roll the result back by +Delta.  Appendix A.1 runs the
// roll and the window partition as separate reshape/permute passes before a
// dense attention backend; here they never touch memory:
//
//   * the roll + partition is the row list of TMA tile::gather4 loads (each
//     load brings 4 arbitrary token rows x 64 columns of Q, K or V into a
//     128-byte-swizzled shared-memory tile), so windows are gathered straight
//     from the [B, T*H*W, heads, d] tensors.  Each producer lane computes the
//     rows of its own gathers and a warp issues all of them in one instruction;
//   * S = Q K^T and O += P V run on tcgen05 tensor cores with S, P and O in
//     tensor memory (TMEM);
//   * softmax is online (running max / sum per query row, one thread per row),
//     with the max kept stale until it grows by more than 2^8 so that O is
//     rarely rescaled;
//   * the inverse roll is the row address of the output store: each query's
//     result is written back to the token row it was gathered from (in the
//     CTA-pair kernel by tile::scatter4 TMA stores from a staging tile, four
//     rows per store, while the softmax warps go on to the next unit).
//
// Two persistent kernels share this pipeline.  A work unit is a run of query
// tiles of one window of one (batch, head); each unit streams the window's
// K/V tiles through a shared-memory ring, and two query tiles per CTA are
// processed in ping-pong (softmax of one tile overlaps the MMAs of the other).
// Unit and slot decoding divide by launch constants through precomputed
// multiply-shift reciprocals (FastDiv), not integer division.
//   * swattn_fwd_pair_kernel (d = 128): clusters of two CTAs issue M = 256
//     MMAs with cta_group::2; each SM loads half of every K/V tile;
//   * swattn_fwd_kernel (any supported d, one CTA per SM): M = 128 MMAs.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_i is
// bf16 over the front of S_i.
//
// Both kernels are templated on <kMem, kRoute>.  A unit's key tiles are those
// of its window, then (kRoute, §3.3 "Content-Adaptive True-Window Routing")
// those of its routed window, then (kMem, §3.2 "K/V-Pooled Global Memory")
// those of an extra K/V segment such as the pooled memory; one online softmax
// runs over all of them.  The routes come from win_desc_kernel (window means
// of Q and K) and route_kernel (top-1 over the spatial neighbour windows), and
// the pooled memory from kv_pool_kernel.
//
// Every mbarrier wait is bounded by a host-set timeout; a wait that runs out
// raises a shared abort flag and a library-wide error word, every role stops
// issuing work, the MMA issuer drains its in-flight MMAs, the producer drains
// its in-flight loads, and TMEM is released before the CTA exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstddef>
#include <math.h>
#include <mutex>
#include <type_traits>
#include <stdint.h>
#include <string.h>

#include "basa_swattn.h"
#include "ptx_sm100.cuh"
#include "softmax_sm100.cuh"

namespace swattn {

constexpr int kThreads = 352;    // 11 warps
constexpr int kTile = 128;       // query rows per tile = key rows per K/V tile
constexpr int kMaxSlots = 8;     // K/V ring depth limit (tiles)
constexpr int kProducerWarp0 = 8;  // warps 8 and 9 each load half of every tile
constexpr int kProducers = 2;
constexpr int kMmaWarp = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;   // S_0 (P_0 in its first 64 columns as bf16 pairs)
constexpr uint32_t kColS1 = 128; // S_1 (P_1 likewise)
constexpr uint32_t kColO0 = 256;
constexpr uint32_t kColO1 = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when the max grows by > 2^8

// ------------------------------------------------------------------ geometry

// Division of 0 <= n < 2^31 by a divisor 1 <= d < 2^31 fixed for a launch, as
// a multiply and a shift: with p = 31 + ceil(log2 d) and m = ceil(2^p / d),
// floor(n * m / 2^p) = floor(n / d), because m * d - 2^p < d makes the error
// term n (m d - 2^p) / (d 2^p) smaller than 1/d.  m < 2^32.
struct FastDiv {
  uint32_t d, m, p;
};

static inline FastDiv make_fastdiv(int d) {
  FastDiv f;
  uint32_t l = 0;
  while ((1ull << l) < static_cast<unsigned long long>(d)) ++l;
  f.d = static_cast<uint32_t>(d);
  f.p = 31 + l;
  f.m = static_cast<uint32_t>(((1ull << f.p) + static_cast<unsigned long long>(d) - 1) / static_cast<unsigned long long>(d));
  return f;
}

__host__ __device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  return static_cast<int>((static_cast<unsigned long long>(static_cast<uint32_t>(n)) * f.m) >> f.p);
}

// Grid, window and shift of one call.  Shared by the kernel, the index-map
// kernel and the host index map, so that all three agree bit for bit.
struct Geometry {
  int n[3];       // extents (T, H, W)
  int w[3];       // window (w_t, w_h, w_w)
  int delta[3];   // shift reduced into [0, n_a)
  int nwin[3];    // ceil(n_a / w_a)
  int n_windows;  // product of nwin
  int nw_max;     // w_t * w_h * w_w
  int N;          // T * H * W
  FastDiv f_nwin[3];   // by nwin[a]
  FastDiv f_w[3];      // by w[a]: a full window's extent
  FastDiv f_tail[3];   // by the extent of the last window along a (n_a - (nwin_a - 1) w_a)
};

// Division by e, the extent along axis a of one of the windows of g.
__host__ __device__ __forceinline__ int div_extent(const Geometry& g, int a, int n, int e) {
  return fdiv(n, e == g.w[a] ? g.f_w[a] : g.f_tail[a]);
}

// Window coordinates m and extents e (truncated at the grid edge) of window `id`
// (raster order over m_t, m_h, m_w).
__host__ __device__ __forceinline__ void window_of(const Geometry& g, int id, int m[3], int e[3]) {
  const int r = fdiv(id, g.f_nwin[2]);
  m[2] = id - r * g.nwin[2];
  m[0] = fdiv(r, g.f_nwin[1]);
  m[1] = r - m[0] * g.nwin[1];
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int left = g.n[a] - m[a] * g.w[a];
    e[a] = left < g.w[a] ? left : g.w[a];
  }
}

// Raster index of the original token that the roll by -Delta places in slot s
// (raster order over s_t, s_h, s_w) of window m: along each axis the rolled
// coordinate m_a*w_a + s_a holds original coordinate (m_a*w_a + s_a + Delta_a) mod n_a.
__host__ __device__ __forceinline__ int slot_token(const Geometry& g, const int m[3],
                                                   const int e[3], int s) {
  const int r = div_extent(g, 2, s, e[2]);
  const int sw = s - r * e[2];
  const int st = div_extent(g, 1, r, e[1]);
  const int sh = r - st * e[1];
  int pt = m[0] * g.w[0] + st + g.delta[0];
  int ph = m[1] * g.w[1] + sh + g.delta[1];
  int pw = m[2] * g.w[2] + sw + g.delta[2];
  if (pt >= g.n[0]) pt -= g.n[0];
  if (ph >= g.n[1]) ph -= g.n[1];
  if (pw >= g.n[2]) pw -= g.n[2];
  return (pt * g.n[1] + ph) * g.n[2] + pw;
}

static int make_geometry(Geometry* g, int T, int H, int W, const int win[3], const int shift[3]) {
  if (!win || !shift || T < 1 || H < 1 || W < 1) return BASA_ERR_INVALID_ARG;
  g->n[0] = T;
  g->n[1] = H;
  g->n[2] = W;
  long long N = 1, nwin = 1, nmax = 1;
  for (int a = 0; a < 3; ++a) {
    if (win[a] < 1 || win[a] > g->n[a]) return BASA_ERR_INVALID_ARG;
    g->w[a] = win[a];
    long long s = shift[a] % g->n[a];
    if (s < 0) s += g->n[a];
    g->delta[a] = static_cast<int>(s);
    g->nwin[a] = (g->n[a] + win[a] - 1) / win[a];
    g->f_nwin[a] = make_fastdiv(g->nwin[a]);
    g->f_w[a] = make_fastdiv(win[a]);
    g->f_tail[a] = make_fastdiv(g->n[a] - (g->nwin[a] - 1) * win[a]);
    N *= g->n[a];
    nwin *= g->nwin[a];
    nmax *= win[a];
  }
  if (N >= (1LL << 31) || nmax >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  g->N = static_cast<int>(N);
  g->n_windows = static_cast<int>(nwin);
  g->nw_max = static_cast<int>(nmax);
  return BASA_OK;
}

// ------------------------------------------------------------------ kernel

struct __align__(64) FwdParams {
  CUtensorMap tq, tk, tv;       // 2D [rows = B*N*heads, cols = d], box {64, 1}, 128B swizzle
  CUtensorMap tkx, tvx;         // extra K/V segment, 2D [rows = B*n_extra*heads, cols = d] (kMem)
  int n_extra;                  // extra keys appended to every window (kMem)
  const int* routed;            // [B, heads, n_windows] routed window of each window, or none (kRoute)
  __nv_bfloat16* out;
  Geometry g;
  int B, heads, d;
  int q_pairs;                  // ceil(nw_max / 256): 256-query units per window
  FastDiv f_qp, f_nw, f_heads;  // by q_pairs, n_windows, heads
  int total_units;              // B * heads * n_windows * q_pairs
  int n_slots;                  // K/V ring depth (tiles)
  float scale_log2;             // scale * log2(e)
  unsigned long long timeout_ns;
  int stall;                    // test hook: the MMA issuer first waits on a barrier nothing arrives on
};

struct SmemCtl {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[kMaxSlots];
  uint64_t kv_empty[kMaxSlots];
  uint64_t s_full[2];           // S_i = Q_i K_j^T is in TMEM
  uint64_t p_full[2];           // P_i is in TMEM and O_i is rescaled
  uint64_t o_final[2];          // last P V of the unit for tile i is done
  uint64_t drained;             // every MMA of the CTA is done
  uint64_t never;               // test hook: never arrived on
  uint32_t tmem_base;
  int abort;
};

static_assert(offsetof(SmemCtl, q_full) % 8 == 0, "mbarriers are 8-byte aligned");

__device__ int g_device_error = 0;

// Waits that drain work already in flight (MMAs, TMA loads) before TMEM is
// released or the CTA exits get at least this long, whatever the caller's
// wait limit: in-flight hardware work always finishes, and cutting these
// waits short would release resources it still uses.
constexpr unsigned long long kDrainMinNs = 200ull * 1000 * 1000;
__device__ __forceinline__ unsigned long long drain_ns(unsigned long long t) {
  return t > kDrainMinNs ? t : kDrainMinNs;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, SmemCtl* ctl,
                                              unsigned long long timeout_ns) {
  if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
  if (mbar_wait_bounded(bar, parity, timeout_ns)) return true;
  *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
  atomicOr(&g_device_error, 1);
  return false;
}

// One unit of work: up to 256 queries (two 128-row tiles) of one window of
// one (batch item, head), attending to every key of that window, then (kRoute)
// to every key of its routed window, then (kMem) to the extra segment.
struct Unit {
  int b, h;
  int m[3], e[3];
  int n_valid;    // tokens in the window
  int q0;         // first query slot of tile 0
  int nkv;        // key tiles: the window's, the routed window's (kRoute), the extra segment's (kMem)
  int nkv_win;    // key tiles of the window
  int nkv_rt;     // key tiles of the routed window (kRoute), else 0
  int rm[3], re[3];  // coordinates and extents of the routed window (kRoute)
  int n_route;    // tokens of the routed window (kRoute), else 0
  int n_extra;    // keys of the extra segment (kMem), else 0
  bool has_q1;    // tile 1 holds at least one query
};

// The routed window of window win_id for the unit's (b, head): an entry
// outside [0, n_windows) (-1 by convention) routes nothing.
__device__ __forceinline__ void route_of(const Geometry& g, const int* routed, int heads, int win_id,
                                         Unit& U) {
  const int r = __ldg(routed + (static_cast<long long>(U.b) * heads + U.h) * g.n_windows + win_id);
  U.n_route = 0;
  U.nkv_rt = 0;
  if (r >= 0 && r < g.n_windows) {
    window_of(g, r, U.rm, U.re);
    U.n_route = U.re[0] * U.re[1] * U.re[2];
    U.nkv_rt = (U.n_route + kTile - 1) / kTile;
  }
}

// Units are numbered with the query pair fastest, then window, then
// (batch, head), so CTAs that run at the same time share K/V in L2.
template <bool kMem, bool kRoute>
__device__ __forceinline__ bool decode_unit(const FwdParams& p, int u, Unit& U) {
  const int r = fdiv(u, p.f_qp);
  const int qp = u - r * p.q_pairs;
  const int bh = fdiv(r, p.f_nw);
  const int win_id = r - bh * p.g.n_windows;
  U.b = fdiv(bh, p.f_heads);
  U.h = bh - U.b * p.heads;
  window_of(p.g, win_id, U.m, U.e);
  U.n_valid = U.e[0] * U.e[1] * U.e[2];
  U.q0 = qp * 2 * kTile;
  if (U.q0 >= U.n_valid) return false;   // a truncated window has fewer query pairs
  U.has_q1 = U.q0 + kTile < U.n_valid;
  U.nkv = (U.n_valid + kTile - 1) / kTile;
  U.nkv_win = U.nkv;
  U.nkv_rt = 0;
  if (kRoute) {
    route_of(p.g, p.routed, p.heads, win_id, U);
    U.nkv += U.nkv_rt;
  }
  U.n_extra = kMem ? p.n_extra : 0;
  if (kMem) U.nkv += (p.n_extra + kTile - 1) / kTile;
  return true;
}

__device__ __forceinline__ int unit_row(const FwdParams& p, const Unit& U, int slot) {
  if (slot >= U.n_valid) slot = U.n_valid - 1;   // padding rows repeat the last token
  return (U.b * p.g.N + slot_token(p.g, U.m, U.e, slot)) * p.heads + U.h;
}

// Key tile j of a unit: segment 0 = the window's tiles, 1 = the routed
// window's (kRoute), 2 = the extra segment's (kMem); *t0 = the first key of
// the tile within its segment.
template <bool kMem, bool kRoute>
__device__ __forceinline__ int seg_of(const Unit& U, int j, int* t0) {
  if ((kMem || kRoute) && j >= U.nkv_win) {
    const int jr = j - U.nkv_win;
    if (kRoute && jr < U.nkv_rt) {
      *t0 = jr * kTile;
      return 1;
    }
    *t0 = (jr - (kRoute ? U.nkv_rt : 0)) * kTile;
    return 2;
  }
  *t0 = j * kTile;
  return 0;
}

// Valid keys of key tile j.
template <bool kMem, bool kRoute>
__device__ __forceinline__ int kv_valid_of(const Unit& U, int j) {
  int t0;
  const int seg = seg_of<kMem, kRoute>(U, j, &t0);
  const int n = seg == 0 ? U.n_valid : (seg == 1 ? U.n_route : U.n_extra);
  const int left = n - t0;
  return left < kTile ? left : kTile;
}

// Rows of the extra segment's tokens s .. s+3 for unit U in the 2D
// [B*n_extra*heads, d] view of the extra K/V: row = (b*n_extra + token)*heads + h;
// tokens at or past n_extra repeat the last one.
__device__ __forceinline__ void extra_rows4(const Unit& U, int heads, int s, int r[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int t = s + k < U.n_extra ? s + k : U.n_extra - 1;
    r[k] = (U.b * U.n_extra + t) * heads + U.h;
  }
}

// Rows of slots s .. s+3 of unit U in the 2D [B*N*heads, d] view of Q/K/V/out,
// row = (b*N + token)*heads + h; slots at or past n_valid repeat the last valid
// slot's row.  The same tokens as slot_token(), slot by slot: the first slot is
// split into (s_t, s_h, s_w) with divisions, the next three step along the
// raster order.
__device__ __forceinline__ void win_rows4(const Geometry& g, int b, int h, const int m[3], const int e[3],
                                          int heads, int s, int r[4]) {
  const int q = div_extent(g, 2, s, e[2]);
  int sw = s - q * e[2];
  int st = div_extent(g, 1, q, e[1]);
  int sh = q - st * e[1];
  const int base_t = m[0] * g.w[0] + g.delta[0];
  const int base_h = m[1] * g.w[1] + g.delta[1];
  const int base_w = m[2] * g.w[2] + g.delta[2];
  const int tok0 = b * g.N;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool pad = st >= e[0];
    int pt = base_t + (pad ? e[0] - 1 : st);
    int ph = base_h + (pad ? e[1] - 1 : sh);
    int pw = base_w + (pad ? e[2] - 1 : sw);
    if (pt >= g.n[0]) pt -= g.n[0];
    if (ph >= g.n[1]) ph -= g.n[1];
    if (pw >= g.n[2]) pw -= g.n[2];
    r[k] = (tok0 + (pt * g.n[1] + ph) * g.n[2] + pw) * heads + h;
    if (++sw == e[2]) {
      sw = 0;
      if (++sh == e[1]) {
        sh = 0;
        ++st;
      }
    }
  }
}

__device__ __forceinline__ void unit_rows4(const Geometry& g, const Unit& U, int heads, int s,
                                           int r[4]) {
  win_rows4(g, U.b, U.h, U.m, U.e, heads, s, r);
}

// Rows of segment seg (0 window, 1 routed window, 2 extra segment) of unit U
// for the segment's keys s .. s+3.
template <bool kMem, bool kRoute>
__device__ __forceinline__ void seg_rows4(const Geometry& g, const Unit& U, int heads, int seg, int s,
                                          int r[4]) {
  if (kMem && seg == 2)
    extra_rows4(U, heads, s, r);
  else if (kRoute && seg == 1)
    win_rows4(g, U.b, U.h, U.rm, U.re, heads, s, r);
  else
    unit_rows4(g, U, heads, s, r);
}

// One key step of the online softmax for the S row of this thread at TMEM
// address tS (128 fp32 columns): the row maximum against the running maximum
// m_run (updated only when it grows by more than kRescaleThreshold; then alpha
// = 2^(m_old - m_new) and need is set), P = 2^(S*sl2 - m_run) in bf16 written
// back over the front of the row, and the fp32 sum of P returned.  The whole
// row comes in one TMEM load and P goes out in two 32-column stores, so S and
// P each sit in one contiguous run of registers; columns >= kv_valid (the last
// tile of a window) are masked, not skipped.
__device__ __forceinline__ float softmax_row_step(uint32_t tS, int kv_valid, float sl2, float& m_run,
                                                  float& alpha, bool& need) {
  float x[kTile];
  {
    uint32_t r[kTile];
    tmem_ld128(tS, r);
    tmem_wait_ld();
    tmem_tie(r);
#pragma unroll
    for (int i = 0; i < kTile; ++i) x[i] = __uint_as_float(r[i]);
  }
  if (kv_valid < kTile) {
#pragma unroll
    for (int i = 0; i < kTile; ++i)
      if (i >= kv_valid) x[i] = -INFINITY;
  }
  const float mx = row_max128(x);
  const float m_new = fmaxf(m_run, mx * sl2);
  need = m_new > m_run + kRescaleThreshold;
  alpha = 1.0f;
  if (need) {
    alpha = ex2_approx(m_run - m_new);
    m_run = m_new;
  }
  const float neg_m = -m_run;
  uint32_t pk[32];
  float rowsum = kv_valid < kTile ? softmax_half_to_pk<true, 0>(x, kv_valid, sl2, neg_m, pk)
                                  : softmax_half_to_pk<false, 0>(x, kv_valid, sl2, neg_m, pk);
  tmem_st32(tS, pk);
  rowsum += kv_valid < kTile ? softmax_half_to_pk<true, 1>(x, kv_valid, sl2, neg_m, pk)
                             : softmax_half_to_pk<false, 1>(x, kv_valid, sl2, neg_m, pk);
  tmem_st32(tS + 32, pk);
  return rowsum;
}

// S_i (+)= Q_i K^T over the head dimension: d/16 MMAs of M=128, N=n_s, K=16.
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr, int d,
                                         int n_s) {
  // Descriptors of the K = 16 slices are the tile's base descriptor plus the
  // slice's byte offset / 16 in the start-address field (shared-memory
  // addresses stay below 2^18, so the field never carries).
  const uint32_t idesc = idesc_bf16_f32(128, n_s, 0, 0);
  const uint64_t qd = smem_desc_sw128(q_addr, 16, 1024), kd = smem_desc_sw128(k_addr, 16, 1024);
  if (d == 64) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      umma_ss(tmem_s, qd + ((kk * 32) >> 4), kd + ((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = ((kk >> 2) * (kTile * 128) + (kk & 3) * 32) >> 4;
      umma_ss(tmem_s, qd + off, kd + off, idesc, kk > 0 ? 1u : 0u);
    }
  }
}

// O_i (+)= P_i V over the keys of one tile: P_i (bf16) sits in TMEM at tmem_p.
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr, int d,
                                         int kv_valid, bool accumulate) {
  const uint32_t idesc = idesc_bf16_f32(128, d, 0, 1);
  const uint64_t vd = smem_desc_sw128(v_addr, kTile * 128, 1024);
  const int ksteps = (kv_valid + 15) >> 4;
  if (ksteps == kTile / 16) {
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      umma_ts(tmem_o, tmem_p + kk * 8, vd + kk * (2048 >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  } else {
    for (int kk = 0; kk < ksteps; ++kk)
      umma_ts(tmem_o, tmem_p + kk * 8, vd + kk * (2048 >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <bool kMem, bool kRoute>
__global__ void __launch_bounds__(kThreads, 1) swattn_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int d = p.d;
  const int tile_bytes = kTile * d * 2;
  const int n_slots = p.n_slots;
  uint8_t* sQ = smem;                           // two query tiles
  uint8_t* sRing = sQ + 2 * tile_bytes;         // K/V ring
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sRing + n_slots * tile_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->q_full[i], kProducers);
      mbar_init(&ctl->q_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->o_final[i], 1);
    }
    for (int s = 0; s < n_slots; ++s) {
      mbar_init(&ctl->kv_full[s], kProducers);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    mbar_init(&ctl->drained, 1);
    mbar_init(&ctl->never, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp0 && lane == 0) {
    prefetch_tensormap(&p.tq);
    prefetch_tensormap(&p.tk);
    prefetch_tensormap(&p.tv);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp >= kProducerWarp0 && warp < kProducerWarp0 + kProducers) {
    // ================================================================ TMA producers
    // A tile is 32 * ncb gathers (4 rows x 64 columns each); gather n covers
    // rows 4 (n / ncb) + [0, 4) and column block n % ncb and belongs to lane
    // n / 2 of producer warp n % 2, which computes its own row coordinates.
    // Every lane with a gather issues it in the same instruction.
    const int pw = warp - kProducerWarp0;
    const int ncb = d / 64;   // 128-byte column blocks per row
    const uint32_t half_bytes = tile_bytes / kProducers;
    uint32_t q_use[2] = {0, 0};
    uint32_t ld = 0;          // loads issued into the ring
    int fill_slot = 0;        // ld % n_slots and ld / n_slots, kept incrementally
    uint32_t fill_use = 0;
    bool ok = true;
    // seg: the segment the tile comes from (0 window, 1 routed window, 2 extra
    // segment); slot0 counts that segment's tokens.
    auto issue = [&](const Unit& U, int slot0, const CUtensorMap* map, uint64_t* bar, uint8_t* tile,
                     int seg) {
      if (elect_one()) mbar_arrive_expect_tx(bar, half_bytes);
      __syncwarp();
      for (int n = pw + kProducers * lane; n < 32 * ncb; n += 32 * kProducers) {
        const int grp = n / ncb, c = n - grp * ncb;
        int r[4];
        seg_rows4<kMem, kRoute>(p.g, U, p.heads, seg, slot0 + 4 * grp, r);
        tma_gather4(map, bar, tile + c * (kTile * 128) + grp * 512, c * 64, r[0], r[1], r[2], r[3]);
      }
      __syncwarp();
    };
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
      Unit U;
      if (!decode_unit<kMem, kRoute>(p, u, U)) continue;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (i == 1 && !U.has_q1) break;
        if (q_use[i] > 0) {
          ok = __all_sync(0xffffffffu,
                          wait_or_abort(&ctl->q_empty[i], (q_use[i] - 1) & 1, ctl, p.timeout_ns));
          if (!ok) break;
        }
        issue(U, U.q0 + i * kTile, &p.tq, &ctl->q_full[i], sQ + i * tile_bytes, 0);
        ++q_use[i];
      }
      for (int j = 0; ok && j < U.nkv; ++j) {
        for (int kv = 0; kv < 2; ++kv) {
          const int slot = fill_slot;
          const uint32_t use = fill_use;
          if (++fill_slot == n_slots) {
            fill_slot = 0;
            ++fill_use;
          }
          if (use > 0) {
            ok = __all_sync(0xffffffffu,
                            wait_or_abort(&ctl->kv_empty[slot], (use - 1) & 1, ctl, p.timeout_ns));
            if (!ok) break;
          }
          int t0;
          const int seg = seg_of<kMem, kRoute>(U, j, &t0);
          const CUtensorMap* map = (kMem && seg == 2) ? (kv == 0 ? &p.tkx : &p.tvx) : (kv == 0 ? &p.tk : &p.tv);
          issue(U, t0, map, &ctl->kv_full[slot], sRing + slot * tile_bytes, seg);
          ++ld;
        }
      }
    }
    // Drain: every load issued has landed before the CTA can exit.  In the
    // normal flow these phases completed long ago and the waits return at once.
    for (int i = 0; i < 2; ++i)
      if (q_use[i] > 0) mbar_wait_bounded(&ctl->q_full[i], (q_use[i] - 1) & 1, drain_ns(p.timeout_ns));
    for (uint32_t x = (ld > static_cast<uint32_t>(n_slots) ? ld - n_slots : 0); x < ld; ++x)
      mbar_wait_bounded(&ctl->kv_full[x % n_slots], (x / n_slots) & 1, drain_ns(p.timeout_ns));
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr[2] = {smem_u32(sQ), smem_u32(sQ + tile_bytes)};
      const uint32_t ring_addr = smem_u32(sRing);
      const uint32_t tS[2] = {tmem + kColS0, tmem + kColS1};
      const uint32_t tO[2] = {tmem + kColO0, tmem + kColO1};
      uint32_t q_use[2] = {0, 0};
      uint32_t p_use[2] = {0, 0};
      // Ring position of the next K/V tile to consume and the parity of its
      // fill, kept incrementally (no division between two MMA batches).
      int kv_slot = 0;
      uint32_t kv_phase = 0;
      auto take = [&](int& slot, uint32_t& phase) {
        slot = kv_slot;
        phase = kv_phase;
        if (++kv_slot == n_slots) {
          kv_slot = 0;
          kv_phase ^= 1u;
        }
      };
      bool ok = !p.stall || wait_or_abort(&ctl->never, 0, ctl, p.timeout_ns);
      for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        Unit U;
        if (!decode_unit<kMem, kRoute>(p, u, U)) continue;
        const int nq = U.has_q1 ? 2 : 1;
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (ok && i < nq) ok = wait_or_abort(&ctl->q_full[i], q_use[i] & 1, ctl, p.timeout_ns);
        if (!ok) break;
        // K_0 -> S_i(0)
        int slot_k;
        uint32_t phase_k;
        take(slot_k, phase_k);
        ok = wait_or_abort(&ctl->kv_full[slot_k], phase_k, ctl, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        {
          const int n_s = (kv_valid_of<kMem, kRoute>(U, 0) + 15) & ~15;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (i >= nq) break;
            issue_qk(tS[i], q_addr[i], ring_addr + slot_k * tile_bytes, d, n_s);
            umma_commit(&ctl->s_full[i]);
            if (U.nkv == 1) umma_commit(&ctl->q_empty[i]);
          }
          umma_commit(&ctl->kv_empty[slot_k]);
        }
        for (int j = 0; j < U.nkv; ++j) {
          int slot_v;
          uint32_t phase_v;
          take(slot_v, phase_v);
          ok = wait_or_abort(&ctl->kv_full[slot_v], phase_v, ctl, p.timeout_ns);
          if (!ok) break;
          const bool more = j + 1 < U.nkv;
          const int kvv = kv_valid_of<kMem, kRoute>(U, j);
          const int n_s = more ? (kv_valid_of<kMem, kRoute>(U, j + 1) + 15) & ~15 : 0;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (i >= nq) break;
            ok = wait_or_abort(&ctl->p_full[i], p_use[i] & 1, ctl, p.timeout_ns);
            if (!ok) break;
            ++p_use[i];
            tc_fence_after();
            issue_pv(tO[i], tS[i], ring_addr + slot_v * tile_bytes, d, kvv, j > 0);
            if (more && i == 0) {
              // K of the next step: waited for here, after this tile's P V
              take(slot_k, phase_k);
              ok = wait_or_abort(&ctl->kv_full[slot_k], phase_k, ctl, p.timeout_ns);
              if (!ok) break;
              tc_fence_after();
            }
            if (more) {
              issue_qk(tS[i], q_addr[i], ring_addr + slot_k * tile_bytes, d, n_s);
              umma_commit(&ctl->s_full[i]);
              if (j + 1 == U.nkv - 1) umma_commit(&ctl->q_empty[i]);
            } else {
              umma_commit(&ctl->o_final[i]);
            }
            if (i == nq - 1) {
              umma_commit(&ctl->kv_empty[slot_v]);
              if (more) umma_commit(&ctl->kv_empty[slot_k]);
            }
          }
          if (!ok) break;
        }
        ++q_use[0];
        if (nq == 2) ++q_use[1];
      }
      // Drain every MMA this thread issued before TMEM is released.
      umma_commit(&ctl->drained);
      mbar_wait_bounded(&ctl->drained, 0, drain_ns(p.timeout_ns));
    }
    __syncwarp();
  } else {
    // ================================================================ softmax (+ correction, epilogue)
    const int wg = warp >> 2;                         // query tile 0 or 1
    const int row = threadIdx.x & 127;                // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + (wg ? kColS1 : kColS0) + lane_off;
    const uint32_t tO = tmem + (wg ? kColO1 : kColO0) + lane_off;
    const float sl2 = p.scale_log2;
    uint32_t s_use = 0, of_use = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
      Unit U;
      if (!decode_unit<kMem, kRoute>(p, u, U)) continue;
      if (wg == 1 && !U.has_q1) continue;
      float m_run = -INFINITY;   // running max of scale*log2(e)*S (possibly stale by < 8)
      float l_run = 0.0f;        // running sum of exp2(x - m_run)
      for (int j = 0; j < U.nkv; ++j) {
        ok = __all_sync(0xffffffffu, wait_or_abort(&ctl->s_full[wg], s_use & 1, ctl, p.timeout_ns));
        if (!ok) break;
        ++s_use;
        tc_fence_after();
        float alpha;
        bool need;
        const float rowsum = softmax_row_step(tS, kv_valid_of<kMem, kRoute>(U, j), sl2, m_run, alpha, need);
        l_run = l_run * alpha + rowsum;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O_i holds P V of tiles 0..j-1 (complete: S_i(j) was issued after
          // them) relative to the old max; rescale the row by alpha.  Done
          // after P so that the S row is no longer live in registers.
          for (int c = 0; c < d / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[wg]);
      }
      if (!ok) break;
      // ---- epilogue: O / l in bf16, stored at the row the query came from
      ok = __all_sync(0xffffffffu, wait_or_abort(&ctl->o_final[wg], of_use & 1, ctl, p.timeout_ns));
      if (!ok) break;
      ++of_use;
      tc_fence_after();
      const int slot = U.q0 + wg * kTile + row;
      const bool valid = slot < U.n_valid;
      __nv_bfloat16* dst = nullptr;
      if (valid)
        dst = p.out + static_cast<size_t>(unit_row(p, U, slot)) * d;
      const float inv_l = 1.0f / l_run;
      for (int c = 0; c < d / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      tc_fence_before();   // O_i reads are ordered before the next unit's P V (via p_full)
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================================
// CTA-pair kernel (head dim 128): the same computation with tcgen05 MMAs of
// M = 256 split over the two CTAs of a cluster.  Each CTA owns 128 query rows
// of every tile and half of every K/V tile (half of the keys of K, half of the
// head dimension of V), so each SM loads half the K/V bytes of the one-CTA
// kernel and each MMA reads half of its B operand from each SM.
//
// Per CTA: warps 0-7 softmax (two query tiles, ping-pong), then the TMA
// producer warps, then the TMEM owner warp, which in the leader CTA (rank 0)
// also issues every MMA of the pair.  Barriers that gate MMAs (q_full, kv_full,
// p_full) live in the leader and count both CTAs; barriers that MMAs signal
// (s_full, o_final, q_empty, kv_empty) are arrived on in both CTAs.
// ============================================================================

#ifndef SWATTN_PAIR_PRODUCERS
#define SWATTN_PAIR_PRODUCERS 3
#endif
constexpr int kPairProducer0 = 8;
constexpr int kPairProducers = SWATTN_PAIR_PRODUCERS;
constexpr int kPairMmaWarp = kPairProducer0 + kPairProducers;
constexpr int kPairThreads = (kPairMmaWarp + 1) * 32;
constexpr int kPairHalfTileBytes = 16384;   // a K half (64 keys x 128) or V half (128 keys x 64)
constexpr int kPairMaxSlots = 12;

struct __align__(64) PairParams {
  CUtensorMap tq, tk, tv;       // 2D [rows = B*N*heads, cols = 128], box {64, 1}, 128B swizzle
  CUtensorMap tkx, tvx;         // extra K/V segment, 2D [rows = B*n_extra*heads, cols = 128] (kMem)
  CUtensorMap to;               // the output, same view as tq (tile::scatter4 stores of the epilogue)
  int n_extra;                  // extra keys appended to every window (kMem)
  const int* routed;            // [B, heads, n_windows] routed window of each window, or none (kRoute)
  __nv_bfloat16* out;
  Geometry g;
  int B, heads;
  int q_quads;                  // ceil(nw_max / 512): 512-query units per window
  FastDiv f_qq, f_nw, f_heads;  // by q_quads, n_windows, heads
  int total_units;
  int n_slots;
  float scale_log2;
  unsigned long long timeout_ns;
  int stall;                    // test hook: the MMA issuer first waits on a barrier nothing arrives on
};

// Query tiles are double-buffered: the units a CTA pair runs alternate between
// two sets of two tiles, so the next unit's queries load while the current one
// runs.  When a unit is done, its set's tile i holds the bf16 output rows of
// tile i on their way to the TMA stores, and is refilled only after those
// stores have read it.
struct PairCtl {
  uint64_t q_full[2][2];        // leader: both CTAs' Q tile i of set s landed
  uint64_t q_free[2][2];        // each CTA: its Q tile i of set s may be refilled
  uint64_t kv_full[kPairMaxSlots];   // leader: both halves of a ring slot landed
  uint64_t kv_empty[kPairMaxSlots];  // both: ring slot may be overwritten
  uint64_t s_full[2];           // both: S_i in TMEM
  uint64_t p_full[2];           // leader: P_i written (and O_i rescaled) in both CTAs
  uint64_t o_final[2];          // both: last P V of the unit for tile i done
  uint64_t drained;             // leader: every MMA done
  uint64_t never;               // test hook: never arrived on
  uint32_t tmem_base;
  int abort;
};

static_assert(offsetof(PairCtl, q_full) % 8 == 0, "mbarriers are 8-byte aligned");

__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, PairCtl* ctl,
                                          unsigned long long timeout_ns, bool cluster_scope) {
  if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
  const bool ok = cluster_scope ? mbar_wait_bounded_cluster(bar, parity, timeout_ns)
                                : mbar_wait_bounded(bar, parity, timeout_ns);
  if (ok) return true;
  *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
  atomicOr(&g_device_error, 1);
  return false;
}

// A pair unit: up to 512 queries; tile i of CTA c holds slots q0 + 256 i + 128 c + [0, 128).
template <bool kMem, bool kRoute>
__device__ __forceinline__ bool decode_pair_unit(const PairParams& p, int u, Unit& U) {
  const int r = fdiv(u, p.f_qq);
  const int qp = u - r * p.q_quads;
  const int bh = fdiv(r, p.f_nw);
  const int win_id = r - bh * p.g.n_windows;
  U.b = fdiv(bh, p.f_heads);
  U.h = bh - U.b * p.heads;
  window_of(p.g, win_id, U.m, U.e);
  U.n_valid = U.e[0] * U.e[1] * U.e[2];
  U.q0 = qp * 4 * kTile;
  if (U.q0 >= U.n_valid) return false;
  U.has_q1 = U.q0 + 2 * kTile < U.n_valid;
  U.nkv = (U.n_valid + kTile - 1) / kTile;
  U.nkv_win = U.nkv;
  U.nkv_rt = 0;
  if (kRoute) {
    route_of(p.g, p.routed, p.heads, win_id, U);
    U.nkv += U.nkv_rt;
  }
  U.n_extra = kMem ? p.n_extra : 0;
  if (kMem) U.nkv += (p.n_extra + kTile - 1) / kTile;
  return true;
}

// Keys of tile j used by the MMAs: all 128, or the valid keys rounded up to 32
// for the last tile (each CTA then holds half of them).
template <bool kMem, bool kRoute>
__device__ __forceinline__ int pair_ns(const Unit& U, int j) {
  const int kvv = kv_valid_of<kMem, kRoute>(U, j);
  return kvv == kTile ? kTile : ((kvv + 31) & ~31);
}

template <bool kMem, bool kRoute>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    swattn_fwd_pair_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kQBytes = kTile * 128 * 2;
  const int n_slots = p.n_slots;
  uint8_t* sQ = smem;                                   // two sets of two own query tiles
  uint8_t* sRing = sQ + 4 * kQBytes;                    // K/V half tiles
  PairCtl* ctl = reinterpret_cast<PairCtl*>(sRing + n_slots * kPairHalfTileBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s)
      for (int i = 0; i < 2; ++i) {
        mbar_init(&ctl->q_full[s][i], 1);
        mbar_init(&ctl->q_free[s][i], 4);
      }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_full[i], 8);
      mbar_init(&ctl->o_final[i], 1);
    }
    for (int s = 0; s < n_slots; ++s) {
      mbar_init(&ctl->kv_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    mbar_init(&ctl->drained, 1);
    mbar_init(&ctl->never, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kPairProducer0 && lane == 0) {
    prefetch_tensormap(&p.tq);
    prefetch_tensormap(&p.tk);
    prefetch_tensormap(&p.tv);
    prefetch_tensormap(&p.to);
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp >= kPairProducer0 && warp < kPairProducer0 + kPairProducers) {
    // ================================================================ TMA producers
    // Gathers of every tile are spread over the producer warps' lanes (see
    // `gathers`).  Loads land in this CTA and are counted on the leader's barriers.
    const int pw = warp - kPairProducer0;
    // Q buffer b = 2 * set + tile: bit b of q_par is the parity of the loads
    // into it so far, bit b of q_loaded is set once it has been loaded
    uint32_t q_par = 0, q_loaded = 0;
    uint32_t ld = 0;
    int fill_slot = 0;                         // ld % n_slots and ld / n_slots, kept incrementally
    uint32_t fill_use = 0;
    uint32_t lu = 0;                           // units of this CTA pair so far
    bool ok = true;
    // `count` gathers numbered 0..count-1 cover slots slot0 + [0, 4 * count / nblk):
    // gather n covers row group n / nblk (slots slot0 + 4 (n / nblk) + [0, 4)) and
    // column block n % nblk, landing at dst + (n / nblk) * 512 + (n % nblk) * blk_stride,
    // columns col0 + 64 * (n % nblk).  Gather n belongs to lane (n / P) mod 32 of
    // producer warp n mod P (P producer warps), which computes its own four row
    // coordinates; every lane with a gather issues it in the same instruction, so
    // a warp puts up to 32 gathers in flight per issue.
    // seg: the segment the rows come from (0 window, 1 routed window, 2 extra
    // segment); slot0 counts that segment's tokens.
    auto gathers = [&](const Unit& U, const CUtensorMap* map, uint32_t bar_leader, uint8_t* dst,
                       int slot0, int count, int nblk, int blk_stride, int col0, int seg) {
      for (int base = 0; base < count; base += 32 * kPairProducers) {
        const int n = base + pw + kPairProducers * lane;
        if (n < count) {
          const int grp = n / nblk, blk = n - grp * nblk;
          int r[4];
          seg_rows4<kMem, kRoute>(p.g, U, p.heads, seg, slot0 + 4 * grp, r);
          tma_gather4_pair(map, bar_leader, dst + grp * 512 + blk * blk_stride, col0 + 64 * blk, r[0],
                           r[1], r[2], r[3]);
        }
      }
      __syncwarp();
    };
    for (int u = cluster_id; ok && u < p.total_units; u += n_clusters) {
      Unit U;
      if (!decode_pair_unit<kMem, kRoute>(p, u, U)) continue;
      const int set = lu & 1;
      ++lu;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (i == 1 && !U.has_q1) break;
        const uint32_t b = 2 * set + i;
        if ((q_loaded >> b) & 1) {
          ok = __all_sync(0xffffffffu, pair_wait(&ctl->q_free[set][i], ((q_par >> b) & 1) ^ 1, ctl,
                                                 p.timeout_ns, false));
          if (!ok) break;
        }
        const uint32_t bar = map_to_rank(smem_u32(&ctl->q_full[set][i]), 0);
        if (leader && pw == 0 && elect_one()) mbar_arrive_expect_tx(&ctl->q_full[set][i], 2 * kQBytes);
        __syncwarp();
        gathers(U, &p.tq, bar, sQ + (2 * set + i) * kQBytes,
                U.q0 + i * 2 * kTile + static_cast<int>(rank) * kTile, 64, 2, kTile * 128, 0, 0);
        q_par ^= 1u << b;
        q_loaded |= 1u << b;
      }
      for (int j = 0; ok && j < U.nkv; ++j) {
        const int ns = pair_ns<kMem, kRoute>(U, j);
        const int half = ns >> 1;
        for (int kv = 0; kv < 2; ++kv) {
          const int slot = fill_slot;
          const uint32_t use = fill_use;
          if (++fill_slot == n_slots) {
            fill_slot = 0;
            ++fill_use;
          }
          if (use > 0) {
            ok = __all_sync(0xffffffffu, pair_wait(&ctl->kv_empty[slot], (use - 1) & 1, ctl,
                                                   p.timeout_ns, false));
            if (!ok) break;
          }
          const uint32_t bar = map_to_rank(smem_u32(&ctl->kv_full[slot]), 0);
          if (leader && pw == 0 && elect_one())
            mbar_arrive_expect_tx(&ctl->kv_full[slot], static_cast<uint32_t>(ns) * 256u);
          __syncwarp();
          uint8_t* dst = sRing + slot * kPairHalfTileBytes;
          // Tiles past the window's come from the routed window (kRoute), then
          // from the extra segment (kMem).
          int t0;
          const int seg = seg_of<kMem, kRoute>(U, j, &t0);
          const bool extra = kMem && seg == 2;
          if (kv == 0)   // K: keys [rank*half, rank*half + half), both column blocks
            gathers(U, extra ? &p.tkx : &p.tk, bar, dst, t0 + static_cast<int>(rank) * half, (half >> 2) * 2, 2,
                    64 * 128, 0, seg);
          else           // V: keys [0, ns), the column block of this CTA's half of d
            gathers(U, extra ? &p.tvx : &p.tv, bar, dst, t0, ns >> 2, 1, 0, 64 * static_cast<int>(rank), seg);
          ++ld;
        }
      }
    }
    // Drain: in the leader, every load of either CTA is counted on these
    // barriers; the final cluster barrier keeps the peer alive until then.
    if (leader) {
      for (int b = 0; b < 4; ++b)
        if ((q_loaded >> b) & 1)
          mbar_wait_bounded(&ctl->q_full[b >> 1][b & 1], ((q_par >> b) & 1) ^ 1, drain_ns(p.timeout_ns));
      for (uint32_t x = (ld > static_cast<uint32_t>(n_slots) ? ld - n_slots : 0); x < ld; ++x)
        mbar_wait_bounded(&ctl->kv_full[x % n_slots], (x / n_slots) & 1, drain_ns(p.timeout_ns));
    }
  } else if (warp == kPairMmaWarp) {
    // ================================================================ MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t ring_addr = smem_u32(sRing);
      const uint32_t idesc_pv = idesc_bf16_f32(256, 128, 0, 1);
      uint32_t q_par = 0;     // bit 2 * set + tile: parity of the uses of that Q buffer so far
      uint32_t p_use[2] = {0, 0};
      // Ring position of the next K/V tile to consume and the parity of its
      // fill, kept incrementally: this thread's code between two MMA batches
      // runs on the critical path, so no division or remainder appears there.
      int kv_slot = 0;
      uint32_t kv_phase = 0;
      auto take = [&](int& slot, uint32_t& phase) {
        slot = kv_slot;
        phase = kv_phase;
        if (++kv_slot == n_slots) {
          kv_slot = 0;
          kv_phase ^= 1u;
        }
      };
      uint32_t lu = 0;
      bool ok = !p.stall || pair_wait(&ctl->never, 0, ctl, p.timeout_ns, false);
      // Descriptors of the K = 16 slices are the tile's base descriptor plus the
      // slice's byte offset / 16 (the start-address field; shared-memory
      // addresses are 16-byte multiples far below 2^18, so the field never
      // carries into its neighbours).
      auto issue_qk = [&](uint32_t q_addr, int i, uint32_t k_addr, int ns) {
        const uint32_t idesc = idesc_bf16_f32(256, ns, 0, 0);
        const uint64_t qd = smem_desc_sw128(q_addr, 16, 1024), kd = smem_desc_sw128(k_addr, 16, 1024);
        const uint32_t tS = tmem + (i ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss_pair(tS, qd + (((kk >> 2) * (kTile * 128) + (kk & 3) * 32) >> 4),
                       kd + (((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int i, uint32_t v_addr, int ns, bool acc) {
        const uint32_t tS = tmem + (i ? kColS1 : kColS0);
        const uint32_t tO = tmem + (i ? kColO1 : kColO0);
        const uint64_t vd = smem_desc_sw128(v_addr, kTile * 128, 1024);
        if (ns == kTile) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts_pair(tO, tS + kk * 8, vd + kk * (2048 >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        } else {
          for (int kk = 0; kk < ns / 16; ++kk)
            umma_ts_pair(tO, tS + kk * 8, vd + kk * (2048 >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      for (int u = cluster_id; ok && u < p.total_units; u += n_clusters) {
        Unit U;
        if (!decode_pair_unit<kMem, kRoute>(p, u, U)) continue;
        const int set = lu & 1;
        ++lu;
        const uint32_t q_addr[2] = {smem_u32(sQ + (2 * set) * kQBytes), smem_u32(sQ + (2 * set + 1) * kQBytes)};
        const int nq = U.has_q1 ? 2 : 1;
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (ok && i < nq)
            ok = pair_wait(&ctl->q_full[set][i], (q_par >> (2 * set + i)) & 1, ctl, p.timeout_ns, false);
        if (!ok) break;
        int slot_k;
        uint32_t phase_k;
        take(slot_k, phase_k);
        ok = pair_wait(&ctl->kv_full[slot_k], phase_k, ctl, p.timeout_ns, false);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (i >= nq) break;
          issue_qk(q_addr[i], i, ring_addr + slot_k * kPairHalfTileBytes, pair_ns<kMem, kRoute>(U, 0));
          umma_commit_pair(&ctl->s_full[i], 3);
        }
        umma_commit_pair(&ctl->kv_empty[slot_k], 3);
        for (int j = 0; j < U.nkv; ++j) {
          // V of this step and K of the next: both are waited for here, before
          // the first P is, so that a tile's P V and Q K^T batches follow each
          // other with nothing in between
          int slot_v;
          uint32_t phase_v;
          take(slot_v, phase_v);
          ok = pair_wait(&ctl->kv_full[slot_v], phase_v, ctl, p.timeout_ns, false);
          if (!ok) break;
          const bool more = j + 1 < U.nkv;
          if (more) {
            take(slot_k, phase_k);
            ok = pair_wait(&ctl->kv_full[slot_k], phase_k, ctl, p.timeout_ns, false);
            if (!ok) break;
          }
          const int ns = pair_ns<kMem, kRoute>(U, j);
          const int ns_next = more ? pair_ns<kMem, kRoute>(U, j + 1) : 0;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (i >= nq) break;
            ok = pair_wait(&ctl->p_full[i], p_use[i] & 1, ctl, p.timeout_ns, false);
            if (!ok) break;
            ++p_use[i];
            tc_fence_after();
            issue_pv(i, ring_addr + slot_v * kPairHalfTileBytes, ns, j > 0);
            if (more) {
              issue_qk(q_addr[i], i, ring_addr + slot_k * kPairHalfTileBytes, ns_next);
              umma_commit_pair(&ctl->s_full[i], 3);
            } else {
              umma_commit_pair(&ctl->o_final[i], 3);
            }
            if (i == nq - 1) {
              umma_commit_pair(&ctl->kv_empty[slot_v], 3);
              if (more) umma_commit_pair(&ctl->kv_empty[slot_k], 3);
            }
          }
          if (!ok) break;
        }
        q_par ^= (nq == 2 ? 3u : 1u) << (2 * set);
      }
      umma_commit_pair(&ctl->drained, 1);
      mbar_wait_bounded(&ctl->drained, 0, drain_ns(p.timeout_ns));
    }
    __syncwarp();
  } else {
    // ================================================================ softmax (+ correction, epilogue)
    const int wg = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + (wg ? kColS1 : kColS0) + lane_off;
    const uint32_t tO = tmem + (wg ? kColO1 : kColO0) + lane_off;
    const uint32_t p_full_leader = map_to_rank(smem_u32(&ctl->p_full[wg]), 0);
    const float sl2 = p.scale_log2;
    uint32_t s_use = 0, of_use = 0;
    uint32_t lu = 0;
    int pending = -1;   // set whose tile wg holds output rows the TMA stores may still be reading
    // Hands tile wg of set `pending` back to the producers once this warp's
    // stores have read it.
    auto release = [&]() {
      if (pending >= 0) {
        bulk_wait_group_read0();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->q_free[pending][wg]);
        pending = -1;
      }
    };
    bool ok = true;
    for (int u = cluster_id; ok && u < p.total_units; u += n_clusters) {
      Unit U;
      if (!decode_pair_unit<kMem, kRoute>(p, u, U)) continue;
      const int set = lu & 1;
      ++lu;
      if (wg == 1 && !U.has_q1) {
        release();
        continue;
      }
      float m_run = -INFINITY;
      float l_run = 0.0f;
      for (int j = 0; j < U.nkv; ++j) {
        ok = __all_sync(0xffffffffu, pair_wait(&ctl->s_full[wg], s_use & 1, ctl, p.timeout_ns, false));
        if (!ok) break;
        ++s_use;
        tc_fence_after();
        float alpha;
        bool need;
        const float rowsum = softmax_row_step(tS, kv_valid_of<kMem, kRoute>(U, j), sl2, m_run, alpha, need);
        l_run = l_run * alpha + rowsum;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(p_full_leader);
        if (j == 0) release();   // the previous unit's stores read their tile long ago
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, pair_wait(&ctl->o_final[wg], of_use & 1, ctl, p.timeout_ns, false));
      if (!ok) break;
      ++of_use;
      tc_fence_after();
      // the unit's window geometry, decoded again rather than held in registers
      // through the key loop
      decode_pair_unit<kMem, kRoute>(p, u, U);
      // ---- epilogue: O / l in bf16 into this tile's (now unused) query buffer,
      // laid out as a load through the same tensor map leaves rows (row r at
      // r * 128 in each 64-column block, 16-byte chunk c at position c ^ (r & 7)),
      // then tile::scatter4 stores put each group of four rows at the rows its
      // queries came from (the inverse roll) while this warp moves on.
      uint8_t* stage = sQ + (2 * set + wg) * kQBytes;
      const float inv_l = 1.0f / l_run;
      uint32_t ra[32], rb[32];
      tmem_ld32(tO, ra);
      tmem_wait_ld();
      tmem_tie(ra);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t(&cur)[32] = (c & 1) ? rb : ra;
        uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
        if (c < 3) tmem_ld32(tO + (c + 1) * 32, nxt);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int q = 4 * c + v4;   // 16-byte chunk of the 256-byte row
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(cur[8 * v4 + 2 * e]) * inv_l,
                                __uint_as_float(cur[8 * v4 + 2 * e + 1]) * inv_l);
          st_shared_v4(stage + (q >> 3) * (kTile * 128) + row * 128 + (((q & 7) ^ (row & 7)) << 4), pk[0], pk[1],
                       pk[2], pk[3]);
        }
        if (c < 3) {
          tmem_wait_ld();
          tmem_tie(nxt);
        }
      }
      tc_fence_before();   // O_i reads are ordered before the next unit's P V (via p_full)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane < 16) {
        // lane l stores rows rbase .. rbase + 3 of this warp's 32, column block l & 1;
        // groups made only of padding rows (past the window's tokens) are not stored,
        // and padding rows inside a group repeat the window's last query, whose own
        // result they equal
        const int rbase = (warp & 3) * 32 + 4 * (lane >> 1);
        const int slot0 = U.q0 + wg * 2 * kTile + static_cast<int>(rank) * kTile + rbase;
        if (slot0 < U.n_valid) {
          int rr[4];
          unit_rows4(p.g, U, p.heads, slot0, rr);
          tma_scatter4(&p.to, stage + (lane & 1) * (kTile * 128) + rbase * 128, 64 * (lane & 1), rr[0], rr[1],
                       rr[2], rr[3]);
        }
        bulk_commit_group();
      }
      pending = set;
    }
    bulk_wait_group0();   // every store of this warp is complete before the CTA exits
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == kPairMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ pooled global memory

// §3.2 "K/V-Pooled Global Memory": xbar[b, g, head, :] = the mean of
// x[b, token, head, :] over the tokens of patch g.  The unshifted grid is cut
// into patches of pool[0] x pool[1] x pool[2] tokens (a truncated last patch
// averages over the tokens it has), numbered in raster order over (g_t, g_h,
// g_w).  One thread per (b, g, head, 8 channels): it sums its 16-byte slice of
// every token row of the patch in fp32 and stores the mean as bf16 (RNE).
// Consecutive threads read consecutive 16-byte pieces of a token row.
struct PoolParams {
  const __nv_bfloat16* x;
  __nv_bfloat16* xbar;
  int B, heads, d, T, H, W;
  int pool[3], G[3];
  long long total;   // B * G * heads * d / 8
};

__global__ void kv_pool_kernel(const PoolParams p) {
  const int chunks = p.d / 8;
  const long long Gt = static_cast<long long>(p.G[0]) * p.G[1] * p.G[2];
  const long long N = static_cast<long long>(p.T) * p.H * p.W;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < p.total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % chunks);
    long long r = idx / chunks;
    const int hd = static_cast<int>(r % p.heads);
    r /= p.heads;
    const long long g = r % Gt;
    const int b = static_cast<int>(r / Gt);
    const int gw = static_cast<int>(g % p.G[2]);
    const int gh = static_cast<int>((g / p.G[2]) % p.G[1]);
    const int gt = static_cast<int>(g / (static_cast<long long>(p.G[1]) * p.G[2]));
    const int t0 = gt * p.pool[0], h0 = gh * p.pool[1], w0 = gw * p.pool[2];
    const int t1 = min(t0 + p.pool[0], p.T), h1 = min(h0 + p.pool[1], p.H), w1 = min(w0 + p.pool[2], p.W);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int t = t0; t < t1; ++t)
      for (int h = h0; h < h1; ++h)
        for (int w = w0; w < w1; ++w) {
          const long long tok = (static_cast<long long>(t) * p.H + h) * p.W + w;
          const uint4 v = *reinterpret_cast<const uint4*>(p.x + ((b * N + tok) * p.heads + hd) * p.d + c * 8);
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(u[i] << 16);
            acc[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
          }
        }
    const float inv = 1.0f / static_cast<float>((t1 - t0) * (h1 - h0) * (w1 - w0));
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    *reinterpret_cast<uint4*>(p.xbar + ((b * Gt + g) * p.heads + hd) * p.d + c * 8) =
        make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ true-window routing

// §3.3 "Content-Adaptive True-Window Routing", descriptors: qbar, kbar[b, head,
// window, :] = the means of Q and K over the window's tokens (fp32).  One CTA
// of 256 threads per (b, window, head), heads fastest so that CTAs running
// together read neighbouring 256-byte pieces of the same token rows.  Thread
// (c, l) sums the 16-byte slice c of the window's tokens l, l + L, l + 2L, ...
// (L = 256 / (d / 8) token lanes); the L partial sums are then added in lane
// order, so the result does not depend on scheduling.
struct DescParams {
  const __nv_bfloat16 *q, *k;
  float *qbar, *kbar;
  Geometry g;
  int B, heads, d;
};

constexpr int kDescThreads = 256;

__global__ void __launch_bounds__(kDescThreads, 2) win_desc_kernel(const DescParams p) {
  __shared__ float red[2][kDescThreads * 8];
  const int chunks = p.d / 8;
  const int lanes = kDescThreads / chunks;
  const int c = threadIdx.x % chunks;
  const int l = threadIdx.x / chunks;
  const int hd = blockIdx.x % p.heads;
  const int rest = blockIdx.x / p.heads;
  const int win = rest % p.g.n_windows;
  const int b = rest / p.g.n_windows;
  int m[3], e[3];
  window_of(p.g, win, m, e);
  const int n = e[0] * e[1] * e[2];
  float aq[8], ak[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) aq[i] = ak[i] = 0.0f;
#pragma unroll 4
  for (int s = l; s < n; s += lanes) {
    const long long row = (static_cast<long long>(b) * p.g.N + slot_token(p.g, m, e, s)) * p.heads + hd;
    const uint4 vq = __ldg(reinterpret_cast<const uint4*>(p.q + row * p.d) + c);
    const uint4 vk = __ldg(reinterpret_cast<const uint4*>(p.k + row * p.d) + c);
    const uint32_t uq[4] = {vq.x, vq.y, vq.z, vq.w}, uk[4] = {vk.x, vk.y, vk.z, vk.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      aq[2 * i] += __uint_as_float(uq[i] << 16);
      aq[2 * i + 1] += __uint_as_float(uq[i] & 0xffff0000u);
      ak[2 * i] += __uint_as_float(uk[i] << 16);
      ak[2 * i + 1] += __uint_as_float(uk[i] & 0xffff0000u);
    }
  }
  // red[t][l * d + channel]
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red[0][l * p.d + c * 8 + i] = aq[i];
    red[1][l * p.d + c * 8 + i] = ak[i];
  }
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(n);
  const long long out0 = ((static_cast<long long>(b) * p.heads + hd) * p.g.n_windows + win) * p.d;
  for (int i = threadIdx.x; i < 2 * p.d; i += kDescThreads) {
    const int t = i / p.d, ch = i - t * p.d;
    float acc = 0.0f;
    for (int j = 0; j < lanes; ++j) acc += red[t][j * p.d + ch];
    (t == 0 ? p.qbar : p.kbar)[out0 + ch] = acc * inv;
  }
}

// §3.3 routing: for each (b, head, window i) the candidate j with the largest
// q_i . k_j (the 1/sqrt(d) factor does not change the order), candidates being
// the other windows of the same temporal window index whose spatial window
// coordinates are within `radius` of i's (no wrap-around); the lowest window
// index wins a tie, -1 when there is no candidate.  One warp per window; the
// dot products are reduced with a fixed butterfly, so every lane sees the
// same value.
struct RouteParams {
  const float *qbar, *kbar;
  int32_t* routed;
  Geometry g;
  long long total;   // B * heads * n_windows
  int d, radius;
};

__global__ void route_kernel(const RouteParams p) {
  const long long wg = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wg >= p.total) return;
  const int nw = p.g.n_windows;
  const int win = static_cast<int>(wg % nw);
  const long long bh = wg / nw;
  const int per = p.d / 32;   // channels per lane (d is 64 or 128)
  float qv[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) qv[c] = c < per ? p.qbar[wg * p.d + lane + 32 * c] : 0.0f;
  int m[3], e[3];
  window_of(p.g, win, m, e);
  const int h0 = max(0, m[1] - p.radius), h1 = min(p.g.nwin[1] - 1, m[1] + p.radius);
  const int w0 = max(0, m[2] - p.radius), w1 = min(p.g.nwin[2] - 1, m[2] + p.radius);
  int best = -1;
  float best_s = -INFINITY;
  for (int jh = h0; jh <= h1; ++jh)
    for (int jw = w0; jw <= w1; ++jw) {
      const int j = (m[0] * p.g.nwin[1] + jh) * p.g.nwin[2] + jw;
      if (j == win) continue;
      const float* kd = p.kbar + (bh * nw + j) * p.d;
      float s = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < per) s = fmaf(qv[c], kd[lane + 32 * c], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (s > best_s) {
        best_s = s;
        best = j;
      }
    }
  if (lane == 0) p.routed[wg] = best;
}

__global__ void index_map_kernel(Geometry g, int32_t* tos) {
  const long long total = static_cast<long long>(g.n_windows) * g.nw_max;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int win = static_cast<int>(i / g.nw_max);
    const int s = static_cast<int>(i % g.nw_max);
    int m[3], e[3];
    window_of(g, win, m, e);
    tos[i] = s < e[0] * e[1] * e[2] ? slot_token(g, m, e, s) : -1;
  }
}

// ------------------------------------------------------------------ host

static std::mutex g_mutex;
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
// Read by every launch, written by the setters below from any host thread.
static std::atomic<unsigned long long> g_timeout_ns{1000000000ull};
static std::atomic<int> g_stall{0};   // test hook, see basa_swattn_set_test_stall
constexpr int kMaxDevices = 64;
static int g_dev_state[kMaxDevices];   // 0 unknown, 1 ready, negative error code

static int slots_for(int d) {
  // K/V ring: as many 128-row tiles as fit next to the two query tiles
  // within about 200 KB, capped at the ring limit.
  const int tile = kTile * d * 2;
  int slots = (200 * 1024 - 2 * tile) / tile;
  return slots > kMaxSlots ? kMaxSlots : slots;
}

static size_t smem_bytes_for(int d) {
  const size_t tile = static_cast<size_t>(kTile) * d * 2;
  size_t bytes = 1024 + tile * (2 + slots_for(d)) + sizeof(SmemCtl);
  // At most one CTA per SM: each CTA takes all 512 TMEM columns.
  const size_t one_per_sm = 120 * 1024;
  return bytes < one_per_sm ? one_per_sm : bytes;
}

static int g_sm_count[kMaxDevices];
static int g_pair_clusters[kMaxDevices];   // co-resident CTA pairs of the pair kernel

// Dynamic shared memory a CTA may use on sm_100 (227 KB).
constexpr size_t kMaxDynSmem = 232448;

static int pair_slots() {
  // K/V ring: as many half tiles as fit next to the four query tiles (two sets)
  const size_t fixed = 1024 + static_cast<size_t>(4 * kTile * 128 * 2) + sizeof(PairCtl);
  const int slots = static_cast<int>((kMaxDynSmem - fixed) / kPairHalfTileBytes);
  return slots > kPairMaxSlots ? kPairMaxSlots : slots;
}

static size_t pair_smem_bytes() {
  return 1024 + static_cast<size_t>(4 * kTile * 128 * 2) +
         static_cast<size_t>(pair_slots()) * kPairHalfTileBytes + sizeof(PairCtl);
}

static int prepare_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BASA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BASA_ERR_UNSUPPORTED;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_dev_state[dev] == 1) return BASA_OK;
  if (g_dev_state[dev] < 0) return g_dev_state[dev];
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return BASA_ERR_CUDA;
  if (major != 10 || minor != 0) {
    g_dev_state[dev] = BASA_ERR_UNSUPPORTED;
    return BASA_ERR_UNSUPPORTED;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return BASA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  size_t smem_max = smem_bytes_for(128) > smem_bytes_for(64) ? smem_bytes_for(128) : smem_bytes_for(64);
  // The four segment variants of each kernel: (kMem, kRoute).
  const void* fwd_kernels[4] = {reinterpret_cast<const void*>(swattn_fwd_kernel<false, false>),
                                reinterpret_cast<const void*>(swattn_fwd_kernel<true, false>),
                                reinterpret_cast<const void*>(swattn_fwd_kernel<false, true>),
                                reinterpret_cast<const void*>(swattn_fwd_kernel<true, true>)};
  const void* pair_kernels[4] = {reinterpret_cast<const void*>(swattn_fwd_pair_kernel<false, false>),
                                 reinterpret_cast<const void*>(swattn_fwd_pair_kernel<true, false>),
                                 reinterpret_cast<const void*>(swattn_fwd_pair_kernel<false, true>),
                                 reinterpret_cast<const void*>(swattn_fwd_pair_kernel<true, true>)};
  for (const void* f : fwd_kernels)
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_max)) !=
        cudaSuccess)
      return BASA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      g_sm_count[dev] < 1)
    return BASA_ERR_CUDA;
  for (const void* f : pair_kernels)
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(pair_smem_bytes())) != cudaSuccess)
      return BASA_ERR_CUDA;
  {
    // How many CTA pairs fit at once (SMs that cannot be paired stay idle),
    // the fewest over the variants so that one grid size serves them all.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * g_sm_count[dev], 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = pair_smem_bytes();
    int least = 0;
    for (const void* f : pair_kernels) {
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, f, &cfg) != cudaSuccess || n < 1) return BASA_ERR_CUDA;
      if (least == 0 || n < least) least = n;
    }
    g_pair_clusters[dev] = least;
  }
  g_dev_state[dev] = 1;
  return BASA_OK;
}

static int encode_rows(CUtensorMap* map, const void* ptr, long long rows, int d) {
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim,
                        gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BASA_OK : BASA_ERR_CUDA;
}

static bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

// [a, a + na) and [b, b + nb) share a byte.
static bool overlaps2(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

}  // namespace swattn

using namespace swattn;

template <typename Kernel, typename Params>
static int launch_variant(Kernel k00, Kernel k10, Kernel k01, Kernel k11, bool mem, bool route, unsigned grid,
                          unsigned threads, size_t smem, void* stream, const Params& p) {
  Kernel f = mem ? (route ? k11 : k10) : (route ? k01 : k00);
  f<<<grid, threads, smem, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// The forward with an optional routed window per window (routed != null,
// [B, heads, n_windows] on the device) and an optional extra K/V segment of E
// tokens per (b, head) appended to every window (routed = null, E = 0: the
// plain forward).
static int launch_fwd(const void* q, const void* k, const void* v, const int* routed, const void* kx,
                      const void* vx, int E, void* out, int B, int heads, int T, int H, int W, int d,
                      const int win[3], const int shift[3], float scale, void* stream) {
  if (!q || !k || !v || !out) return BASA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1 || E < 0) return BASA_ERR_INVALID_ARG;
  if (E > 0 && (!kx || !vx)) return BASA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return BASA_ERR_INVALID_ARG;
  if (scale < 0.0f) return BASA_ERR_UNSUPPORTED;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(B) * g.N * heads;
  const long long xrows = static_cast<long long>(B) * E * heads;
  if (rows >= (1LL << 31) || xrows >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  const void* ptrs[6] = {q, k, v, out, E > 0 ? kx : q, E > 0 ? vx : q};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) & 15) return BASA_ERR_ALIGNMENT;
  if (routed && (reinterpret_cast<uintptr_t>(routed) & 3)) return BASA_ERR_ALIGNMENT;
  const size_t bytes = static_cast<size_t>(rows) * d * 2;
  const size_t xbytes = static_cast<size_t>(xrows) * d * 2;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
    return BASA_ERR_ALIAS;
  if (E > 0 && (overlaps2(out, bytes, kx, xbytes) || overlaps2(out, bytes, vx, xbytes)))
    return BASA_ERR_ALIAS;
  const size_t rbytes = static_cast<size_t>(B) * heads * g.n_windows * sizeof(int);
  if (routed && overlaps2(out, bytes, routed, rbytes)) return BASA_ERR_ALIAS;
  const long long q_pairs = (g.nw_max + 2 * kTile - 1) / (2 * kTile);
  const long long units = static_cast<long long>(B) * heads * g.n_windows * q_pairs;
  if (units >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;

  int dev = 0;
  rc = prepare_device(&dev);
  if (rc) return rc;

  if (d == 128) {
    // CTA-pair kernel: units of up to 512 queries, one cluster of two CTAs each.
    const long long q_quads = (g.nw_max + 4 * kTile - 1) / (4 * kTile);
    const long long punits = static_cast<long long>(B) * heads * g.n_windows * q_quads;
    if (punits >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
    PairParams pp;
    memset(&pp, 0, sizeof(pp));
    if (encode_rows(&pp.tq, q, rows, d) || encode_rows(&pp.tk, k, rows, d) ||
        encode_rows(&pp.tv, v, rows, d) || encode_rows(&pp.to, out, rows, d))
      return BASA_ERR_CUDA;
    if (E > 0 && (encode_rows(&pp.tkx, kx, xrows, d) || encode_rows(&pp.tvx, vx, xrows, d)))
      return BASA_ERR_CUDA;
    pp.n_extra = E;
    pp.routed = routed;
    pp.out = static_cast<__nv_bfloat16*>(out);
    pp.g = g;
    pp.B = B;
    pp.heads = heads;
    pp.q_quads = static_cast<int>(q_quads);
    pp.f_qq = make_fastdiv(pp.q_quads);
    pp.f_nw = make_fastdiv(g.n_windows);
    pp.f_heads = make_fastdiv(heads);
    pp.total_units = static_cast<int>(punits);
    pp.n_slots = pair_slots();
    pp.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    pp.timeout_ns = g_timeout_ns.load();
    pp.stall = g_stall.load();
    const long long clusters = punits < g_pair_clusters[dev] ? punits : g_pair_clusters[dev];
    return launch_variant(swattn_fwd_pair_kernel<false, false>, swattn_fwd_pair_kernel<true, false>,
                          swattn_fwd_pair_kernel<false, true>, swattn_fwd_pair_kernel<true, true>, E > 0,
                          routed != nullptr, static_cast<unsigned>(2 * clusters), kPairThreads,
                          pair_smem_bytes(), stream, pp);
  }

  FwdParams p;
  memset(&p, 0, sizeof(p));
  if (encode_rows(&p.tq, q, rows, d) || encode_rows(&p.tk, k, rows, d) ||
      encode_rows(&p.tv, v, rows, d))
    return BASA_ERR_CUDA;
  if (E > 0 && (encode_rows(&p.tkx, kx, xrows, d) || encode_rows(&p.tvx, vx, xrows, d)))
    return BASA_ERR_CUDA;
  p.n_extra = E;
  p.routed = routed;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.g = g;
  p.B = B;
  p.heads = heads;
  p.d = d;
  p.q_pairs = static_cast<int>(q_pairs);
  p.f_qp = make_fastdiv(p.q_pairs);
  p.f_nw = make_fastdiv(g.n_windows);
  p.f_heads = make_fastdiv(heads);
  p.total_units = static_cast<int>(units);
  p.n_slots = slots_for(d);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.stall = g_stall.load();
  // Persistent: one CTA per SM, each walking the units with a stride of the grid.
  const long long grid = units < g_sm_count[dev] ? units : g_sm_count[dev];
  return launch_variant(swattn_fwd_kernel<false, false>, swattn_fwd_kernel<true, false>,
                        swattn_fwd_kernel<false, true>, swattn_fwd_kernel<true, true>, E > 0,
                        routed != nullptr, static_cast<unsigned>(grid), kThreads, smem_bytes_for(d), stream, p);
}

extern "C" int basa_swattn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                               int heads, int T, int H, int W, int d, const int win[3],
                               const int shift[3], float scale, void* stream) {
  return launch_fwd(q, k, v, nullptr, nullptr, nullptr, 0, out, B, heads, T, H, W, d, win, shift, scale,
                    stream);
}

extern "C" int basa_swattn_fwd_mem(const void* q, const void* k, const void* v, const void* kx,
                                   const void* vx, int E, void* out, int B, int heads, int T, int H,
                                   int W, int d, const int win[3], const int shift[3], float scale,
                                   void* stream) {
  return launch_fwd(q, k, v, nullptr, kx, vx, E, out, B, heads, T, H, W, d, win, shift, scale, stream);
}

extern "C" int basa_swattn_fwd_route(const void* q, const void* k, const void* v, const int32_t* routed,
                                     const void* kx, const void* vx, int E, void* out, int B, int heads,
                                     int T, int H, int W, int d, const int win[3], const int shift[3],
                                     float scale, void* stream) {
  if (!routed) return BASA_ERR_INVALID_ARG;
  return launch_fwd(q, k, v, routed, kx, vx, E, out, B, heads, T, H, W, d, win, shift, scale, stream);
}

extern "C" int basa_route_workspace_bytes(int B, int heads, int T, int H, int W, int d, const int win[3],
                                          size_t* bytes) {
  if (!bytes || B < 1 || heads < 1) return BASA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  const int zero[3] = {0, 0, 0};
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, zero);
  if (rc) return rc;
  *bytes = 2 * static_cast<size_t>(B) * heads * g.n_windows * d * sizeof(float);
  return BASA_OK;
}

extern "C" int basa_route(const void* q, const void* k, int B, int heads, int T, int H, int W, int d,
                          const int win[3], const int shift[3], int radius, void* workspace,
                          size_t workspace_bytes, int32_t* routed, void* stream) {
  if (!q || !k || !workspace || !routed || B < 1 || heads < 1 || radius < 0) return BASA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  size_t need = 0;
  rc = basa_route_workspace_bytes(B, heads, T, H, W, d, win, &need);
  if (rc) return rc;
  if (workspace_bytes < need) return BASA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * g.N * heads;
  const long long descs = static_cast<long long>(B) * heads * g.n_windows;
  if (rows >= (1LL << 31) || descs >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  const void* ptrs[3] = {q, k, workspace};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) & 15) return BASA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(routed) & 3) return BASA_ERR_ALIGNMENT;
  const size_t in_bytes = static_cast<size_t>(rows) * d * 2;
  const size_t rbytes = static_cast<size_t>(descs) * sizeof(int32_t);
  if (overlaps2(workspace, need, q, in_bytes) || overlaps2(workspace, need, k, in_bytes) ||
      overlaps2(routed, rbytes, q, in_bytes) || overlaps2(routed, rbytes, k, in_bytes) ||
      overlaps2(routed, rbytes, workspace, need))
    return BASA_ERR_ALIAS;
  // A radius past the window grid selects the same candidates as the grid's
  // extent; clamping keeps the kernel's window arithmetic inside int.
  const int rmax = g.nwin[1] > g.nwin[2] ? g.nwin[1] : g.nwin[2];
  if (radius > rmax) radius = rmax;
  int dev = 0;
  rc = prepare_device(&dev);
  if (rc) return rc;
  DescParams dp;
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.k = static_cast<const __nv_bfloat16*>(k);
  dp.qbar = static_cast<float*>(workspace);
  dp.kbar = dp.qbar + descs * d;
  dp.g = g;
  dp.B = B;
  dp.heads = heads;
  dp.d = d;
  win_desc_kernel<<<static_cast<unsigned>(descs), kDescThreads, 0, static_cast<cudaStream_t>(stream)>>>(dp);
  RouteParams rp;
  rp.qbar = dp.qbar;
  rp.kbar = dp.kbar;
  rp.routed = routed;
  rp.g = g;
  rp.total = descs;
  rp.d = d;
  rp.radius = radius;
  const long long blocks = (descs * 32 + 255) / 256;
  route_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(rp);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// ------------------------------------------------------------------ routing without allocation
//
// basa_route_noalloc is basa_route for callers that cannot allocate device
// memory: code running inside another framework's execution step (a plugin's
// enqueue, a serving loop with a fixed memory budget) where cudaMalloc is
// forbidden or would stall the device.  Its window descriptors live in this
// file-scope array instead of a caller's workspace.  Every GPU that loads the
// library holds the array until the process exits, and every call on a device
// shares it: calls whose work overlaps on the GPU (two streams, or two host
// threads) race on it.  Each call overwrites every descriptor it reads, so
// nothing needs clearing between calls.
constexpr size_t kRouteScratchBytes = BASA_ROUTE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];
// Device address of g_route_scratch on each device (host code cannot use the
// array's name as a device address), found on the first call on that device.
static void* g_route_scratch_addr[kMaxDevices];

static int route_scratch_address(int dev, void** addr) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_route_scratch_addr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_route_scratch) != cudaSuccess || !a) return BASA_ERR_CUDA;
    g_route_scratch_addr[dev] = a;
  }
  *addr = g_route_scratch_addr[dev];
  return BASA_OK;
}

extern "C" int basa_route_noalloc(const void* q, const void* k, int B, int heads, int T, int H, int W, int d,
                                  const int win[3], const int shift[3], int radius, int32_t* routed,
                                  void* stream) {
  if (!q || !k || !routed || B < 1 || heads < 1 || radius < 0) return BASA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  const long long rows = static_cast<long long>(B) * g.N * heads;
  const long long descs = static_cast<long long>(B) * heads * g.n_windows;
  if (rows >= (1LL << 31) || descs >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  // two fp32 descriptor arrays (window means of Q and of K)
  if (static_cast<unsigned long long>(descs) * d * 2 * sizeof(float) > kRouteScratchBytes)
    return BASA_ERR_SCRATCH_LIMIT;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(k) & 15)) return BASA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(routed) & 3) return BASA_ERR_ALIGNMENT;
  const size_t in_bytes = static_cast<size_t>(rows) * d * 2;
  const size_t rbytes = static_cast<size_t>(descs) * sizeof(int32_t);
  if (overlaps2(routed, rbytes, q, in_bytes) || overlaps2(routed, rbytes, k, in_bytes)) return BASA_ERR_ALIAS;
  const int rmax = g.nwin[1] > g.nwin[2] ? g.nwin[1] : g.nwin[2];
  if (radius > rmax) radius = rmax;
  int dev = 0;
  rc = prepare_device(&dev);
  if (rc) return rc;
  void* scratch = nullptr;
  rc = route_scratch_address(dev, &scratch);
  if (rc) return rc;
  DescParams dp;
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.k = static_cast<const __nv_bfloat16*>(k);
  dp.qbar = static_cast<float*>(scratch);
  dp.kbar = dp.qbar + descs * d;
  dp.g = g;
  dp.B = B;
  dp.heads = heads;
  dp.d = d;
  win_desc_kernel<<<static_cast<unsigned>(descs), kDescThreads, 0, static_cast<cudaStream_t>(stream)>>>(dp);
  RouteParams rp;
  rp.qbar = dp.qbar;
  rp.kbar = dp.kbar;
  rp.routed = routed;
  rp.g = g;
  rp.total = descs;
  rp.d = d;
  rp.radius = radius;
  const long long blocks = (descs * 32 + 255) / 256;
  route_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(rp);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

extern "C" int basa_swattn_index_map(int T, int H, int W, const int win[3], const int shift[3],
                                     int32_t* d_token_of_slot, void* stream) {
  if (!d_token_of_slot) return BASA_ERR_INVALID_ARG;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  const long long total = static_cast<long long>(g.n_windows) * g.nw_max;
  if (total >= (1LL << 40)) return BASA_ERR_UNSUPPORTED;
  long long blocks = (total + 255) / 256;
  if (blocks > 65535) blocks = 65535;
  index_map_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      g, d_token_of_slot);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

extern "C" int basa_swattn_index_map_host(int T, int H, int W, const int win[3],
                                          const int shift[3], int32_t* token_of_slot) {
  if (!token_of_slot) return BASA_ERR_INVALID_ARG;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  for (int wid = 0; wid < g.n_windows; ++wid) {
    int m[3], e[3];
    window_of(g, wid, m, e);
    const int nv = e[0] * e[1] * e[2];
    for (int s = 0; s < g.nw_max; ++s)
      token_of_slot[static_cast<size_t>(wid) * g.nw_max + s] = s < nv ? slot_token(g, m, e, s) : -1;
  }
  return BASA_OK;
}

extern "C" int basa_swattn_flops(int B, int heads, int T, int H, int W, int d, const int win[3],
                                 double* flops) {
  if (!flops || B < 1 || heads < 1 || d < 1) return BASA_ERR_INVALID_ARG;
  const int zero[3] = {0, 0, 0};
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, zero);
  if (rc) return rc;
  // sum over windows of n_m^2 factorises into per-axis sums of squared extents
  double s2 = 1.0;
  for (int a = 0; a < 3; ++a) {
    double acc = 0.0;
    for (int mi = 0; mi < g.nwin[a]; ++mi) {
      const int left = g.n[a] - mi * g.w[a];
      const double ext = left < g.w[a] ? left : g.w[a];
      acc += ext * ext;
    }
    s2 *= acc;
  }
  *flops = 4.0 * s2 * d * static_cast<double>(B) * heads;
  return BASA_OK;
}

extern "C" int basa_kv_pool_tokens(int T, int H, int W, const int pool[3], int* G) {
  if (!pool || !G || T < 1 || H < 1 || W < 1) return BASA_ERR_INVALID_ARG;
  const int n[3] = {T, H, W};
  long long g = 1;
  for (int a = 0; a < 3; ++a) {
    if (pool[a] < 1) return BASA_ERR_INVALID_ARG;
    g *= (n[a] + pool[a] - 1) / pool[a];
  }
  if (g >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  *G = static_cast<int>(g);
  return BASA_OK;
}

extern "C" int basa_kv_pool(const void* k, const void* v, void* kbar, void* vbar, int B, int heads,
                            int T, int H, int W, int d, const int pool[3], void* stream) {
  if (!k || !v || !kbar || !vbar || !pool || B < 1 || heads < 1) return BASA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  int G = 0;
  int rc = basa_kv_pool_tokens(T, H, W, pool, &G);
  if (rc) return rc;
  const long long N = static_cast<long long>(T) * H * W;
  const long long rows = static_cast<long long>(B) * N * heads;
  const long long grows = static_cast<long long>(B) * G * heads;
  if (rows >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  const void* ptrs[4] = {k, v, kbar, vbar};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) & 15) return BASA_ERR_ALIGNMENT;
  const size_t in_bytes = static_cast<size_t>(rows) * d * 2, out_bytes = static_cast<size_t>(grows) * d * 2;
  if (overlaps2(kbar, out_bytes, k, in_bytes) || overlaps2(kbar, out_bytes, v, in_bytes) ||
      overlaps2(vbar, out_bytes, k, in_bytes) || overlaps2(vbar, out_bytes, v, in_bytes) ||
      overlaps2(kbar, out_bytes, vbar, out_bytes))
    return BASA_ERR_ALIAS;
  int dev = 0;
  rc = prepare_device(&dev);
  if (rc) return rc;
  PoolParams pp;
  pp.B = B;
  pp.heads = heads;
  pp.d = d;
  pp.T = T;
  pp.H = H;
  pp.W = W;
  const int n[3] = {T, H, W};
  for (int a = 0; a < 3; ++a) {
    pp.pool[a] = pool[a];
    pp.G[a] = (n[a] + pool[a] - 1) / pool[a];
  }
  pp.total = grows * (d / 8);
  const long long want = (pp.total + 255) / 256;
  const long long cap = 8LL * g_sm_count[dev];
  const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
  for (int t = 0; t < 2; ++t) {
    pp.x = static_cast<const __nv_bfloat16*>(t == 0 ? k : v);
    pp.xbar = static_cast<__nv_bfloat16*>(t == 0 ? kbar : vbar);
    kv_pool_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(pp);
  }
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

extern "C" int basa_shift_schedule(int L, const int win[3], const int step_offset[3], int* shifts) {
  if (L < 1 || !win || !step_offset || !shifts) return BASA_ERR_INVALID_ARG;
  for (int a = 0; a < 3; ++a)
    if (win[a] < 1) return BASA_ERR_INVALID_ARG;
  const int K = (L + 1) / 2;
  for (int a = 0; a < 3; ++a) {
    const long long w = win[a];
    const long long delta = w / L > 1 ? w / L : 1;
    long long c = step_offset[a] % w;
    if (c < 0) c += w;
    for (int l = 0; l < L; ++l) {
      // b_l: even positions take a_0, a_1, ... (first half), odd positions
      // a_K, a_{K+1}, ... (second half).
      const long long i = (l % 2 == 0) ? l / 2 : K + l / 2;
      const long long b = (i * delta) % w;
      shifts[3 * l + a] = static_cast<int>((b + c) % w);
    }
  }
  return BASA_OK;
}

extern "C" int basa_swattn_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BASA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return BASA_ERR_CUDA;
  if (v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return BASA_ERR_CUDA;
    return BASA_ERR_DEVICE;
  }
  return BASA_OK;
}

extern "C" int basa_swattn_set_wait_timeout_ns(unsigned long long ns) {
  g_timeout_ns.store(ns);
  return BASA_OK;
}

extern "C" int basa_swattn_set_test_stall(int on) {
  g_stall.store(on ? 1 : 0);
  return BASA_OK;
}

extern "C" const char* basa_strerror(int code) {
  switch (code) {
    case BASA_OK: return "ok";
    case BASA_ERR_INVALID_ARG: return "invalid argument";
    case BASA_ERR_UNSUPPORTED: return "unsupported configuration";
    case BASA_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
    case BASA_ERR_CUDA: return "CUDA call failed";
    case BASA_ERR_DEVICE: return "a device-side wait timed out";
    case BASA_ERR_ALIAS: return "out overlaps an input";
    case BASA_ERR_SCRATCH_LIMIT: return "problem needs more than the library's fixed device scratch";
    default: return "unknown error";
  }
}
