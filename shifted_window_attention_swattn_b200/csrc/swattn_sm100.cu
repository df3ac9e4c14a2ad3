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
//     load brings 4 arbitrary token rows of Q, K or V into a 128-byte-swizzled
//     shared-memory tile), so windows are gathered straight from the
//     [B, T*H*W, heads, d] tensors;
//   * S = Q K^T and O += P V run on tcgen05 tensor cores with S, P and O in
//     tensor memory (TMEM);
//   * softmax is online (running max / sum per query row, one thread per row),
//     with the max kept stale until it grows by more than 2^8 so that O is
//     rarely rescaled;
//   * the inverse roll is the row address of the output store: each query's
//     result is written back to the token row it was gathered from.
//
// One CTA handles one 128-query tile of one window of one (batch, head):
//   warps 0-3  softmax, O correction and epilogue (thread t owns query row t)
//   warp  4    TMA producer (Q once, then K/V tiles through a 2-stage ring)
//   warp  5    TMEM owner and MMA issuer (one elected lane)
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d) P0 [384,448) P1 [448,512).
//
// Every mbarrier wait is bounded by a host-set timeout; a wait that runs out
// raises a shared abort flag and a library-wide error word, every role stops
// issuing work, the MMA issuer drains its in-flight MMAs, the producer drains
// its in-flight loads, and TMEM is released before the CTA exits.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <math.h>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "basa_swattn.h"
#include "ptx_sm100.cuh"

namespace swattn {

constexpr int kThreads = 192;
constexpr int kTile = 128;       // query rows per CTA tile = key rows per K/V tile
constexpr int kStages = 2;       // K/V ring depth
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S buffer b at kColS + 128 * b
constexpr uint32_t kColO = 256;
constexpr uint32_t kColP = 384;   // P buffer b at kColP + 64 * b
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when the max grows by > 2^8

// ------------------------------------------------------------------ geometry

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
};

// Window coordinates m and extents e (truncated at the grid edge) of window `id`
// (raster order over m_t, m_h, m_w).
__host__ __device__ __forceinline__ void window_of(const Geometry& g, int id, int m[3], int e[3]) {
  m[2] = id % g.nwin[2];
  const int r = id / g.nwin[2];
  m[1] = r % g.nwin[1];
  m[0] = r / g.nwin[1];
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
  const int sw = s % e[2];
  const int r = s / e[2];
  const int sh = r % e[1];
  const int st = r / e[1];
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
  __nv_bfloat16* out;
  Geometry g;
  int B, heads, d;
  int q_tiles;                  // ceil(nw_max / 128)
  float scale_log2;             // scale * log2(e)
  unsigned long long timeout_ns;
};

struct SmemCtl {
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t v_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;              // P V of every tile but the last
  uint64_t o_final;             // P V of the last tile
  uint64_t drained;             // every MMA of the CTA
  uint32_t tmem_base;
  int abort;
};

__device__ int g_device_error = 0;

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, SmemCtl* ctl,
                                              unsigned long long timeout_ns) {
  if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
  if (mbar_wait_bounded(bar, parity, timeout_ns)) return true;
  *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
  atomicOr(&g_device_error, 1);
  return false;
}

__device__ __forceinline__ int token_row(const FwdParams& p, int b, int h, int token) {
  return (b * p.g.N + token) * p.heads + h;
}

__global__ void __launch_bounds__(kThreads, 1) swattn_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int d = p.d;
  const int tile_bytes = kTile * d * 2;
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + tile_bytes;
  uint8_t* sV = sK + kStages * tile_bytes;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sV + kStages * tile_bytes);

  // ---- work unit: (batch*head, window, query tile), query tile fastest
  int unit = blockIdx.x;
  const int qt = unit % p.q_tiles;
  unit /= p.q_tiles;
  const int win_id = unit % p.g.n_windows;
  const int bh = unit / p.g.n_windows;
  const int b = bh / p.heads;
  const int h = bh % p.heads;
  int m[3], e[3];
  window_of(p.g, win_id, m, e);
  const int n_valid = e[0] * e[1] * e[2];
  const int q0 = qt * kTile;
  if (q0 >= n_valid) return;   // a truncated window has fewer query tiles (CTA-uniform)
  const int nkv = (n_valid + kTile - 1) / kTile;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_full[i], kSoftmaxWarps);
    }
    mbar_init(&ctl->o_done, 1);
    mbar_init(&ctl->o_final, 1);
    mbar_init(&ctl->drained, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
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

  if (warp == kProducerWarp) {
    // ================================================================ producer
    const int ncb = d / 64;   // 64-column (128-byte) blocks per row
    int last_tile_in_stage[kStages];
    for (int s = 0; s < kStages; ++s) last_tile_in_stage[s] = -1;
    int r[4];
    // Q tile: slots q0 .. q0+127, rows past the window repeat its last token
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int s = q0 + 4 * lane + i;
      if (s >= n_valid) s = n_valid - 1;
      r[i] = token_row(p, b, h, slot_token(p.g, m, e, s));
    }
    if (lane == 0) mbar_arrive_expect_tx(&ctl->q_full, tile_bytes);
    __syncwarp();
    for (int c = 0; c < ncb; ++c)
      tma_gather4(&p.tq, &ctl->q_full, sQ + c * (kTile * 128) + lane * 512, c * 64, r[0], r[1],
                  r[2], r[3]);
    for (int j = 0; j < nkv; ++j) {
      const int s = j % kStages;
      if (j >= kStages) {
        bool ok = wait_or_abort(&ctl->kv_empty[s], ((j / kStages) - 1) & 1, ctl, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int sl = j * kTile + 4 * lane + i;
        if (sl >= n_valid) sl = n_valid - 1;
        r[i] = token_row(p, b, h, slot_token(p.g, m, e, sl));
      }
      uint8_t* dk = sK + s * tile_bytes;
      uint8_t* dv = sV + s * tile_bytes;
      if (lane == 0) mbar_arrive_expect_tx(&ctl->k_full[s], tile_bytes);
      __syncwarp();
      for (int c = 0; c < ncb; ++c)
        tma_gather4(&p.tk, &ctl->k_full[s], dk + c * (kTile * 128) + lane * 512, c * 64, r[0],
                    r[1], r[2], r[3]);
      if (lane == 0) mbar_arrive_expect_tx(&ctl->v_full[s], tile_bytes);
      __syncwarp();
      for (int c = 0; c < ncb; ++c)
        tma_gather4(&p.tv, &ctl->v_full[s], dv + c * (kTile * 128) + lane * 512, c * 64, r[0],
                    r[1], r[2], r[3]);
      last_tile_in_stage[s] = j;
    }
    // Drain: every load this warp issued has landed before the CTA can exit.
    // (In the normal flow these phases are long complete and return at once.)
    mbar_wait_bounded(&ctl->q_full, 0, p.timeout_ns);
    for (int s = 0; s < kStages; ++s) {
      const int j = last_tile_in_stage[s];
      if (j >= 0) {
        mbar_wait_bounded(&ctl->k_full[s], (j / kStages) & 1, p.timeout_ns);
        mbar_wait_bounded(&ctl->v_full[s], (j / kStages) & 1, p.timeout_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      const uint32_t idesc_pv = idesc_bf16_f32(128, d, 0, 1);
      const int ksteps_qk = d / 16;
      bool ok = wait_or_abort(&ctl->q_full, 0, ctl, p.timeout_ns);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j % kStages;
          const int bb = j & 1;
          ok = wait_or_abort(&ctl->k_full[s], (j / kStages) & 1, ctl, p.timeout_ns);
          if (!ok) break;
          tc_fence_after();
          int kv_valid = n_valid - j * kTile;
          if (kv_valid > kTile) kv_valid = kTile;
          const int n_s = (kv_valid + 15) & ~15;
          const uint32_t idesc_s = idesc_bf16_f32(128, n_s, 0, 0);
          const uint32_t kbase = k_addr + s * tile_bytes;
          for (int kk = 0; kk < ksteps_qk; ++kk) {
            const uint32_t off = (kk >> 2) * (kTile * 128) + (kk & 3) * 32;
            umma_ss(tmem + kColS + 128u * bb, smem_desc_sw128(q_addr + off, 16, 1024),
                    smem_desc_sw128(kbase + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full[bb]);
        }
        if (j >= 1) {
          const int jp = j - 1;
          const int sp = jp % kStages;
          const int bp = jp & 1;
          ok = wait_or_abort(&ctl->p_full[bp], (jp >> 1) & 1, ctl, p.timeout_ns);
          if (!ok) break;
          ok = wait_or_abort(&ctl->v_full[sp], (jp / kStages) & 1, ctl, p.timeout_ns);
          if (!ok) break;
          tc_fence_after();
          int kv_valid = n_valid - jp * kTile;
          if (kv_valid > kTile) kv_valid = kTile;
          const int ksteps = (kv_valid + 15) >> 4;
          const uint32_t vbase = v_addr + sp * tile_bytes;
          for (int kk = 0; kk < ksteps; ++kk) {
            umma_ts(tmem + kColO, tmem + kColP + 64u * bp + kk * 8,
                    smem_desc_sw128(vbase + kk * 2048, kTile * 128, 1024), idesc_pv,
                    (jp > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&ctl->kv_empty[sp]);
          umma_commit(jp == nkv - 1 ? &ctl->o_final : &ctl->o_done);
        }
      }
      // Drain every MMA this thread issued before TMEM is released.
      umma_commit(&ctl->drained);
      mbar_wait_bounded(&ctl->drained, 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int bb = j & 1;
      ok = wait_or_abort(&ctl->s_full[bb], (j >> 1) & 1, ctl, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      int kv_valid = n_valid - j * kTile;
      if (kv_valid > kTile) kv_valid = kTile;
      const int nchunks = (kv_valid + 31) >> 5;

      float x[kTile];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < nchunks) {
          uint32_t r[32];
          tmem_ld32(tmem + kColS + 128u * bb + lane_off + c * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(r[i]);
        }
      }
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kTile; ++i) {
        x[i] = (i < kv_valid) ? x[i] * sl2 : -INFINITY;
        mx = fmaxf(mx, x[i]);
      }
      const float m_new = fmaxf(m_run, mx);
      const bool need = m_new > m_run + kRescaleThreshold;
      float alpha = 1.0f;
      if (need) {
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      float rowsum = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < nchunks) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2_approx(x[c * 32 + 2 * i] - m_run);
            const float p1 = ex2_approx(x[c * 32 + 2 * i + 1] - m_run);
            rowsum += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tmem + kColP + 64u * bb + lane_off + c * 16, pk);
        }
      }
      l_run = l_run * alpha + rowsum;
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        // O holds P V of tiles 0..j-1 relative to the old max: wait for the
        // last of them to finish, then scale the row by alpha.
        bool ok2 = wait_or_abort(&ctl->o_done, (j - 1) & 1, ctl, p.timeout_ns);
        ok2 = __all_sync(0xffffffffu, ok2);
        if (!ok2) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < d / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + kColO + lane_off + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tmem + kColO + lane_off + c * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[bb]);
    }
    // ---- epilogue: O / l, bf16, stored at the row the query came from
    if (ok) {
      ok = wait_or_abort(&ctl->o_final, 0, ctl, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int slot = q0 + static_cast<int>(threadIdx.x);
      const bool valid = slot < n_valid;
      __nv_bfloat16* dst = nullptr;
      if (valid)
        dst = p.out + static_cast<size_t>(token_row(p, b, h, slot_token(p.g, m, e, slot))) * d;
      const float inv_l = 1.0f / l_run;
      for (int c = 0; c < d / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + kColO + lane_off + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                              __uint_as_float(r[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
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
static unsigned long long g_timeout_ns = 1000000000ull;
constexpr int kMaxDevices = 64;
static int g_dev_state[kMaxDevices];   // 0 unknown, 1 ready, negative error code

static size_t smem_bytes_for(int d) {
  const size_t tile = static_cast<size_t>(kTile) * d * 2;
  size_t bytes = 1024 + tile * (1 + 2 * kStages) + sizeof(SmemCtl);
  // At most one CTA per SM: each CTA takes all 512 TMEM columns.
  const size_t one_per_sm = 120 * 1024;
  return bytes < one_per_sm ? one_per_sm : bytes;
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
  if (cudaFuncSetAttribute(swattn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem_bytes_for(128))) != cudaSuccess)
    return BASA_ERR_CUDA;
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

}  // namespace swattn

using namespace swattn;

extern "C" int basa_swattn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                               int heads, int T, int H, int W, int d, const int win[3],
                               const int shift[3], float scale, void* stream) {
  if (!q || !k || !v || !out) return BASA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1) return BASA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return BASA_ERR_INVALID_ARG;
  Geometry g;
  int rc = make_geometry(&g, T, H, W, win, shift);
  if (rc) return rc;
  if (d != 64 && d != 128) return BASA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(B) * g.N * heads;
  if (rows >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;
  const void* ptrs[4] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) & 15) return BASA_ERR_ALIGNMENT;
  const size_t bytes = static_cast<size_t>(rows) * d * 2;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
    return BASA_ERR_ALIAS;
  const long long q_tiles = (g.nw_max + kTile - 1) / kTile;
  const long long grid = static_cast<long long>(B) * heads * g.n_windows * q_tiles;
  if (grid >= (1LL << 31)) return BASA_ERR_UNSUPPORTED;

  int dev = 0;
  rc = prepare_device(&dev);
  if (rc) return rc;

  FwdParams p;
  memset(&p, 0, sizeof(p));
  if (encode_rows(&p.tq, q, rows, d) || encode_rows(&p.tk, k, rows, d) ||
      encode_rows(&p.tv, v, rows, d))
    return BASA_ERR_CUDA;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.g = g;
  p.B = B;
  p.heads = heads;
  p.d = d;
  p.q_tiles = static_cast<int>(q_tiles);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns;
  swattn_fwd_kernel<<<static_cast<unsigned>(grid), kThreads, smem_bytes_for(d),
                      static_cast<cudaStream_t>(stream)>>>(p);
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
  std::lock_guard<std::mutex> lock(g_mutex);
  g_timeout_ns = ns;
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
    default: return "unknown error";
  }
}
