// Backward pass of exact softmax attention for B200 (sm_100a): dQ, dK, dV of
// L = sum(O * dO) for O = softmax(scale * Q K^T [+ causal mask]) V, with the
// probabilities recomputed tile by tile from Q, K and the forward's LSE
// instead of being stored ("selected recomputation in the backward pass",
// lihaoran.work, "The intermediate matrix comes first"; liminalml.com
// "FlashAttention", "Why use it?").  The N x N matrices never reach memory.
//
// With P = e^(scale q.k - LSE) recomputed per tile:
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   bwd_rowdot   D = rowsum(dO * O), one warp per row (HBM-bound).
//   bwd_dkdv     one CTA per 128-key tile: S^T = K Q^T and dP^T = V dO^T into
//                TMEM, P^T and dS^T formed in place (bf16), then
//                dV += P^T dO and dK += dS^T Q accumulate in TMEM over the
//                query tiles (tcgen05, A operands from TMEM).
//   bwd_dq       one CTA per 128-query tile: S = Q K^T and dP = dO V^T, dS in
//                place, dQ += dS K over the key tiles.
// CTA layout of the two tiled kernels (384 threads): warp 0 TMA producer,
// warp 1 TMEM owner and MMA issuer, warps 4-11 elementwise step and epilogue
// (two threads per TMEM lane, i.e. per row of the tile, 64 columns each).
// Every wait is bounded as in the forward kernel.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fa.h"
#include "host_util.h"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kTile = 128;   // rows of a query tile, keys of a key tile
constexpr int kThreads = 384;
constexpr int kElemWarp0 = 4;
constexpr int kElemThreads = 256;  // warps 4-11: two threads per row, 64 columns each
constexpr uint32_t kTmemCols = 512;
constexpr int kChunkBytes = kTile * 64 * 2;  // one 64-wide, 128-row swizzled box

enum : uint32_t { kSiteLoad = 0, kSiteStage = 1, kSiteS = 2, kSiteDs = 3, kSiteO = 4 };

struct BwdParams {
  const float* lse;  // [BH][N] natural-log LSE of the forward
  const float* dd;   // [BH][N] D = rowsum(dO * O)
  int N;
  int BH;
  int n_tiles;       // ceil(N / 128)
  int group_heads;   // heads whose CTAs are scheduled together
  float scale;       // multiplier of q.k
  float scale_log2;  // scale * log2(e)
  uint64_t timeout_ns;
};

__device__ uint32_t g_bwd_status;

// TMEM column maps (both kernels): S or S^T at [0,128), dP or dP^T at
// [128,256), accumulators from 256.  P / dS (bf16 pairs) overwrite their own
// tile: the 32 values of columns 32c..32c+31 go, packed, to columns
// 32c..32c+15, so each thread only overwrites what it has already read.
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;

// TMEM column of the packed bf16 operand for K-step kk (16 keys or queries)
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk >> 1) * 32 + (kk & 1) * 8; }

// Work order shared by the tiled kernels: heads in groups, inside a group the
// tiles with the most work first, cycling over the group's heads.
__device__ __forceinline__ void tile_of(const BwdParams& p, bool heavy_high, int* bh, int* tile) {
  const int per_group = p.group_heads * p.n_tiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int rem = static_cast<int>(blockIdx.x) % per_group;
  const int gh = min(p.group_heads, p.BH - grp * p.group_heads);
  *bh = grp * p.group_heads + rem % gh;
  const int k = rem / gh;
  *tile = heavy_high ? p.n_tiles - 1 - k : k;
}

// Elementwise step over 64 of the 128 columns (chunks c0, c0+1 of 32) of the
// calling thread's row: p = 2^(s * scale log2e - lse2), masked to 0 where
// `allowed` fails; ds = p * (dp - dsub).  P (optional) and dS are written as
// bf16 pairs into the first half of each chunk's own columns.
template <bool WRITE_P, typename ColLse, typename ColDsub, typename Allowed>
__device__ __forceinline__ void p_ds_tile(uint32_t tS, uint32_t tDP, int c0, float sl2, ColLse col_lse2,
                                          ColDsub col_dsub, Allowed allowed) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = c0 + cc;
    uint32_t s[32], dp[32];
    tmem_ld32(tS + c * 32, s);
    tmem_ld32(tDP + c * 32, dp);
    tmem_wait_ld();
    uint32_t pk[16], dk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int col0 = c * 32 + e, col1 = col0 + 1;
      float p0 = ex2_approx(fmaf(__uint_as_float(s[e]), sl2, -col_lse2(col0)));
      float p1 = ex2_approx(fmaf(__uint_as_float(s[e + 1]), sl2, -col_lse2(col1)));
      if (!allowed(col0)) p0 = 0.f;
      if (!allowed(col1)) p1 = 0.f;
      const float d0 = p0 * (__uint_as_float(dp[e]) - col_dsub(col0));
      const float d1 = p1 * (__uint_as_float(dp[e + 1]) - col_dsub(col1));
      pk[e >> 1] = pack_bf16x2(p0, p1);
      dk[e >> 1] = pack_bf16x2(d0, d1);
    }
    if (WRITE_P) tmem_st16(tS + c * 32, pk);
    tmem_st16(tDP + c * 32, dk);
  }
}

// Store 32-column chunks [cb, ce) of a 128 x D tile held in TMEM (this
// thread's row r, fp32) as bf16 into the 128-byte-swizzled staging buffer
// that a TMA store then writes out.
template <int D>
__device__ __forceinline__ void store_tile(uint32_t tAcc, float mul, uint8_t* stage, int r, int cb,
                                           int ce) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    if (c < cb || c >= ce) continue;
    uint32_t o[32];
    tmem_ld32(tAcc + c * 32, o);
    tmem_wait_ld();
    uint8_t* rowp = stage + (c >> 1) * kChunkBytes + r * 128;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint4 v;
      v.x = pack_bf16x2(__uint_as_float(o[8 * g + 0]) * mul, __uint_as_float(o[8 * g + 1]) * mul);
      v.y = pack_bf16x2(__uint_as_float(o[8 * g + 2]) * mul, __uint_as_float(o[8 * g + 3]) * mul);
      v.z = pack_bf16x2(__uint_as_float(o[8 * g + 4]) * mul, __uint_as_float(o[8 * g + 5]) * mul);
      v.w = pack_bf16x2(__uint_as_float(o[8 * g + 6]) * mul, __uint_as_float(o[8 * g + 7]) * mul);
      const int gran = ((c & 1) * 4 + g) ^ (r & 7);
      *reinterpret_cast<uint4*>(rowp + gran * 16) = v;
    }
  }
}

// ---------------------------------------------------------------------------
// D = rowsum(dO * O)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                      float* __restrict__ dd, long long rows) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat162* o = reinterpret_cast<const __nv_bfloat162*>(O + row * D + lane * kPer);
  const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(dO + row * D + lane * kPer);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < kPer / 2; ++i) {
    const float2 a = __bfloat1622float2(o[i]);
    const float2 b = __bfloat1622float2(g[i]);
    acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dd[row] = acc;
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per key tile
// ---------------------------------------------------------------------------
template <int D>
struct DkdvCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = D == 128 ? 2 : 3;      // each stage: Q_i and dO_i
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmemTiles = 2 * kTileBytes + kStages * kStageBytes;  // K, V, ring
  static constexpr int kNumBars = 1 + 2 * kStages + 1 + 1 + 1 + 1;
  static constexpr int kSmemBytes = kSmemTiles + 2 * 2 * kTile * 4 + kNumBars * 8 + 16 + 1024;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const BwdParams p) {
  using C = DkdvCfg<D>;
  constexpr int S = C::kStages;
  constexpr int TB = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + TB;
  uint8_t* sRing = smem + 2 * TB;  // stage s: Q at +0, dO at +TB
  float* sLse = reinterpret_cast<float*>(smem + C::kSmemTiles);  // [2][128] log2 units
  float* sD = sLse + 2 * kTile;                                   // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sD + 2 * kTile);
  uint64_t* kv_full = bars;            // K_j, V_j landed
  uint64_t* st_full = bars + 1;        // [S] Q_i, dO_i landed
  uint64_t* st_empty = st_full + S;    // [S] MMA done with a stage
  uint64_t* s_full = st_empty + S;     // S^T and dP^T in TMEM
  uint64_t* ds_ready = s_full + 1;     // P^T and dS^T in TMEM (128 arrivals)
  uint64_t* acc_done = ds_ready + 1;   // dK, dV final
  uint64_t* mma_done = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* status = &g_bwd_status;
  const uint64_t tmo = p.timeout_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, j;
  tile_of(p, /*heavy_high=*/false, &bh, &j);  // causal: low key tiles see the most queries
  const int i_first = CAUSAL ? j : 0;         // query tiles that see this key tile
  const int n_iter = p.n_tiles - i_first;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_ready, kElemThreads);
    mbar_init(acc_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(kv_full, 2 * TB);
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d(sK + c * kChunkBytes, &tmK, kv_full, c * 64, j * kTile, bh);
        tma_load_3d(sV + c * kChunkBytes, &tmV, kv_full, c * 64, j * kTile, bh);
      }
      int it = 0;
      for (; it < n_iter && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        ok = mbar_wait(&st_empty[s], ph ^ 1u, abort_flag, status, tmo, kSiteStage);
        if (!ok) break;
        const int i = i_first + it;
        uint8_t* st = sRing + s * C::kStageBytes;
        mbar_arrive_expect_tx(&st_full[s], 2 * TB);
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(st + c * kChunkBytes, &tmQ, &st_full[s], c * 64, i * kTile, bh);
          tma_load_3d(st + TB + c * kChunkBytes, &tmdO, &st_full[s], c * 64, i * kTile, bh);
        }
      }
      if (!ok) {
        for (int s = 0; s < S && s < it; ++s) {
          const int last = s + ((it - 1 - s) / S) * S;
          mbar_wait_drain(&st_full[s], static_cast<uint32_t>(last / S) & 1u, tmo);
        }
        mbar_wait_drain(kv_full, 0, tmo);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kTile, kTile, false);
      constexpr uint32_t idAcc = idesc_bf16_f32(kTile, D, true);
      const uint32_t sk = smem_addr(sK), sv = smem_addr(sV), sr = smem_addr(sRing);
      // X^T = A B^T with A, B both [128 rows][d] K-major tiles
      auto issue_abt = [&](uint32_t d_tmem, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          mma_ss(d_tmem, sw128_desc(a + off, 16, 1024), sw128_desc(b + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      // acc (+)= A[tmem, 128 x 128 queries] * B[queries x d] (B MN-major)
      auto issue_acc = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          mma_ts(d_tmem, a_tmem + packed_col(kk), sw128_desc(b + kk * 2048, kChunkBytes, 1024), idAcc,
                 (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, status, tmo, kSiteLoad);
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it % S;
        if (!(ok = mbar_wait(&st_full[s], static_cast<uint32_t>(it / S) & 1u, abort_flag, status, tmo, kSiteLoad))) break;
        tc_fence_after();
        const uint32_t q = sr + s * C::kStageBytes, dO = q + TB;
        issue_abt(tmem + kColS, sk, q);   // S^T = K Q^T
        issue_abt(tmem + kColDP, sv, dO); // dP^T = V dO^T
        mma_commit(s_full);
        if (!(ok = mbar_wait(ds_ready, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteDs))) break;
        tc_fence_after();
        issue_acc(tmem + kColAcc, tmem + kColS, dO, it > 0);      // dV += P^T dO
        issue_acc(tmem + kColAcc + D, tmem + kColDP, q, it > 0);  // dK += dS^T Q
        mma_commit(&st_empty[s]);
      }
      if (ok) mma_commit(acc_done);
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, tmo);
    }
  } else if (warp >= kElemWarp0) {
    const int half = (warp - kElemWarp0) >> 2;  // which 64 of the 128 query columns
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key row inside the tile
    const int key = j * kTile + r;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + kColS, tDP = tmem + lane_base + kColDP;
    const float sl2 = p.scale_log2;
    const float* lse_g = p.lse + static_cast<size_t>(bh) * p.N;
    const float* d_g = p.dd + static_cast<size_t>(bh) * p.N;
    // LSE (log2 units; first half of the threads) and D (second half) of the
    // 128 queries of a tile, staged in shared memory (two buffers); queries
    // past N get LSE = +inf, so P = 0 there.
    auto fetch = [&](int i) {
      const int qi = i * kTile + r;
      if (half == 0) return qi < p.N ? lse_g[qi] * 1.4426950408889634f : INFINITY;
      return qi < p.N ? d_g[qi] : 0.f;
    };
    float* stage_buf = half == 0 ? sLse : sD;
    float nxt = n_iter > 0 ? fetch(i_first) : 0.f;
    stage_buf[r] = nxt;
    named_bar_sync(1, kElemThreads);
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int i = i_first + it;
      const int buf = it & 1;
      if (it + 1 < n_iter) nxt = fetch(i + 1);  // next tile's, early
      const bool good = __all_sync(
          0xffffffffu, mbar_wait(s_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteS));
      if (good) {
        tc_fence_after();
        const float* lt = sLse + buf * kTile;
        const float* dt = sD + buf * kTile;
        const bool diag = CAUSAL && i == j;
        p_ds_tile<true>(
            tS, tDP, 2 * half, sl2, [&](int c) { return lt[c]; }, [&](int c) { return dt[c]; },
            [&](int c) { return !diag || i * kTile + c >= key; });
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_ready);
      }
      stage_buf[(buf ^ 1) * kTile + r] = nxt;
      // one barrier per iteration for every thread: it publishes the next
      // tile's LSE/D and makes a give-up decision uniform across the warps
      if (named_bar_or(1, kElemThreads, !good)) {
        ok = false;
        break;
      }
    }
    if (ok) ok = mbar_wait(acc_done, 0, abort_flag, status, tmo, kSiteO);
    const bool failed = named_bar_or(2, kElemThreads, !ok);
    if (!failed && n_iter > 0) {
      tc_fence_after();
      // K and V are no longer read by any MMA: they stage dK (first half of
      // the threads) and dV (second half)
      if (half == 0)
        store_tile<D>(tmem + lane_base + kColAcc + D, p.scale, sK, r, 0, D / 32);
      else
        store_tile<D>(tmem + lane_base + kColAcc, 1.f, sV, r, 0, D / 32);
      fence_proxy_async_smem();
      named_bar_sync(1, kElemThreads);
      if (half == 0 && r == 0) {
        for (int c = 0; c < C::kChunks; ++c) {
          tma_store_3d(&tmdK, sK + c * kChunkBytes, c * 64, j * kTile, bh);
          tma_store_3d(&tmdV, sV + c * kChunkBytes, c * 64, j * kTile, bh);
        }
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per query tile
// ---------------------------------------------------------------------------
template <int D>
struct DqCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = D == 128 ? 2 : 3;      // each stage: K_j and V_j
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmemTiles = 2 * kTileBytes + kStages * kStageBytes;  // Q, dO, ring
  static constexpr int kNumBars = 1 + 2 * kStages + 1 + 1 + 1 + 1;
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + 1024;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, const BwdParams p) {
  using C = DqCfg<D>;
  constexpr int S = C::kStages;
  constexpr int TB = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = smem + TB;
  uint8_t* sRing = smem + 2 * TB;  // stage s: K at +0, V at +TB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* q_full = bars;
  uint64_t* st_full = bars + 1;
  uint64_t* st_empty = st_full + S;
  uint64_t* s_full = st_empty + S;
  uint64_t* ds_ready = s_full + 1;
  uint64_t* acc_done = ds_ready + 1;
  uint64_t* mma_done = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* status = &g_bwd_status;
  const uint64_t tmo = p.timeout_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, i;
  tile_of(p, /*heavy_high=*/true, &bh, &i);  // causal: high query tiles see the most keys
  const int n_iter = CAUSAL ? i + 1 : p.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_ready, kElemThreads);
    mbar_init(acc_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(q_full, 2 * TB);
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d(sQ + c * kChunkBytes, &tmQ, q_full, c * 64, i * kTile, bh);
        tma_load_3d(sdO + c * kChunkBytes, &tmdO, q_full, c * 64, i * kTile, bh);
      }
      int it = 0;
      for (; it < n_iter && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        ok = mbar_wait(&st_empty[s], ph ^ 1u, abort_flag, status, tmo, kSiteStage);
        if (!ok) break;
        const int jt = it;  // key tile
        uint8_t* st = sRing + s * C::kStageBytes;
        mbar_arrive_expect_tx(&st_full[s], 2 * TB);
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(st + c * kChunkBytes, &tmK, &st_full[s], c * 64, jt * kTile, bh);
          tma_load_3d(st + TB + c * kChunkBytes, &tmV, &st_full[s], c * 64, jt * kTile, bh);
        }
      }
      if (!ok) {
        for (int s = 0; s < S && s < it; ++s) {
          const int last = s + ((it - 1 - s) / S) * S;
          mbar_wait_drain(&st_full[s], static_cast<uint32_t>(last / S) & 1u, tmo);
        }
        mbar_wait_drain(q_full, 0, tmo);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kTile, kTile, false);
      constexpr uint32_t idAcc = idesc_bf16_f32(kTile, D, true);
      const uint32_t sq = smem_addr(sQ), sdo = smem_addr(sdO), sr = smem_addr(sRing);
      auto issue_abt = [&](uint32_t d_tmem, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          mma_ss(d_tmem, sw128_desc(a + off, 16, 1024), sw128_desc(b + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, status, tmo, kSiteLoad);
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it % S;
        if (!(ok = mbar_wait(&st_full[s], static_cast<uint32_t>(it / S) & 1u, abort_flag, status, tmo, kSiteLoad))) break;
        tc_fence_after();
        const uint32_t k = sr + s * C::kStageBytes, v = k + TB;
        issue_abt(tmem + kColS, sq, k);    // S = Q K^T
        issue_abt(tmem + kColDP, sdo, v);  // dP = dO V^T
        mma_commit(s_full);
        if (!(ok = mbar_wait(ds_ready, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteDs))) break;
        tc_fence_after();
        // dQ += dS K: A = dS in TMEM (over dP), B = K tile as [keys][d] (MN-major)
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          mma_ts(tmem + kColAcc, tmem + kColDP + packed_col(kk), sw128_desc(k + kk * 2048, kChunkBytes, 1024),
                 idAcc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&st_empty[s]);
      }
      if (ok) mma_commit(acc_done);
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, tmo);
    }
  } else if (warp >= kElemWarp0) {
    const int half = (warp - kElemWarp0) >> 2;  // which 64 of the 128 key columns
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // query row inside the tile
    const int row = i * kTile + r;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + kColS, tDP = tmem + lane_base + kColDP;
    const float sl2 = p.scale_log2;
    // this row's LSE (log2 units) and D; rows past N get P = 0
    const float lse2 = row < p.N ? p.lse[static_cast<size_t>(bh) * p.N + row] * 1.4426950408889634f : INFINITY;
    const float dsub = row < p.N ? p.dd[static_cast<size_t>(bh) * p.N + row] : 0.f;
    const int key_limit = CAUSAL ? min(row, p.N - 1) : p.N - 1;
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(s_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteS));
      if (!ok) break;
      tc_fence_after();
      const int kbase = it * kTile;
      const bool masked = (kbase + kTile > p.N) || (CAUSAL && kbase + kTile - 1 > i * kTile);
      p_ds_tile<false>(
          tS, tDP, 2 * half, sl2, [&](int) { return lse2; }, [&](int) { return dsub; },
          [&](int c) { return !masked || kbase + c <= key_limit; });
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_ready);
    }
    if (ok) ok = mbar_wait(acc_done, 0, abort_flag, status, tmo, kSiteO);
    const bool failed = named_bar_or(2, kElemThreads, !ok);
    if (!failed) {
      tc_fence_after();
      // Q is no longer read by any MMA: it stages dQ, each half of the
      // threads taking half of the columns
      store_tile<D>(tmem + lane_base + kColAcc, p.scale, sQ, r, half * (D / 64), (half + 1) * (D / 64));
      fence_proxy_async_smem();
      named_bar_sync(1, kElemThreads);
      if (half == 0 && r == 0) {
        for (int c = 0; c < C::kChunks; ++c) tma_store_3d(&tmdQ, sQ + c * kChunkBytes, c * 64, i * kTile, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

std::mutex g_attr_mutex;
bool g_attr_set[64][8] = {};

template <typename Kern>
fa_status set_smem(Kern kern, int bytes, int slot) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return host::cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  if (!g_attr_set[dev & 63][slot]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return host::cuda_fail(e, "cudaFuncSetAttribute");
    g_attr_set[dev & 63][slot] = true;
  }
  return FA_OK;
}

template <int D, bool CAUSAL>
fa_status launch_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     void* dQ, void* dK, void* dV, float* dd, BwdParams prm, cudaStream_t st) {
  const int N = prm.N, BH = prm.BH;
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
  if (!host::make_map(&mq, Q, D, N, BH, kTile) || !host::make_map(&mk, K, D, N, BH, kTile) ||
      !host::make_map(&mv, V, D, N, BH, kTile) || !host::make_map(&mdo, dO, D, N, BH, kTile) ||
      !host::make_map(&mdq, dQ, D, N, BH, kTile) || !host::make_map(&mdk, dK, D, N, BH, kTile) ||
      !host::make_map(&mdv, dV, D, N, BH, kTile)) {
    snprintf(host::g_last_error, sizeof(host::g_last_error), "cuTensorMapEncodeTiled failed");
    return FA_ERR_CUDA;
  }
  const long long rows = static_cast<long long>(BH) * N;
  bwd_rowdot_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), dd, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd rowdot launch");
  const unsigned grid = static_cast<unsigned>(static_cast<long long>(BH) * prm.n_tiles);
  const int slot = (D == 128 ? 4 : 0) + (CAUSAL ? 2 : 0);
  fa_status r = set_smem(bwd_dkdv_kernel<D, CAUSAL>, DkdvCfg<D>::kSmemBytes, slot);
  if (r != FA_OK) return r;
  r = set_smem(bwd_dq_kernel<D, CAUSAL>, DqCfg<D>::kSmemBytes, slot + 1);
  if (r != FA_OK) return r;
  bwd_dkdv_kernel<D, CAUSAL><<<grid, kThreads, DkdvCfg<D>::kSmemBytes, st>>>(mq, mk, mv, mdo, mdk, mdv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd dkdv launch");
  bwd_dq_kernel<D, CAUSAL><<<grid, kThreads, DqCfg<D>::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd dq launch");
  return FA_OK;
}

}  // namespace

// Read and clear the backward kernels' status word (fa_get_device_status
// reports it together with the forward's).
cudaError_t read_and_clear_status(uint32_t* v) {
  *v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(v, g_bwd_status, sizeof(*v));
  if (e != cudaSuccess || *v == 0) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_bwd_status, &zero, sizeof(zero));
}

}  // namespace bwd
}  // namespace fa

extern "C" {

size_t fa_bwd_workspace_bytes(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return static_cast<size_t>(B) * H * N * 4;
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                 size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                 void* stream) {
  using namespace fa;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace) return FA_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || !std::isfinite(scale)) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  const long long n_tiles = (static_cast<long long>(N) + bwd::kTile - 1) / bwd::kTile;
  if (BH > (1ll << 30) || BH * n_tiles > 0x7fffffffll || BH * N > 0x7fffffffll * 8ll) return FA_ERR_SHAPE;
  auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis16(Q) || mis16(K) || mis16(V) || mis16(O) || mis16(dO) || mis16(dQ) || mis16(dK) ||
      mis16(dV) || mis16(workspace) || (reinterpret_cast<uintptr_t>(LSE) & 3u))
    return FA_ERR_ALIGN;
  const size_t need = fa_bwd_workspace_bytes(B, H, N);
  if (workspace_bytes < need) return FA_ERR_WORKSPACE;
  const size_t nb = static_cast<size_t>(BH) * N * d * 2;
  const size_t lb = static_cast<size_t>(BH) * N * 4;
  const void* ins[6] = {Q, K, V, O, dO, LSE};
  const size_t insz[6] = {nb, nb, nb, nb, nb, lb};
  void* outs[4] = {dQ, dK, dV, workspace};
  const size_t outsz[4] = {nb, nb, nb, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (host::overlaps(outs[a], outsz[a], ins[b], insz[b])) return FA_ERR_ALIAS;
    for (int b = a + 1; b < 4; ++b)
      if (host::overlaps(outs[a], outsz[a], outs[b], outsz[b])) return FA_ERR_ALIAS;
  }
  fa_status st0 = host::require_sm100();
  if (st0 != FA_OK) return st0;
  bwd::BwdParams prm{};
  prm.lse = LSE;
  prm.dd = static_cast<const float*>(workspace);
  prm.N = N;
  prm.BH = static_cast<int>(BH);
  prm.n_tiles = static_cast<int>(n_tiles);
  {
    // keep the Q, dO, K, V of one group of heads (8*N*d bytes per head) within ~48 MB of L2
    const long long per_head = 8ll * N * d;
    long long g = (48ll << 20) / per_head;
    prm.group_heads = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
  }
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  prm.timeout_ns = host::wait_timeout_ns();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* dd = static_cast<float*>(workspace);
  if (d == 128)
    return causal ? bwd::launch_bwd<128, true>(Q, K, V, O, dO, dQ, dK, dV, dd, prm, st)
                  : bwd::launch_bwd<128, false>(Q, K, V, O, dO, dQ, dK, dV, dd, prm, st);
  return causal ? bwd::launch_bwd<64, true>(Q, K, V, O, dO, dQ, dK, dV, dd, prm, st)
                : bwd::launch_bwd<64, false>(Q, K, V, O, dO, dQ, dK, dV, dd, prm, st);
}

}  // extern "C"
