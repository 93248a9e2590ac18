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
//   bwd_rowdot   D = rowsum(dO * O) and LSE * log2(e), one warp per row,
//                into a workspace padded to whole 128-row tiles, and the fp32
//                dQ accumulator set to zero (HBM-bound).
//   bwd_dkdv     one CTA per 128-key tile, over the query tiles that see it:
//                S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T formed
//                in place (bf16); dV += P^T dO and dK += dS^T Q accumulate in
//                TMEM; dQ_i = dS K, the tile's share of the query tile's dQ,
//                is formed in TMEM and added into the fp32 accumulator in
//                global memory (reductions at L2).  Every product of the
//                gradient is computed once.
//   bwd_dq_convert  dQ = scale * accumulator, to bf16.
// CTA layout of bwd_dkdv (384 threads): warp 0 TMA producer, warp 1 TMEM
// owner and MMA issuer, warps 4-11 elementwise step, dQ reductions and
// epilogue (two threads per TMEM lane, i.e. per row).  The elementwise
// threads work through each tile a quarter (32 columns) at a time
// and release every quarter to the MMA issuer on its own barrier, so that the
// accumulating products of one quarter overlap the elementwise step of the
// next.  The MMAs are N = 128 (S, dP) or N = d (accumulators): an M = 128
// tcgen05.mma costs about the same at N = 64 as at N = 128.
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

constexpr int kTile = 128;  // query rows and keys per tile
constexpr int kQuarter = 32;  // columns released to the MMAs at a time
constexpr int kThreads = 384;
constexpr int kElemWarp0 = 4;      // warps 4-11: two threads per row, 16 columns of each quarter each
constexpr int kElemThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kChunkBytes = kTile * 64 * 2;  // one 64-wide, 128-row swizzled box: 16 KB

enum : uint32_t { kSiteLoad = 0, kSiteStage = 1, kSiteS = 2, kSiteDs = 3, kSiteO = 4, kSiteDq = 5 };

struct BwdParams {
  const float* lse2;  // [BH][n_pad] the forward's LSE times log2(e); +inf past N
  const float* dd;    // [BH][n_pad] D = rowsum(dO * O); 0 past N
  float* dq_acc;      // [BH][n_pad][d] fp32: dS K summed over the key tiles by reduce-adds
  int N;
  int n_pad;          // N rounded up to a multiple of 128
  int BH;
  int n_tiles;        // n_pad / 128
  int group_heads;    // heads whose CTAs are scheduled together
  float scale;        // multiplier of q.k
  float scale_log2;   // scale * log2(e)
  uint64_t timeout_ns;
};

__device__ uint32_t g_bwd_status;

// Optional phase trace (build with -DFA_TRACE): SM clock stamps of the
// producer, the MMA issuer and two elementwise threads, for the first CTAs
// of each tiled kernel (k = 0: dK/dV, 1: dQ).
#ifdef FA_TRACE
constexpr int kTraceCtas = 16;
constexpr int kTraceIters = 64;
__device__ unsigned long long* g_bwd_trace;  // [2][kTraceCtas][4 roles][kTraceIters][8 events]
// (the clock is read before the buffer's address is loaded, so that the load
// cannot delay the stamp)
#define BWD_TRACE(k, role, iter, ev)                                                                   \
  do {                                                                                                 \
    const unsigned long long now_ = clock64();                                                         \
    if (blockIdx.x < kTraceCtas && (iter) < kTraceIters && g_bwd_trace != nullptr)                     \
      g_bwd_trace[(((static_cast<size_t>(k) * kTraceCtas + blockIdx.x) * 4 + (role)) * kTraceIters +   \
                   (iter)) * 8 + (ev)] = now_;                                                          \
  } while (0)
#else
#define BWD_TRACE(k, role, iter, ev) \
  do {                               \
  } while (0)
#endif

// TMEM columns (both tiled kernels): S (or S^T) at [0,128), dP (or dP^T) at
// [128,256), accumulators from 256.  P and dS (bf16 pairs) overwrite their own
// columns: the 16 values a thread forms in columns c..c+15 go, packed, to
// columns c..c+7.
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;
// TMEM column of the packed bf16 operand for K-step kk (16 queries or keys):
// quarter kk / 2, half kk % 2
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk >> 1) * 32 + (kk & 1) * 16; }

// *p += v, four fp32 adds performed at L2 (no value returned)
__device__ __forceinline__ void red_add_v4(float* p, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

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

// tcgen05.wait::ld naming one 16-register destination of the loads it waits
// for, so that no use of it can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld_reg16(uint32_t (&a)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
        "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]),
        "+r"(a[15])
      :
      : "memory");
}

// Exponentials of 16 columns c0..c0+15 of the calling thread's row, from
// scores s in registers: p = 2^(s * scale log2e - lse2), 0 where `allowed`
// fails (MASK only).  col(c, l4, d4) gives lse2 and D of columns c..c+3.
template <bool MASK, typename Col, typename Allowed>
__device__ __forceinline__ void p_16(const uint32_t (&s)[16], int c0, float sl2, Col col, Allowed allowed,
                                     float (&p)[16]) {
  const float2 sl2v = make_float2(sl2, sl2);
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    float4 l4, d4;
    col(c0 + e, l4, d4);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 sv = make_float2(__uint_as_float(s[e + u]), __uint_as_float(s[e + u + 1]));
      const float2 lv = u == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w);
      const float2 x = ffma2(sv, sl2v, lv);
      p[e + u] = ex2_approx(x.x);
      p[e + u + 1] = ex2_approx(x.y);
      if (MASK) {
        if (!allowed(c0 + e + u)) p[e + u] = 0.f;
        if (!allowed(c0 + e + u + 1)) p[e + u + 1] = 0.f;
      }
    }
  }
}

// ds = p * (dp - D) for the same 16 columns; P and dS packed to bf16 pairs.
template <typename Col>
__device__ __forceinline__ void ds_16(const float (&p)[16], const uint32_t (&dp)[16], int c0, Col col,
                                      uint32_t (&pk)[8], uint32_t (&dk)[8]) {
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    float4 l4, d4;
    col(c0 + e, l4, d4);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 dv = u == 0 ? make_float2(-d4.x, -d4.y) : make_float2(-d4.z, -d4.w);
      const float2 pv = make_float2(p[e + u], p[e + u + 1]);
      const float2 g = fadd2(make_float2(__uint_as_float(dp[e + u]), __uint_as_float(dp[e + u + 1])), dv);
      const float2 dsv = fmul2(pv, g);
      pk[(e + u) >> 1] = pack_bf16x2(pv.x, pv.y);
      dk[(e + u) >> 1] = pack_bf16x2(dsv.x, dsv.y);
    }
  }
}

// The calling thread's share of one tile: 16 columns of each quarter
// (column h*16 of quarters 0..3), quarter by quarter.  Only S is needed for
// the exponentials, so quarter 0's run while the dP product may still be in
// the tensor core; dp_ready() waits for it (false: give up) before dP is
// first read.  The scores of the next quarter are loaded while the current
// one is computed, and its dP while the current stores drain; P (optional)
// and dS go back as bf16 pairs over the first 8 of each thread's 16 columns,
// and each quarter is released on ready[q] once its stores have completed.
// DS_SMEM: dS also goes to shared memory as the A operand of dQ_i = dS K:
// [keys][queries] (query-contiguous, two 64-query chunks of 128-byte rows in
// the 128-byte swizzle), row r = the thread's key; ds_row points at row r of
// the first chunk.  each_quarter(q) runs at the start of quarter q (other
// work to interleave with the quarters).
template <bool WRITE_P, bool MASK, bool DS_SMEM, typename Col, typename Allowed, typename Wait,
          typename Each>
__device__ __forceinline__ bool p_ds_tile(uint32_t tS, uint32_t tDP, int h, float sl2, Col col,
                                          Allowed allowed, uint64_t* ready, Wait dp_ready, Each each_quarter,
                                          uint8_t* ds_row = nullptr, int r = 0) {
  uint32_t s[2][16], dp[16];
  tmem_ld16(tS + h * 16, s[0]);
  tmem_wait_ld_reg16(s[0]);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c0 = q * kQuarter + h * 16;
    if (q < 3) tmem_ld16(tS + c0 + kQuarter, s[(q + 1) & 1]);
    each_quarter(q);
    float pv[16];
    p_16<MASK>(s[q & 1], c0, sl2, col, allowed, pv);
    if (q == 0) {
      if (!dp_ready()) return false;
      tc_fence_after();
      tmem_ld16(tDP + c0, dp);
      tmem_wait_ld_regs(dp, s[1]);
    }
    uint32_t pk[8], dk[8];
    ds_16(pv, dp, c0, col, pk, dk);
    if (q < 3) tmem_ld16(tDP + c0 + kQuarter, dp);
    if (WRITE_P) tmem_st8(tS + c0, pk);
    tmem_st8(tDP + c0, dk);
    if (DS_SMEM) {
      // queries c0..c0+15 = 16-byte granules gb, gb + 1 of the row in chunk q / 2
      uint8_t* rowp = ds_row + (q >> 1) * kChunkBytes;
      const int gb = (q & 1) * 4 + h * 2;
      *reinterpret_cast<uint4*>(rowp + ((gb ^ (r & 7)) * 16)) = make_uint4(dk[0], dk[1], dk[2], dk[3]);
      *reinterpret_cast<uint4*>(rowp + (((gb + 1) ^ (r & 7)) * 16)) = make_uint4(dk[4], dk[5], dk[6], dk[7]);
      fence_proxy_async_smem();  // visible to the tensor core's reads
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&ready[q]);
    if (q < 3) tmem_wait_ld_regs(dp, s[(q + 1) & 1]);
  }
  return true;
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
// D = rowsum(dO * O) and LSE in log2 units, padded to n_pad rows per head
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                      const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dd,
                      float* __restrict__ dq_acc, int N, int n_pad, long long rows_pad) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows_pad) return;
  // the dQ accumulator row starts at zero (padding rows too: they receive
  // reduce-adds of zeros)
  {
    float* z = dq_acc + row * D + lane * kPer;
    if constexpr (kPer == 4)
      *reinterpret_cast<float4*>(z) = make_float4(0.f, 0.f, 0.f, 0.f);
    else
      *reinterpret_cast<float2*>(z) = make_float2(0.f, 0.f);
  }
  const long long bh = row / n_pad;
  const int q = static_cast<int>(row - bh * n_pad);
  if (q >= N) {  // padding: P = 0 there
    if (lane == 0) {
      lse2[row] = INFINITY;
      dd[row] = 0.f;
    }
    return;
  }
  const long long src = bh * N + q;
  const __nv_bfloat162* o = reinterpret_cast<const __nv_bfloat162*>(O + src * D + lane * kPer);
  const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(dO + src * D + lane * kPer);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < kPer / 2; ++i) {
    const float2 a = __bfloat1622float2(o[i]);
    const float2 b = __bfloat1622float2(g[i]);
    acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dd[row] = acc;
    lse2[row] = lse[src] * 1.4426950408889634f;
  }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per 128-key tile
// ---------------------------------------------------------------------------
template <int D>
struct DkdvCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = D == 128 ? 2 : 4;  // each stage: Q_i and dO_i (+ LSE2_i, D_i)
  static constexpr int kStageBytes = 2 * kTileBytes;
  // dS of the current tile (bf16, [keys][queries] in two 64-query chunks):
  // the A operand of dQ_i = dS K; once that product has finished, the
  // elementwise warps transpose dQ_i's rows through it, one 32-row x
  // 32-column (fp32) box per warp at a time
  static constexpr int kDsBytes = 2 * kChunkBytes;
  static constexpr int kBoxBytes = 32 * 128;
  static_assert((kElemThreads / 32) * kBoxBytes <= kDsBytes, "the transposition boxes fit the dS buffer");
  static constexpr int kSmemTiles = 2 * kTileBytes + kStages * kStageBytes + kDsBytes;  // K, V, ring, dS
  static constexpr int kLdBytes = kStages * 2 * kTile * 4;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 4 + 1 + 1 + 2;
  // No alignment slack: at d = 128 it would not fit in 227 KB.  The kernel
  // checks that its dynamic shared memory starts 1024-aligned instead.
  static constexpr int kSmemBytes = kSmemTiles + kLdBytes + kNumBars * 8 + 16;
  // the dQ_i product in TMEM: over S^T at d = 128 (all 512 columns are
  // otherwise in use), in the 128 columns past the accumulators at d = 64
  static constexpr uint32_t kColDQ = D == 128 ? kColS : kColAcc + 2 * D;
  static_assert(kColDQ + D <= kTmemCols, "dQ_i fits in TMEM");
};

// One CTA per 128-key tile j; per query tile i (the ones that see tile j):
//   S^T = K Q_i^T and dP^T = V dO_i^T (N = 128) into TMEM;
//   the elementwise threads form P^T and dS^T a quarter (32 queries) at a
//   time and release each quarter on its own barrier, so that dV += P^T dO_i
//   and dK += dS^T Q_i run on one quarter while the next is being formed;
//   they also write dS to shared memory, and dQ_i = dS K (the tile's share of
//   dQ for query tile i) is then formed in TMEM, read out by the elementwise
//   warps and added into the fp32 dQ accumulator in global memory by
//   reductions at L2.  So every product of the gradient is computed once: no
//   second pass recomputes S and dP for dQ.
// tcgen05 MMAs of one thread run in issue order, so dP^T of tile i+1 may be
// issued right after the products that read tile i's dS^T, and S^T of tile
// i+1 right after dQ_i has been read out of the columns they share (d = 128).
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const BwdParams p) {
  using C = DkdvCfg<D>;
  constexpr int S = C::kStages;
  constexpr int TB = C::kTileBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment and there is no slack to
  // align by hand: refuse to run otherwise (uniformly, before any barrier)
  if ((smem_addr(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_bwd_status, kStatusBounds);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;
  uint8_t* sV = smem + TB;
  uint8_t* sRing = smem + 2 * TB;  // stage s: Q_i at +0, dO_i at +TB
  uint8_t* sDs = sRing + S * C::kStageBytes;
  float* sLd = reinterpret_cast<float*>(smem + C::kSmemTiles);  // stage s: LSE2 [128], D [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles + C::kLdBytes);
  uint64_t* kv_full = bars;           // K, V landed
  uint64_t* st_full = bars + 1;       // [S] Q_i, dO_i, LSE2_i, D_i landed
  uint64_t* st_empty = st_full + S;   // [S] MMA done with a stage
  uint64_t* s_full = st_empty + S;    // S^T in TMEM
  uint64_t* dp_full = s_full + 1;     // dP^T in TMEM
  uint64_t* ds_ready = dp_full + 1;   // [4] quarter q of P^T and dS^T in TMEM, dS in SMEM (256 arrivals)
  uint64_t* acc_done = ds_ready + 4;  // dK, dV final
  uint64_t* mma_done = acc_done + 1;
  uint64_t* dq_full = mma_done + 1;     // dQ_i in TMEM (dS no longer read)
  uint64_t* dq_drained = dq_full + 1;   // dQ_i read out of TMEM (one arrival per elementwise warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dq_drained + 1);
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
    mbar_init(dp_full, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&ds_ready[q], kElemThreads);
    mbar_init(acc_done, 1);
    mbar_init(mma_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_drained, kElemThreads / 32);
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
      const size_t ld_row = static_cast<size_t>(bh) * p.n_pad;
      int it = 0;
      for (; it < n_iter && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        ok = mbar_wait(&st_empty[s], ph ^ 1u, abort_flag, status, tmo, kSiteStage);
        if (!ok) break;
        BWD_TRACE(0, 3, it, 0);
        const int i = i_first + it;
        uint8_t* st = sRing + s * C::kStageBytes;
        float* ld = sLd + s * 2 * kTile;
        mbar_arrive_expect_tx(&st_full[s], 2 * TB + 2 * kTile * 4);
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(st + c * kChunkBytes, &tmQ, &st_full[s], c * 64, i * kTile, bh);
          tma_load_3d(st + TB + c * kChunkBytes, &tmdO, &st_full[s], c * 64, i * kTile, bh);
        }
        bulk_load(ld, p.lse2 + ld_row + i * kTile, kTile * 4, &st_full[s]);
        bulk_load(ld + kTile, p.dd + ld_row + i * kTile, kTile * 4, &st_full[s]);
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
      constexpr uint32_t idDq = idesc_bf16_f32(kTile, D, true, true);
      const uint32_t sk = smem_addr(sK), sv = smem_addr(sV), sr = smem_addr(sRing), sds = smem_addr(sDs);
      // X^T = A B^T with A, B both [128 rows][d] K-major tiles
      auto issue_abt = [&](uint32_t d_tmem, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          mma_ss(d_tmem, sw128_desc(a + off, 16, 1024), sw128_desc(b + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      // acc (+)= A[tmem, 128 x 32 queries of quarter q] * B[those queries x d] (B MN-major)
      auto issue_acc_q = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b, int q, bool accumulate) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int kk = 2 * q + h;
          mma_ts(d_tmem, a_tmem + packed_col(kk), sw128_desc(b + kk * 2048, kChunkBytes, 1024), idAcc,
                 (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      // dQ_i = dS K: A = dS [keys][queries] (M = queries contiguous), B = K
      // [keys][d] (N = d contiguous); 16 keys (rows) = 2 KB per K-step
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ss(tmem + C::kColDQ, sw128_desc(sds + kk * 2048, kChunkBytes, 1024),
                 sw128_desc(sk + kk * 2048, kChunkBytes, 1024), idDq, kk > 0 ? 1u : 0u);
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, status, tmo, kSiteLoad);
      if (ok && n_iter > 0 && (ok = mbar_wait(&st_full[0], 0, abort_flag, status, tmo, kSiteLoad))) {
        tc_fence_after();
        issue_abt(tmem + kColS, sk, sr);        // S^T = K Q^T
        mma_commit(s_full);
        issue_abt(tmem + kColDP, sv, sr + TB);  // dP^T = V dO^T
        mma_commit(dp_full);
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it % S;
        const uint32_t q = sr + s * C::kStageBytes, dO = q + TB;
        BWD_TRACE(0, 0, it, 1);
        for (int qq = 0; qq < 4 && ok; ++qq) {
          if (!(ok = mbar_wait(&ds_ready[qq], static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteDs)))
            break;
          if (qq == 0) BWD_TRACE(0, 0, it, 2);
          BWD_TRACE(0, 0, it, 4 + qq);
          tc_fence_after();
          issue_acc_q(tmem + kColAcc, tmem + kColS, dO, qq, it > 0);      // dV += P^T dO
          issue_acc_q(tmem + kColAcc + D, tmem + kColDP, q, qq, it > 0);  // dK += dS^T Q
        }
        if (!ok) break;
        // at d = 64 dQ_i has columns of its own: the previous one must have been read out
        if (D == 64 && it > 0 &&
            !(ok = mbar_wait(dq_drained, static_cast<uint32_t>(it - 1) & 1u, abort_flag, status, tmo, kSiteDq)))
          break;
        issue_dq();
        mma_commit(dq_full);
        mma_commit(&st_empty[s]);
        BWD_TRACE(0, 0, it, 3);
        if (it + 1 < n_iter) {
          const int s1 = (it + 1) % S;
          const uint32_t q1 = sr + s1 * C::kStageBytes;
          if (!(ok = mbar_wait(&st_full[s1], static_cast<uint32_t>((it + 1) / S) & 1u, abort_flag, status, tmo,
                               kSiteLoad)))
            break;
          BWD_TRACE(0, 0, it + 1, 0);
          tc_fence_after();
          issue_abt(tmem + kColDP, sv, q1 + TB);  // dP^T of the next tile: dK has read this dS^T
          mma_commit(dp_full);
          // at d = 128 the next S^T goes where dQ_i is: wait until it is read out
          if (D == 128 &&
              !(ok = mbar_wait(dq_drained, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteDq)))
            break;
          tc_fence_after();
          issue_abt(tmem + kColS, sk, q1);
          mma_commit(s_full);
        }
      }
      if (ok) mma_commit(acc_done);
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, tmo);
    }
  } else if (warp >= kElemWarp0) {
    const int e = warp - kElemWarp0;  // elementwise warp 0..7
    const int h = e >> 2;              // which 16 columns of every quarter; which half of dQ_i's columns
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key row inside the tile; query row of dQ_i
    const int key = j * kTile + r;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + kColS, tDP = tmem + lane_base + kColDP;
    const uint32_t tDQ = tmem + lane_base + C::kColDQ;
    uint8_t* box = sDs + e * C::kBoxBytes;  // this warp's transposition box
    const float sl2 = p.scale_log2;
    const bool tr = lane == 0 && wq == 0;
    // A tile's share of dQ is added into the fp32 accumulator while the next
    // tile is formed: 3/16 of it in each quarter and the last quarter of it
    // while the dQ product of that tile is in the tensor core, so that the
    // reductions reach L2 as a steady stream under the arithmetic instead of
    // a burst the warps would stall on.  pend holds it transposed (see
    // below); pend_base is its accumulator rows, null when nothing is
    // pending.
    constexpr int kRounds = D / 64;     // 32-column groups of this thread's half of a row
    constexpr int kReds = kRounds * 8;  // reduction instructions per tile and thread
    constexpr int kPerQuarter = kReds * 3 / 16;
    float4 pend[kReds];
    float* pend_base = nullptr;
    auto flush = [&](int from, int to) {
      if (pend_base == nullptr) return;
#pragma unroll
      for (int k = 0; k < kReds; ++k) {
        if (k < from || k >= to) continue;
        const int row = (k & 7) * 4 + (lane >> 3), g = lane & 7;
        red_add_v4(pend_base + static_cast<size_t>(row) * D + (k >> 3) * 32 + g * 4, pend[k]);
      }
    };
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int s = it % S;
      const int i = i_first + it;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(s_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteS));
      // the stage's LSE2 and D come from the bulk copy engine: observe its barrier too
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait(&st_full[s], static_cast<uint32_t>(it / S) & 1u, abort_flag,
                                               status, tmo, kSiteLoad));
      if (!ok) break;
      if (tr) BWD_TRACE(0, 1 + h, it, 0);
      tc_fence_after();
      const float4* l4p = reinterpret_cast<const float4*>(sLd + s * 2 * kTile);
      const float4* d4p = l4p + kTile / 4;
      auto col = [&](int c, float4& l4, float4& d4) {
        l4 = l4p[c >> 2];
        d4 = d4p[c >> 2];
      };
      const int q0 = i * kTile;
      auto allowed = [&](int c) { return q0 + c >= key; };
      const bool diag = CAUSAL && i == j;
      auto dp_ready = [&]() {
        return __all_sync(0xffffffffu, mbar_wait(dp_full, static_cast<uint32_t>(it) & 1u, abort_flag, status,
                                                 tmo, kSiteS));
      };
      // (the previous tile's transposition is over: every warp passed the
      // barrier that ends it)
      uint8_t* ds_row = sDs + r * 128;
      auto each_quarter = [&](int q) { flush(q * kPerQuarter, (q + 1) * kPerQuarter); };
      ok = diag ? p_ds_tile<true, true, true>(tS, tDP, h, sl2, col, allowed, ds_ready, dp_ready, each_quarter,
                                              ds_row, r)
                : p_ds_tile<true, false, true>(tS, tDP, h, sl2, col, allowed, ds_ready, dp_ready, each_quarter,
                                               ds_row, r);
      if (tr) BWD_TRACE(0, 1 + h, it, 1);
      if (!ok) break;
      flush(4 * kPerQuarter, kReds);
      // dQ_i: this thread's query row r, columns [h d/2, (h+1) d/2), 32 at a time
      ok = __all_sync(0xffffffffu,
                      mbar_wait(dq_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, tmo, kSiteDq));
      if (!ok) break;
      tc_fence_after();
      uint32_t o[kRounds][32];
#pragma unroll
      for (int rd = 0; rd < kRounds; ++rd) tmem_ld32(tDQ + h * (D / 2) + rd * 32, o[rd]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_drained);
      // Transposed 32 columns at a time through this warp's box (the dQ_i
      // product has finished, so dS is no longer read and its buffer holds
      // the boxes): each lane writes its row (128 bytes, 16-byte granules
      // rotated by the row to spread the banks), then the warp reads the box
      // back four rows per instruction, eight lanes per row, so that every
      // reduction instruction covers four whole 128-byte lines of the
      // accumulator.
#pragma unroll
      for (int rd = 0; rd < kRounds; ++rd) {
#pragma unroll
        for (int g = 0; g < 8; ++g)
          *reinterpret_cast<uint4*>(box + lane * 128 + ((g ^ (lane & 7)) * 16)) =
              make_uint4(o[rd][4 * g], o[rd][4 * g + 1], o[rd][4 * g + 2], o[rd][4 * g + 3]);
        __syncwarp();
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const int row = k4 * 4 + (lane >> 3), g = lane & 7;
          pend[rd * 8 + k4] = *reinterpret_cast<const float4*>(box + row * 128 + ((g ^ (row & 7)) * 16));
        }
        __syncwarp();  // the box is read before the next round overwrites it
      }
      pend_base = p.dq_acc + (static_cast<size_t>(bh) * p.n_pad + i * kTile + wq * 32) * D + h * (D / 2);
      // the next tile's dS goes into the same buffer: every warp must have
      // read its boxes back first
      named_bar_sync(3, kElemThreads);
      if (tr) BWD_TRACE(0, 1 + h, it, 2);
    }
    if (ok) flush(0, kReds);  // the last tile's share
    if (ok) ok = mbar_wait(acc_done, 0, abort_flag, status, tmo, kSiteO);
    const bool failed = named_bar_or(2, kElemThreads, !ok);
    if (!failed && n_iter > 0) {
      tc_fence_after();
      // K and V are no longer read by any MMA (the last dQ_i has finished):
      // they stage dK (warps 4-7) and dV (warps 8-11)
      if (h == 0)
        store_tile<D>(tmem + lane_base + kColAcc + D, p.scale, sK, r, 0, D / 32);
      else
        store_tile<D>(tmem + lane_base + kColAcc, 1.f, sV, r, 0, D / 32);
      fence_proxy_async_smem();
      named_bar_sync(1, kElemThreads);
      if (h == 0 && r == 0) {
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

// dQ = scale * (sum over the key tiles of dS K), fp32 -> bf16, rows < N; one
// warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dQ, float scale,
                          int N, int n_pad, long long rows) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const long long bh = row / N;
  const long long q = row - bh * N;
  const float* src = dq_acc + (bh * n_pad + q) * D + lane * kPer;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(dQ + row * D + lane * kPer);
  if constexpr (kPer == 4) {
    const float4 v = *reinterpret_cast<const float4*>(src);
    dst[0] = __floats2bfloat162_rn(v.x * scale, v.y * scale);
    dst[1] = __floats2bfloat162_rn(v.z * scale, v.w * scale);
  } else {
    const float2 v = *reinterpret_cast<const float2*>(src);
    dst[0] = __floats2bfloat162_rn(v.x * scale, v.y * scale);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

// dynamic shared-memory attribute set per (device, kernel); the call is
// idempotent, so threads that race on an unset flag both make it, harmlessly
std::atomic<bool> g_attr_set[64][8] = {};

template <typename Kern>
fa_status set_smem(Kern kern, int bytes, int slot) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return host::cuda_fail(e, "cudaGetDevice");
  if (!g_attr_set[dev & 63][slot].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return host::cuda_fail(e, "cudaFuncSetAttribute");
    g_attr_set[dev & 63][slot].store(true, std::memory_order_release);
  }
  return FA_OK;
}

template <int D, bool CAUSAL>
fa_status launch_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const float* LSE, void* dQ, void* dK, void* dV, float* lse2, float* dd, BwdParams prm,
                     cudaStream_t st) {
  const int N = prm.N, BH = prm.BH;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (!host::make_map_cached(&mq, Q, D, N, BH, kTile) || !host::make_map_cached(&mk, K, D, N, BH, kTile) ||
      !host::make_map_cached(&mv, V, D, N, BH, kTile) || !host::make_map_cached(&mdo, dO, D, N, BH, kTile) ||
      !host::make_map_cached(&mdk, dK, D, N, BH, kTile) || !host::make_map_cached(&mdv, dV, D, N, BH, kTile)) {
    snprintf(host::g_last_error, sizeof(host::g_last_error), "cuTensorMapEncodeTiled failed");
    return FA_ERR_CUDA;
  }
  const long long rows_pad = static_cast<long long>(BH) * prm.n_pad;
  bwd_rowdot_kernel<D><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), LSE, lse2, dd, prm.dq_acc,
      N, prm.n_pad, rows_pad);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd rowdot launch");
  const unsigned grid = static_cast<unsigned>(static_cast<long long>(BH) * prm.n_tiles);
  const int slot = (D == 128 ? 4 : 0) + (CAUSAL ? 2 : 0);
  fa_status r = set_smem(bwd_dkdv_kernel<D, CAUSAL>, DkdvCfg<D>::kSmemBytes, slot);
  if (r != FA_OK) return r;
  bwd_dkdv_kernel<D, CAUSAL><<<grid, kThreads, DkdvCfg<D>::kSmemBytes, st>>>(mq, mk, mv, mdo, mdk, mdv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd dkdv launch");
  const long long rows = static_cast<long long>(BH) * N;
  bwd_dq_convert_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      prm.dq_acc, static_cast<__nv_bfloat16*>(dQ), prm.scale, N, prm.n_pad, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail(e, "bwd dq convert launch");
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

#ifdef FA_TRACE
// Trace builds only: device buffer of 2*16*4*64*8 uint64 (or NULL).
int fa_bwd_trace_set(void* device_buffer) {
  return cudaMemcpyToSymbol(fa::bwd::g_bwd_trace, &device_buffer, sizeof(device_buffer)) == cudaSuccess ? 0 : 1;
}
#endif

size_t fa_bwd_workspace_bytes(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  // LSE * log2(e) and D = rowsum(dO * O), fp32, each [B][H][N rounded up to
  // 128]; then the fp32 dQ accumulator [B][H][N rounded up][d], sized for
  // the largest head dimension (128)
  const size_t n_pad = (static_cast<size_t>(N) + fa::bwd::kTile - 1) / fa::bwd::kTile * fa::bwd::kTile;
  return (2 + 128) * static_cast<size_t>(B) * H * n_pad * 4;
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
  prm.N = N;
  prm.n_tiles = static_cast<int>(n_tiles);
  prm.n_pad = prm.n_tiles * bwd::kTile;
  prm.BH = static_cast<int>(BH);
  float* lse2 = static_cast<float*>(workspace);
  float* dd = lse2 + static_cast<size_t>(BH) * prm.n_pad;
  prm.lse2 = lse2;
  prm.dd = dd;
  prm.dq_acc = dd + static_cast<size_t>(BH) * prm.n_pad;  // 1024-byte aligned: n_pad is a multiple of 128
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
  if (d == 128)
    return causal ? bwd::launch_bwd<128, true>(Q, K, V, O, dO, LSE, dQ, dK, dV, lse2, dd, prm, st)
                  : bwd::launch_bwd<128, false>(Q, K, V, O, dO, LSE, dQ, dK, dV, lse2, dd, prm, st);
  return causal ? bwd::launch_bwd<64, true>(Q, K, V, O, dO, LSE, dQ, dK, dV, lse2, dd, prm, st)
                : bwd::launch_bwd<64, false>(Q, K, V, O, dO, LSE, dQ, dK, dV, lse2, dd, prm, st);
}

}  // extern "C"
