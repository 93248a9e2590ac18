// Fused exact softmax attention forward for B200 (sm_100a), and the C ABI
// declared in include/fa.h.
//
// What it computes: O = softmax(scale * Q K^T [+ causal mask]) V and the
// row log-sum-exp (lihaoran.work "FlashAttention: the intermediate matrix
// comes first", the opening formula).  How: the online block update of
// liminalml.com "FlashAttention" -- per query row a running maximum m,
// denominator l and unnormalised numerator u; a tile whose scores raise the
// maximum rescales u and l by e^(m - m') before its own terms are added
// (the 5 -> 10 question on the same page), and the output is u / l after the
// last tile.  Scores and probabilities live only in tensor memory; the N x N
// matrix never reaches HBM (sadullah.online "Flash Attention Explained",
// fused tiled computation; interactiveml.org "FlashAttention saves the
// matrix, not the quadratic work").
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0      TMA producer: Q tiles once, then K/V tiles through a ring of
//               shared-memory stages guarded by full/empty mbarriers.
//   warp 1      TMEM owner and MMA issuer (one thread): S_t = Q_t K^T
//               (SS MMA, M=128 N=128 K=d) and O_t += P_t V (TS MMA, P from
//               TMEM, M=128 N=d K=128), completion signalled by tcgen05.commit.
//   warps 2-3   idle.
//   warps 4-7   softmax + epilogue for query tile 0 (one thread per row).
//   warps 8-11  softmax + epilogue for query tile 1.
// Each CTA owns 2 query tiles of 128 rows (256 rows of one head) so that the
// softmax of one tile overlaps the MMAs of the other.
//
// Tensor memory (512 columns x 128 lanes of 32 bit):
//   [0,128)      S_0, fp32; P_0 (bf16 pairs) overwrites its first 64 columns
//   [128,256)    S_1 / P_1
//   [256,256+d)  O_0 accumulator, fp32
//   [256+d, 256+2d) O_1 accumulator
//
// Softmax runs in base 2 with log2(e) folded into the scale: x = s * scale *
// log2 e, p = 2^(x - m).  The reference maximum m is only raised when a tile
// exceeds it by more than 8 (a factor 256), so most tiles skip the O rescale;
// p <= 256 stays exact enough in bf16 and the final u / l uses the same m,
// so the result is unchanged.
//
// Every wait is bounded: a wait that runs out sets an abort flag in shared
// memory and a bit in the device status word; all roles then unwind, copies
// in flight are drained, and TMEM is released.  Nothing traps.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "fa.h"
#include "host_util.h"
#include "sm100.cuh"

namespace fa {
namespace bwd {
cudaError_t read_and_clear_status(uint32_t* v);  // fa_bwd.cu
}

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // keys per tile (default; 64 is built for the tile-size sweep)
constexpr int kQTiles = 2;     // query tiles per CTA
static_assert(FA_BLOCK_Q == kQTiles * kBM && FA_BLOCK_K == kBN,
              "a block-sparse block is one CTA's query rows by one key tile");
constexpr int kThreads = 384;  // 12 warps
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;
// wait sites reported in the device status word (bit 8 + site)
enum : uint32_t {
  kSiteKvEmpty = 0, kSiteQ = 1, kSiteKvFull = 2, kSiteS = 3, kSiteP = 4,  // 4..5: p_full[0..1]
  kSiteO = 8, kSiteDebug = 9,
};
constexpr int kChunkBytes = kBM * 64 * 2;  // one 64-wide, 128-row swizzled box: 16 KB

struct FwdParams {
  float* lse;           // [BH][N] or nullptr
  int N;                // sequence length
  int BH;               // batch * heads
  int group_heads;      // heads whose CTAs are scheduled together
  int n_qblk;           // ceil(N / 256)
  int n_kv;             // ceil(N / key tile)
  float scale_log2;     // scale * log2(e)
  uint64_t timeout_ns;  // bound on every wait
  uint32_t debug;       // bit 0: stall the softmax warps on a barrier nobody signals
  // split-KV only: the key tiles of a query block are divided into
  // num_splits ranges of kv_per_split tiles; each CTA writes the normalised
  // partial output and partial LSE of its range (fp32, row-major)
  int num_splits;
  int kv_per_split;
  float* o_part;    // [num_splits][BH][N][d]
  float* lse_part;  // [num_splits][BH][N]
  // block-sparse only: the key tiles each 256-row query block retains, as
  // CSR lists (strictly ascending within a block), shared by every head
  const int* blk_row_ptr;  // [n_qblk + 1]
  const int* blk_col_idx;  // [blk_nnz]
  int blk_nnz;
};

__device__ uint32_t g_device_status;

// Index checks of the debug build (compiled with -DFA_DEBUG): every shared
// memory, tensor memory and global index the kernels compute at run time is
// checked before the access it guards.  A failed check raises kStatusBounds
// and bit 16 + site in the device status word, the access is skipped, and the
// CTA unwinds as after a wait that gave up; nothing traps.  In the normal
// build the checks compile to nothing.
enum : uint32_t {
  kCheckQLoad = 0, kCheckKvLoad = 1, kCheckLse = 2, kCheckPartial = 3, kCheckStage = 4,
  kCheckStore = 5, kCheckMerge = 6, kCheckTmem = 7,
};
#ifdef FA_DEBUG
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t site) {
  if (!ok) atomicOr(&g_device_status, kStatusBounds | (1u << (16 + (site & 15u))));
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(bool, uint32_t) { return true; }
#endif

// Optional phase trace (build with -DFA_TRACE): SM clock stamps of the MMA
// issuer and of one thread per softmax warpgroup, for the first CTAs.
#ifdef FA_TRACE
constexpr int kTraceCtas = 16;
constexpr int kTraceIters = 64;
__device__ unsigned long long* g_trace;  // [kTraceCtas][4 roles][kTraceIters][8 events]
// The buffer's address is read once per thread at the start of the kernel
// (FA_TRACE_INIT): a stamp is then a clock read and a store, with no load in
// front of the clock that could delay it.
#define FA_TRACE_INIT() unsigned long long* const trace_buf = blockIdx.x < kTraceCtas ? g_trace : nullptr
#define FA_TRACE_MARK(role, iter, ev)                                                        \
  do {                                                                                       \
    if (trace_buf != nullptr && (iter) < kTraceIters) {                                      \
      const unsigned long long now = clock64();                                              \
      trace_buf[((static_cast<size_t>(blockIdx.x) * 4 + (role)) * kTraceIters + (iter)) * 8 + \
                (ev)] = now;                                                                 \
    }                                                                                        \
  } while (0)
#else
#define FA_TRACE_INIT() \
  do {                  \
  } while (0)
#define FA_TRACE_MARK(role, iter, ev) \
  do {                                \
  } while (0)
#endif

template <int D, int BN = kBN>
struct Cfg {
  static_assert(BN == 128 || BN == 64, "key tiles of 128 or 64");
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = kBM * D * 2;  // one query tile (reused as O staging)
  static constexpr int kStageBytes = BN * D * 2;  // one ring stage: a whole K or V tile
  static constexpr int kKChunkBytes = BN * 128;   // one 64-wide d chunk of a K stage
  static constexpr int kVChunkBytes = BN * 128;   // one 64-wide d chunk of a V stage
  // the same ring bytes whatever the tile: more stages for smaller tiles
  static constexpr int kStages = (D == 64 ? 8 : 4) * (128 / BN);
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 1 + 1;
  static constexpr int kSmemTiles = kQTiles * kQBytes + kStages * kStageBytes;
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + 1024;
  static constexpr uint32_t kColO = 256;
};

// One CTA owns two 128-row query tiles of one head and issues M=128 MMAs.
template <int D, bool CAUSAL, bool SPLIT, bool SPARSE, int BN, int QT>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = Cfg<D, BN>;
  constexpr int S = C::kStages;
  constexpr int QB = C::kQBytes;
  static_assert(BN == 128 || !(SPLIT || SPARSE), "split-KV and block-sparse use 128-key tiles");
  // QT = query tiles per CTA: 2 (the two tiles ping-pong), or 1 for the
  // tile-size sweep (tile slot 0 stays empty, slot 1 holds the CTA's rows)
  static_assert(QT == 2 || (QT == 1 && !SPLIT && !SPARSE), "one query tile per CTA: plain forward only");
  constexpr int SB = C::kStageBytes;
  static_assert(!(SPARSE && SPLIT), "block-sparse uses the unsplit shape");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                  // kQTiles query tiles (reused as O staging)
  uint8_t* sKV = smem + kQTiles * QB;  // S ring stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* q_full = bars;            // [2] Q tile landed
  uint64_t* kv_full = q_full + 2;     // [S] K/V stage landed
  uint64_t* kv_empty = kv_full + S;   // [S] MMA -> producer
  uint64_t* s_full = kv_empty + S;    // [2] MMA -> softmax
  uint64_t* p_full = s_full + 2;      // [2] softmax -> MMA
  uint64_t* o_full = p_full + 2;      // [2] MMA -> epilogue
  uint64_t* mma_done = o_full + 2;    // [1] MMA -> itself, before TMEM release
  uint64_t* never = mma_done + 1;     // [1] debug: nothing arrives here
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* status = &g_device_status;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FA_TRACE_INIT();
  const int split = SPLIT ? static_cast<int>(blockIdx.x % p.num_splits) : 0;
  const int unit = SPLIT ? static_cast<int>(blockIdx.x / p.num_splits) : static_cast<int>(blockIdx.x);
  // Work order: heads in groups of p.group_heads; inside a group, query
  // blocks from the heaviest (last rows: most keys when causal) to the
  // lightest, cycling over the group's heads.  Blocks that run together then
  // share the K/V of a few heads in L2, and light blocks end the grid.
  const int per_group = p.group_heads * p.n_qblk;
  const int grp = unit / per_group;
  const int rem = unit % per_group;
  const int grp_heads = min(p.group_heads, p.BH - grp * p.group_heads);
  const int bh = grp * p.group_heads + rem % grp_heads;
  const int qblk = p.n_qblk - 1 - rem / grp_heads;
  const int q0 = qblk * QT * kBM - (2 - QT) * kBM;  // first row of slot 0
  // last key tile each query tile needs (the causal diagonal, or the end)
  int j_last[2];
#pragma unroll
  for (int t = 0; t < 2; ++t)
    j_last[t] = CAUSAL ? min(q0 + (t + 1) * kBM - 1, p.N - 1) / BN : p.n_kv - 1;
  // key tiles [kv_lo, kv_end) of this CTA (all of them unless split), visited
  // from kv_end-1 down to kv_lo
  const int kv_lo = SPLIT ? split * p.kv_per_split : 0;
  const int kv_end = SPLIT ? min(j_last[1] + 1, kv_lo + p.kv_per_split) : j_last[1] + 1;
  int n_iter = max(0, kv_end - kv_lo);
  // iterations before a query tile's first unmasked key tile are skipped for
  // it; a tile whose first iteration is past n_iter has no keys in this range
  int first_it[2] = {kv_end - 1 - min(j_last[0], kv_end - 1), 0};
  // Block-sparse: this block's retained key tiles, visited from the last
  // entry down.  Entries past tile 1's diagonal are seen by no row and are
  // dropped; leading visits past tile 0's diagonal are skipped for tile 0.
  // A malformed list raises kStatusLayout; out-of-range or out-of-order
  // entries are then masked out entirely (no memory outside the tensors is
  // touched), and the outputs are not meaningful.
  const int* blk = nullptr;
  if (SPARSE) {
    int beg = __ldg(p.blk_row_ptr + qblk), end = __ldg(p.blk_row_ptr + qblk + 1);
    if (!(0 <= beg && beg <= end && end <= p.blk_nnz)) {
      if (threadIdx.x == 0) atomicOr(&g_device_status, kStatusLayout);
      beg = end = 0;
    }
    blk = p.blk_col_idx + beg;
    int n = end - beg;
    while (n > 0 && __ldg(blk + n - 1) > j_last[1]) {
      if (threadIdx.x == 0 && __ldg(blk + n - 1) >= p.n_kv) atomicOr(&g_device_status, kStatusLayout);
      --n;
    }
    int skip = 0;
    while (skip < n && __ldg(blk + n - 1 - skip) > j_last[0]) ++skip;
    n_iter = n;
    first_it[0] = skip;
  }
  if (QT == 1) first_it[0] = n_iter;  // slot 0 unused
  const bool tile_active[2] = {first_it[0] < n_iter, n_iter > 0};
  // key tile of iteration it
  auto kv_tile = [&](int it) { return SPARSE ? __ldg(blk + n_iter - 1 - it) : kv_end - 1 - it; };
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], kBM);
      mbar_init(&o_full[t], 1);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  static_assert(2 * BN <= C::kColO && C::kColO + 2 * D <= kTmemCols, "S_0, S_1, O_0, O_1 fit the allocation");
  // (all 512 columns are allocated, so the base column is 0)
  if (threadIdx.x == 0) in_bounds((tmem & 0xffffu) == 0, kCheckTmem);

  // rows of this CTA's query tile t
  auto tile_row0 = [&](int t) { return q0 + t * kBM; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_iter > 0) {
      bool ok = true;
      bool q_issued[2] = {false, false};
      if (tile_active[0]) {
        if (in_bounds(tile_row0(0) >= 0 && tile_row0(0) < p.n_qblk * QT * kBM && bh < p.BH, kCheckQLoad)) {
          q_issued[0] = true;
          mbar_arrive_expect_tx(&q_full[0], QB);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sQ + c * kChunkBytes, &tmQ, &q_full[0], c * 64, tile_row0(0), bh);
        } else {
          ok = false;
          *abort_flag = 1;
        }
      }
      int i = 0;  // loads issued into the ring, in consumption order K0 V0 K1 V1 ...
      for (int it = 0; it < n_iter && ok; ++it) {
        // (a block-sparse entry out of range is loaded clamped and masked)
        const int j = SPARSE ? min(max(kv_tile(it), 0), p.n_kv - 1) : kv_tile(it);
        for (int kv = 0; kv < 2; ++kv) {
          const int s = i % S;
          const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
          ok = mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, status, tmo, kSiteKvEmpty);
          if (!ok) break;
          if (!in_bounds(j >= 0 && j < p.n_kv && s < S && bh < p.BH, kCheckKvLoad)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], SB);
          uint8_t* st = sKV + s * SB;
          const CUtensorMap* map = kv == 0 ? &tmK : &tmV;
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(st + c * C::kKChunkBytes, map, &kv_full[s], c * 64, j * BN, bh);
          ++i;
          if (it == 0 && kv == 0) {
            if (!in_bounds(tile_row0(1) >= 0 && tile_row0(1) < p.n_qblk * QT * kBM, kCheckQLoad)) {
              ok = false;
              *abort_flag = 1;
              break;
            }
            q_issued[1] = true;
            mbar_arrive_expect_tx(&q_full[1], QB);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sQ + QB + c * kChunkBytes, &tmQ, &q_full[1], c * 64, tile_row0(1), bh);
          }
        }
      }
      if (!ok) {
        // Unwinding: wait for every copy this CTA issued, so that none lands
        // in shared memory after the CTA has ended.
        for (int s = 0; s < S && s < i; ++s) {
          const int last = s + ((i - 1 - s) / S) * S;
          mbar_wait_drain(&kv_full[s], static_cast<uint32_t>(last / S) & 1u, tmo);
        }
        for (int t = 0; t < 2; ++t)
          if (q_issued[t]) mbar_wait_drain(&q_full[t], 0, tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, BN, false);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, true);
      const uint32_t sq = smem_addr(sQ);
      const uint32_t skv = smem_addr(sKV);
      // The issuing thread is on the critical path between the softmax and
      // the next S (an MMA is accepted only about as fast as the tensor core
      // retires the one before), so at d = 128 each operand's descriptor is
      // built once per product and advanced by a constant per K-step (the
      // start-address field counts 16-byte units and shared-memory addresses
      // stay below 2^18, so adding the offset never carries out of it).
      // Measured on B200: +2.6% at d = 128, -1.5% at d = 64 (kept off there).
      constexpr bool kAdvanceDesc = D == 128;
      // S_t = Q_t K^T: A = Q_t (K-major), B = K stage (K-major); 16 columns of
      // d per instruction, 32 bytes apart inside each 128-byte swizzled row.
      auto issue_s = [&](int t, int s) {
        const uint64_t a0 = sw128_desc(sq + t * QB, 16, 1024);
        const uint64_t b0 = sw128_desc(skv + s * SB, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * C::kKChunkBytes + (kk & 3) * 32;
          const uint64_t ad = kAdvanceDesc ? a0 + (aoff >> 4) : sw128_desc(sq + t * QB + aoff, 16, 1024);
          const uint64_t bd = kAdvanceDesc ? b0 + (boff >> 4) : sw128_desc(skv + s * SB + boff, 16, 1024);
          mma_ss(tmem + t * BN, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V: A = P_t in TMEM (8 columns per 16 keys), B = V stage
      // stored d-contiguous (MN-major): 16 keys = 2 KB apart, d halves 16 KB apart.
      auto issue_pv = [&](int t, int s, bool accumulate) {
        const uint64_t v0 = sw128_desc(skv + s * SB, C::kVChunkBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = kAdvanceDesc ? v0 + static_cast<uint32_t>(kk * (2048 >> 4))
                                           : sw128_desc(skv + s * SB + kk * 2048, C::kVChunkBytes, 1024);
          const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::kColO + t * D, tmem + t * BN + kk * 8, bd, idO, acc);
        }
      };
      auto commit = [&](uint64_t* bar) { mma_commit(bar); };
      bool ok = mbar_wait(&kv_full[0], 0, abort_flag, status, tmo, kSiteKvFull);
      bool q_ready[2] = {false, false};
      for (int t = 0; t < 2 && ok; ++t) {
        if (first_it[t] != 0) continue;
        ok = mbar_wait(&q_full[t], 0, abort_flag, status, tmo, kSiteQ);
        if (!ok) break;
        q_ready[t] = true;
        tc_fence_after();
        issue_s(t, 0);
        commit(&s_full[t]);
      }
      if (ok) commit(&kv_empty[0]);
      for (int it = 0; it < n_iter && ok; ++it) {
        const int iv = 2 * it + 1, ik = 2 * it + 2;
        const int sv = iv % S, sk = ik % S;
        const bool last = it == n_iter - 1;
        if (!(ok = mbar_wait(&kv_full[sv], static_cast<uint32_t>(iv / S) & 1u, abort_flag, status, tmo, kSiteKvFull))) break;
        FA_TRACE_MARK(3, it, 0);
        // the next K tile too, here rather than between a PV and an S
        // product: it has normally landed long before, but the wait itself
        // costs the issuing thread time that the tensor core then idles
        if (!last && !(ok = mbar_wait(&kv_full[sk], static_cast<uint32_t>(ik / S) & 1u, abort_flag, status, tmo,
                                      kSiteKvFull)))
          break;
        FA_TRACE_MARK(3, it, 1);
        for (int t = 0; t < 2; ++t) {
          if (it >= first_it[t]) {
            const uint32_t ph = static_cast<uint32_t>(it - first_it[t]) & 1u;
            const bool acc = it > first_it[t];
            if (!(ok = mbar_wait(&p_full[t], ph, abort_flag, status, tmo, kSiteP + t))) break;
            FA_TRACE_MARK(0, it, 3 * t);
            tc_fence_after();
            issue_pv(t, sv, acc);
            FA_TRACE_MARK(0, it, 3 * t + 1);
            if (last) commit(&o_full[t]);
          }
          if (!last && it + 1 >= first_it[t]) {
            if (!q_ready[t]) {
              if (!(ok = mbar_wait(&q_full[t], 0, abort_flag, status, tmo, kSiteQ))) break;
              q_ready[t] = true;
            }
            tc_fence_after();
            issue_s(t, sk);
            commit(&s_full[t]);
            FA_TRACE_MARK(0, it, 3 * t + 2);
          }
        }
        if (!ok) break;
        commit(&kv_empty[sv]);
        if (!last) commit(&kv_empty[sk]);
      }
      // every MMA issued here has finished before TMEM is released
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, tmo);
    }
  } else if (warp >= kSoftmaxWarp0 && (QT == 2 || warp >= kSoftmaxWarp0 + 4)) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - kSoftmaxWarp0) >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;                    // TMEM lane quarter
    const int r = wq * 32 + lane;               // row inside the tile
    const int row0 = tile_row0(t);
    const int row = row0 + r;                   // query index in the head
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * BN;
    const uint32_t tO = tmem + lane_base + C::kColO + t * D;
    const float sl2 = p.scale_log2;
    // last key this row may see
    const int key_limit = CAUSAL ? min(row, p.N - 1) : p.N - 1;
    // O_t holds the product through the previous tile (that MMA finished
    // before S_t of this tile was committed): rescale this thread's row of
    // it in place, before P of this tile releases the next PV product.
    auto rescale_o_rows = [&](uint32_t taddr, float a) {
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t o[16];
        tmem_ld16(taddr + c * 16, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
        tmem_st16(taddr + c * 16, o);
      }
    };

    float m_ref = -INFINITY;  // reference maximum, log2 units of scaled scores
    float l_sum = 0.f;        // running denominator relative to m_ref
    bool ok = true;
    if (p.debug & 1u) {
      ok = __all_sync(0xffffffffu, mbar_wait(never, 0, abort_flag, status, tmo, kSiteDebug));
    }
    for (int it = first_it[t]; it < n_iter && ok; ++it) {
      const int li = it - first_it[t];
      int j = kv_tile(it);
      // a block-sparse entry out of range or out of order contributes nothing
      bool bad = false;
      if (SPARSE) {
        bad = j < 0 || j >= p.n_kv || (it > 0 && j >= kv_tile(it - 1));
        if (bad) {
          if ((threadIdx.x & 127) == 0) atomicOr(&g_device_status, kStatusLayout);
          j = 0;
        }
      }
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&s_full[t], static_cast<uint32_t>(li) & 1u, abort_flag, status, tmo, kSiteS));
      if (!ok) break;
      const bool tr = lane == 0 && (warp & 3) == 0;
      if (tr) FA_TRACE_MARK(1 + t, it, 0);
      tc_fence_after();
      constexpr int kQ32 = BN / 32;  // 32-key groups of a tile
      uint32_t sr[kQ32][32];
#pragma unroll
      for (int q = 0; q < kQ32; ++q) tmem_ld32(tS + q * 32, sr[q]);
      tmem_wait_ld();
      if (tr) FA_TRACE_MARK(1 + t, it, 1);

      const int kbase = j * BN;
      const bool masked = bad || (kbase + BN > p.N) || (CAUSAL && kbase + BN - 1 > row0);
      if (masked) {
        const int lim = bad ? -1 : key_limit;
#pragma unroll
        for (int q = 0; q < kQ32; ++q)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (kbase + q * 32 + c > lim) sr[q][c] = __float_as_uint(-INFINITY);
      }
      // row maximum of the raw scores (scale > 0 keeps the argmax): BN/16
      // independent chains of three-input maxima
      constexpr int kChains = BN / 16;
      float mx[kChains];
#pragma unroll
      for (int k = 0; k < kChains; ++k) mx[k] = __uint_as_float(sr[k >> 1][(k & 1) * 16]);
#pragma unroll
      for (int k = 0; k < kChains; ++k) {
        const uint32_t* v = &sr[k >> 1][(k & 1) * 16];
#pragma unroll
        for (int c = 1; c < 15; c += 2)
          mx[k] = fmax3(mx[k], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
        mx[k] = fmaxf(mx[k], __uint_as_float(v[15]));
      }
      float m_all;
      if constexpr (kChains == 8)
        m_all = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      else
        m_all = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]);
      const float m_tile = m_all * sl2;
      if (tr) FA_TRACE_MARK(1 + t, it, 2);
      // raise the reference maximum only when this tile exceeds it by > 2^8
      const bool raise = m_tile > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (raise) {
        alpha = ex2_approx(m_ref - m_tile);  // 0 while m_ref is -inf
        m_ref = m_tile;
      }
      const bool rescale_o = li > 0 && __any_sync(0xffffffffu, raise);
      const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const float2 sl2v = make_float2(sl2, sl2);
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 ps2[kQ32];
      // p = 2^(s * scale * log2 e - m), written as bf16 pairs over the first
      // BN/2 columns of S_t, 64 keys at a time, and published whole on
      // p_full[t].
#pragma unroll
      for (int h = 0; h < BN / 64; ++h) {
        // keys [64h, 64h + 64) -> 32 columns of bf16 pairs at column 32h
        uint32_t pk[32];
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int q = 2 * h + qq;
          ps2[q] = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(sr[q][c]), __uint_as_float(sr[q][c + 1])),
                                   sl2v, nm2);
            float2 pv;
            pv.x = ex2_approx(x.x);
            pv.y = ex2_approx(x.y);
            ps2[q] = fadd2(ps2[q], pv);
            pk[qq * 16 + (c >> 1)] = pack_bf16x2(pv.x, pv.y);
          }
        }
        tmem_st32(tS + h * 32, pk);
        if (tr && h == 0) FA_TRACE_MARK(1 + t, it, 3);
      }
      // the rescale waits until the scores have left the registers
      if (rescale_o) rescale_o_rows(tO, alpha);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      float2 psum;
      if constexpr (kQ32 == 4)
        psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
      else
        psum = fadd2(ps2[0], ps2[1]);
      l_sum = l_sum * alpha + (psum.x + psum.y);
      if (tr) FA_TRACE_MARK(1 + t, it, 4);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && tile_active[t]) ok = mbar_wait(&o_full[t], 0, abort_flag, status, tmo, kSiteO);
    const bool failed = named_bar_or(1 + t, kBM, !ok);
    if (!failed && SPLIT) {
      // partial state of this key range: u / l (fp32) and its LSE; a range
      // with no allowed key for this row gives LSE = -inf and weight 0 in
      // the merge
      tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const float lse_val = l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.69314718055994530942f : -INFINITY;
      const size_t prow = (static_cast<size_t>(split) * p.BH + bh) * p.N + row;
      float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
      const bool row_ok =
          row < p.N &&
          in_bounds(split < p.num_splits && bh < p.BH && prow < static_cast<size_t>(p.num_splits) * p.BH * p.N,
                    kCheckPartial);
      if (row_ok) p.lse_part[prow] = lse_val;
      if (tile_active[t]) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int g = 0; g < 8; ++g)
              dst[c * 8 + g] = make_float4(__uint_as_float(o[4 * g]) * inv_l, __uint_as_float(o[4 * g + 1]) * inv_l,
                                           __uint_as_float(o[4 * g + 2]) * inv_l, __uint_as_float(o[4 * g + 3]) * inv_l);
          }
        }
      } else if (row_ok) {
#pragma unroll
        for (int g = 0; g < D / 4; ++g) dst[g] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    } else if (!failed) {
      tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      if (p.lse != nullptr && row < p.N && in_bounds(bh < p.BH && row >= 0, kCheckLse)) {
        const float lse2 = l_sum > 0.f ? m_ref + log2f(l_sum) : -INFINITY;
        p.lse[static_cast<size_t>(bh) * p.N + row] = lse2 * 0.69314718055994530942f;
      }
      // O_t / l -> bf16 -> the Q_t buffer (no MMA reads it any more), laid
      // out as the 128-byte-swizzled boxes the store tensor map expects.
      uint8_t* stage = sQ + t * QB;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (tile_active[t]) {
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
        } else {  // no retained key (block-sparse): O = 0
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        uint8_t* rowp = stage + (c >> 1) * kChunkBytes + r * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * g + 0]) * inv_l, __uint_as_float(o[8 * g + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * g + 2]) * inv_l, __uint_as_float(o[8 * g + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * g + 4]) * inv_l, __uint_as_float(o[8 * g + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * g + 6]) * inv_l, __uint_as_float(o[8 * g + 7]) * inv_l);
          const int gran = ((c & 1) * 4 + g) ^ (r & 7);
          if (in_bounds(rowp + gran * 16 >= stage && rowp + gran * 16 + 16 <= stage + QB, kCheckStage))
            *reinterpret_cast<uint4*>(rowp + gran * 16) = v;
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + t, kBM);
      if (r == 0 && row0 < p.N) {
        for (int c = 0; c < C::kChunks; ++c)
          if (in_bounds(row0 >= 0 && bh < p.BH, kCheckStore))
            tma_store_3d(&tmO, stage + c * kChunkBytes, c * 64, row0, bh);
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

// Merge of the split-KV partial states of every row: with M = max_s LSE_s
// and w_s = e^(LSE_s - M) (0 for an empty range), O = sum_s w_s O_s / sum_s
// w_s and LSE = M + ln sum_s w_s -- the block update applied to whole states
// (liminalml.com "FlashAttention", m' = max(m, max s) and the rescale of
// both numerator and denominator; interactiveml.org, the merge with the
// guard for m = -inf).  One warp per row; each lane owns d/32 columns.
template <int D>
__global__ void __launch_bounds__(256)
    fa_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                    __nv_bfloat16* __restrict__ O, float* __restrict__ LSE, long long rows,
                    int num_splits) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = 0; s < num_splits; ++s) m = fmaxf(m, lse_part[s * rows + row]);
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < num_splits; ++s) {
    if (!in_bounds(s * rows + row < num_splits * rows, kCheckMerge)) break;
    const float l = lse_part[s * rows + row];
    const float w = (l == -INFINITY) ? 0.f : ex2_approx((l - m) * 1.4426950408889634f);
    wsum += w;
    const float* src = o_part + (s * rows + row) * D + lane * kPer;
    if (kPer == 4) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
      acc[2] += w * v.z;
      acc[3] += w * v.w;
    } else {
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += w * src[i];
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = O + row * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; i += 2) {
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  }
  if (LSE != nullptr && lane == 0) LSE[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace host {
thread_local char g_last_error[256] = "";
unsigned int g_debug_flags = 0;
unsigned long long g_timeout_ns = 0;
}  // namespace host

namespace {

using host::cuda_fail;
using host::g_debug_flags;
using host::g_last_error;
using host::g_timeout_ns;
using host::kDefaultTimeoutNs;
using host::make_map_cached;
using host::overlaps;

// Per-device facts found on first use.  No lock is held while launching: the
// attribute call is idempotent, so two threads that both find it unset both
// make it, harmlessly.
struct DeviceInfo {
  std::atomic<int> sm100{0};  // 0 unknown, 1 yes, -1 no
  std::atomic<bool> attr_set[128] = {};
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];

template <int D, bool CAUSAL, bool SPLIT, bool SPARSE = false, int BN = kBN, int QT = kQTiles>
fa_status launch(const void* Q, const void* K, const void* V, void* O, FwdParams prm, int N, int BH,
                 cudaStream_t stream, DeviceInfo& dev) {
  using C = Cfg<D, BN>;
  prm.n_kv = (N + BN - 1) / BN;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_cached(&mq, Q, D, N, BH, kBM) || !make_map_cached(&mk, K, D, N, BH, BN) ||
      !make_map_cached(&mv, V, D, N, BH, BN) || !make_map_cached(&mo, O, D, N, BH, kBM)) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed");
    return FA_ERR_CUDA;
  }
  const long long rows_per_block = static_cast<long long>(QT) * kBM;
  prm.n_qblk = static_cast<int>((N + rows_per_block - 1) / rows_per_block);
  const long long units = static_cast<long long>(BH) * prm.n_qblk;
  const long long grid = units * (SPLIT ? prm.num_splits : 1);
  if (grid > 0x7fffffffll) return FA_ERR_SHAPE;
  constexpr int slot = (QT == 1 ? 64 : 0) + (BN == 64 ? 32 : 0) + (SPARSE ? 16 : 0) + (D == 128 ? 8 : 0) +
                       (CAUSAL ? 4 : 0) + (SPLIT ? 1 : 0);
  auto kern = fa_fwd_kernel<D, CAUSAL, SPLIT, SPARSE, BN, QT>;
  if (!dev.attr_set[slot].load(std::memory_order_acquire)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    dev.attr_set[slot].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, prm);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return FA_OK;
}

template <int D>
fa_status launch_merge(const float* o_part, const float* lse_part, void* O, float* LSE, long long rows,
                       int num_splits, cudaStream_t stream) {
  constexpr int kWarps = 8;
  const long long blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffll) return FA_ERR_SHAPE;
  fa_merge_kernel<D><<<static_cast<unsigned>(blocks), kWarps * 32, 0, stream>>>(
      o_part, lse_part, static_cast<__nv_bfloat16*>(O), LSE, rows, num_splits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" {

const char* fa_version(void) { return "0.1.0"; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
    case FA_ERR_SHAPE: return "FA_ERR_SHAPE: bad B/H/N, size overflow or non-finite scale";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: d must be 64 or 128, scale > 0, sm_100 GPU";
    case FA_ERR_ALIGN: return "FA_ERR_ALIGN: Q/K/V/O need 16-byte, LSE 4-byte alignment";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call or kernel launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    case FA_ERR_ALIAS: return "FA_ERR_ALIAS: O, LSE or the workspace overlaps an input or each other";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: the workspace is smaller than required";
    case FA_ERR_LAYOUT: return "FA_ERR_LAYOUT: a block-sparse list was out of range or out of order";
    case FA_ERR_BOUNDS: return "FA_ERR_BOUNDS: an index check of the debug build failed";
  }
  return "unknown fa_status";
}

const char* fa_last_cuda_error(void) { return fa::g_last_error; }

#ifdef FA_TRACE
// Trace builds only: device buffer of kTraceCtas*4*kTraceIters*8 uint64 (or NULL).
int fa_trace_set(void* device_buffer) {
  return cudaMemcpyToSymbol(fa::g_trace, &device_buffer, sizeof(device_buffer)) == cudaSuccess ? 0 : 1;
}
#endif

void fa_set_debug(unsigned int flags, unsigned long long timeout_ns) {
  fa::g_debug_flags = flags;
  fa::g_timeout_ns = timeout_ns;
}

}  // extern "C"

namespace fa {
namespace {

// Argument checks shared by the forward entry points (host only).
fa_status check_args(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                     int B, int H, int N, int d, float scale) {
  if (!Q || !K || !V || !O) return FA_ERR_NULL;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  if (!std::isfinite(scale)) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  const long long n_qblk = (static_cast<long long>(N) + kBM - 1) / kBM;  // 128-row query tiles (any kernel shape)
  if (BH > (1ll << 30) || BH * n_qblk > 0x7fffffffll) return FA_ERR_SHAPE;
  auto mis16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (mis16(Q) || mis16(K) || mis16(V) || mis16(O)) return FA_ERR_ALIGN;
  if (LSE && (reinterpret_cast<uintptr_t>(LSE) & 3u) != 0) return FA_ERR_ALIGN;
  const size_t nbytes = static_cast<size_t>(BH) * N * d * 2;
  const size_t lbytes = static_cast<size_t>(BH) * N * 4;
  if (overlaps(O, nbytes, Q, nbytes) || overlaps(O, nbytes, K, nbytes) ||
      overlaps(O, nbytes, V, nbytes))
    return FA_ERR_ALIAS;
  if (LSE && (overlaps(LSE, lbytes, Q, nbytes) || overlaps(LSE, lbytes, K, nbytes) ||
              overlaps(LSE, lbytes, V, nbytes) || overlaps(LSE, lbytes, O, nbytes)))
    return FA_ERR_ALIAS;
  return FA_OK;
}

// After check_args: the current device must be an sm_100 GPU; fills *prm
// (all but n_qblk and the split fields) and *dev.
fa_status prepare(const float* LSE, int B, int H, int N, int d, float scale, FwdParams* prm,
                  DeviceInfo** dev) {
  const long long BH = static_cast<long long>(B) * H;
  int dev_id = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev_id < 0 || dev_id >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  *dev = &g_devices[dev_id];
  if ((*dev)->sm100.load(std::memory_order_acquire) == 0) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev_id);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    (*dev)->sm100.store(major == 10 ? 1 : -1, std::memory_order_release);
  }
  if ((*dev)->sm100.load(std::memory_order_acquire) != 1) return FA_ERR_UNSUPPORTED;

  *prm = FwdParams{};
  prm->lse = const_cast<float*>(LSE);
  prm->N = N;
  prm->n_qblk = 0;  // set per kernel shape in launch()
  prm->n_kv = (N + kBN - 1) / kBN;
  prm->BH = static_cast<int>(BH);
  {
    // keep the K/V of one group of heads (4*N*d bytes per head) within ~48 MB of L2
    const long long per_head = 4ll * N * d;
    long long g = (48ll << 20) / per_head;
    prm->group_heads = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
  }
  prm->scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  prm->timeout_ns = g_timeout_ns ? g_timeout_ns : kDefaultTimeoutNs;
  prm->debug = g_debug_flags;
  prm->num_splits = 1;
  return FA_OK;
}

constexpr int kMaxSplits = 256;

long long splitkv_rows(int B, int H, int N) { return static_cast<long long>(B) * H * N; }

size_t splitkv_bytes(int B, int H, int N, int d, int num_splits) {
  const long long rows = splitkv_rows(B, H, N);
  return static_cast<size_t>(num_splits) * static_cast<size_t>(rows) * (static_cast<size_t>(d) + 1) * 4;
}

int default_splits(int B, int H, int N, bool causal) {
  const long long units = static_cast<long long>(B) * H * ((N + kQTiles * kBM - 1) / (kQTiles * kBM));
  const int n_kv = (N + kBN - 1) / kBN;
  // non-causal: as many ranges as fit in one wave of 148 SMs without starting
  // a second; causal (uneven ranges): at least one and a half waves; at least
  // two key tiles per range.  Chosen from measurements on B200.
  long long s = causal ? (222 + units - 1) / units : 148 / units;
  const long long cap = n_kv / 2 > 1 ? n_kv / 2 : 1;
  if (s > cap) s = cap;
  if (s > kMaxSplits) s = kMaxSplits;
  return static_cast<int>(s < 1 ? 1 : s);
}

// The range count a split-KV call really runs: num_splits <= 0 picks the
// default; ranges are ceil(n_kv / num_splits) key tiles each, and trailing
// empty ranges are dropped.  0 when num_splits exceeds kMaxSplits.
int effective_splits(int B, int H, int N, bool causal, int num_splits) {
  if (num_splits <= 0) num_splits = default_splits(B, H, N, causal);
  if (num_splits > kMaxSplits) return 0;
  const int n_kv = (N + kBN - 1) / kBN;
  const int kv_per_split = (n_kv + num_splits - 1) / num_splits;
  return (n_kv + kv_per_split - 1) / kv_per_split;
}

// Workspace bytes of a split-KV call that runs `splits` ranges: none for a
// single range (the fused kernel writes O and LSE directly).
size_t splitkv_need(int B, int H, int N, int d, int splits) {
  return splits > 1 ? splitkv_bytes(B, H, N, d, splits) : 0;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
                 int N, int d, float scale, int causal, void* stream) {
  using namespace fa;
  FwdParams prm;
  DeviceInfo* dev = nullptr;
  fa_status st0 = check_args(Q, K, V, O, LSE, B, H, N, d, scale);
  if (st0 == FA_OK) st0 = prepare(LSE, B, H, N, d, scale, &prm, &dev);
  if (st0 != FA_OK) return st0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bh = prm.BH;
  if (d == 128)
    return causal ? launch<128, true, false>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<128, false, false>(Q, K, V, O, prm, N, bh, st, *dev);
  return causal ? launch<64, true, false>(Q, K, V, O, prm, N, bh, st, *dev)
                : launch<64, false, false>(Q, K, V, O, prm, N, bh, st, *dev);
}

fa_status fa_fwd_tile_config(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                             int H, int N, int d, float scale, int causal, int query_rows, int key_tile,
                             void* stream) {
  using namespace fa;
  if (query_rows == 0) query_rows = kQTiles * kBM;
  if (key_tile == 0) key_tile = kBN;
  if (query_rows == kQTiles * kBM && key_tile == kBN)
    return fa_fwd(Q, K, V, O, LSE, B, H, N, d, scale, causal, stream);
  FwdParams prm;
  DeviceInfo* dev = nullptr;
  fa_status st0 = check_args(Q, K, V, O, LSE, B, H, N, d, scale);
  if (st0 != FA_OK) return st0;
  if ((query_rows != 128 && query_rows != 256) || (key_tile != 64 && key_tile != 128)) return FA_ERR_UNSUPPORTED;
  st0 = prepare(LSE, B, H, N, d, scale, &prm, &dev);
  if (st0 != FA_OK) return st0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bh = prm.BH;
  // (query rows, key tile) in {(256, 64), (128, 128), (128, 64)}; (256, 128) is fa_fwd
  if (query_rows == 256) {
    if (d == 128)
      return causal ? launch<128, true, false, false, 64, 2>(Q, K, V, O, prm, N, bh, st, *dev)
                    : launch<128, false, false, false, 64, 2>(Q, K, V, O, prm, N, bh, st, *dev);
    return causal ? launch<64, true, false, false, 64, 2>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<64, false, false, false, 64, 2>(Q, K, V, O, prm, N, bh, st, *dev);
  }
  if (key_tile == 128) {
    if (d == 128)
      return causal ? launch<128, true, false, false, 128, 1>(Q, K, V, O, prm, N, bh, st, *dev)
                    : launch<128, false, false, false, 128, 1>(Q, K, V, O, prm, N, bh, st, *dev);
    return causal ? launch<64, true, false, false, 128, 1>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<64, false, false, false, 128, 1>(Q, K, V, O, prm, N, bh, st, *dev);
  }
  if (d == 128)
    return causal ? launch<128, true, false, false, 64, 1>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<128, false, false, false, 64, 1>(Q, K, V, O, prm, N, bh, st, *dev);
  return causal ? launch<64, true, false, false, 64, 1>(Q, K, V, O, prm, N, bh, st, *dev)
                : launch<64, false, false, false, 64, 1>(Q, K, V, O, prm, N, bh, st, *dev);
}

int fa_fwd_splitkv_default_splits(int B, int H, int N, int d, int causal) {
  (void)d;
  if (B < 1 || H < 1 || N < 1) return 1;
  return fa::default_splits(B, H, N, causal != 0);
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int causal, int num_splits) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  const int splits = fa::effective_splits(B, H, N, causal != 0, num_splits);
  return splits == 0 ? 0 : fa::splitkv_need(B, H, N, d, splits);
}

fa_status fa_fwd_splitkv(const void* Q, const void* K, const void* V, void* O, float* LSE,
                         void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                         float scale, int causal, int num_splits, void* stream) {
  using namespace fa;
  FwdParams prm;
  DeviceInfo* dev = nullptr;
  fa_status st0 = check_args(Q, K, V, O, LSE, B, H, N, d, scale);
  if (st0 != FA_OK) return st0;
  // equal ranges of key tiles; trailing empty ranges are dropped
  num_splits = effective_splits(B, H, N, causal != 0, num_splits);
  if (num_splits == 0) return FA_ERR_UNSUPPORTED;
  const int n_kv = (N + kBN - 1) / kBN;
  const int kv_per_split = (n_kv + num_splits - 1) / num_splits;
  const size_t need = splitkv_need(B, H, N, d, num_splits);
  if (need > 0) {
    if (workspace == nullptr) return FA_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return FA_ERR_ALIGN;
    if (workspace_bytes < need) return FA_ERR_WORKSPACE;
    const size_t nbytes = static_cast<size_t>(B) * H * N * d * 2;
    if (overlaps(workspace, need, Q, nbytes) || overlaps(workspace, need, K, nbytes) ||
        overlaps(workspace, need, V, nbytes) || overlaps(workspace, need, O, nbytes) ||
        (LSE && overlaps(workspace, need, LSE, static_cast<size_t>(B) * H * N * 4)))
      return FA_ERR_ALIAS;
  }
  st0 = prepare(LSE, B, H, N, d, scale, &prm, &dev);
  if (st0 != FA_OK) return st0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bh = prm.BH;
  if (num_splits == 1) {
    // one range: the fused kernel writes O and LSE directly
    if (d == 128)
      return causal ? launch<128, true, false>(Q, K, V, O, prm, N, bh, st, *dev)
                    : launch<128, false, false>(Q, K, V, O, prm, N, bh, st, *dev);
    return causal ? launch<64, true, false>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<64, false, false>(Q, K, V, O, prm, N, bh, st, *dev);
  }
  const long long rows = splitkv_rows(B, H, N);
  prm.num_splits = num_splits;
  prm.kv_per_split = kv_per_split;
  prm.o_part = static_cast<float*>(workspace);
  prm.lse_part = prm.o_part + static_cast<size_t>(num_splits) * rows * d;
  fa_status r;
  if (d == 128)
    r = causal ? launch<128, true, true>(Q, K, V, O, prm, N, bh, st, *dev)
               : launch<128, false, true>(Q, K, V, O, prm, N, bh, st, *dev);
  else
    r = causal ? launch<64, true, true>(Q, K, V, O, prm, N, bh, st, *dev)
               : launch<64, false, true>(Q, K, V, O, prm, N, bh, st, *dev);
  if (r != FA_OK) return r;
  return d == 128 ? launch_merge<128>(prm.o_part, prm.lse_part, O, LSE, rows, num_splits, st)
                  : launch_merge<64>(prm.o_part, prm.lse_part, O, LSE, rows, num_splits, st);
}

fa_status fa_fwd_block_sparse(const void* Q, const void* K, const void* V, void* O, float* LSE,
                              const int* block_row_ptr, const int* block_col_idx, int nnz, int B,
                              int H, int N, int d, float scale, int causal, void* stream) {
  using namespace fa;
  FwdParams prm;
  DeviceInfo* dev = nullptr;
  fa_status st0 = check_args(Q, K, V, O, LSE, B, H, N, d, scale);
  if (st0 != FA_OK) return st0;
  if (block_row_ptr == nullptr || (nnz > 0 && block_col_idx == nullptr)) return FA_ERR_NULL;
  if (nnz < 0) return FA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(block_row_ptr) & 3u) || (reinterpret_cast<uintptr_t>(block_col_idx) & 3u))
    return FA_ERR_ALIGN;
  const size_t n_blocks = static_cast<size_t>((N + FA_BLOCK_Q - 1) / FA_BLOCK_Q);
  const size_t rp_bytes = (n_blocks + 1) * 4, ci_bytes = static_cast<size_t>(nnz) * 4;
  const size_t nbytes = static_cast<size_t>(B) * H * N * d * 2;
  const size_t lbytes = static_cast<size_t>(B) * H * N * 4;
  if (overlaps(O, nbytes, block_row_ptr, rp_bytes) || (nnz > 0 && overlaps(O, nbytes, block_col_idx, ci_bytes)) ||
      (LSE && (overlaps(LSE, lbytes, block_row_ptr, rp_bytes) ||
               (nnz > 0 && overlaps(LSE, lbytes, block_col_idx, ci_bytes)))))
    return FA_ERR_ALIAS;
  st0 = prepare(LSE, B, H, N, d, scale, &prm, &dev);
  if (st0 != FA_OK) return st0;
  prm.blk_row_ptr = block_row_ptr;
  prm.blk_col_idx = block_col_idx;
  prm.blk_nnz = nnz;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bh = prm.BH;
  if (d == 128)
    return causal ? launch<128, true, false, true>(Q, K, V, O, prm, N, bh, st, *dev)
                  : launch<128, false, false, true>(Q, K, V, O, prm, N, bh, st, *dev);
  return causal ? launch<64, true, false, true>(Q, K, V, O, prm, N, bh, st, *dev)
                : launch<64, false, false, true>(Q, K, V, O, prm, N, bh, st, *dev);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// split-KV without any allocation
// ---------------------------------------------------------------------------
// Some callers cannot allocate device memory at the moment they need
// attention: code running inside a CUDA stream capture that must not add
// allocation nodes, real-time or embedded runtimes that forbid allocation
// after start-up, or hosts whose memory pool is owned by another framework.
// For them the split-KV forward can run on a workspace that is part of this
// library: a fixed array in device memory, allocated once when the library's
// code is loaded on a GPU and held by every GPU that loads it until the
// process exits.
namespace fa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on each device.  In host code the
// array's name is only a stand-in for the symbol, never an address a kernel
// may use; the real address is looked up once per device, with that device
// current.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_fwd_splitkv_noalloc(const void* Q, const void* K, const void* V, void* O, float* LSE,
                                 int B, int H, int N, int d, float scale, int causal, int num_splits,
                                 void* stream) {
  using namespace fa;
  // argument errors are reported exactly as fa_fwd_splitkv reports them
  fa_status st0 = check_args(Q, K, V, O, LSE, B, H, N, d, scale);
  if (st0 != FA_OK) return st0;
  // the ranges this call really runs: a single range needs no scratch at all
  const int splits = effective_splits(B, H, N, causal != 0, num_splits);
  if (splits == 0) return FA_ERR_UNSUPPORTED;
  const size_t need = splitkv_need(B, H, N, d, splits);
  if (need > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES)) return FA_ERR_WORKSPACE;
  int dev_id = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev_id < 0 || dev_id >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev_id] == nullptr) {
      // first call on this device: find the array's device address
      e = cudaGetSymbolAddress(&g_noalloc_ptr[dev_id], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_ptr[dev_id] = nullptr;
        return cuda_fail(e, "cudaGetSymbolAddress");
      }
    }
    scratch = g_noalloc_ptr[dev_id];
  }
  // Every partial state the merge reads is written first by the same call,
  // so nothing in the scratch has to start at zero.
  return fa_fwd_splitkv(Q, K, V, O, LSE, scratch, static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES), B,
                        H, N, d, scale, causal, splits, stream);
}

fa_status fa_get_device_status_word(void* stream, unsigned int* word) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (word) *word = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fa::cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(v));
  if (e != cudaSuccess) return fa::cuda_fail(e, "cudaMemcpyFromSymbol");
  uint32_t vb = 0;
  e = fa::bwd::read_and_clear_status(&vb);
  if (e != cudaSuccess) return fa::cuda_fail(e, "backward status");
  v |= vb;
  if (word) *word = v;
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(zero));  // backward's already cleared
    if (e != cudaSuccess) return fa::cuda_fail(e, "cudaMemcpyToSymbol");
    if (v & fa::kStatusTimeout) return FA_ERR_DEVICE_TIMEOUT;
    return (v & fa::kStatusBounds) ? FA_ERR_BOUNDS : FA_ERR_LAYOUT;
  }
  return FA_OK;
}

fa_status fa_get_device_status(void* stream) { return fa_get_device_status_word(stream, nullptr); }

}  // extern "C"
