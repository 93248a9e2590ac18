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
// CTA layout (384 threads, one persistent CTA per SM):
//   warp 0      TMA producer: Q tiles, then K/V tiles through a ring of
//               shared-memory stages guarded by full/empty mbarriers.
//   warp 1      TMEM owner and MMA issuer (one thread): S_t = Q_t K^T
//               (SS MMA, M=128 N=128 K=d) and O_t += P_t V (TS MMA, P from
//               TMEM, M=128 N=d K=128), completion signalled by tcgen05.commit.
//   warps 2-3   idle.
//   warps 4-7   softmax + epilogue for query tile 0 (one thread per row).
//   warps 8-11  softmax + epilogue for query tile 1.
// Warps 0-3 give registers up to the softmax warpgroups (setmaxnreg): 136
// and 184 per thread (152 and 176 for d = 64 causal) against the 168 of the
// launch.
// A work item is 2 query tiles of 128 rows (256 rows of one head) so that the
// softmax of one tile overlaps the MMAs of the other.  Each CTA takes items
// gridDim.x apart until none is left; the next item's loads and first score
// products overlap the previous item's last products and epilogue.
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
// Registers per thread after the split between warpgroup 0 (producer, MMA,
// two idle warps) and the two softmax warpgroups, with 128 * control + 256 *
// softmax = 384 * 168, the 64K register file at the launch's 168 per thread:
// the smallest control share that compiles without spills in every
// variant (found with -Xptxas -v), the rest to the softmax.
template <int D, bool CAUSAL, bool SPLIT, bool SPARSE>
__host__ __device__ constexpr uint32_t regs_control() {
  return 136;
}
template <int D, bool CAUSAL, bool SPLIT, bool SPARSE>
__host__ __device__ constexpr uint32_t regs_softmax() {
  return (kThreads * 168 - 128 * regs_control<D, CAUSAL, SPLIT, SPARSE>()) / 256;
}
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// a tile whose row sum of p (against the lagging reference maximum) stays
// within 2^30 keeps the reference (2^16 redid tiles often when Q ~ N(0, 4^2):
// 2.5-3.4% slower there)
constexpr float kLazySum = 1073741824.0f;
constexpr uint32_t kTmemCols = 512;
// wait sites reported in the device status word (bit 8 + site)
enum : uint32_t {
  kSiteKvEmpty = 0, kSiteQ = 1, kSiteKvFull = 2, kSiteS = 3, kSiteP = 4,  // 4..5: p_full[0..1]
  kSiteQFree = 6, kSiteSched = 7, kSiteO = 8, kSiteDebug = 9,
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
  static constexpr int kQBytes = kBM * D * 2;  // one query tile
  static constexpr int kStageBytes = BN * D * 2;  // one ring stage: a whole K or V tile
  static constexpr int kKChunkBytes = BN * 128;   // one 64-wide d chunk of a K stage
  static constexpr int kVChunkBytes = BN * 128;   // one 64-wide d chunk of a V stage
  // the same ring bytes whatever the tile: more stages for smaller tiles
  static constexpr int kStages = (D == 64 ? 8 : 4) * (128 / BN);
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 2 + 1 + 1 + 2 + 2 + 1;
  // O staging: one 32-row x 64-column bf16 box (128-byte rows) per softmax warp
  static constexpr int kOStageBytes = 32 * 128;
  static constexpr int kSmemTiles = kQTiles * kQBytes + kStages * kStageBytes + 8 * kOStageBytes;
  // control block: launch-cancel answer (16 B), barriers, next-item slots,
  // TMEM base and abort flag (16 B), and the slack for 1024-byte alignment
  static constexpr int kSmemBytes = kSmemTiles + 16 + kNumBars * 8 + 16 + 1024;
  static constexpr uint32_t kColO = 256;
};

// The work of one unit: a 256-row query block (two 128-row tiles, or one
// for the tile-size sweep) of one head, and for split-KV one key range.
struct Unit {
  int bh, qblk, split, q0;
  int j_last[2];
  int kv_lo, kv_end, n_iter;
  int first_it[2];
  bool active[2];
  const int* blk;  // block-sparse: this block's retained key tiles
};

// Work item w, in heavy-first order: heads in groups of p.group_heads;
// inside a group, query blocks from the heaviest (last rows: most keys when
// causal) to the lightest, cycling over the group's heads, so that blocks
// running together share the K/V of a few heads in L2; split-KV ranges of one
// block are adjacent.
template <bool CAUSAL, bool SPLIT, bool SPARSE, int BN, int QT>
__device__ __forceinline__ Unit unit_of(const FwdParams& p, int w) {
  Unit u;
  u.split = SPLIT ? w % p.num_splits : 0;
  const int unit = SPLIT ? w / p.num_splits : w;
  const int per_group = p.group_heads * p.n_qblk;
  const int grp = unit / per_group;
  const int rem = unit % per_group;
  const int grp_heads = min(p.group_heads, p.BH - grp * p.group_heads);
  u.bh = grp * p.group_heads + rem % grp_heads;
  u.qblk = p.n_qblk - 1 - rem / grp_heads;
  u.q0 = u.qblk * QT * kBM - (2 - QT) * kBM;  // first row of slot 0
  // last key tile each query tile needs (the causal diagonal, or the end)
#pragma unroll
  for (int t = 0; t < 2; ++t)
    u.j_last[t] = CAUSAL ? min(u.q0 + (t + 1) * kBM - 1, p.N - 1) / BN : p.n_kv - 1;
  // key tiles [kv_lo, kv_end) of this unit (all of them unless split),
  // visited from kv_end - 1 down to kv_lo
  u.kv_lo = SPLIT ? u.split * p.kv_per_split : 0;
  u.kv_end = SPLIT ? min(u.j_last[1] + 1, u.kv_lo + p.kv_per_split) : u.j_last[1] + 1;
  u.n_iter = max(0, u.kv_end - u.kv_lo);
  // iterations before a query tile's first unmasked key tile are skipped for
  // it; a tile whose first iteration is past n_iter has no keys in this range
  u.first_it[0] = u.kv_end - 1 - min(u.j_last[0], u.kv_end - 1);
  u.first_it[1] = 0;
  u.blk = nullptr;
  // Block-sparse: this block's retained key tiles, visited from the last
  // entry down.  Entries past tile 1's diagonal are seen by no row and are
  // dropped; leading visits past tile 0's diagonal are skipped for tile 0.
  // A malformed list raises kStatusLayout; out-of-range or out-of-order
  // entries are then masked out entirely (no memory outside the tensors is
  // touched), and the outputs are not meaningful.
  if (SPARSE) {
    int beg = __ldg(p.blk_row_ptr + u.qblk), end = __ldg(p.blk_row_ptr + u.qblk + 1);
    if (!(0 <= beg && beg <= end && end <= p.blk_nnz)) {
      if (threadIdx.x == 0) atomicOr(&g_device_status, kStatusLayout);
      beg = end = 0;
    }
    u.blk = p.blk_col_idx + beg;
    int n = end - beg;
    while (n > 0 && __ldg(u.blk + n - 1) > u.j_last[1]) {
      if (threadIdx.x == 0 && __ldg(u.blk + n - 1) >= p.n_kv) atomicOr(&g_device_status, kStatusLayout);
      --n;
    }
    int skip = 0;
    while (skip < n && __ldg(u.blk + n - 1 - skip) > u.j_last[0]) ++skip;
    u.n_iter = n;
    u.first_it[0] = skip;
  }
  if (QT == 1) u.first_it[0] = u.n_iter;  // slot 0 unused
  u.active[0] = u.first_it[0] < u.n_iter;
  u.active[1] = u.n_iter > 0;
  return u;
}

// One CTA is launched per work item, in heavy-first order, but a CTA does
// not end with its item: its producer thread asks the hardware to cancel the
// launch of the next pending CTA (cluster launch control) and takes that
// CTA's item over, until none is left.  The SMs so take the items in launch
// order, as free SMs would take new CTAs (greedy longest-first), while each
// CTA keeps its tensor memory, barriers and pipeline: every barrier counts
// its phases on from one item to the next, and the next item's Q and K/V
// tiles load, and its first score products run, while the previous item's
// last products and epilogue finish.
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
  uint8_t* sQ = smem;                  // kQTiles query tiles
  uint8_t* sKV = smem + kQTiles * QB;  // S ring stages
  uint8_t* sO = sKV + S * SB;          // O staging, one box per softmax warp
  uint8_t* ctrl = smem + C::kSmemTiles;
  void* clc_resp = ctrl;              // 16 B: answer of the last launch-cancel request
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl + 16);
  uint64_t* q_full = bars;            // [2] Q tile landed
  uint64_t* kv_full = q_full + 2;     // [S] K/V stage landed
  uint64_t* kv_empty = kv_full + S;   // [S] MMA -> producer
  uint64_t* s_full = kv_empty + S;    // [2] MMA -> softmax
  uint64_t* p_full = s_full + 2;      // [2] softmax -> MMA
  uint64_t* o_full = p_full + 2;      // [2] MMA -> epilogue
  uint64_t* q_free = o_full + 2;      // [2] MMA -> producer: an item's last S product of tile t is done
  uint64_t* mma_done = q_free + 2;    // [1] MMA -> itself, before TMEM release
  uint64_t* never = mma_done + 1;     // [1] debug: nothing arrives here
  uint64_t* sched_full = never + 1;   // [2] producer -> MMA, softmax: next item id written
  uint64_t* sched_empty = sched_full + 2;  // [2] MMA, softmax -> producer: id read
  uint64_t* clc_bar = sched_empty + 2;     // [1] launch-cancel answer landed
  volatile int* sched_item = reinterpret_cast<volatile int*>(clc_bar + 1);  // [2] next item, -1: none
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(sched_item) + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* status = &g_device_status;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FA_TRACE_INIT();
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], kBM / 32);  // one arrival per softmax warp
      mbar_init(&o_full[t], 1);
      mbar_init(&q_free[t], 1);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(never, 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(&sched_full[k], 1);
      // the MMA thread and every softmax warp read each id
      mbar_init(&sched_empty[k], 1 + (kBM / 32) * QT);
    }
    mbar_init(clc_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (!SPLIT) tma_prefetch_desc(&tmO);
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
  // Every warp, converged, inside its role's branch (so that the role's code
  // is compiled for its count): warpgroup 0 gives registers up, the softmax
  // warpgroups take them.
  constexpr uint32_t kRegsControl = regs_control<D, CAUSAL, SPLIT, SPARSE>();
  constexpr uint32_t kRegsSoftmax = regs_softmax<D, CAUSAL, SPLIT, SPARSE>();
  static_assert(kRegsControl % 8 == 0 && kRegsSoftmax % 8 == 0 &&
                    128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * 168,
                "the split fits the launch's registers");
  if (warp < kSoftmaxWarp0) regs_dealloc<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int i = 0;                     // loads issued into the ring, over all items
      int q_loads[2] = {0, 0};       // loads issued into each Q buffer
      bool clc_open = true;          // launches may be left to take over
      bool clc_pending = false;      // a request whose answer is not read yet
      uint32_t clc_phase = 0;
      int w = static_cast<int>(blockIdx.x);
      // Asks for the next item.  Asked at the start of this item's last
      // loads, about two iterations before the CTA finishes it (the loads
      // run that far ahead of the products), so that items go to CTAs in the
      // order in which they finish, as with new CTAs on free SMs; asked at
      // the start of an item, the second round of items would be dealt out
      // before any CTA is near its end (measured: 10% slower on causal
      // N = 8192).  The answer is read once the item's loads are issued.
      auto request_next = [&]() {
        if (clc_open && !clc_pending) {
          mbar_arrive_expect_tx(clc_bar, 16);
          clc_try_cancel(clc_resp, clc_bar);
          clc_pending = true;
        }
      };
      for (int k = 0; ok; ++k) {
        const Unit u = unit_of<CAUSAL, SPLIT, SPARSE, BN, QT>(p, w);
        // Q tile t of this item, once the previous item's last S product of
        // tile t (the last reader of the buffer) has finished
        auto load_q = [&](int t) {
          if (q_loads[t] > 0 &&
              !mbar_wait(&q_free[t], static_cast<uint32_t>(q_loads[t] - 1) & 1u, abort_flag, status, tmo, kSiteQFree))
            return false;
          const int row0 = u.q0 + t * kBM;
          if (!in_bounds(row0 >= 0 && row0 < p.n_qblk * QT * kBM && u.bh < p.BH, kCheckQLoad)) {
            *abort_flag = 1;
            return false;
          }
          ++q_loads[t];
          mbar_arrive_expect_tx(&q_full[t], QB);
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_3d(sQ + t * QB + ch * kChunkBytes, &tmQ, &q_full[t], ch * 64, row0, u.bh);
          return true;
        };
        if (u.active[0] && !(ok = load_q(0))) break;
        // loads of this item in consumption order K0 V0 K1 V1 ... (none
        // when the item has no key tile)
        for (int it = 0; it < u.n_iter && ok; ++it) {
          if (it == u.n_iter - 1) request_next();
          // (a block-sparse entry out of range is loaded clamped and masked)
          const int j = SPARSE ? min(max(__ldg(u.blk + u.n_iter - 1 - it), 0), p.n_kv - 1) : u.kv_end - 1 - it;
          for (int kv = 0; kv < 2; ++kv) {
            const int s = i % S;
            const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
            ok = mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, status, tmo, kSiteKvEmpty);
            if (!ok) break;
            if (!in_bounds(j >= 0 && j < p.n_kv && s < S && u.bh < p.BH, kCheckKvLoad)) {
              ok = false;
              *abort_flag = 1;
              break;
            }
            mbar_arrive_expect_tx(&kv_full[s], SB);
            uint8_t* st = sKV + s * SB;
            const CUtensorMap* map = kv == 0 ? &tmK : &tmV;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_3d(st + ch * C::kKChunkBytes, map, &kv_full[s], ch * 64, j * BN, u.bh);
            ++i;
            if (it == 0 && kv == 0 && !(ok = load_q(1))) break;
          }
        }
        if (!ok) break;
        request_next();  // (an item without key tiles)
        int next = -1;
        if (clc_pending) {
          if (!(ok = mbar_wait(clc_bar, clc_phase, abort_flag, status, tmo, kSiteSched))) break;
          clc_phase ^= 1u;
          clc_pending = false;
          uint32_t x;
          if (clc_query(clc_resp, &x))
            next = static_cast<int>(x);
          else
            clc_open = false;  // no launch left: no further request may be made
        }
        // hand the next item (or the end, -1) to the MMA and softmax roles
        if (!(ok = mbar_wait(&sched_empty[k & 1], (static_cast<uint32_t>(k >> 1) & 1u) ^ 1u, abort_flag, status,
                             tmo, kSiteSched)))
          break;
        sched_item[k & 1] = next;
        mbar_arrive(&sched_full[k & 1]);
        if (next < 0) break;
        w = next;
      }
      if (!ok) {
        // Unwinding: wait for every copy this CTA issued, so that none lands
        // in shared memory after the CTA has ended.
        for (int s = 0; s < S && s < i; ++s) {
          const int last = s + ((i - 1 - s) / S) * S;
          mbar_wait_drain(&kv_full[s], static_cast<uint32_t>(last / S) & 1u, tmo);
        }
        for (int t = 0; t < 2; ++t)
          if (q_loads[t] > 0) mbar_wait_drain(&q_full[t], static_cast<uint32_t>(q_loads[t] - 1) & 1u, tmo);
        // and for the answer of a launch-cancel request still on its way
        if (clc_pending) mbar_wait_drain(clc_bar, clc_phase, tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, BN, false);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, true);
      const uint32_t sq = smem_addr(sQ);
      const uint32_t skv = smem_addr(sKV);
      // The issuing thread is on the critical path between the softmax and
      // the next S (an MMA is accepted only about as fast as the tensor core
      // retires the one before), so each operand's descriptor is built once
      // per product and advanced by a constant per K-step (the start-address
      // field counts 16-byte units and shared-memory addresses stay below
      // 2^18, so adding the offset never carries out of it).  Measured on
      // B200: +2.6% at d = 128, +1.2% at d = 64.
      // S_t = Q_t K^T: A = Q_t (K-major), B = K stage (K-major); 16 columns of
      // d per instruction, 32 bytes apart inside each 128-byte swizzled row.
      auto issue_s = [&](int t, int s) {
        const uint64_t a0 = sw128_desc(sq + t * QB, 16, 1024);
        const uint64_t b0 = sw128_desc(skv + s * SB, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * C::kKChunkBytes + (kk & 3) * 32;
          mma_ss(tmem + t * BN, a0 + (aoff >> 4), b0 + (boff >> 4), idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V: A = P_t in TMEM (8 columns per 16 keys), B = V stage
      // stored d-contiguous (MN-major): 16 keys = 2 KB apart, d halves 16 KB apart.
      auto issue_pv = [&](int t, int s, bool accumulate) {
        const uint64_t v0 = sw128_desc(skv + s * SB, C::kVChunkBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = v0 + static_cast<uint32_t>(kk * (2048 >> 4));
          const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::kColO + t * D, tmem + t * BN + kk * 8, bd, idO, acc);
        }
      };
      bool ok = true;
      int i = 0;                     // ring loads consumed, over all items
      int q_seen[2] = {0, 0};        // Q loads consumed per buffer
      int p_seen[2] = {0, 0};        // P publications consumed per tile
      int trace_it = 0;              // iterations over all items (trace stamps)
      int w = static_cast<int>(blockIdx.x);
      for (int k = 0; ok; ++k) {
        const Unit u = unit_of<CAUSAL, SPLIT, SPARSE, BN, QT>(p, w);
        const int n_iter = u.n_iter;
        if (n_iter > 0) {
          // the ring stage of load number n, waited for
          auto wait_load = [&](int n) {
            return mbar_wait(&kv_full[n % S], static_cast<uint32_t>(n / S) & 1u, abort_flag, status, tmo, kSiteKvFull);
          };
          auto wait_q = [&](int t) {
            if (!mbar_wait(&q_full[t], static_cast<uint32_t>(q_seen[t]) & 1u, abort_flag, status, tmo, kSiteQ))
              return false;
            ++q_seen[t];
            return true;
          };
          const int i0 = i;  // this item's first load: K0 at i0, V0 at i0 + 1, K1 at i0 + 2, ...
          bool q_ready[2] = {false, false};
          if (!(ok = wait_load(i0))) break;
  #pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || u.first_it[t] != 0) continue;
            if (!(ok = wait_q(t))) break;
            q_ready[t] = true;
            tc_fence_after();
            issue_s(t, i0 % S);
            mma_commit(&s_full[t]);
            if (n_iter == 1) mma_commit(&q_free[t]);  // the item's last S product of tile t
          }
          if (!ok) break;
          mma_commit(&kv_empty[i0 % S]);
          for (int it = 0; it < n_iter && ok; ++it) {
            const int iv = i0 + 2 * it + 1, ik = i0 + 2 * it + 2;
            const int sv = iv % S, sk = ik % S;
            const bool last = it == n_iter - 1;
            // At d = 64 each V after the item's first is waited for earlier,
            // between the previous key tile's PV and S products of query tile
            // 1 (+1.7% there; -2.9% at d = 128, where that wait delays the S
            // products of the longer PV/S blocks)
            constexpr bool kEarlyV = D == 64;
            if ((!kEarlyV || it == 0) && !(ok = wait_load(iv))) break;
            FA_TRACE_MARK(3, trace_it + it, 0);
            // the next K tile too, here rather than between a PV and an S
            // product: it has normally landed long before, but the wait itself
            // costs the issuing thread time that the tensor core then idles
            if (!last && !(ok = wait_load(ik))) break;
            FA_TRACE_MARK(3, trace_it + it, 1);
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok) continue;
              if (it >= u.first_it[t]) {
                // (the first PV of an item overwrites O_t; the softmax threads
                // that publish its P have read the previous item's O_t out
                // of TMEM before, in their epilogue)
                if (!(ok = mbar_wait(&p_full[t], static_cast<uint32_t>(p_seen[t]) & 1u, abort_flag, status, tmo,
                                     kSiteP + t)))
                  break;
                ++p_seen[t];
                FA_TRACE_MARK(0, trace_it + it, 3 * t);
                tc_fence_after();
                issue_pv(t, sv, it > u.first_it[t]);
                FA_TRACE_MARK(0, trace_it + it, 3 * t + 1);
                if (last) mma_commit(&o_full[t]);
              }
              // the V stage is free once the second tile's PV has read it,
              // ahead of that tile's next S product (+1.3% on causal N = 8192
              // against releasing it with the K stage after that S)
              if (t == 1) mma_commit(&kv_empty[sv]);
              if (kEarlyV && t == 1 && !last && !(ok = wait_load(iv + 2))) break;
              if (!last && it + 1 >= u.first_it[t]) {
                if (!q_ready[t]) {
                  if (!(ok = wait_q(t))) break;
                  q_ready[t] = true;
                }
                tc_fence_after();
                issue_s(t, sk);
                mma_commit(&s_full[t]);
                if (it + 1 == n_iter - 1) mma_commit(&q_free[t]);  // the item's last S product of tile t
                FA_TRACE_MARK(0, trace_it + it, 3 * t + 2);
              }
            }
            if (!ok) break;
            if (!last) mma_commit(&kv_empty[sk]);
          }
          i = i0 + 2 * n_iter;
          trace_it += n_iter;
        }
        if (!ok) break;
        // the next item
        if (!(ok = mbar_wait(&sched_full[k & 1], static_cast<uint32_t>(k >> 1) & 1u, abort_flag, status, tmo,
                             kSiteSched)))
          break;
        const int next = sched_item[k & 1];
        mbar_arrive(&sched_empty[k & 1]);
        if (next < 0) break;
        w = next;
      }
      // every MMA issued here has finished before TMEM is released
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, tmo);
    }
  } else if (warp >= kSoftmaxWarp0) {
    regs_alloc<kRegsSoftmax>();
    if (QT == 2 || warp >= kSoftmaxWarp0 + 4) {  // (with one query tile, slot 0 is unused)
      // ------------------------------------------------------------ softmax
      const int t = (warp - kSoftmaxWarp0) >> 2;  // query tile of this warpgroup
      const int wq = warp & 3;                    // TMEM lane quarter
      const int r = wq * 32 + lane;               // row inside the tile
      const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tS = tmem + lane_base + t * BN;
      const uint32_t tO = tmem + lane_base + C::kColO + t * D;
      const float sl2 = p.scale_log2;
      // O_t holds the product through the previous tile (that MMA finished
      // before S_t of this tile was committed): rescale this thread's row of
      // it in place, before P of this tile releases the next PV product.
      auto rescale_o_rows = [&](uint32_t taddr, float a) {
  #pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t o[16];
          tmem_ld16(taddr + cc * 16, o);
          tmem_wait_ld();
  #pragma unroll
          for (int kx = 0; kx < 16; ++kx) o[kx] = __float_as_uint(__uint_as_float(o[kx]) * a);
          tmem_st16(taddr + cc * 16, o);
        }
      };

      bool ok = true;
      if (p.debug & 1u) {
        ok = __all_sync(0xffffffffu, mbar_wait(never, 0, abort_flag, status, tmo, kSiteDebug));
      }
      int s_seen = 0;   // S_t products consumed, over all items
      int o_seen = 0;   // O_t completions consumed, over all items
      int trace_it = 0;
      int w = static_cast<int>(blockIdx.x);
      for (int k = 0;; ++k) {
        const Unit u = unit_of<CAUSAL, SPLIT, SPARSE, BN, QT>(p, w);
        const int row0 = u.q0 + t * kBM;
        const int row = row0 + r;  // query index in the head
        const int bh = u.bh;
        const int n_iter = u.n_iter;
        const int first = t ? u.first_it[1] : u.first_it[0];
        const bool active = t ? u.active[1] : u.active[0];
        const int kv_top = SPARSE ? 0 : u.kv_end - 1;
        const int* const blk = u.blk;
        // last key this row may see
        const int key_limit = CAUSAL ? min(row, p.N - 1) : p.N - 1;
        auto kv_tile = [&](int it) { return SPARSE ? __ldg(blk + n_iter - 1 - it) : kv_top - it; };
        float m_ref = -INFINITY;  // reference maximum, log2 units of scaled scores
        float l_sum = 0.f;        // running denominator relative to m_ref
        for (int it = first; it < n_iter && ok; ++it) {
          const int li = it - first;
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
                          mbar_wait(&s_full[t], static_cast<uint32_t>(s_seen) & 1u, abort_flag, status, tmo, kSiteS));
          if (!ok) break;
          ++s_seen;
          const bool tr = lane == 0 && (warp & 3) == 0;
          if (tr) FA_TRACE_MARK(1 + t, trace_it + it, 0);
          tc_fence_after();
          constexpr int kQ32 = BN / 32;  // 32-key groups of a tile
          uint32_t sr[kQ32][32];
  #pragma unroll
          for (int q = 0; q < kQ32; ++q) tmem_ld32(tS + q * 32, sr[q]);
          tmem_wait_ld();
          if (tr) FA_TRACE_MARK(1 + t, trace_it + it, 1);

          const int kbase = j * BN;
          const bool masked = bad || (kbase + BN > p.N) || (CAUSAL && kbase + BN - 1 > row0);
          if (masked) {
            const int lim = bad ? -1 : key_limit;
  #pragma unroll
            for (int q = 0; q < kQ32; ++q)
  #pragma unroll
              for (int cc = 0; cc < 32; ++cc)
                if (kbase + q * 32 + cc > lim) sr[q][cc] = __float_as_uint(-INFINITY);
          }
          // row maximum of the raw scores (scale > 0 keeps the argmax): BN/16
          // independent chains of three-input maxima; log2 units of scaled scores
          auto tile_max = [&]() {
            constexpr int kChains = BN / 16;
            float mx[kChains];
  #pragma unroll
            for (int kx = 0; kx < kChains; ++kx) mx[kx] = __uint_as_float(sr[kx >> 1][(kx & 1) * 16]);
  #pragma unroll
            for (int kx = 0; kx < kChains; ++kx) {
              const uint32_t* v = &sr[kx >> 1][(kx & 1) * 16];
  #pragma unroll
              for (int cc = 1; cc < 15; cc += 2)
                mx[kx] = fmax3(mx[kx], __uint_as_float(v[cc]), __uint_as_float(v[cc + 1]));
              mx[kx] = fmaxf(mx[kx], __uint_as_float(v[15]));
            }
            float m_all;
            if constexpr (kChains == 8)
              m_all = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            else
              m_all = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]);
            return m_all * sl2;
          };
          const float2 sl2v = make_float2(sl2, sl2);
          float2 ps2[kQ32];
          // p = 2^(s * scale * log2 e - m_ref), written as bf16 pairs over the
          // first BN/2 columns of S_t, 64 keys at a time, and published whole
          // on p_full[t]; ps2 gets the row sums of the fp32 p.  The keys are
          // taken from the top down, so that the scores of keys [0, BN/2),
          // whose columns the P stores overwrite, are the last ones read:
          // they stay in registers for a redo (below), while those of keys
          // [BN/2, BN) remain in TMEM.
          auto exponentials = [&]() {
            const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
            const float2 nm2 = make_float2(neg_m, neg_m);
  #pragma unroll
            for (int h = BN / 64 - 1; h >= 0; --h) {
              // keys [64h, 64h + 64) -> 32 columns of bf16 pairs at column 32h
              uint32_t pk[32];
  #pragma unroll
              for (int qq = 1; qq >= 0; --qq) {
                const int q = 2 * h + qq;
                ps2[q] = make_float2(0.f, 0.f);
  #pragma unroll
                for (int cc = 0; cc < 32; cc += 2) {
                  const float2 x = ffma2(make_float2(__uint_as_float(sr[q][cc]), __uint_as_float(sr[q][cc + 1])),
                                         sl2v, nm2);
                  float2 pv;
                  pv.x = ex2_approx(x.x);
                  pv.y = ex2_approx(x.y);
                  ps2[q] = fadd2(ps2[q], pv);
                  pk[qq * 16 + (cc >> 1)] = pack_bf16x2(pv.x, pv.y);
                }
              }
              tmem_st32(tS + h * 32, pk);
              if (tr && h == BN / 64 - 1) FA_TRACE_MARK(1 + t, trace_it + it, 3);
            }
          };
          auto row_sum = [&]() {
            float2 psum;
            if constexpr (kQ32 == 4)
              psum = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
            else
              psum = fadd2(ps2[0], ps2[1]);
            return psum.x + psum.y;
          };
          // The reference maximum m_ref lags the row maximum: it is raised
          // only when a tile's scores exceed it by more than
          // kRescaleThreshold.  In a row block's first tile the maximum is
          // taken before the exponentials.  After that it is not: the
          // exponentials run against m_ref, and a row sum of at most kLazySum
          // (2^30) bounds every p of the tile by it, so m_ref may stay (fp32
          // and bf16 hold such p with their full relative precision).  Only
          // a warp with a larger sum (or a row still without a reference)
          // takes the maximum and redoes the tile.
          float alpha = 1.f;
          bool raise = false;
          bool maxed = li == 0;  // the tile's maximum was taken (only then may a row raise)
          auto raise_ref = [&]() {
            const float m_tile = tile_max();
            raise = m_tile > m_ref + kRescaleThreshold;
            if (raise) {
              alpha = ex2_approx(m_ref - m_tile);  // 0 while m_ref is -inf
              m_ref = m_tile;
            }
          };
          if (li == 0) {
            raise_ref();
            if (tr) FA_TRACE_MARK(1 + t, trace_it + it, 2);
            exponentials();
          } else {
            if (tr) FA_TRACE_MARK(1 + t, trace_it + it, 2);
            exponentials();
            const float sum = row_sum();
            if (__any_sync(0xffffffffu, !(sum <= kLazySum) || m_ref == -INFINITY)) {
              maxed = true;
              // the scores of keys [BN/2, BN) back from TMEM (their columns
              // hold no P)
  #pragma unroll
              for (int q = kQ32 / 2; q < kQ32; ++q) tmem_ld32(tS + q * 32, sr[q]);
              tmem_wait_ld();
              if (masked) {
                const int lim = bad ? -1 : key_limit;
  #pragma unroll
                for (int q = kQ32 / 2; q < kQ32; ++q)
  #pragma unroll
                  for (int cc = 0; cc < 32; ++cc)
                    if (kbase + q * 32 + cc > lim) sr[q][cc] = __float_as_uint(-INFINITY);
              }
              raise_ref();
              // (the stores of P are warp-wide: every lane writes its row again)
              if (__any_sync(0xffffffffu, raise)) exponentials();
            }
          }
          // (no vote when no row could have raised: +0.7% on causal N = 8192)
          const bool rescale_o = li > 0 && maxed && __any_sync(0xffffffffu, raise);
          // the rescale waits until the scores have left the registers
          if (rescale_o) rescale_o_rows(tO, alpha);
          // every lane's stores have completed; one arrival per warp
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[t]);
          if (lane == 0 && wq != 0) FA_TRACE_MARK(1 + t, trace_it + it, 4 + wq);
          l_sum = l_sum * alpha + row_sum();
          if (tr) FA_TRACE_MARK(1 + t, trace_it + it, 4);
        }
        trace_it += n_iter;

        // ---------------------------------------------------------- epilogue
        if (ok && active) {
          ok = mbar_wait(&o_full[t], static_cast<uint32_t>(o_seen) & 1u, abort_flag, status, tmo, kSiteO);
          ++o_seen;
        }
        if (named_bar_or(1 + t, kBM, !ok)) break;
        tc_fence_after();
        const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
        const float lse2 = l_sum > 0.f ? m_ref + log2f(l_sum) : -INFINITY;
        if (SPLIT) {
          // partial state of this key range: u / l (fp32) and its LSE; a range
          // with no allowed key for this row gives LSE = -inf and weight 0 in
          // the merge
          const size_t prow = (static_cast<size_t>(u.split) * p.BH + bh) * p.N + row;
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
          const bool row_ok =
              row < p.N &&
              in_bounds(u.split < p.num_splits && bh < p.BH && prow < static_cast<size_t>(p.num_splits) * p.BH * p.N,
                        kCheckPartial);
          if (row_ok) p.lse_part[prow] = lse2 * 0.69314718055994530942f;
  #pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            if (active) {
              tmem_ld32(tO + cc * 32, o);
              tmem_wait_ld();
            } else {
  #pragma unroll
              for (int kx = 0; kx < 32; ++kx) o[kx] = 0u;
            }
            if (row_ok) {
  #pragma unroll
              for (int g = 0; g < 8; ++g)
                dst[cc * 8 + g] = make_float4(__uint_as_float(o[4 * g]) * inv_l, __uint_as_float(o[4 * g + 1]) * inv_l,
                                              __uint_as_float(o[4 * g + 2]) * inv_l, __uint_as_float(o[4 * g + 3]) * inv_l);
            }
          }
        } else {
          if (p.lse != nullptr && row < p.N && in_bounds(bh < p.BH && row >= 0, kCheckLse))
            p.lse[static_cast<size_t>(bh) * p.N + row] = lse2 * 0.69314718055994530942f;
          // O_t / l -> bf16, 64 columns at a time through this warp's staging
          // box (its 32 rows, laid out as the 128-byte swizzle of the store
          // tensor map), written out by a TMA store; rows past N are clipped
          // by the store.  The Q buffers stay free for the next item's loads.
          uint8_t* stage = sO + (warp - kSoftmaxWarp0) * C::kOStageBytes;
          const int wrow0 = row0 + wq * 32;
          uint8_t* rowp = stage + lane * 128;
  #pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
  #pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t o[32];
              if (active) {
                tmem_ld32(tO + ch * 64 + h * 32, o);
                tmem_wait_ld();
              } else {  // no retained key (block-sparse): O = 0
  #pragma unroll
                for (int kx = 0; kx < 32; ++kx) o[kx] = 0u;
              }
              if (h == 0) {
                // the previous store from this box has been read out
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
              }
  #pragma unroll
              for (int gg = 0; gg < 4; ++gg) {
                const uint32_t* src = &o[gg * 8];
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(src[0]) * inv_l, __uint_as_float(src[1]) * inv_l);
                v.y = pack_bf16x2(__uint_as_float(src[2]) * inv_l, __uint_as_float(src[3]) * inv_l);
                v.z = pack_bf16x2(__uint_as_float(src[4]) * inv_l, __uint_as_float(src[5]) * inv_l);
                v.w = pack_bf16x2(__uint_as_float(src[6]) * inv_l, __uint_as_float(src[7]) * inv_l);
                const int gran = (h * 4 + gg) ^ (lane & 7);
                if (in_bounds(rowp + gran * 16 >= stage && rowp + gran * 16 + 16 <= stage + C::kOStageBytes,
                              kCheckStage))
                  *reinterpret_cast<uint4*>(rowp + gran * 16) = v;
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && wrow0 < p.N && in_bounds(wrow0 >= 0 && bh < p.BH, kCheckStore)) {
              tma_store_3d(&tmO, stage, ch * 64, wrow0, bh);
              bulk_commit_group();
            }
          }
        }
        // the next item; the warps of this warpgroup agree on going on
        // before any of them reaches the next item's barriers
        const bool got =
            __all_sync(0xffffffffu, mbar_wait(&sched_full[k & 1], static_cast<uint32_t>(k >> 1) & 1u, abort_flag,
                                              status, tmo, kSiteSched));
        const int next = got ? sched_item[k & 1] : -1;
        __syncwarp();
        if (got && lane == 0) mbar_arrive(&sched_empty[k & 1]);
        if (named_bar_or(1 + t, kBM, !got) || next < 0) break;
        w = next;
      }
      // the staging box has been read out before the CTA's shared memory goes
      if (!SPLIT && lane == 0) bulk_wait_group_read0();
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
      !make_map_cached(&mv, V, D, N, BH, BN) || (!SPLIT && !make_map_cached(&mo, O, D, N, BH, 32))) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed");
    return FA_ERR_CUDA;
  }
  const long long rows_per_block = static_cast<long long>(QT) * kBM;
  prm.n_qblk = static_cast<int>((N + rows_per_block - 1) / rows_per_block);
  const long long units = static_cast<long long>(BH) * prm.n_qblk;
  const long long items = units * (SPLIT ? prm.num_splits : 1);
  if (items > 0x7fffffffll) return FA_ERR_SHAPE;
  // one CTA per item; each running CTA takes over the items of CTAs not yet
  // launched, so in practice one CTA per SM runs them all
  const long long grid = items;
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
  if (SPLIT) mo = mq;  // (unused: the partial states are plain stores)
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
