// Microbenchmark: cycles per tcgen05.mma (M=128, N=128, K=16, bf16 -> fp32)
// issued back to back by one thread per SM, in the forward's order and TMEM
// layout, alone and beside the kinds of work the forward runs around it.
//
// One CTA of 256 threads per SM (148 CTAs). Shared memory holds a 128 x 128
// Q tile and a K tile (K-major, 128-byte swizzle) and a V tile (MN-major);
// TMEM holds S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512). Thread 0
// issues 16 rounds of 32 products and waits for them; the CTA's elapsed
// SM cycles / 512 is reported, averaged over the CTAs. Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../csrc/sm100.cuh"

using namespace fa;

namespace {

constexpr int kRounds = 16;
constexpr int kCtas = 148;
constexpr int kThreads = 256;
constexpr int kOperandBytes = 96 * 1024;   // Q [0,32K), K [32K,64K), V [64K,96K)
constexpr int kLandingOffset = 128 * 1024;  // bulk-copy landing area [128K,160K)
constexpr int kSmem = 200 * 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum Pattern {
  kSSOnly,             // S0 S1 S0 S1
  kTSOnly,             // PV0 PV1 PV0 PV1
  kForward,            // PV0 S0 PV1 S1: P_t read, then S_t written over it
  kForwardNoOverlap,   // the same mix, PV's A operand never written by S
  kForwardCommits,     // kForward + a commit after each tile
  kForwardWait,        // kForward + a wait on a completed barrier before each group of 8
  kForwardFence,       // kForward + tcgen05.fence::after_thread_sync before each group
  kWithTmemLoads,      // kForwardNoOverlap + 4 warps streaming tcgen05.ld
  kWithTmemStores,     // kForwardNoOverlap + 4 warps streaming tcgen05.st
  kWithEx2,            // kForwardNoOverlap + 6 warps running ex2 chains
  kWithBulkCopies,     // kForward + one thread streaming 32 KB bulk copies into shared memory
  kWithPolling,        // kForwardWait + 6 warps polling a barrier that never completes
};

template <int P>
__global__ void __launch_bounds__(kThreads, 1)
    mma_issue_kernel(unsigned long long* cycles, uint32_t* status, const uint8_t* gsrc, int random_operands) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOperandBytes);  // [0] done [1] commits [2] completed [3] copies [4] never
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 8);
  volatile int* abort = reinterpret_cast<volatile int*>(slot + 1);
  volatile int* stop = reinterpret_cast<volatile int*>(slot + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kOperandBytes / 4; i += blockDim.x) {
    uint32_t w = 0x3f803f80u;  // bf16 1.0 pairs
    if (random_operands) {     // bf16 values in +-[0.5, 1) from an integer hash
      uint32_t h = static_cast<uint32_t>(i) * 2654435761u + blockIdx.x * 97u;
      h ^= h >> 15;
      h *= 2246822519u;
      h ^= h >> 13;
      w = (0x3f00u | (h & 0x807fu)) | ((0x3f00u | ((h >> 16) & 0x807fu)) << 16);
    }
    reinterpret_cast<uint32_t*>(smem)[i] = w;
  }
  if (threadIdx.x == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(&bar[b], 1);
    *abort = 0;
    *stop = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) mbar_arrive(&bar[2]);  // phase 0 of bar[2] completes here
  __syncthreads();
  const uint32_t tmem = *slot;
  constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
  constexpr uint32_t idO = idesc_bf16_f32(128, 128, true);
  const uint32_t sq = smem_addr(smem), sk = sq + 32768, sv = sq + 65536;
  const unsigned long long t0 = clock64();
  if (threadIdx.x == 0) {
    auto S = [&](uint32_t dcol) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_ss(tmem + dcol, sw128_desc(sq + off, 16, 1024), sw128_desc(sk + off, 16, 1024), idS, kk > 0);
      }
    };
    auto PV = [&](uint32_t dcol, uint32_t acol) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + dcol, tmem + acol + kk * 8, sw128_desc(sv + kk * 2048, 16384, 1024), idO, 1);
    };
    auto gate = [&]() {
      if (P == kForwardWait || P == kWithPolling) mbar_wait(&bar[2], 0, abort, status, kTimeoutNs, 0);
      if (P == kForwardFence) tc_fence_after();
    };
    for (int r = 0; r < kRounds; ++r) {
      switch (P) {
        case kSSOnly: S(0); S(128); S(0); S(128); break;
        case kTSOnly: PV(256, 0); PV(384, 128); PV(256, 0); PV(384, 128); break;
        case kForwardNoOverlap:
        case kWithTmemLoads:
        case kWithTmemStores:
        case kWithEx2: PV(256, 192); S(0); PV(384, 192); S(0); break;
        case kForwardCommits:
          PV(256, 0); S(0); mma_commit(&bar[1]);
          PV(384, 128); S(128); mma_commit(&bar[1]);
          break;
        case kForwardWait:
        case kForwardFence:
        case kWithPolling:
          gate(); PV(256, 0); gate(); S(0); gate(); PV(384, 128); gate(); S(128);
          break;
        default: PV(256, 0); S(0); PV(384, 128); S(128); break;  // kForward, kWithBulkCopies
      }
    }
    mma_commit(&bar[0]);
    mbar_wait(&bar[0], 0, abort, status, kTimeoutNs, 0);
    *stop = 1;
  } else if (P == kWithBulkCopies && warp == 1 && lane == 0) {
    const uint8_t* src = gsrc + static_cast<size_t>(blockIdx.x) * 32768;
    for (int i = 0; i < 4000 && !*stop; ++i) {
      mbar_arrive_expect_tx(&bar[3], 32768);
      bulk_load(smem + kLandingOffset, src, 32768, &bar[3]);
      if (!mbar_wait(&bar[3], i & 1, abort, status, kTimeoutNs, 1)) break;
    }
  } else if (P == kWithPolling && warp >= 2) {
    const uint32_t a = smem_addr(&bar[4]);
    for (int i = 0; i < 2000000 && !*stop; ++i)
      if (mbar_try_wait<false>(a, 0)) break;
  } else if ((P == kWithTmemLoads || P == kWithTmemStores) && warp >= 4) {
    // this warp's lane quarter; loads read S, stores write [128,192), which no product touches here
    const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t r[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) r[k] = k;
    uint32_t acc = 0;
    for (int i = 0; i < 20000 && !*stop; ++i) {
      if (P == kWithTmemLoads) {
        tmem_ld32(tmem + lanes + (i & 3) * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) acc += r[k];
      } else {
        tmem_st32(tmem + lanes + 128 + (i & 1) * 32, r);
        tmem_wait_st();
      }
    }
    if (acc == 0x12345678u) cycles[kCtas + blockIdx.x] = acc;
  } else if (P == kWithEx2 && warp >= 2) {
    float x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = -0.001f * (threadIdx.x + k);
    for (int i = 0; i < 200000 && !*stop; ++i) {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = ex2_approx(x[k]) * -0.5f;
    }
    if (x[0] == 12345.f) cycles[kCtas + blockIdx.x] = 1;
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int P>
int run(const char* name, int random_operands, unsigned long long* d, uint32_t* st, const uint8_t* g) {
  cudaMemset(st, 0, 4);
  cudaFuncSetAttribute(mma_issue_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  for (int rep = 0; rep < 3; ++rep) mma_issue_kernel<P><<<kCtas, kThreads, kSmem>>>(d, st, g, random_operands);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    std::printf("%s: %s\n", name, cudaGetErrorString(e));
    return 1;
  }
  std::vector<unsigned long long> h(kCtas);
  uint32_t s = 0;
  cudaMemcpy(h.data(), d, kCtas * 8, cudaMemcpyDeviceToHost);
  cudaMemcpy(&s, st, 4, cudaMemcpyDeviceToHost);
  double avg = 0;
  for (auto x : h) avg += static_cast<double>(x);
  avg /= kCtas;
  std::printf("{\"pattern\": \"%s\", \"random_operands\": %d, \"status\": %u, \"cycles_per_product\": %.1f}\n", name,
              random_operands, s, avg / (kRounds * 32));
  return s != 0;
}

}  // namespace

int main() {
  unsigned long long* d = nullptr;
  uint32_t* st = nullptr;
  uint8_t* g = nullptr;
  if (cudaMalloc(&d, 2 * kCtas * 8) != cudaSuccess || cudaMalloc(&st, 4) != cudaSuccess ||
      cudaMalloc(&g, static_cast<size_t>(kCtas) * 32768) != cudaSuccess) {
    std::printf("allocation failed\n");
    return 1;
  }
  cudaMemset(g, 0, static_cast<size_t>(kCtas) * 32768);
  int bad = 0;
  bad |= run<kSSOnly>("SS only", 0, d, st, g);
  bad |= run<kTSOnly>("TS only", 0, d, st, g);
  bad |= run<kForward>("forward order PV0 S0 PV1 S1", 0, d, st, g);
  bad |= run<kForward>("forward order, random operands", 1, d, st, g);
  bad |= run<kForwardNoOverlap>("same mix, S never overwrites P", 0, d, st, g);
  bad |= run<kForwardCommits>("forward order + commit per tile", 0, d, st, g);
  bad |= run<kForwardFence>("forward order + fence per group of 8", 0, d, st, g);
  bad |= run<kForwardWait>("forward order + completed-barrier wait per group of 8", 0, d, st, g);
  bad |= run<kWithTmemLoads>("+ 4 warps streaming tcgen05.ld", 0, d, st, g);
  bad |= run<kWithTmemStores>("+ 4 warps streaming tcgen05.st", 0, d, st, g);
  bad |= run<kWithEx2>("+ 6 warps running ex2 chains", 0, d, st, g);
  bad |= run<kWithBulkCopies>("+ 32 KB bulk copies streaming into shared memory", 0, d, st, g);
  bad |= run<kWithPolling>("wait per group + 6 warps polling a barrier", 0, d, st, g);
  cudaFree(d);
  cudaFree(st);
  cudaFree(g);
  return bad;
}
