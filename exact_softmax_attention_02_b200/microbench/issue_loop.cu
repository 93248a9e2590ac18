// Microbenchmark: the forward's MMA issue loop with stand-in roles, to find
// what the issuing thread waits for. One CTA of 384 threads per SM (148
// CTAs), 64 iterations of 32 products (M=128, N=128, K=16) each:
//   warp 0      stand-in producer: fills a 4-stage K/V ring (plain arrivals,
//               32 KB bulk copies, or the forward's own tiled TMA loads)
//   warp 1      the issuer, one thread, with the forward's order, barriers and
//               commits: PV_t, then the next S_t, for t = 0, 1
//   warps 4-11  stand-in softmax warpgroups: wait for S_t, publish P_t at once
// Reports SM cycles per iteration, averaged over the CTAs. Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <vector>

#include "../csrc/host_util.h"
#include "../csrc/sm100.cuh"

using namespace fa;

namespace {

constexpr int kIters = 64, kStages = 4, kQBytes = 32768, kStageBytes = 32768;
constexpr int kCtas = 148, kThreads = 384, kGroups = kCtas / 8 + 1;  // 8 CTAs share K/V
constexpr int kSmem = 2 * kQBytes + kStages * kStageBytes + 1024 + 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum Variant {
  kHandshakes,   // plain arrivals for K/V; stand-ins poll S with every lane
  kLaneZeroPoll, // stand-ins poll S with lane 0 only
  kNoPWait,      // the issuer does not wait for P
  kKVOnly,       // the issuer waits for K/V only; stand-ins arrive without waiting
  kLoadS,        // stand-ins also load S (4 x tcgen05.ld.x32) before publishing P
  kBulkKV,       // K/V moved by 32 KB bulk copies from L2/HBM
  kTmaKV,        // K/V moved by the forward's tiled TMA loads (two 64-column boxes, 128-byte swizzle)
};

template <int V>
__global__ void __launch_bounds__(kThreads, 1)
    issue_loop_kernel(const __grid_constant__ CUtensorMap tm, unsigned long long* cycles, uint32_t* status,
                      const uint8_t* gsrc) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + 2 * kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kStages * kStageBytes);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* mma_done = p_full + 2;
  uint32_t* slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (2 * kQBytes + kStages * kStageBytes) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem)[i] = 0x3f803f80u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const unsigned long long t0 = clock64();
  if (warp == 0) {
    if (lane == 0) {
      // ring slots in the issuer's order: K0, then V_it, K_it+1 per iteration
      for (int i = 0; i < 2 * kIters; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&kv_empty[s], ((i / kStages) & 1) ^ 1, abort, status, kTimeoutNs, 0)) break;
        if (V == kBulkKV) {
          const uint8_t* src = gsrc + (static_cast<size_t>(blockIdx.x / 8) * (2 * kIters) + i) * kStageBytes;
          mbar_arrive_expect_tx(&kv_full[s], kStageBytes);
          bulk_load(sKV + s * kStageBytes, src, kStageBytes, &kv_full[s]);
        } else if (V == kTmaKV) {
          mbar_arrive_expect_tx(&kv_full[s], kStageBytes);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sKV + s * kStageBytes + c * 16384, &tm, &kv_full[s], c * 64, ((i / 2) % 64) * 128,
                        blockIdx.x / 8);
        } else {
          mbar_arrive(&kv_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, 128, true);
      const uint32_t sq = smem_addr(sQ), skv = smem_addr(sKV);
      auto issue_s = [&](int t, int s) {
        const uint64_t a0 = sw128_desc(sq + t * kQBytes, 16, 1024), b0 = sw128_desc(skv + s * kStageBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss(tmem + t * 128, a0 + off, b0 + off, idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint64_t v0 = sw128_desc(skv + s * kStageBytes, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, v0 + kk * 128, idO, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&kv_full[0], 0, abort, status, kTimeoutNs, 1);
      for (int t = 0; t < 2 && ok; ++t) {
        tc_fence_after();
        issue_s(t, 0);
        mma_commit(&s_full[t]);
      }
      if (ok) mma_commit(&kv_empty[0]);
      for (int it = 0; it < kIters && ok; ++it) {
        const int iv = 2 * it + 1, ik = 2 * it + 2, sv = iv % kStages, sk = ik % kStages;
        const bool last = it == kIters - 1;
        if (!(ok = mbar_wait(&kv_full[sv], (iv / kStages) & 1, abort, status, kTimeoutNs, 2))) break;
        bool k_ready = false;
        for (int t = 0; t < 2; ++t) {
          if (V != kNoPWait && V != kKVOnly)
            if (!(ok = mbar_wait(&p_full[t], it & 1, abort, status, kTimeoutNs, 3 + t))) break;
          tc_fence_after();
          issue_pv(t, sv, it > 0);
          if (!last) {
            if (!k_ready) {
              if (!(ok = mbar_wait(&kv_full[sk], (ik / kStages) & 1, abort, status, kTimeoutNs, 5))) break;
              k_ready = true;
            }
            tc_fence_after();
            issue_s(t, sk);
            mma_commit(&s_full[t]);
          }
        }
        if (!ok) break;
        mma_commit(&kv_empty[sv]);
        if (!last) mma_commit(&kv_empty[sk]);
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, kTimeoutNs);
    }
  } else if (warp >= 4) {
    const int t = (warp - 4) >> 2;
    const uint32_t tS = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + t * 128;
    bool ok = true;
    for (int li = 0; li < kIters && ok; ++li) {
      if (V == kLaneZeroPoll) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&s_full[t], li & 1, abort, status, kTimeoutNs, 6);
        ok = __shfl_sync(0xffffffffu, w, 0);
      } else if (V != kKVOnly) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], li & 1, abort, status, kTimeoutNs, 6));
      }
      if (!ok) break;
      tc_fence_after();
      if (V == kLoadS) {
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, r[q]);
        tmem_wait_ld();
        if (r[0][0] == 0x12345678u && r[3][31] == 1u) cycles[kCtas + blockIdx.x] = 1;
      }
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
  }
  tc_fence_before();
  __syncthreads();
  const unsigned long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int V>
int run(const char* name, const CUtensorMap& tm, unsigned long long* d, uint32_t* st, const uint8_t* g) {
  cudaMemset(st, 0, 4);
  cudaFuncSetAttribute(issue_loop_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  for (int rep = 0; rep < 3; ++rep) issue_loop_kernel<V><<<kCtas, kThreads, kSmem>>>(tm, d, st, g);
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
  std::printf("{\"variant\": \"%s\", \"status\": %u, \"cycles_per_iteration\": %.0f, \"cycles_per_product\": %.1f}\n",
              name, s, avg / kIters, avg / kIters / 32);
  return s != 0;
}

}  // namespace

int main() {
  unsigned long long* d = nullptr;
  uint32_t* st = nullptr;
  uint8_t* g = nullptr;
  // K/V source: kGroups x 128 stages of 32 KB (80 MB), also viewed as
  // [kGroups][8192][128] bf16 for the tiled loads
  const size_t gbytes = static_cast<size_t>(kGroups) * 2 * kIters * kStageBytes;
  if (cudaMalloc(&d, 2 * kCtas * 8) != cudaSuccess || cudaMalloc(&st, 4) != cudaSuccess ||
      cudaMalloc(&g, gbytes) != cudaSuccess) {
    std::printf("allocation failed\n");
    return 1;
  }
  cudaMemset(g, 0, gbytes);
  CUtensorMap tm;
  if (!fa::host::make_map(&tm, g, 128, 8192, kGroups, 128)) {
    std::printf("tensor map encoding failed\n");
    return 1;
  }
  int bad = 0;
  bad |= run<kHandshakes>("forward handshakes, stand-ins publish P at once", tm, d, st, g);
  bad |= run<kLaneZeroPoll>("stand-ins poll with lane 0", tm, d, st, g);
  bad |= run<kLoadS>("stand-ins also load S", tm, d, st, g);
  bad |= run<kNoPWait>("issuer does not wait for P", tm, d, st, g);
  bad |= run<kKVOnly>("issuer waits for K/V only", tm, d, st, g);
  bad |= run<kBulkKV>("K/V by 32 KB bulk copies from L2/HBM", tm, d, st, g);
  bad |= run<kTmaKV>("K/V by the forward's tiled TMA loads", tm, d, st, g);
  cudaFree(d);
  cudaFree(st);
  cudaFree(g);
  return bad;
}
