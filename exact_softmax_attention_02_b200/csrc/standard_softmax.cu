// Row softmax over a materialised score matrix: the middle step of standard
// (non-fused) attention, kept as a comparator for the fused kernel.
//
// Standard attention writes the N x N score matrix to global memory, reads it
// back for the softmax, writes the probabilities, and reads them again for
// the product with V (sadullah.online "Flash Attention Explained", "The real
// bottleneck isn't FLOPs, it's memory movement"; interactiveml.org: standard
// implementations write the square table of scores to HBM and read it back).
// This kernel is that softmax: fp32 scores S [BH][N][N] in, bf16
// probabilities P [BH][N][N] and the row log-sum-exp out.  The two products
// around it are plain library GEMMs.
//
// One CTA per row.  Pass 1 runs over the row once with a per-thread running
// maximum and denominator (rescaled when the maximum rises), then combines
// the threads' (m, l) pairs; pass 2 reads the row again (mostly from L2) and
// writes p = e^(scale*s - m) / l.  Causal rows stop at the diagonal; the
// masked tail of P is written as zeros.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>

#include "fa.h"

namespace fa_std {

constexpr int kThreads = 256;

__device__ __forceinline__ void combine(float& m, float& l, float m2, float l2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // both empty
  l = (m == -INFINITY ? 0.f : l * exp2f(m - mn)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - mn));
  m = mn;
}

__global__ void __launch_bounds__(kThreads)
    softmax_rows_kernel(const float* __restrict__ S, __nv_bfloat16* __restrict__ P,
                        float* __restrict__ LSE, int N, float scale_log2, int causal) {
  const long long row_id = blockIdx.x;  // (bh, i) flattened
  const int i = static_cast<int>(row_id % N);
  const float* s = S + row_id * N;
  __nv_bfloat16* p = P + row_id * N;
  const int n_valid = causal ? i + 1 : N;  // keys 0 .. n_valid-1 are allowed

  // pass 1: running maximum and denominator, log2 units
  float m = -INFINITY, l = 0.f;
  for (int j = threadIdx.x; j < n_valid; j += kThreads) {
    const float x = s[j] * scale_log2;
    if (x > m) {
      l = (m == -INFINITY ? 0.f : l * exp2f(m - x)) + 1.f;
      m = x;
    } else {
      l += exp2f(x - m);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
    combine(m, l, m2, l2);
  }
  __shared__ float sm[kThreads / 32], sl[kThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sm[warp] = m;
    sl[warp] = l;
  }
  __syncthreads();
  m = sm[0];
  l = sl[0];
  for (int w = 1; w < kThreads / 32; ++w) combine(m, l, sm[w], sl[w]);
  const float inv_l = 1.f / l;
  if (threadIdx.x == 0 && LSE != nullptr) LSE[row_id] = (m + log2f(l)) * 0.69314718055994530942f;

  // pass 2: probabilities, two per store
  for (int j = 2 * threadIdx.x; j < N; j += 2 * kThreads) {
    const float x0 = j < n_valid ? exp2f(s[j] * scale_log2 - m) * inv_l : 0.f;
    const float x1 = (j + 1 < n_valid) ? exp2f(s[j + 1] * scale_log2 - m) * inv_l : 0.f;
    if (j + 1 < N) {
      *reinterpret_cast<__nv_bfloat162*>(p + j) = __floats2bfloat162_rn(x0, x1);
    } else {
      p[j] = __float2bfloat16_rn(x0);
    }
  }
}

}  // namespace fa_std

extern "C" fa_status fa_softmax_rows(const float* S, void* P, float* LSE, int BH, int N, float scale,
                                     int causal, void* stream) {
  if (!S || !P) return FA_ERR_NULL;
  if (BH < 1 || N < 1 || !std::isfinite(scale)) return FA_ERR_SHAPE;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(S) & 3u) || (reinterpret_cast<uintptr_t>(P) & 3u) ||
      (LSE && (reinterpret_cast<uintptr_t>(LSE) & 3u)))
    return FA_ERR_ALIGN;
  if ((N & 1) != 0) return FA_ERR_UNSUPPORTED;  // bf16 pairs keep 4-byte alignment per row
  const long long rows = static_cast<long long>(BH) * N;
  if (rows > 0x7fffffffll) return FA_ERR_SHAPE;
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  fa_std::softmax_rows_kernel<<<static_cast<unsigned>(rows), fa_std::kThreads, 0,
                                static_cast<cudaStream_t>(stream)>>>(
      S, static_cast<__nv_bfloat16*>(P), LSE, N, scale_log2, causal);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}
