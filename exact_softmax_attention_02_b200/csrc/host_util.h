// Host-side helpers shared by the library's translation units (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fa.h"

namespace fa {
namespace host {

// message behind fa_last_cuda_error(), per calling thread (defined in fa_fwd.cu)
extern thread_local char g_last_error[256];
// fa_set_debug() state (defined in fa_fwd.cu)
extern unsigned int g_debug_flags;
extern unsigned long long g_timeout_ns;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;

inline unsigned long long wait_timeout_ns() { return g_timeout_ns ? g_timeout_ns : kDefaultTimeoutNs; }

inline fa_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  return FA_ERR_CUDA;
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [BH][N][d] bf16 viewed as a 3-D tensor (d fastest); boxes of 64 x box_rows
// x 1 with the 128-byte swizzle.  Rows past N read as zero and are not stored.
inline bool make_map(CUtensorMap* map, const void* base, int d, int N, int BH, int box_rows) {
  auto enc = encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// make_map through a small per-thread cache.  A tensor map holds only the
// base address, the extents, the strides and the box, so an entry keyed by
// exactly those stays valid for as long as the process runs, whatever happens
// to the memory in between (a buffer freed and reallocated at the same address
// with the same shape gets the same map).  Per thread, so no lock is taken.
inline bool make_map_cached(CUtensorMap* map, const void* base, int d, int N, int BH, int box_rows) {
  struct Entry {
    const void* base;
    int d, N, BH, box_rows;
    unsigned stamp;
    CUtensorMap map;
  };
  constexpr int kEntries = 16;
  thread_local Entry cache[kEntries] = {};
  thread_local unsigned clock = 0;
  if (++clock == 0) ++clock;  // 0 marks an empty entry
  int victim = 0;
  for (int i = 0; i < kEntries; ++i) {
    Entry& e = cache[i];
    if (e.stamp != 0 && e.base == base && e.d == d && e.N == N && e.BH == BH && e.box_rows == box_rows) {
      e.stamp = clock;
      *map = e.map;
      return true;
    }
    if (e.stamp < cache[victim].stamp) victim = i;
  }
  if (!make_map(map, base, d, N, BH, box_rows)) return false;
  Entry& e = cache[victim];
  e.base = base;
  e.d = d;
  e.N = N;
  e.BH = BH;
  e.box_rows = box_rows;
  e.stamp = clock;
  e.map = *map;
  return true;
}

inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// FA_OK when the current device is an sm_100 GPU.
inline fa_status require_sm100() {
  static std::mutex mu;
  static signed char known[64] = {};  // 0 unknown, 1 yes, -1 no
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (known[dev] == 0) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    known[dev] = (major == 10) ? 1 : -1;
  }
  return known[dev] == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

}  // namespace host
}  // namespace fa
