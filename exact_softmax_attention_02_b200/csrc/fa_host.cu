// Host-buffer forward: Q, K, V in host memory in, O and LSE back to host
// memory, with the copies and the kernels pipelined over groups of heads.
//
// Attention of one (batch, head) pair needs only that pair's Q, K and V
// (lihaoran.work, the opening formula: every output row is a softmax over
// its own head's keys), so the heads can be moved and computed in chunks.
// Three streams per device carry the work: chunk c is copied in on the first
// while chunk c-1 is computed on the second and chunk c-2 is copied out on
// the third.  PCIe is full duplex, so a step costs about the longer of the
// two copy directions instead of the sum of copies and compute.
//
// The library allocates no device memory: the caller passes a device
// workspace that holds the device copies of Q, K, V, O and LSE.  The streams
// and events are created once per device, on first use, and kept.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fa.h"
#include "host_util.h"

namespace fa {
namespace hostpipe {

constexpr int kMaxDevices = 64;
constexpr int kMaxChunks = 64;
constexpr int kDefaultChunks = 8;

struct Pipeline {
  bool ready = false;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kMaxChunks] = {}, kern[kMaxChunks] = {};
};

Pipeline g_pipes[kMaxDevices];
std::mutex g_pipe_mutex;

fa_status make_pipeline(Pipeline& p) {
  if (p.ready) return FA_OK;
  cudaError_t e = cudaSuccess;
  auto mk_stream = [&](cudaStream_t* s) {
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
  };
  auto mk_event = [&](cudaEvent_t* ev) {
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  };
  mk_stream(&p.h2d);
  mk_stream(&p.comp);
  mk_stream(&p.d2h);
  mk_event(&p.start);
  mk_event(&p.done);
  for (int c = 0; c < kMaxChunks; ++c) {
    mk_event(&p.in[c]);
    mk_event(&p.kern[c]);
  }
  if (e != cudaSuccess) return host::cuda_fail(e, "stream/event creation");
  p.ready = true;
  return FA_OK;
}

size_t tensor_bytes(int B, int H, int N, int d) { return static_cast<size_t>(B) * H * N * d * 2; }

}  // namespace hostpipe
}  // namespace fa

extern "C" {

size_t fa_fwd_host_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  const size_t nb = fa::hostpipe::tensor_bytes(B, H, N, d);
  return 4 * nb + static_cast<size_t>(B) * H * N * 4;
}

fa_status fa_fwd_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, float* LSEh,
                      void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
                      int causal, int chunks, void* stream) {
  using namespace fa::hostpipe;
  if (!Qh || !Kh || !Vh || !Oh || !workspace) return FA_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || !std::isfinite(scale)) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return FA_ERR_ALIGN;
  const size_t need = fa_fwd_host_workspace_bytes(B, H, N, d);
  if (workspace_bytes < need) return FA_ERR_WORKSPACE;
  // the host arguments must be host memory (pinned or pageable); the
  // workspace must be device memory
  const void* host_args[5] = {Qh, Kh, Vh, Oh, LSEh};
  for (const void* ptr : host_args) {
    if (ptr == nullptr) continue;
    cudaPointerAttributes at{};
    cudaError_t e = cudaPointerGetAttributes(&at, ptr);
    if (e != cudaSuccess) return fa::host::cuda_fail(e, "cudaPointerGetAttributes");
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return FA_ERR_UNSUPPORTED;
  }
  {
    cudaPointerAttributes at{};
    cudaError_t e = cudaPointerGetAttributes(&at, workspace);
    if (e != cudaSuccess) return fa::host::cuda_fail(e, "cudaPointerGetAttributes");
    if (at.type != cudaMemoryTypeDevice) return FA_ERR_UNSUPPORTED;
  }
  const long long BH = static_cast<long long>(B) * H;
  if (BH > (1ll << 30)) return FA_ERR_SHAPE;
  if (chunks <= 0) chunks = kDefaultChunks;
  if (chunks > kMaxChunks) chunks = kMaxChunks;
  if (chunks > BH) chunks = static_cast<int>(BH);
  const long long per = (BH + chunks - 1) / chunks;  // heads per chunk
  chunks = static_cast<int>((BH + per - 1) / per);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fa::host::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  Pipeline& p = g_pipes[dev];
  fa_status st = make_pipeline(p);
  if (st != FA_OK) return st;

  const size_t nb = tensor_bytes(B, H, N, d);
  const size_t head_bytes = static_cast<size_t>(N) * d * 2;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t *Qd = ws, *Kd = ws + nb, *Vd = ws + 2 * nb, *Od = ws + 3 * nb;
  float* Ld = reinterpret_cast<float*>(ws + 4 * nb);
  const uint8_t* qh = static_cast<const uint8_t*>(Qh);
  const uint8_t* kh = static_cast<const uint8_t*>(Kh);
  const uint8_t* vh = static_cast<const uint8_t*>(Vh);
  uint8_t* oh = static_cast<uint8_t*>(Oh);
  cudaStream_t caller = static_cast<cudaStream_t>(stream);

  // everything starts after the work already queued on the caller's stream
  // (a previous call may still be reading the workspace)
  auto ck = [&](cudaError_t err, const char* what) {
    if (err != cudaSuccess && e == cudaSuccess) {
      e = err;
      fa::host::cuda_fail(err, what);
    }
  };
  ck(cudaEventRecord(p.start, caller), "cudaEventRecord");
  ck(cudaStreamWaitEvent(p.h2d, p.start, 0), "cudaStreamWaitEvent");
  ck(cudaStreamWaitEvent(p.comp, p.start, 0), "cudaStreamWaitEvent");
  ck(cudaStreamWaitEvent(p.d2h, p.start, 0), "cudaStreamWaitEvent");
  if (e != cudaSuccess) return FA_ERR_CUDA;
  // On an error after work was enqueued: join all three streams back into the
  // caller's stream before returning, so that no copy into the caller's host
  // buffers and no read of the workspace outlives what the caller's stream
  // orders after this call.  Errors of these joining calls are not reported
  // over the first one.
  auto fail = [&](fa_status result) {
    cudaEventRecord(p.start, p.h2d);
    cudaStreamWaitEvent(p.d2h, p.start, 0);
    cudaEventRecord(p.start, p.comp);
    cudaStreamWaitEvent(p.d2h, p.start, 0);
    cudaEventRecord(p.done, p.d2h);
    cudaStreamWaitEvent(caller, p.done, 0);
    return result;
  };
  for (int c = 0; c < chunks; ++c) {
    const long long h0 = c * per, h1 = (h0 + per < BH) ? h0 + per : BH;
    const size_t off = static_cast<size_t>(h0) * head_bytes;
    const size_t len = static_cast<size_t>(h1 - h0) * head_bytes;
    ck(cudaMemcpyAsync(Qd + off, qh + off, len, cudaMemcpyHostToDevice, p.h2d), "cudaMemcpyAsync Q");
    ck(cudaMemcpyAsync(Kd + off, kh + off, len, cudaMemcpyHostToDevice, p.h2d), "cudaMemcpyAsync K");
    ck(cudaMemcpyAsync(Vd + off, vh + off, len, cudaMemcpyHostToDevice, p.h2d), "cudaMemcpyAsync V");
    ck(cudaEventRecord(p.in[c], p.h2d), "cudaEventRecord");
    ck(cudaStreamWaitEvent(p.comp, p.in[c], 0), "cudaStreamWaitEvent");
    if (e != cudaSuccess) return fail(FA_ERR_CUDA);
    // the heads of this chunk are one [1][h1-h0][N][d] problem
    st = fa_fwd(Qd + off, Kd + off, Vd + off, Od + off, LSEh ? Ld + h0 * N : nullptr, 1,
                static_cast<int>(h1 - h0), N, d, scale, causal, p.comp);
    if (st != FA_OK) return fail(st);
    ck(cudaEventRecord(p.kern[c], p.comp), "cudaEventRecord");
    ck(cudaStreamWaitEvent(p.d2h, p.kern[c], 0), "cudaStreamWaitEvent");
    ck(cudaMemcpyAsync(oh + off, Od + off, len, cudaMemcpyDeviceToHost, p.d2h), "cudaMemcpyAsync O");
    if (LSEh)
      ck(cudaMemcpyAsync(LSEh + h0 * N, Ld + h0 * N, static_cast<size_t>(h1 - h0) * N * 4,
                         cudaMemcpyDeviceToHost, p.d2h),
         "cudaMemcpyAsync LSE");
    if (e != cudaSuccess) return fail(FA_ERR_CUDA);
  }
  // the caller's stream resumes once every copy out has landed
  ck(cudaEventRecord(p.done, p.d2h), "cudaEventRecord");
  ck(cudaStreamWaitEvent(caller, p.done, 0), "cudaStreamWaitEvent");
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
