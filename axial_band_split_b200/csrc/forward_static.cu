// mrf_forward_static: the fp16 forward with its per-call workspace in a fixed device array
// compiled into the library, for callers that must not allocate device memory when they
// run the model (for instance a real-time audio callback, or a host framework that owns
// every device allocation and forbids others while it processes).  The handle (weights)
// is created beforehand with mrf_create; this call itself allocates nothing.
#include <cuda_runtime.h>

#include <cstdio>
#include <string>

#include "mrf_handle.h"

namespace mrf {

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB on every device that loads the library

// Zero at load; afterwards it keeps whatever the last call left in it.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the array on the current device.  Looked up on every call (the lookup
// allocates nothing), so no address outlives the context it was taken in.
cudaError_t scratch_address(void **out) { return cudaGetSymbolAddress(out, g_static_scratch); }

}  // namespace
}  // namespace mrf

using namespace mrf;

extern "C" mrf_status mrf_forward_static(mrf_handle *h, const float *in, float *out, int B, int T, void *stream) {
  if (!h) return MRF_EINVAL;
  if (!in || !out) { h->err = "null stft_repr or masks pointer"; return MRF_EINVAL; }
  if (h->cfg.compute != MRF_FP16 || !h->f16) {
    h->err = "mrf_forward_static runs the fp16 schedule only";
    return MRF_EUNSUPPORTED;
  }
  if (B < 1 || B > h->cfg.max_batch || T < 1 || T > h->cfg.max_frames) {
    h->err = "B or T outside [1, max_batch] x [1, max_frames]";
    return MRF_ESHAPE;
  }
  if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15) {
    h->err = "stft_repr and masks must be 16-byte aligned";
    return MRF_EINVAL;
  }
  const size_t io = (size_t)B * h->tab.n_freqs * h->tab.channels * T * 2 * sizeof(float);
  const char *a = reinterpret_cast<const char *>(in), *b = reinterpret_cast<const char *>(out);
  if (a < b + io * h->cfg.num_stems && b < a + io) { h->err = "stft_repr and masks overlap"; return MRF_EINVAL; }
  const size_t need = fp16_workspace_layout(h, nullptr, false, nullptr, nullptr, nullptr);
  if (need > kStaticScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "the handle's workspace (%.1f MiB for max_batch x max_frames = %d x %d) exceeds the %zu MiB static "
             "scratch of mrf_forward_static; create the handle with a smaller max_batch x max_frames",
             need / 1048576.0, h->cfg.max_batch, h->cfg.max_frames, kStaticScratchBytes >> 20);
    h->err = buf;
    return MRF_ESHAPE;
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    h->err = "the handle's device must be current";
    return MRF_EINVAL;
  }
  void *base = nullptr;
  e = scratch_address(&base);
  if (e != cudaSuccess) {
    cudaGetLastError();
    h->err = std::string("cudaGetSymbolAddress failed: ") + cudaGetErrorString(e);
    return MRF_ECUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaGetLastError();
  // The schedule clears the accumulators it needs at zero (the row sums of squares) on every
  // call.  Rows of the activation buffers past this call's B*T keep what an earlier call left
  // (possibly another handle's, in another layout): ragged GEMM tiles read them, but a GEMM
  // row only feeds the same output row, which the epilogue drops, so they never reach a
  // result.  The masks are written, never multiplied into stft_repr (apply_masks is a
  // property of the handle's last mrf_forward_separate, not of this call).
  Fp16Workspace saved{};
  fp16_workspace_layout(h, base, true, &saved, nullptr, nullptr);
  const bool timing = h->timing, apply = h->apply_masks;
  h->timing = false;
  h->apply_masks = false;
  h->cur_stream = st;
  h->launch_counter = 0;
  h->sched_error.clear();
  schedule_fp16(h, in, out, B, T);
  h->timing = timing;
  h->apply_masks = apply;
  fp16_restore_workspace(h, saved);
  h->last_launches = h->launch_counter;
  h->last_B = B;
  h->last_T = T;
  h->last_static = true;
  if (!h->sched_error.empty()) { h->err = h->sched_error; return MRF_ECUDA; }
  e = cudaGetLastError();
  if (e != cudaSuccess) { h->err = std::string("kernel launch: ") + cudaGetErrorString(e); return MRF_ECUDA; }
  return MRF_OK;
}
