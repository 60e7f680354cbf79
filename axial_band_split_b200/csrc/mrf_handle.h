// The handle behind the C ABI: configuration, band tables, device weights, workspace,
// captured CUDA graphs and kernel-timing events.
#pragma once
#include <cuda_runtime.h>

#include <map>
#include <string>
#include <vector>

#include "mrf_internal.h"

namespace mrf {

struct TrF32 {  // one transformer, fp32 (debug schedule)
  float *g_attn = nullptr, *wqkv = nullptr, *wg = nullptr, *bg = nullptr, *wo = nullptr;
  float *g_ff = nullptr, *w1 = nullptr, *b1 = nullptr, *w2 = nullptr, *b2 = nullptr, *g_out = nullptr;
};

struct MaskF32 {  // the mask heads, one per stem: w[stem][layer]
  std::vector<std::vector<float *>> w, b;
  std::vector<float *> w_last, b_last;
  SimtGroup *g_first = nullptr, *g_mid = nullptr, *g_last = nullptr;
};

struct Workspace {  // fp32 debug schedule
  float *X = nullptr, *Xa = nullptr, *QKV = nullptr, *G = nullptr, *Q = nullptr, *K = nullptr,
        *V = nullptr, *O = nullptr, *Hf = nullptr, *H1 = nullptr, *H2 = nullptr, *Mg = nullptr;
};

struct GraphKey {
  int B, T;
  const float *in;
  float *out;
  bool apply;  // masks applied to stft_repr (mrf_forward_separate) rather than written
  bool operator==(const GraphKey &o) const {
    return B == o.B && T == o.T && in == o.in && out == o.out && apply == o.apply;
  }
};

struct GraphEntry {
  GraphKey key;
  cudaGraphExec_t exec;
  int launches;
};

struct PendingTiming {
  const char *name;
  cudaEvent_t e0, e1;
};

struct Fp16State;  // sched_fp16.cu

// A weight read from the caller's table, converted to fp32.
struct HostW {
  std::vector<float> v;
  std::vector<int64_t> shape;
};
using WeightMap = std::map<std::string, HostW>;

}  // namespace mrf

struct mrf_handle {
  mrf_config cfg{};
  mrf::BandTables tab;
  int device = 0;
  std::string err;

  // allocation bookkeeping (every device buffer is freed by mrf_destroy)
  int fail_alloc_after = -1;
  int n_allocs = 0;
  std::vector<void *> allocs;
  void *alloc_bytes(size_t bytes);
  template <class T>
  T *alloc(size_t n) { return static_cast<T *>(alloc_bytes(n * sizeof(T))); }
  bool upload(void *dst, const void *src, size_t bytes);

  // tables
  int32_t *d_feat_row = nullptr, *d_feat_c = nullptr, *d_src0 = nullptr, *d_src1 = nullptr;
  float *d_row_weight = nullptr;
  mrf::BandDesc *d_bands = nullptr;
  std::vector<mrf::BandDesc> bands;
  int max_width = 0;
  float2 *d_rope = nullptr;
  float *w_bs = nullptr, *b_bs = nullptr;
  unsigned *status = nullptr;

  // fp32 debug schedule
  std::vector<mrf::TrF32> trf;
  mrf::MaskF32 mf;
  mrf::SimtGroup *d_tgroups = nullptr;
  mrf::Workspace ws;

  // fp16 tensor-core schedule
  mrf::Fp16State *f16 = nullptr;

  // execution
  bool timing = false, use_graph = true;
  bool apply_masks = false;  // the schedule being recorded multiplies stft_repr by the masks
  bool stall_test = false;   // test hook: the next fp16 schedule's first GEMM stalls (bounded)
  cudaStream_t cur_stream = nullptr, cap_stream = nullptr;
  std::vector<mrf::PendingTiming> pending;
  std::vector<mrf::GraphEntry> graphs;
  int launch_counter = 0, last_launches = -1, last_B = -1, last_T = -1;
  bool last_static = false;  // the last forward ran in mrf_forward_static's shared scratch
  // host-buffer entry points: two device input/output slots used in turn, one copy stream
  // per direction, and the events that order copies and forwards (mrf_api.cu, host_pipe)
  float *io_in[2] = {nullptr, nullptr}, *io_out[2] = {nullptr, nullptr};
  cudaStream_t h2d_stream = nullptr, d2h_stream = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_fwd[2] = {nullptr, nullptr},
              ev_out[2] = {nullptr, nullptr}, ev_join = nullptr, ev_start = nullptr;
  int io_next = 0;
  bool pipe_open = false;  // a batch of host-buffer calls has begun and not been joined
  // spectral front / back end (signal_api.cu): FFT tables of n_fft and grow-only scratch
  float2 *d_tw = nullptr;
  float *d_win = nullptr;
  std::vector<std::pair<void *, size_t>> sig_scratch;
  std::string sched_error;  // set by a schedule that refused to launch

  void begin(const char *name);
  void end();
};

namespace mrf {
using Handle = ::mrf_handle;

// sched_fp16.cu
std::string fp16_supported(const mrf_config &c, const BandTables &t);
mrf_status pack_fp16(mrf_handle *h, WeightMap &W);
void schedule_fp16(mrf_handle *h, const float *in, float *out, int B, int T);
void destroy_fp16(mrf_handle *h);
bool debug_buffer_fp16(mrf_handle *h, const std::string &name, const void **ptr, size_t *bytes);

// The fp16 schedule's per-forward workspace pointers, and their layout in one
// caller-provided region (sched_fp16.cu); used by mrf_forward_static.
struct Fp16Workspace {
  float *ss;
  __half *Xh, *QKV, *O, *Hh, *H1, *H2, *A_bs;
  float *ssx, *ssg;
};
size_t fp16_workspace_layout(mrf_handle *h, void *base, bool apply, Fp16Workspace *saved, size_t *qkv_offset,
                             size_t *qkv_bytes);
void fp16_restore_workspace(mrf_handle *h, const Fp16Workspace &s);
}  // namespace mrf
