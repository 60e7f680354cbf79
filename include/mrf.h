/*
 * mrf.h - C ABI of the Mel-Band RoFormer core forward on NVIDIA B200 (sm_100a).
 *
 * The library computes the network between STFT and iSTFT of Mel-Band RoFormer:
 * a complex stereo STFT in, per-bin complex masks out.  The contract follows the model
 * card "musetric/vocal-separation-roformer-onnx", section "Signature": stft_repr float32
 * [B, F*2, T, 2] (batch, freq*2 + channel, time, re/im) in, masks float32 of the same
 * shape out, "already gathered/averaged" from the mel bands.  The method is described in
 * "Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility", section
 * "The forward chain" (mel-band gather, BandSplit, depth x (time transformer, band
 * transformer), mask estimator, overlap scatter-add and average), and as a GPU-oriented
 * rewrite in "@audio/neural-separate 0.4.0 → 0.5.0", package/scripts/export-roformer.py,
 * class Core.
 *
 * Conventions for every entry point:
 *  - A status code is returned; nothing is thrown, nothing aborts.  mrf_last_error()
 *    gives a text for the last failure.
 *  - Host pointers are read during the call only; the caller keeps ownership.
 *  - Device pointers (stft_repr, masks) are owned by the caller and must stay valid until
 *    the work queued on the stream has finished.
 *  - A handle may be used by one host thread at a time.
 */
#ifndef MRF_H
#define MRF_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MRF_OK = 0,
  MRF_EINVAL = -1,        /* null pointer or value out of range */
  MRF_ESHAPE = -2,        /* B or T outside [1, max_batch] x [1, max_frames], or a weight shape mismatch */
  MRF_ENOMEM = -3,        /* device or host allocation failed (nothing leaked) */
  MRF_ECUDA = -4,         /* a CUDA runtime call failed; mrf_last_error has its text */
  MRF_EUNSUPPORTED = -5,  /* configuration the kernels do not implement */
  MRF_ETIMEOUT = -6,      /* a device-side bounded wait expired; the kernel returned early */
  MRF_EWEIGHTS = -7       /* a required weight is missing, duplicated or has the wrong dtype */
} mrf_status;

typedef enum {
  MRF_FP16 = 0,           /* fp16 operands, fp32 accumulation on tcgen05 tensor cores; the residual
                             stream between the GEMMs is stored in fp16 */
  MRF_BF16 = 1,           /* the same schedule with bf16 operands and activations (weights rounded
                             to bf16 once), fp32 accumulation; the residual stream also keeps an
                             fp32 master copy */
  MRF_FP32_DEBUG = 2      /* fp32 CUDA-core schedule, unfused, for debugging and tight parity */
} mrf_compute;

typedef enum { MRF_DTYPE_F32 = 0, MRF_DTYPE_F16 = 1 } mrf_dtype;

/* Model configuration: the fields of the checkpoint's config.json.  All sizes explicit. */
typedef struct {
  int sample_rate;       /* 44100: defines the Slaney mel band edges */
  int n_fft;             /* 2048 -> F = n_fft/2 + 1 = 1025 bins */
  int audio_channels;    /* 2 (stereo; rows are f*2 + s) */
  int num_bands;         /* 60 mel bands */
  int dim;               /* 384 */
  int depth;             /* 6 axial blocks, each a time and a band transformer */
  int heads;             /* 8 */
  int dim_head;          /* 64: depth of q and k per head (and of v unless dim_head_v is set) */
  int ff_mult;           /* 4: feed-forward inner width ff_mult*dim */
  int mask_hidden;       /* 4*dim: hidden width of the mask MLP */
  int mask_depth;        /* 2: tanh layers of the mask MLP before its GLU layer */
  int num_stems;         /* 1..4: one mask estimator per stem over the shared trunk */
  int zero_dc;           /* 0: DC rows averaged like any other; 1: DC mask weight 0 */
  int max_batch;         /* workspace is sized for max_batch x max_frames at create */
  int max_frames;
  float rope_theta;      /* 10000 */
  int compute;           /* mrf_compute */
  int ff_act;            /* feed-forward activation: 0 GELU (the pages' models); 1 GEGLU, a variant
                            whose first projection is [2*ff, dim] with halves (value, gate) and
                            whose hidden is value * gelu(gate) */
  int dim_head_v;        /* width of v per head; 0: dim_head.  A value below dim_head gives the
                            attention whose q and k are deeper than v ("evaluation.md",
                            section "BS PolarFormer: the same quality for a quarter of the
                            arithmetic": q and k 128 deep against v 64; rotary positions on q and
                            k): to_qkv is then [heads*(2*dim_head + dim_head_v), dim] with
                            features q (head, d), k (head, d), v (head, d), and to_out is
                            [dim, heads*dim_head_v].  The softmax scale stays dim_head^-1/2. */
} mrf_config;

/* One named weight, PyTorch [out, in] layout, contiguous, in host memory. */
typedef struct {
  const char *name;      /* checkpoint path, e.g. "layers.0.1.layers.0.0.to_qkv.weight" */
  int dtype;             /* mrf_dtype */
  int ndim;              /* 1 or 2 */
  int64_t shape[4];
  const void *host_data;
} mrf_tensor;

typedef struct mrf_handle mrf_handle;

/*
 * mrf_create - validate the configuration and the weight table, build the band tables
 * (Slaney mel bank binarised, DC into band 0, Nyquist into the last band: "Mel-Band
 * RoFormer — architecture, inference hot path & RTX 3050 feasibility", section "The
 * mel-band split, exactly"), repack and upload the weights, allocate the workspace for
 * max_batch x max_frames on the current device.
 *
 * Weight names (n_w entries, any order): for each band k,
 *   band_split.to_features.{k}.0.gamma [d_in_k], .1.weight [dim, d_in_k], .1.bias [dim];
 * for each block l and axis a (0 = time, 1 = band), under layers.{l}.{a}.:
 *   layers.0.0.norm.gamma [dim], layers.0.0.to_qkv.weight [heads*(2*dim_head + dv), dim],
 *   layers.0.0.to_gates.weight [heads, dim], layers.0.0.to_gates.bias [heads],
 *   layers.0.0.to_out.0.weight [dim, heads*dv] (dv = dim_head_v, or dim_head when 0),
 *   layers.0.1.net.0.gamma [dim], layers.0.1.net.1.weight [ff, dim], .net.1.bias [ff],
 *   layers.0.1.net.4.weight [dim, ff], .net.4.bias [dim], norm.gamma [dim];
 * for each stem s and band k: mask_estimators.{s}.to_freqs.{k}.0.{0,2,4}.{weight,bias}.
 * d_in_k = 2 * bins_k * audio_channels.  Weights are host memory owned by the caller and
 * are not referenced after the call.  On failure *out is NULL and nothing is leaked.
 * Errors: MRF_EINVAL, MRF_EUNSUPPORTED, MRF_EWEIGHTS, MRF_ESHAPE, MRF_ENOMEM, MRF_ECUDA.
 */
mrf_status mrf_create(const mrf_config *cfg, const mrf_tensor *w, int n_w, mrf_handle **out);

/*
 * mrf_forward - masks = core(stft_repr), queued on `stream` (a cudaStream_t; NULL is the
 * legacy default stream).  stft_repr: device float32 [B, F*C, T, 2], contiguous, 16-byte
 * aligned; masks: device float32 [B, num_stems, F*C, T, 2] (for one stem the shape of
 * stft_repr), must not overlap stft_repr.  B in [1, max_batch], T in [1, max_frames].
 * Arguments are checked before anything is launched; on error nothing is queued.
 * Asynchronous: returns once the work is queued.  Device-side failures (a bounded wait
 * that expired) surface through mrf_sync_status.
 */
mrf_status mrf_forward(mrf_handle *h, const float *stft_repr, float *masks, int B, int T,
                       void *stream);

/*
 * mrf_forward_separate - the separated spectra: the forward's masks multiplied into the
 * complex stft_repr, spec[b, s, r, t] = masks[b, s, r, t] * stft_repr[b, r, t] (complex
 * product of the (re, im) pairs), computed in the overlap-average kernel so the masks are
 * never written ("Mel-Band RoFormer — architecture, inference hot path & RTX 3050
 * feasibility", section "The forward chain": multiply the original complex STFT).  Same arguments,
 * layout, checks and errors as mrf_forward, with spec in place of masks.
 */
mrf_status mrf_forward_separate(mrf_handle *h, const float *stft_repr, float *spec, int B, int T,
                                void *stream);

/*
 * mrf_stft - the model's STFT ("Mel-Band RoFormer — architecture, inference hot path & RTX
 * 3050 feasibility", section "The forward chain": torch.stft, periodic Hann window of n_fft,
 * center=True with reflect padding of n_fft/2, unnormalised).  audio: device float32
 * [B, C, L] (C = audio_channels), L > n_fft/2; stft_repr: device float32 [B, (n_fft/2+1)*C,
 * 1 + L/hop, 2], row f*C + c, (re, im).  n_fft must be a power of two <= 4096.  Queued on
 * `stream`.  Errors: MRF_EINVAL, MRF_ESHAPE, MRF_EUNSUPPORTED, MRF_ENOMEM, MRF_ECUDA.
 */
mrf_status mrf_stft(mrf_handle *h, const float *audio, float *stft_repr, int B, int L, int hop, void *stream);

/*
 * mrf_istft - torch.istft of the same STFT: per frame the inverse real FFT times the window,
 * overlap-added at hop, divided by the overlap-added squared window; the first n_fft/2
 * samples dropped, `length` kept.  spec: device float32 [S, (n_fft/2+1)*C, T, 2]; audio:
 * device float32 [S, C, length].  Allocates (once, grown on demand) an S*C*T*n_fft scratch.
 */
mrf_status mrf_istft(mrf_handle *h, const float *spec, float *audio, int S, int T, int hop, int length,
                     void *stream);

/*
 * mrf_separate_audio - full separation of one mix: the chunk loop of "Mel-Band RoFormer —
 * ...", section "Verified inference hot path" (8 s chunks at a stride of 0.9 chunk; the mix
 * reflect-padded by the border chunk - stride when longer than two borders; a short last chunk
 * padded by reflection when more than half a chunk remains, by zeros otherwise; linear fades
 * of chunk/10 samples, the first chunk's fade-in and the last chunk's fade-out forced to 1;
 * out += estimate * window, counter += window; out / max(counter, 1e-8), border cropped),
 * each chunk through mrf_stft, mrf_forward_separate and mrf_istft, up to min(max_batch, 16)
 * chunks per forward.  mix: device float32 [C, L]; stems: device float32 [num_stems, C, L].
 * max_frames must hold 1 + 8 sample_rate / hop frames.  Allocates its buffers on first use
 * (grown on demand, freed by mrf_destroy).
 */
mrf_status mrf_separate_audio(mrf_handle *h, const float *mix, float *stems, int L, int hop, void *stream);

/*
 * mrf_separate_audio_chunked - mrf_separate_audio with a chunk of chunk_samples samples instead of
 * 8 s (0: 8 s), the stride, border and fades scaling with it (stride 0.9 chunk, fades chunk / 10).
 * The pages fix the 8 s chunk of their checkpoints and leave the chunk length open ("Mel-Band
 * RoFormer — ...", section "Gaps and open questions"); this entry point serves that sweep.
 * max_frames must hold 1 + chunk_samples / hop frames.  MRF_EINVAL for chunk_samples below 10 or
 * not above n_fft / 2; otherwise as mrf_separate_audio.
 */
mrf_status mrf_separate_audio_chunked(mrf_handle *h, const float *mix, float *stems, int L, int hop,
                                      int chunk_samples, void *stream);

/*
 * mrf_forward_host - the same forward from and to HOST memory: copies stft_repr to the
 * device, runs mrf_forward, copies the masks back ([B, num_stems, F*C, T, 2] floats), and
 * waits for the stream.  For the
 * fastest copies the host buffers should be pinned (cudaHostAlloc / torch pin_memory).
 */
mrf_status mrf_forward_host(mrf_handle *h, const float *stft_repr_host, float *masks_host,
                            int B, int T, void *stream);

/*
 * mrf_forward_host_async - mrf_forward_host without the wait, for a caller that feeds a
 * stream of inputs from host memory (a file or a live source cut into windows): each call
 * enqueues the host-to-device copy of stft_repr_host, the forward and the device-to-host copy
 * of the masks, and returns.  Copies run on two streams of the handle's own (one per
 * direction) and the forward on `stream`; the handle keeps two device input/output slots that
 * calls use in turn, so call k+1's input copy and call k-1's output copy run while call k
 * computes.  Events order the three: a slot's input is overwritten only after the forward that
 * read it ended, and its output only after its copy to the host ended.  (The pages have no
 * counterpart: this is an integration entry point, not a step of the method.)
 *
 * Shapes and layouts as for mrf_forward_host.  Ownership: the caller keeps both host buffers
 * alive and unchanged (stft_repr_host) and unread (masks_host) until mrf_host_join's wait has
 * returned.  Calls between two joins form a batch: the batch's first copy starts after the work
 * enqueued on `stream` before that call (so CUDA events recorded on `stream` before the batch and
 * after its join bracket every copy); a later call's copy starts as soon as its slot is free,
 * possibly before work enqueued on `stream` since the batch began has run, so stft_repr_host must
 * hold its data when the call is made.  For copies that overlap compute both
 * buffers must be pinned (cudaHostAlloc / torch pin_memory): a pageable output buffer makes the
 * copy wait for its forward inside the call.  Not for use while `stream` is being captured.
 * Errors: MRF_EINVAL / MRF_ESHAPE for bad arguments (nothing enqueued), MRF_ECUDA if a copy or
 * the forward could not be enqueued; a device-side expired wait surfaces at mrf_sync_status.
 */
mrf_status mrf_forward_host_async(mrf_handle *h, const float *stft_repr_host, float *masks_host,
                                  int B, int T, void *stream);

/*
 * mrf_host_join - makes `stream` wait (on the device; the host does not block) until every
 * copy that mrf_forward_host_async has enqueued so far has ended, and closes the batch (the
 * next call's copy again follows the work on its stream).  After it, a
 * cudaStreamSynchronize of `stream` (or mrf_sync_status, which does one and checks the status
 * word) means every masks_host buffer of those calls holds its result.  Work enqueued on
 * `stream` after the join is ordered after those copies, so CUDA events recorded on `stream`
 * around a batch of calls and the join time the whole pipeline, copies included.  A join with
 * no call pending does nothing.  Errors: MRF_EINVAL for a null handle, MRF_ECUDA if the wait
 * could not be enqueued.
 */
mrf_status mrf_host_join(mrf_handle *h, void *stream);

/*
 * mrf_forward_static - the same fp16 forward as mrf_forward, for callers that must not
 * allocate device memory while they run the model: a real-time audio callback that may not
 * block in the allocator, or a host framework that owns every device allocation and
 * forbids others during processing.  (The pages have no counterpart: this is an
 * integration entry point, not a step of the method.)
 *
 * The per-call workspace lives in a 64 MiB array compiled into the library (every device
 * that loads the library holds it until the process exits); nothing is allocated by this
 * call: no cudaMalloc, no cudaFree, no graph instantiation (it launches eagerly).  The
 * handle must come from mrf_create with compute = MRF_FP16, and its whole workspace for
 * max_batch x max_frames must fit in 64 MiB, else MRF_ESHAPE with the size in the message
 * (the tiny model fits at T <= ~2000; the vocals model only at a few tens of frames).
 * stft_repr and masks as for mrf_forward; the handle's device must be current.
 *
 * Each call looks up the array's device address (cudaGetSymbolAddress, which allocates
 * nothing) with the handle's device current; the first lookup on a device may load the
 * library's device code there, so make the first call before any stream capture.  Every
 * call uses the same array, which keeps the last call's contents: each call clears the
 * accumulators it needs at zero; rows past this call's B*T may hold an earlier call's bytes,
 * which feed only rows that are dropped.  Calls that overlap on the GPU, from any handle or
 * thread, race and corrupt each other's results: serialise them (one stream, or events).
 * This call always writes masks (never the separated spectra of mrf_forward_separate), and
 * mrf_debug_buffer does not read its buffers (it returns MRF_EINVAL after it).
 */
mrf_status mrf_forward_static(mrf_handle *h, const float *stft_repr, float *masks, int B, int T,
                              void *stream);

/*
 * mrf_sync_status - wait for `stream`, then report the device status word: MRF_OK, or
 * MRF_ETIMEOUT if a kernel's bounded wait expired (the word is cleared on read), or
 * MRF_ECUDA for a CUDA error.
 */
mrf_status mrf_sync_status(mrf_handle *h, void *stream);

/* mrf_destroy - free everything the handle owns.  NULL is a no-op. */
void mrf_destroy(mrf_handle *h);

/* Text of the handle's last error, or of the calling thread's last create/table error for NULL. */
const char *mrf_last_error(const mrf_handle *h);

/*
 * mrf_band_tables - host-only test hook: the band tables the library builds for cfg
 * (fields sample_rate, n_fft, audio_channels, num_bands, zero_dc).  Any output may be NULL.
 *   first_bin, last_bin [num_bands]; width [num_bands] (d_in_k);
 *   feat_row [sum d_in]: stft_repr row of each band feature (band order, feature
 *   (j*C + s)*2 + c for the j-th bin of the band); row_weight [F*C]: 1 / (bands covering
 *   the row's bin), 0 at DC when zero_dc.  *n_feat receives sum d_in.
 */
mrf_status mrf_band_tables(const mrf_config *cfg, int32_t *first_bin, int32_t *last_bin,
                           int32_t *width, int32_t *feat_row, float *row_weight, int32_t *n_feat);

/*
 * mrf_chunk_plan - host-only test hook: the geometry mrf_separate_audio_chunked uses for a mix of L
 * samples at sample_rate with chunks of chunk_samples samples (0: 8 s; no device work, no
 * handle).  *chunk = chunk_samples (or 8 * sample_rate), the stride 0.9 chunk (truncated), *border
 * = chunk - stride when L > 2 * (chunk - stride) (the mix is then reflect-padded by it on both
 * sides) else 0, *padded_length = L + 2 * border, and chunks at offsets 0, stride, 2 stride, ...
 * below padded_length: off[i], valid[i] = min(chunk, padded_length - off[i]) samples, mode[i] = 0
 * (full), 1 (tail padded by reflection: more than half a chunk valid) or 2 (tail padded by zeros).
 * Writes at most max_chunks entries of each array (any array may be NULL); *n_chunks receives the
 * count.  MRF_EINVAL for sample_rate < 1, L < 2, chunk_samples < 0 or in 1..9, or a NULL scalar
 * output.
 */
mrf_status mrf_chunk_plan(int sample_rate, int chunk_samples, int L, int *chunk, int *border, int *padded_length,
                          int *n_chunks, int32_t *off, int32_t *valid, int32_t *mode, int max_chunks);

/* Kernel timing, for measurement.  When enabled, mrf_forward launches eagerly (no CUDA
 * graph) and records a CUDA event pair around every kernel on the forward's stream;
 * mrf_kernel_times waits for the events and returns, per kernel kind, the number of
 * launches and the summed milliseconds since the last reset. */
typedef struct { char name[32]; int launches; double ms; } mrf_kernel_time;
mrf_status mrf_set_timing(mrf_handle *h, int enable);
mrf_status mrf_kernel_times(mrf_handle *h, mrf_kernel_time *out, int max_n, int *n_out);

/* Enable (1, default) or disable (0) CUDA graph capture of the forward schedule. */
mrf_status mrf_set_graph(mrf_handle *h, int enable);

/*
 * mrf_debug_stall_next - test hook of the failure path: in the next fp16 forward, CTA 0 of the
 * first tensor-core GEMM issues no loads (a flag nothing sets), so its bounded waits expire
 * (about 2 s), record their site in the device status word and return; the forward's other
 * work runs on.  mrf_sync_status then returns MRF_ETIMEOUT and clears the status word, and the
 * handle stays usable.  The stalled forward runs without a CUDA graph, so no captured graph
 * holds the stall.  No fault, trap or hang is involved.
 */
mrf_status mrf_debug_stall_next(mrf_handle *h);

/*
 * mrf_debug_buffer - test hook: wait for the device, then copy the start of an internal
 * buffer of the last forward to host memory.  "X": the residual stream after the last
 * transformer, float32 [B*T*num_bands, dim], token (b*T + t)*num_bands + k; "M" (MRF_FP32_DEBUG
 * only: the fp16 schedule averages the mask features into the masks without storing them): the
 * mask estimator output before the overlap average, float32 [B*T, sum d_in].  At most
 * max_bytes are copied; *bytes_out receives the number copied.  MRF_EINVAL when no forward
 * has run, or when the last one was mrf_forward_static (its buffers are not the handle's).
 */
mrf_status mrf_debug_buffer(mrf_handle *h, const char *name, void *host_dst, size_t max_bytes,
                            size_t *bytes_out);

/* Number of kernels one mrf_forward launches for (B, T). */
int mrf_launches_per_forward(const mrf_handle *h, int B, int T);

#ifdef __cplusplus
}
#endif
#endif /* MRF_H */
