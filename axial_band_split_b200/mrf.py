"""Python binding of libmrf (include/mrf.h): argument marshalling only.

Every step of the forward runs in the library's CUDA kernels; PyTorch is used here for
device memory and streams.  The binding raises if libmrf.so is missing or a call fails:
there is no fallback path.

    from axial_band_split_b200 import mrf
    model = mrf.Model(cfg, weights, max_batch=1, max_frames=1100)   # weights: name -> ndarray
    masks = model.forward(stft_repr)            # torch CUDA float32 [B, F*2, T, 2]
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmrf.so")

MRF_FP16 = 0
MRF_BF16 = 1
MRF_FP32_DEBUG = 2
STATUS = {0: "MRF_OK", -1: "MRF_EINVAL", -2: "MRF_ESHAPE", -3: "MRF_ENOMEM", -4: "MRF_ECUDA",
          -5: "MRF_EUNSUPPORTED", -6: "MRF_ETIMEOUT", -7: "MRF_EWEIGHTS"}

# every symbol include/mrf.h declares
EXPORTS = ["mrf_create", "mrf_forward", "mrf_forward_separate", "mrf_stft", "mrf_istft", "mrf_separate_audio",
           "mrf_forward_host", "mrf_forward_host_async", "mrf_host_join", "mrf_sync_status", "mrf_destroy",
           "mrf_last_error", "mrf_band_tables", "mrf_set_timing", "mrf_kernel_times",
           "mrf_set_graph", "mrf_launches_per_forward", "mrf_debug_buffer", "mrf_forward_static",
           "mrf_debug_stall_next", "mrf_chunk_plan", "mrf_separate_audio_chunked"]


class MrfError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class mrf_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "sample_rate", "n_fft", "audio_channels", "num_bands", "dim", "depth", "heads", "dim_head",
        "ff_mult", "mask_hidden", "mask_depth", "num_stems", "zero_dc", "max_batch", "max_frames")] + \
        [("rope_theta", ctypes.c_float), ("compute", ctypes.c_int), ("ff_act", ctypes.c_int),
         ("dim_head_v", ctypes.c_int)]


class mrf_tensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int),
                ("shape", ctypes.c_int64 * 4), ("host_data", ctypes.c_void_p)]


class mrf_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int), ("ms", ctypes.c_double)]


_lib = None


def lib():
    """The loaded libmrf.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: run `python -m axial_band_split_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, V = ctypes.c_void_p, ctypes.c_int, None
        L.mrf_create.argtypes = [ctypes.POINTER(mrf_config), ctypes.POINTER(mrf_tensor), I, ctypes.POINTER(P)]
        L.mrf_create.restype = I
        L.mrf_forward.argtypes = [P, P, P, I, I, P]
        L.mrf_forward.restype = I
        L.mrf_forward_separate.argtypes = [P, P, P, I, I, P]
        L.mrf_forward_separate.restype = I
        L.mrf_stft.argtypes = [P, P, P, I, I, I, P]
        L.mrf_stft.restype = I
        L.mrf_istft.argtypes = [P, P, P, I, I, I, I, P]
        L.mrf_istft.restype = I
        L.mrf_separate_audio.argtypes = [P, P, P, I, I, P]
        L.mrf_separate_audio.restype = I
        L.mrf_separate_audio_chunked.argtypes = [P, P, P, I, I, I, P]
        L.mrf_separate_audio_chunked.restype = I
        L.mrf_forward_static.argtypes = [P, P, P, I, I, P]
        L.mrf_forward_static.restype = I
        L.mrf_forward_host.argtypes = [P, P, P, I, I, P]
        L.mrf_forward_host.restype = I
        L.mrf_forward_host_async.argtypes = [P, P, P, I, I, P]
        L.mrf_forward_host_async.restype = I
        L.mrf_host_join.argtypes = [P, P]
        L.mrf_host_join.restype = I
        L.mrf_sync_status.argtypes = [P, P]
        L.mrf_sync_status.restype = I
        L.mrf_destroy.argtypes = [P]
        L.mrf_destroy.restype = V
        L.mrf_last_error.argtypes = [P]
        L.mrf_last_error.restype = ctypes.c_char_p
        L.mrf_band_tables.argtypes = [ctypes.POINTER(mrf_config)] + [P] * 6
        L.mrf_band_tables.restype = I
        L.mrf_set_timing.argtypes = [P, I]
        L.mrf_set_timing.restype = I
        L.mrf_set_graph.argtypes = [P, I]
        L.mrf_set_graph.restype = I
        L.mrf_kernel_times.argtypes = [P, ctypes.POINTER(mrf_kernel_time), I, ctypes.POINTER(I)]
        L.mrf_kernel_times.restype = I
        L.mrf_debug_buffer.argtypes = [P, ctypes.c_char_p, P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]
        L.mrf_debug_buffer.restype = I
        L.mrf_debug_stall_next.argtypes = [P]
        L.mrf_debug_stall_next.restype = I
        L.mrf_launches_per_forward.argtypes = [P, I, I]
        L.mrf_launches_per_forward.restype = I
        IP = ctypes.POINTER(I)
        L.mrf_chunk_plan.argtypes = [I, I, I, IP, IP, IP, IP, P, P, P, I]
        L.mrf_chunk_plan.restype = I
        _lib = L
    return _lib


def _check(status, handle=None):
    if status != 0:
        raise MrfError(status, lib().mrf_last_error(handle).decode(errors="replace"))


def make_config(cfg, max_batch=1, max_frames=1100, compute=MRF_FP16):
    """mrf_config from any object with the model fields (sample_rate, n_fft, ...)."""
    c = mrf_config()
    c.sample_rate, c.n_fft, c.audio_channels = cfg.sample_rate, cfg.n_fft, cfg.audio_channels
    c.num_bands, c.dim, c.depth, c.heads, c.dim_head = cfg.num_bands, cfg.dim, cfg.depth, cfg.heads, cfg.dim_head
    c.ff_mult, c.mask_hidden, c.mask_depth = cfg.ff_mult, cfg.dim * cfg.mask_hidden_mult, cfg.mask_depth
    c.num_stems, c.zero_dc = cfg.num_stems, int(cfg.zero_dc)
    c.max_batch, c.max_frames = max_batch, max_frames
    c.rope_theta, c.compute = cfg.rope_theta, compute
    c.ff_act = getattr(cfg, "ff_act", 0)
    c.dim_head_v = getattr(cfg, "dim_head_v", 0)
    return c


def band_tables(cfg):
    """The library's band tables for cfg: dict of numpy arrays (first_bin, last_bin, width,
    feat_row, row_weight)."""
    c = make_config(cfg)
    n_feat = ctypes.c_int(0)
    _check(lib().mrf_band_tables(ctypes.byref(c), None, None, None, None, None, ctypes.byref(n_feat)))
    nb, rows = cfg.num_bands, (cfg.n_fft // 2 + 1) * cfg.audio_channels
    out = {"first_bin": np.zeros(nb, np.int32), "last_bin": np.zeros(nb, np.int32),
           "width": np.zeros(nb, np.int32), "feat_row": np.zeros(n_feat.value, np.int32),
           "row_weight": np.zeros(rows, np.float32)}
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().mrf_band_tables(ctypes.byref(c), ptr(out["first_bin"]), ptr(out["last_bin"]),
                                 ptr(out["width"]), ptr(out["feat_row"]), ptr(out["row_weight"]), None))
    return out


def chunk_plan(sample_rate, length, chunk_samples=0):
    """mrf_chunk_plan: the separation loop's geometry for a mix of `length` samples (chunks of
    chunk_samples, 0: 8 s): dict with chunk, border, padded_length and the per-chunk arrays off,
    valid, mode (0 full, 1 reflect tail, 2 zero tail)."""
    vals = [ctypes.c_int(0) for _ in range(4)]
    _check(lib().mrf_chunk_plan(sample_rate, chunk_samples, length, *[ctypes.byref(v) for v in vals], None, None,
                                None, 0))
    n = vals[3].value
    out = {k: np.zeros(n, np.int32) for k in ("off", "valid", "mode")}
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().mrf_chunk_plan(sample_rate, chunk_samples, length, *[ctypes.byref(v) for v in vals],
                                ptr(out["off"]), ptr(out["valid"]), ptr(out["mode"]), n))
    out.update(chunk=vals[0].value, border=vals[1].value, padded_length=vals[2].value)
    return out


def _stream_ptr(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


class Model:
    """A created libmrf handle: weights on the device, workspace for max_batch x max_frames."""

    def __init__(self, cfg, weights, max_batch=1, max_frames=1100, compute=MRF_FP16):
        self.cfg = cfg
        self.rows = (cfg.n_fft // 2 + 1) * cfg.audio_channels
        c = make_config(cfg, max_batch, max_frames, compute)
        keep, table = [], (mrf_tensor * len(weights))()
        for i, (name, a) in enumerate(weights.items()):
            a = np.ascontiguousarray(a)
            if a.dtype not in (np.float32, np.float16):
                a = a.astype(np.float32)
            keep.append(a)
            bname = name.encode()
            keep.append(bname)
            t = table[i]
            t.name = bname
            t.dtype = 0 if a.dtype == np.float32 else 1
            t.ndim = a.ndim
            for d in range(a.ndim):
                t.shape[d] = a.shape[d]
            t.host_data = a.ctypes.data
        h = ctypes.c_void_p()
        _check(lib().mrf_create(ctypes.byref(c), table, len(weights), ctypes.byref(h)))
        self._h = h
        self._host_pending = []  # (input, output) host tensors of forward_host_async calls not yet synced

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            lib().mrf_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check_input(self, x):
        """stft_repr must be a contiguous CUDA float32 [B, F*C, T, 2] of this model's rows."""
        import torch
        assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous(), "stft_repr: contiguous CUDA float32"
        assert x.dim() == 4 and x.shape[1] == self.rows and x.shape[3] == 2, \
            f"stft_repr must be [B, {self.rows}, T, 2], got {tuple(x.shape)}"

    def _check_host_input(self, x):
        """stft_repr for the host-buffer entry points: a contiguous host float32 [B, F*C, T, 2]."""
        import torch
        assert not x.is_cuda and x.dtype == torch.float32 and x.is_contiguous(), "stft_repr: contiguous host float32"
        assert x.dim() == 4 and x.shape[1] == self.rows and x.shape[3] == 2, \
            f"stft_repr must be [B, {self.rows}, T, 2], got {tuple(x.shape)}"

    def _check_out(self, x, out):
        """`out` must hold exactly B * num_stems * rows * T * 2 floats, on x's device."""
        import torch
        B, R, T, _ = x.shape
        need = B * self.cfg.num_stems * R * T * 2
        assert out.dtype == torch.float32 and out.is_contiguous(), "out: contiguous float32"
        assert out.device == x.device and out.is_cuda == x.is_cuda, "out must be on stft_repr's device"
        assert out.numel() == need, f"out holds {out.numel()} floats, the forward writes {need}"

    def _out_like(self, x, out):
        """[B, F*2, T, 2] for one stem, [B, stems, F*2, T, 2] for more."""
        import torch
        if out is not None:
            self._check_out(x, out)
            return out
        B, R, T, two = x.shape
        stems = self.cfg.num_stems
        shape = (B, R, T, two) if stems == 1 else (B, stems, R, T, two)
        return torch.empty(shape, dtype=x.dtype, device=x.device, pin_memory=not x.is_cuda and x.is_pinned())

    def forward(self, stft_repr, out=None, stream=None):
        """masks for a CUDA float32 tensor [B, F*2, T, 2] (queued on `stream`)."""
        self._check_input(stft_repr)
        B, R, T, two = stft_repr.shape
        out = self._out_like(stft_repr, out)
        _check(lib().mrf_forward(self._h, ctypes.c_void_p(stft_repr.data_ptr()),
                                 ctypes.c_void_p(out.data_ptr()), B, T, _stream_ptr(stream)), self._h)
        return out

    def separate(self, stft_repr, out=None, stream=None):
        """mrf_forward_separate: the separated spectra (masks times stft_repr, complex), same
        shape as forward's masks."""
        self._check_input(stft_repr)
        B, R, T, two = stft_repr.shape
        out = self._out_like(stft_repr, out)
        _check(lib().mrf_forward_separate(self._h, ctypes.c_void_p(stft_repr.data_ptr()),
                                          ctypes.c_void_p(out.data_ptr()), B, T, _stream_ptr(stream)), self._h)
        return out

    def stft(self, audio, hop, out=None, stream=None):
        """mrf_stft: CUDA float32 audio [B, C, L] -> stft_repr [B, (n_fft/2+1) C, 1 + L // hop, 2]."""
        import torch
        assert audio.is_cuda and audio.dtype == torch.float32 and audio.is_contiguous()
        B, C, L = audio.shape
        if out is None:
            out = torch.empty((B, (self.cfg.n_fft // 2 + 1) * C, 1 + L // hop, 2), dtype=audio.dtype,
                              device=audio.device)
        _check(lib().mrf_stft(self._h, ctypes.c_void_p(audio.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, L,
                              hop, _stream_ptr(stream)), self._h)
        return out

    def istft(self, spec, hop, length, out=None, stream=None):
        """mrf_istft: CUDA float32 spectra [..., (n_fft/2+1) C, T, 2] -> audio [..., C, length]."""
        import torch
        assert spec.is_cuda and spec.dtype == torch.float32 and spec.is_contiguous()
        lead, FC, T = spec.shape[:-3], spec.shape[-3], spec.shape[-2]
        C = self.cfg.audio_channels
        S = int(np.prod(lead)) if lead else 1
        if out is None:
            out = torch.empty(tuple(lead) + (C, length), dtype=spec.dtype, device=spec.device)
        _check(lib().mrf_istft(self._h, ctypes.c_void_p(spec.data_ptr()), ctypes.c_void_p(out.data_ptr()), S, T,
                               hop, length, _stream_ptr(stream)), self._h)
        return out

    def separate_audio(self, mix, hop, out=None, stream=None, chunk_samples=0):
        """mrf_separate_audio(_chunked): CUDA float32 mix [C, L] -> stems [num_stems, C, L], in chunks
        of chunk_samples samples (0: 8 s)."""
        import torch
        assert mix.is_cuda and mix.dtype == torch.float32 and mix.is_contiguous()
        C, L = mix.shape
        if out is None:
            out = torch.empty((self.cfg.num_stems, C, L), dtype=mix.dtype, device=mix.device)
        assert out.is_cuda and out.dtype == torch.float32 and out.is_contiguous() and \
            out.numel() == self.cfg.num_stems * C * L
        _check(lib().mrf_separate_audio_chunked(self._h, ctypes.c_void_p(mix.data_ptr()),
                                                ctypes.c_void_p(out.data_ptr()), L, hop, chunk_samples,
                                                _stream_ptr(stream)), self._h)
        return out

    def forward_static(self, stft_repr, out, stream=None):
        """mrf_forward_static: the same forward with the library's fixed device scratch
        instead of the handle's workspace; allocates nothing (out must be given)."""
        self._check_input(stft_repr)
        self._check_out(stft_repr, out)
        B, R, T, _ = stft_repr.shape
        _check(lib().mrf_forward_static(self._h, ctypes.c_void_p(stft_repr.data_ptr()),
                                        ctypes.c_void_p(out.data_ptr()), B, T, _stream_ptr(stream)), self._h)
        return out

    def forward_host(self, stft_repr, out=None, stream=None):
        """masks for a host float32 array/tensor, copies inside the call; waits for the stream."""
        import torch
        x = stft_repr if isinstance(stft_repr, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(stft_repr))
        self._check_host_input(x)
        B, R, T, _ = x.shape
        out = self._out_like(x, out)
        _check(lib().mrf_forward_host(self._h, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                      B, T, _stream_ptr(stream)), self._h)
        return out

    def forward_host_async(self, stft_repr, out, stream=None):
        """enqueues H2D copy, forward and D2H copy of one host tensor and returns; `out` holds the
        masks once host_join and a stream synchronize (or sync_status) have followed.  Both
        tensors are kept referenced here until then; pin them for copies that overlap compute."""
        x = stft_repr
        self._check_host_input(x)
        self._check_out(x, out)
        B, R, T, _ = x.shape
        _check(lib().mrf_forward_host_async(self._h, ctypes.c_void_p(stft_repr.data_ptr()),
                                            ctypes.c_void_p(out.data_ptr()), B, T, _stream_ptr(stream)), self._h)
        self._host_pending.append((stft_repr, out))
        return out

    def host_join(self, stream=None):
        """makes `stream` wait for every copy forward_host_async enqueued (no host wait)."""
        _check(lib().mrf_host_join(self._h, _stream_ptr(stream)), self._h)

    def sync_status(self, stream=None):
        _check(lib().mrf_sync_status(self._h, _stream_ptr(stream)), self._h)
        self._host_pending = []

    def set_timing(self, on: bool):
        _check(lib().mrf_set_timing(self._h, int(on)), self._h)

    def set_graph(self, on: bool):
        _check(lib().mrf_set_graph(self._h, int(on)), self._h)

    def kernel_times(self):
        """{kernel name: (launches, total ms)} since the last call (timing mode)."""
        n = ctypes.c_int(0)
        buf = (mrf_kernel_time * 64)()
        _check(lib().mrf_kernel_times(self._h, buf, 64, ctypes.byref(n)), self._h)
        return {buf[i].name.decode(): (buf[i].launches, buf[i].ms) for i in range(n.value)}

    def debug_buffer(self, name, count):
        """First `count` float32 values of an internal buffer of the last forward ("X", "M")."""
        out = np.zeros(count, np.float32)
        n = ctypes.c_size_t(0)
        _check(lib().mrf_debug_buffer(self._h, name.encode(), out.ctypes.data_as(ctypes.c_void_p),
                                      out.nbytes, ctypes.byref(n)), self._h)
        return out[: n.value // 4]

    def debug_stall_next(self):
        """mrf_debug_stall_next: the next fp16 forward's first GEMM lets its bounded waits expire."""
        _check(lib().mrf_debug_stall_next(self._h), self._h)

    def launches_per_forward(self, B, T):
        return lib().mrf_launches_per_forward(self._h, B, T)
