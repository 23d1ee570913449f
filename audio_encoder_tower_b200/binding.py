"""ctypes binding of the encoder C ABI (include/enc.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of libenc_b200.so. PyTorch provides device memory and streams.
The library must be built (python -m audio_encoder_tower_b200.build); there is
no fallback of any kind when it is missing.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libenc_b200.so")

ENC_OK, ENC_ERR_INVALID_ARG, ENC_ERR_UNSUPPORTED, ENC_ERR_OOM, ENC_ERR_CUDA, ENC_ERR_TIMEOUT, \
    ENC_ERR_DEVICE_CHECK = range(7)
ENC_DTYPE_BF16, ENC_DTYPE_FP32 = 0, 1

EXPORTED = ["enc_create", "enc_forward", "enc_output_positions", "enc_get_status", "enc_destroy",
            "enc_status_string", "enc_device_bytes", "enc_linear_bf16", "enc_attention_bf16",
            "enc_profile_enable", "enc_profile_collect", "enc_launch_count", "enc_forward_static_scratch",
            "enc_frontend_create", "enc_frontend_log_mel", "enc_frontend_destroy",
            "enc_cache_create", "enc_forward_cached", "enc_cache_size", "enc_cache_destroy", "enc_cache_content_keys",
            "enc_clip_flops", "enc_shard_plan", "enc_selftest_timeout", "enc_check_guards",
            "enc_guard_selftest"]
ENC_FLAG_GUARD = 1

KERNEL_CLASSES = ["mel", "conv1", "conv2", "ln", "qkv", "attn", "out", "fc1", "fc2", "final", "proj1", "proj2",
                  "zero"]


class EncError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class EncConfig(ctypes.Structure):
    _fields_ = [("n_mels", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn_dim", ctypes.c_int32),
                ("max_frames", ctypes.c_int32), ("max_batch", ctypes.c_int32), ("pool_step", ctypes.c_int32),
                ("proj_hidden", ctypes.c_int32), ("proj_out", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32), ("attn_chunk", ctypes.c_int32)]


_VP = ctypes.c_void_p
_VPP = ctypes.POINTER(ctypes.c_void_p)
LAYER_FIELDS = ["ln1_g", "ln1_b", "q_w", "q_b", "k_w", "k_b", "v_w", "v_b", "o_w", "o_b", "ln2_g", "ln2_b",
                "fc1_w", "fc1_b", "fc2_w", "fc2_b"]


class EncKernelTimes(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * 13), ("flops", ctypes.c_double * 13), ("launches", ctypes.c_int64 * 13)]


class EncWeights(ctypes.Structure):
    _fields_ = ([("conv1_w", _VP), ("conv1_b", _VP), ("conv2_w", _VP), ("conv2_b", _VP)] +
                [(f, _VPP) for f in LAYER_FIELDS] +
                [("lnpost_g", _VP), ("lnpost_b", _VP), ("proj1_w", _VP), ("proj1_b", _VP),
                 ("proj2_w", _VP), ("proj2_b", _VP)])


_LIB = None


def load_library(path: str = LIB_PATH):
    """Load libenc_b200.so and declare the signatures of every exported call."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m audio_encoder_tower_b200.build`")
    lib = ctypes.CDLL(path)
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.enc_create.argtypes = [ctypes.POINTER(EncConfig), ctypes.POINTER(EncWeights), ctypes.POINTER(ctypes.c_void_p)]
    lib.enc_create.restype = ctypes.c_int
    lib.enc_forward.argtypes = [_VP, _VP, i32p, ctypes.c_int32, _VP, _VP]
    lib.enc_forward.restype = ctypes.c_int
    lib.enc_output_positions.argtypes = [_VP, ctypes.c_int32, i32p, i32p, i32p, i32p]
    lib.enc_output_positions.restype = ctypes.c_int
    lib.enc_get_status.argtypes = [_VP, _VP]
    lib.enc_get_status.restype = ctypes.c_int
    lib.enc_destroy.argtypes = [_VP]
    lib.enc_destroy.restype = None
    lib.enc_status_string.argtypes = [ctypes.c_int]
    lib.enc_status_string.restype = ctypes.c_char_p
    lib.enc_device_bytes.argtypes = [_VP]
    lib.enc_device_bytes.restype = ctypes.c_size_t
    lib.enc_linear_bf16.argtypes = [_VP, _VP, _VP, _VP, _VP, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_int32, _VP, _VP]
    lib.enc_linear_bf16.restype = ctypes.c_int
    lib.enc_attention_bf16.argtypes = [_VP, _VP, _VP, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, _VP, _VP]
    lib.enc_attention_bf16.restype = ctypes.c_int
    lib.enc_profile_enable.argtypes = [_VP, ctypes.c_int32]
    lib.enc_profile_enable.restype = ctypes.c_int
    lib.enc_profile_collect.argtypes = [_VP, ctypes.POINTER(EncKernelTimes)]
    lib.enc_profile_collect.restype = ctypes.c_int
    lib.enc_launch_count.argtypes = [_VP]
    lib.enc_launch_count.restype = ctypes.c_int64
    lib.enc_forward_static_scratch.argtypes = [_VP, _VP, i32p, ctypes.c_int32, _VP, _VP]
    lib.enc_forward_static_scratch.restype = ctypes.c_int
    lib.enc_frontend_create.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p)]
    lib.enc_frontend_create.restype = ctypes.c_int
    lib.enc_frontend_log_mel.argtypes = [_VP, _VP, ctypes.c_int32, _VP, ctypes.c_int32, _VP]
    lib.enc_frontend_log_mel.restype = ctypes.c_int
    lib.enc_frontend_destroy.argtypes = [_VP]
    lib.enc_frontend_destroy.restype = None
    lib.enc_cache_create.argtypes = [_VP, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p)]
    lib.enc_cache_create.restype = ctypes.c_int
    lib.enc_forward_cached.argtypes = [_VP, _VP, i32p, ctypes.POINTER(ctypes.c_uint64), ctypes.c_int32, _VP, i32p,
                                       _VP]
    lib.enc_forward_cached.restype = ctypes.c_int
    lib.enc_cache_content_keys.argtypes = [_VP, _VP, i32p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint64), _VP]
    lib.enc_cache_content_keys.restype = ctypes.c_int
    lib.enc_cache_size.argtypes = [_VP]
    lib.enc_cache_size.restype = ctypes.c_int32
    lib.enc_cache_destroy.argtypes = [_VP]
    lib.enc_cache_destroy.restype = None
    lib.enc_check_guards.argtypes = [_VP, ctypes.c_char_p, ctypes.c_size_t]
    lib.enc_check_guards.restype = ctypes.c_int
    lib.enc_guard_selftest.argtypes = [_VP, ctypes.c_int32, ctypes.c_int64]
    lib.enc_guard_selftest.restype = ctypes.c_int
    lib.enc_selftest_timeout.argtypes = [_VP, ctypes.c_int64, _VP]
    lib.enc_selftest_timeout.restype = ctypes.c_int
    lib.enc_clip_flops.argtypes = [ctypes.POINTER(EncConfig), ctypes.c_int32, ctypes.POINTER(ctypes.c_double)]
    lib.enc_clip_flops.restype = ctypes.c_int
    lib.enc_shard_plan.argtypes = [ctypes.POINTER(EncConfig), i32p, ctypes.c_int32, ctypes.c_int32, i32p, i32p, i32p,
                                   ctypes.POINTER(ctypes.c_double)]
    lib.enc_shard_plan.restype = ctypes.c_int
    _LIB = lib
    return lib


def status_string(code: int) -> str:
    return load_library().enc_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != ENC_OK:
        raise EncError(code, what)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def encoder_config(*, n_mels, d_model, n_layers, n_heads, ffn_dim, max_frames, max_batch, dtype="bf16",
                   pool_step=1, proj_hidden=0, proj_out=0, ln_eps=1e-5, head_dim=64, attn_chunk=0,
                   guard=False) -> EncConfig:
    """The enc_config struct of a tower geometry (dtype "bf16" or "fp32"); guard sets ENC_FLAG_GUARD."""
    return EncConfig(n_mels, d_model, n_layers, n_heads, head_dim, ffn_dim, max_frames, max_batch, pool_step,
                     proj_hidden, proj_out, ln_eps, ENC_DTYPE_BF16 if dtype == "bf16" else ENC_DTYPE_FP32,
                     ENC_FLAG_GUARD if guard else 0, attn_chunk)


def clip_flops(cfg: EncConfig, length: int) -> float:
    """Algorithmic FLOPs of one clip of `length` valid frames (enc_clip_flops)."""
    v = ctypes.c_double()
    _check(load_library().enc_clip_flops(ctypes.byref(cfg), int(length), ctypes.byref(v)), "enc_clip_flops")
    return float(v.value)


def shard_plan(cfg: EncConfig, lengths, world: int):
    """Split clips over `world` ranks of cfg.max_batch clips each (enc_shard_plan).

    lengths: [B] valid frames per clip, or an int B for B full-length clips.
    Returns (rank_of [B], index_of [B], rank_count [world], rank_flops [world]).
    """
    i32p = ctypes.POINTER(ctypes.c_int32)
    if isinstance(lengths, (int, np.integer)):
        B, ln = int(lengths), None
    else:
        ln = np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
        B = int(ln.shape[0])
    rank_of = np.zeros(B, np.int32)
    index_of = np.zeros(B, np.int32)
    count = np.zeros(max(int(world), 1), np.int32)
    flops = np.zeros(max(int(world), 1), np.float64)
    _check(load_library().enc_shard_plan(ctypes.byref(cfg), None if ln is None else ln.ctypes.data_as(i32p), B,
                                         int(world), rank_of.ctypes.data_as(i32p), index_of.ctypes.data_as(i32p),
                                         count.ctypes.data_as(i32p),
                                         flops.ctypes.data_as(ctypes.POINTER(ctypes.c_double))), "enc_shard_plan")
    return rank_of, index_of, count, flops


class Encoder:
    """One encoder handle (enc_create / enc_forward / enc_destroy).

    weights: dict of device tensors in PyTorch layouts named as in enc.h
    ("conv1_w", "layers.{l}.q_w", "lnpost_g", "proj1_w", ...), dtype matching
    `dtype` ("bf16" or "fp32"). They may be freed after construction.
    """

    def __init__(self, *, n_mels, d_model, n_layers, n_heads, ffn_dim, max_frames, max_batch, dtype="bf16",
                 pool_step=1, proj_hidden=0, proj_out=0, ln_eps=1e-5, head_dim=64, attn_chunk=0, guard=False,
                 weights: dict):
        self.lib = load_library()
        self.cfg = encoder_config(n_mels=n_mels, d_model=d_model, n_layers=n_layers, n_heads=n_heads,
                                  ffn_dim=ffn_dim, max_frames=max_frames, max_batch=max_batch, dtype=dtype,
                                  pool_step=pool_step, proj_hidden=proj_hidden, proj_out=proj_out, ln_eps=ln_eps,
                                  head_dim=head_dim, attn_chunk=attn_chunk, guard=guard)
        w = EncWeights()
        for f in ("conv1_w", "conv1_b", "conv2_w", "conv2_b", "lnpost_g", "lnpost_b",
                  "proj1_w", "proj1_b", "proj2_w", "proj2_b"):
            setattr(w, f, _ptr(weights.get(f)))
        keep = []
        for f in LAYER_FIELDS:
            arr = (ctypes.c_void_p * max(n_layers, 1))()
            for l in range(n_layers):
                arr[l] = _ptr(weights.get(f"layers.{l}.{f}"))
            keep.append(arr)
            setattr(w, f, ctypes.cast(arr, _VPP))
        h = ctypes.c_void_p()
        _check(self.lib.enc_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(h)), "enc_create")
        self.handle = h
        self.dtype = dtype

    # ----------------------------------------------------------- geometry
    def output_positions(self, B: int, lengths=None):
        """(n_out [B] int32, p_out, d_out) for a batch, from the library."""
        n_out = np.zeros(B, np.int32)
        p = ctypes.c_int32()
        dd = ctypes.c_int32()
        lp = None
        if lengths is not None:
            lengths = np.ascontiguousarray(lengths, dtype=np.int32)
            lp = lengths.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        _check(self.lib.enc_output_positions(self.handle, B, lp, n_out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                             ctypes.byref(p), ctypes.byref(dd)), "enc_output_positions")
        return n_out, p.value, dd.value

    # ------------------------------------------------------------ forward
    def forward(self, mel, lengths=None, out=None, stream=None):
        """Enqueue the forward pass of mel [B, n_mels, T] (device) on `stream`.

        Returns `out` [B, P_out, d_out] (allocated with torch when not given).
        """
        import torch
        B = int(mel.shape[0])
        if out is None:
            _, p_out, d_out = self.output_positions(B, lengths)
            out = torch.empty((B, p_out, d_out), dtype=mel.dtype, device=mel.device)
        lp = None
        if lengths is not None:
            self._len = np.ascontiguousarray(lengths, dtype=np.int32)
            lp = self._len.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        _check(self.lib.enc_forward(self.handle, _ptr(mel), lp, B, _ptr(out), _stream_handle(stream)),
               "enc_forward")
        return out

    def forward_static_scratch(self, mel, lengths=None, out=None, stream=None):
        """enc_forward_static_scratch: the same forward with its workspace in the
        library's fixed 64 MiB static device array (no device allocation in the call).

        `out` must be given by callers that cannot allocate; when omitted it is
        allocated here with torch for convenience.
        """
        import torch
        B = int(mel.shape[0])
        if out is None:
            _, p_out, d_out = self.output_positions(B, lengths)
            out = torch.empty((B, p_out, d_out), dtype=mel.dtype, device=mel.device)
        lp = None
        if lengths is not None:
            self._len = np.ascontiguousarray(lengths, dtype=np.int32)
            lp = self._len.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        _check(self.lib.enc_forward_static_scratch(self.handle, _ptr(mel), lp, B, _ptr(out),
                                                   _stream_handle(stream)), "enc_forward_static_scratch")
        return out

    def status(self, stream=None):
        """Synchronise `stream` and raise if a device-side check or wait failed."""
        _check(self.lib.enc_get_status(self.handle, _stream_handle(stream)), "enc_get_status")

    def check_guards(self):
        """enc_check_guards (handles created with guard=True): raise EncError naming the
        buffer and offset if a kernel wrote into a guard region around a workspace buffer."""
        msg = ctypes.create_string_buffer(256)
        code = self.lib.enc_check_guards(self.handle, msg, 256)
        if code != ENC_OK:
            raise EncError(code, "enc_check_guards: " + msg.value.decode())

    def guard_selftest(self, buffer: int, offset: int):
        """enc_guard_selftest: one guard byte changed from the host is reported, then restored."""
        _check(self.lib.enc_guard_selftest(self.handle, int(buffer), int(offset)), "enc_guard_selftest")

    def selftest_timeout(self, limit_ns: int, stream=None):
        """Enqueue the failure-detection self-test (enc_selftest_timeout): a bounded
        wait that runs out after limit_ns; the next status() raises ENC_ERR_TIMEOUT."""
        _check(self.lib.enc_selftest_timeout(self.handle, int(limit_ns), _stream_handle(stream)),
               "enc_selftest_timeout")

    def profile(self, enable: bool):
        """Bracket every kernel of the following forwards with CUDA events."""
        _check(self.lib.enc_profile_enable(self.handle, 1 if enable else 0), "enc_profile_enable")

    def collect_profile(self) -> dict:
        """{class: (ms, flops, launches)} summed since the last collect (waits for the events)."""
        t = EncKernelTimes()
        _check(self.lib.enc_profile_collect(self.handle, ctypes.byref(t)), "enc_profile_collect")
        return {k: (t.ms[i], t.flops[i], int(t.launches[i])) for i, k in enumerate(KERNEL_CLASSES)
                if t.launches[i]}

    def launch_count(self) -> int:
        return int(self.lib.enc_launch_count(self.handle))

    def device_bytes(self) -> int:
        return int(self.lib.enc_device_bytes(self.handle))

    def close(self):
        if getattr(self, "handle", None):
            self.lib.enc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------- single-kernel calls
def linear_bf16(A, W, bias=None, out=None, resid=None, gelu=False, status=None, stream=None):
    """out = act(A W^T + bias) on the tensor cores (bf16 in/out), or resid += A W^T + bias."""
    import torch
    M, K = A.shape
    N = W.shape[0]
    if out is None and resid is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(load_library().enc_linear_bf16(_ptr(A), _ptr(W), _ptr(bias), _ptr(out), _ptr(resid), M, N, K,
                                          1 if gelu else 0, _ptr(status), _stream_handle(stream)),
           "enc_linear_bf16")
    return out if resid is None else resid


def attention_bf16(qkv, cu, max_n, n_heads, out=None, status=None, stream=None):
    """Packed-clip bidirectional attention: qkv [R, 3d] bf16, cu device int32 [B+1]."""
    import torch
    R = qkv.shape[0]
    d = 64 * n_heads
    if out is None:
        out = torch.empty((R, d), dtype=torch.bfloat16, device=qkv.device)
    _check(load_library().enc_attention_bf16(_ptr(qkv), _ptr(out), _ptr(cu), int(R), int(cu.numel()) - 1,
                                             int(max_n), int(n_heads), _ptr(status), _stream_handle(stream)),
           "enc_attention_bf16")
    return out


class Frontend:
    """Log-mel front end (enc_frontend_create / enc_frontend_log_mel / enc_frontend_destroy):
    30 s clips of 16 kHz audio, fp32 [B, 480000] on the device -> [B, n_mels, 3000]."""

    SAMPLES, FRAMES = 480000, 3000

    def __init__(self, n_mels: int = 128, max_batch: int = 16):
        self.lib = load_library()
        h = ctypes.c_void_p()
        _check(self.lib.enc_frontend_create(int(n_mels), int(max_batch), ctypes.byref(h)), "enc_frontend_create")
        self.h, self.n_mels, self.max_batch = h, int(n_mels), int(max_batch)

    def log_mel(self, audio, out=None, dtype="bf16", stream=None):
        import torch
        B = audio.shape[0]
        if audio.dtype != torch.float32 or tuple(audio.shape[1:]) != (self.SAMPLES,) or not audio.is_contiguous():
            raise ValueError("audio must be a contiguous fp32 [B, 480000] device tensor")
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        if out is None:
            out = torch.empty((B, self.n_mels, self.FRAMES), dtype=tdt, device=audio.device)
        _check(self.lib.enc_frontend_log_mel(self.h, _ptr(audio), int(B), _ptr(out), 0 if dtype == "bf16" else 1,
                                             _stream_handle(stream)), "enc_frontend_log_mel")
        return out

    def close(self):
        if self.h:
            self.lib.enc_frontend_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cache:
    """Embeddings cache in front of an Encoder (enc_cache_create / enc_forward_cached):
    outputs looked up by a 64-bit key per clip that identifies its mel and length."""

    def __init__(self, encoder: "Encoder", capacity: int):
        self.lib = load_library()
        self.encoder = encoder
        h = ctypes.c_void_p()
        _check(self.lib.enc_cache_create(encoder.handle, int(capacity), ctypes.byref(h)), "enc_cache_create")
        self.h = h

    def content_keys(self, mel, lengths=None, stream=None) -> np.ndarray:
        """enc_cache_content_keys: [B] uint64 keys hashed from each clip's length and
        valid mel frames on the device (waits for `stream`)."""
        B = int(mel.shape[0])
        ln = None if lengths is None else np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
        keys = np.zeros(B, dtype=np.uint64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        _check(self.lib.enc_cache_content_keys(self.h, _ptr(mel), None if ln is None else ln.ctypes.data_as(i32p),
                                               B, keys.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)),
                                               _stream_handle(stream)), "enc_cache_content_keys")
        return keys

    def forward(self, mel, keys=None, lengths=None, out=None, stream=None):
        """Returns (out, hits): hits[b] = 1 where clip b's output came from the cache.
        keys=None derives each clip's key from its content (content_keys)."""
        import torch
        B = int(mel.shape[0])
        if keys is None:
            keys = self.content_keys(mel, lengths, stream)
        if out is None:
            _, p_out, d_out = self.encoder.output_positions(B, lengths)
            out = torch.empty((B, p_out, d_out), dtype=mel.dtype, device=mel.device)
        k = np.ascontiguousarray(np.asarray(keys, dtype=np.uint64))
        if k.shape != (B,):
            raise ValueError("one key per clip")
        ln = None if lengths is None else np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
        hits = np.zeros(B, dtype=np.int32)
        i32p = ctypes.POINTER(ctypes.c_int32)
        _check(self.lib.enc_forward_cached(self.h, _ptr(mel), None if ln is None else ln.ctypes.data_as(i32p),
                                           k.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)), int(B), _ptr(out),
                                           hits.ctypes.data_as(i32p), _stream_handle(stream)), "enc_forward_cached")
        return out, hits

    def size(self) -> int:
        return int(self.lib.enc_cache_size(self.h))

    def close(self):
        if self.h:
            self.lib.enc_cache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
