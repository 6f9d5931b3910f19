"""Python binding of the ARL2 C ABI (include/arl2.h), through ctypes.

Argument marshalling only: each function checks shapes, dtypes and devices of torch
tensors and passes raw pointers and the current CUDA stream to libarl2.so, where every
step of the layer runs in hand-written sm_100a kernels. There is no fallback: if the
library is missing or cannot load, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarl2.so")

ARL2_OK, ARL2_ERR_INVALID_ARG, ARL2_ERR_UNSUPPORTED, ARL2_ERR_OOM = 0, 1, 2, 3
ARL2_ERR_CUDA, ARL2_ERR_TIMEOUT, ARL2_ERR_STATE = 4, 5, 6
STATUS_NAMES = {
    0: "ARL2_OK", 1: "ARL2_ERR_INVALID_ARG", 2: "ARL2_ERR_UNSUPPORTED", 3: "ARL2_ERR_OOM",
    4: "ARL2_ERR_CUDA", 5: "ARL2_ERR_TIMEOUT", 6: "ARL2_ERR_STATE",
}

_P, _I, _S, _U64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
# name -> (restype, argtypes); the names and order follow include/arl2.h.
SIGNATURES = {
    "arl2_create": (_S, [_I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
    "arl2_set_feature_maps": (_S, [_P, _P, _P, _P, _P]),
    "arl2_frame_query": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_frame_commit": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_frame_query_host": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_frame_commit_host": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_frame_clean_pass": (_S, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "arl2_set_clean_split": (_S, [_P, _I]),
    "arl2_clean_split": (_I, [_P]),
    "arl2_frame_query_token": (_S, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "arl2_frame_commit_token": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_set_gate_weights": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_frame_gates": (_S, [_P, _P, _P, _P, _P]),
    "arl2_frame_commit_gated": (_S, [_P, _P, _P, _P, _P]),
    "arl2_reset": (_S, [_P, _P]),
    "arl2_get_state": (_S, [_P, _P, _P]),
    "arl2_set_state": (_S, [_P, _P, _P]),
    "arl2_frame_index": (_I, [_P]),
    "arl2_get_status": (_S, [_P]),
    "arl2_set_wait_timeout_ns": (_S, [_P, _U64]),
    "arl2_test_stall_next_query": (_S, [_P]),
    "arl2_set_launch_overlap": (_S, [_P, ctypes.c_int]),
    "arl2_memory_bytes": (_SZ, [_P]),
    "arl2_destroy": (None, [_P]),
    "arl2_frame_commit_noalloc": (_S, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "arl2_kvcache_create": (_S, [_I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
    "arl2_kvcache_query": (_S, [_P, _P, _P, _P, _P, _P]),
    "arl2_kvcache_commit": (_S, [_P, _P, _P, _P]),
    "arl2_kvcache_reset": (_S, [_P]),
    "arl2_kvcache_frames": (_I, [_P]),
    "arl2_kvcache_get_status": (_S, [_P]),
    "arl2_kvcache_memory_bytes": (_SZ, [_P]),
    "arl2_kvcache_destroy": (None, [_P]),
}

_lib: Optional[ctypes.CDLL] = None


class Arl2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {STATUS_NAMES.get(status, status)}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libarl2.so and declare its signatures. Raises ImportError if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m softmax_attention_ar_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != ARL2_OK:
        raise Arl2Error(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, shape, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    return t.data_ptr()


def _cuda(t: torch.Tensor, dtype: torch.dtype, shape, name: str) -> int:
    """_dev for arguments that must be device memory (the kernels read them through TMA)."""
    p = _dev(t, dtype, shape, name)
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    return p


def _host(t: torch.Tensor, dtype: torch.dtype, shape, name: str) -> int:
    """_dev for arguments of the host-buffer calls, which must be host memory."""
    p = _dev(t, dtype, shape, name)
    if t.is_cuda:
        raise ValueError(f"{name}: expected a host (CPU) tensor")
    return p


# ------------------------------------------------------------------ raw C-ABI mirrors
def arl2_create(H: int, T: int, d_k: int, d_v: int, B: int) -> ctypes.c_void_p:
    out = _P()
    _check(load_library().arl2_create(H, T, d_k, d_v, B, ctypes.byref(out)), "arl2_create")
    return out


def arl2_destroy(ctx) -> None:
    load_library().arl2_destroy(ctx)


class ARL2Layer:
    """One ARL2 hybrid attention layer for B streams of H heads, T tokens per frame, head dim d.

    ``query`` is one denoising (or clean) pass of the current frame: it reads the state of
    the previous frame and never writes it. ``commit`` is the clean-pass state update that
    closes the frame. All tensors are CUDA tensors: q, k, v, o bf16 [B, T, H, d]; alpha,
    beta fp32 [B, H, T]; the state fp32 [B, H, d, d]; feature maps bf16 [H, d, d].
    """

    def __init__(self, H: int, T: int, d: int, B: int = 1):
        self.H, self.T, self.d, self.B = H, T, d, B
        self._lib = load_library()
        self._ctx = arl2_create(H, T, d, d, B)

    # -- shapes
    @property
    def act_shape(self):
        return (self.B, self.T, self.H, self.d)

    @property
    def gate_shape(self):
        return (self.B, self.H, self.T)

    @property
    def state_shape(self):
        return (self.B, self.H, self.d, self.d)

    def close(self) -> None:
        if self._ctx is not None:
            self._lib.arl2_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_feature_maps(self, Wq, Wk, Wv, stream=None) -> None:
        shp = (self.H, self.d, self.d)
        _check(self._lib.arl2_set_feature_maps(self._ctx, _dev(Wq, torch.bfloat16, shp, "Wq"),
                                               _dev(Wk, torch.bfloat16, shp, "Wk"),
                                               _dev(Wv, torch.bfloat16, shp, "Wv"), _stream(stream)),
               "arl2_set_feature_maps")

    def query(self, q, k, v, out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(self.act_shape, dtype=torch.bfloat16, device=q.device)
        s = self.act_shape
        _check(self._lib.arl2_frame_query(self._ctx, _cuda(q, torch.bfloat16, s, "q"), _cuda(k, torch.bfloat16, s, "k"),
                                          _cuda(v, torch.bfloat16, s, "v"), _cuda(out, torch.bfloat16, s, "o"),
                                          _stream(stream)), "arl2_frame_query")
        return out

    def commit(self, k, v, alpha, beta, stream=None) -> None:
        s, g = self.act_shape, self.gate_shape
        _check(self._lib.arl2_frame_commit(self._ctx, _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
                                           _cuda(alpha, torch.float32, g, "alpha"), _cuda(beta, torch.float32, g, "beta"),
                                           _stream(stream)), "arl2_frame_commit")

    def clean_pass(self, q, k, v, alpha, beta, out=None, stream=None) -> torch.Tensor:
        """The clean pass in one launch: out = the query of (q, k, v) on S_{N-1}, and the commit
        of (k, v, alpha, beta) into S_N."""
        if out is None:
            out = torch.empty(self.act_shape, dtype=torch.bfloat16, device=q.device)
        s, g = self.act_shape, self.gate_shape
        _check(self._lib.arl2_frame_clean_pass(self._ctx, _cuda(q, torch.bfloat16, s, "q"),
                                               _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
                                               _cuda(out, torch.bfloat16, s, "o"),
                                               _cuda(alpha, torch.float32, g, "alpha"),
                                               _cuda(beta, torch.float32, g, "beta"), _stream(stream)),
               "arl2_frame_clean_pass")
        return out

    def set_clean_split(self, commit_sms: int) -> None:
        """SMs the clean pass gives the commit (0: chosen by the library's cost model)."""
        _check(self._lib.arl2_set_clean_split(self._ctx, int(commit_sms)), "arl2_set_clean_split")

    @property
    def clean_split(self) -> int:
        """SMs the clean pass currently gives the commit."""
        return self._lib.arl2_clean_split(self._ctx)

    def query_token(self, q, k, v, alpha, beta, out=None, stream=None) -> torch.Tensor:
        """Token-level access: intra attention plus the token-by-token readout of this pass."""
        if out is None:
            out = torch.empty(self.act_shape, dtype=torch.bfloat16, device=q.device)
        s, g = self.act_shape, self.gate_shape
        _check(self._lib.arl2_frame_query_token(self._ctx, _cuda(q, torch.bfloat16, s, "q"),
                                                _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
                                                _cuda(out, torch.bfloat16, s, "o"),
                                                _cuda(alpha, torch.float32, g, "alpha"),
                                                _cuda(beta, torch.float32, g, "beta"), _stream(stream)),
               "arl2_frame_query_token")
        return out

    def commit_token(self, k, v, alpha, beta, stream=None) -> None:
        """Token-level access: S_N = the state after the clean pass's last token."""
        s, g = self.act_shape, self.gate_shape
        _check(self._lib.arl2_frame_commit_token(self._ctx, _cuda(k, torch.bfloat16, s, "k"),
                                                 _cuda(v, torch.bfloat16, s, "v"),
                                                 _cuda(alpha, torch.float32, g, "alpha"),
                                                 _cuda(beta, torch.float32, g, "beta"), _stream(stream)),
               "arl2_frame_commit_token")

    def query_host(self, q, k, v, out, stream=None) -> torch.Tensor:
        """Host-buffer query: q, k, v, out are CPU tensors (pinned for asynchrony)."""
        s = self.act_shape
        _check(self._lib.arl2_frame_query_host(self._ctx, _host(q, torch.bfloat16, s, "q"),
                                               _host(k, torch.bfloat16, s, "k"), _host(v, torch.bfloat16, s, "v"),
                                               _host(out, torch.bfloat16, s, "o"), _stream(stream)),
               "arl2_frame_query_host")
        return out

    def commit_host(self, k, v, alpha, beta, stream=None) -> None:
        s, g = self.act_shape, self.gate_shape
        _check(self._lib.arl2_frame_commit_host(self._ctx, _host(k, torch.bfloat16, s, "k"),
                                                _host(v, torch.bfloat16, s, "v"),
                                                _host(alpha, torch.float32, g, "alpha"),
                                                _host(beta, torch.float32, g, "beta"), _stream(stream)),
               "arl2_frame_commit_host")

    def set_gate_weights(self, Wa, Wb, ba, bb, stream=None) -> None:
        """Gate projections for gates produced from the hidden state: Wa, Wb bf16 [H, H*d];
        ba, bb fp32 [H]."""
        D = self.H * self.d
        _check(self._lib.arl2_set_gate_weights(self._ctx, _dev(Wa, torch.bfloat16, (self.H, D), "Wa"),
                                               _dev(Wb, torch.bfloat16, (self.H, D), "Wb"),
                                               _dev(ba, torch.float32, (self.H,), "ba"),
                                               _dev(bb, torch.float32, (self.H,), "bb"), _stream(stream)),
               "arl2_set_gate_weights")

    def gates(self, x, alpha=None, beta=None, stream=None):
        """alpha, beta fp32 [B, H, T] from the hidden state x bf16 [B, T, H*d]."""
        if alpha is None:
            alpha = torch.empty(self.gate_shape, dtype=torch.float32, device=x.device)
        if beta is None:
            beta = torch.empty(self.gate_shape, dtype=torch.float32, device=x.device)
        xs, g = (self.B, self.T, self.H * self.d), self.gate_shape
        _check(self._lib.arl2_frame_gates(self._ctx, _cuda(x, torch.bfloat16, xs, "x"),
                                          _cuda(alpha, torch.float32, g, "alpha"),
                                          _cuda(beta, torch.float32, g, "beta"), _stream(stream)),
               "arl2_frame_gates")
        return alpha, beta

    def commit_gated(self, x, k, v, stream=None) -> None:
        """The clean-pass commit with its gates produced from the hidden state x."""
        xs, s = (self.B, self.T, self.H * self.d), self.act_shape
        _check(self._lib.arl2_frame_commit_gated(self._ctx, _cuda(x, torch.bfloat16, xs, "x"),
                                                 _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
                                                 _stream(stream)), "arl2_frame_commit_gated")

    def reset(self, stream=None) -> None:
        _check(self._lib.arl2_reset(self._ctx, _stream(stream)), "arl2_reset")

    def get_state(self, out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(self.state_shape, dtype=torch.float32, device="cuda")
        _check(self._lib.arl2_get_state(self._ctx, _dev(out, torch.float32, self.state_shape, "dst"),
                                        _stream(stream)), "arl2_get_state")
        return out

    def set_state(self, S, stream=None) -> None:
        _check(self._lib.arl2_set_state(self._ctx, _dev(S, torch.float32, self.state_shape, "src"), _stream(stream)),
               "arl2_set_state")

    @property
    def frame_index(self) -> int:
        return self._lib.arl2_frame_index(self._ctx)

    def status(self) -> int:
        """Synchronise and return (and clear) the device status (ARL2_OK, ARL2_ERR_TIMEOUT, ...)."""
        return self._lib.arl2_get_status(self._ctx)

    def set_wait_timeout_ns(self, ns: int) -> None:
        _check(self._lib.arl2_set_wait_timeout_ns(self._ctx, int(ns)), "arl2_set_wait_timeout_ns")

    def set_launch_overlap(self, enable: bool) -> None:
        """Queries and commits may start behind the previous kernel in their stream (see arl2.h)."""
        _check(self._lib.arl2_set_launch_overlap(self._ctx, int(bool(enable))), "arl2_set_launch_overlap")

    def test_stall_next_query(self) -> None:
        """Failure-detection hook: the next query's bounded wait runs out (no GPU fault)."""
        _check(self._lib.arl2_test_stall_next_query(self._ctx), "arl2_test_stall_next_query")

    @property
    def memory_bytes(self) -> int:
        return self._lib.arl2_memory_bytes(self._ctx)


def frame_commit_noalloc(k, v, alpha, beta, Wk, Wv, S_prev, S_next, status, stream=None) -> None:
    """Commit without a context or any allocation (arl2_frame_commit_noalloc).

    For callers that cannot allocate device memory: the library's fixed scratch array is
    used instead. k, v bf16 [B, T, H, d]; alpha, beta fp32 [B, H, T]; Wk, Wv bf16 [H, d, d];
    S_prev, S_next fp32 [B, H, d, d] (S_next may be S_prev); status an int32 [1] device word
    the caller zeroed, which reads nonzero after the call if a bounded wait ran out.
    """
    B, T, H, d = k.shape
    s, g, w, st = (B, T, H, d), (B, H, T), (H, d, d), (B, H, d, d)
    if status is None or status.dtype != torch.int32 or status.numel() != 1 or not status.is_cuda:
        raise ValueError("status: expected one int32 element in device memory")
    status_ptr = status.data_ptr()
    _check(load_library().arl2_frame_commit_noalloc(
        B, H, T, d, _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
        _cuda(alpha, torch.float32, g, "alpha"), _cuda(beta, torch.float32, g, "beta"),
        _cuda(Wk, torch.bfloat16, w, "Wk"), _cuda(Wv, torch.bfloat16, w, "Wv"),
        _cuda(S_prev, torch.float32, st, "S_prev"), _cuda(S_next, torch.float32, st, "S_next"),
        status_ptr, _stream(stream)), "arl2_frame_commit_noalloc")


class KVCacheBaseline:
    """The growing-KV-cache full-softmax baseline (comparison only); see arl2_kvcache_* in arl2.h."""

    def __init__(self, H: int, T: int, d: int, B: int = 1, max_frames: int = 1):
        self.H, self.T, self.d, self.B, self.max_frames = H, T, d, B, max_frames
        self._lib = load_library()
        out = _P()
        _check(self._lib.arl2_kvcache_create(H, T, d, B, max_frames, ctypes.byref(out)), "arl2_kvcache_create")
        self._c = out

    @property
    def act_shape(self):
        return (self.B, self.T, self.H, self.d)

    def close(self) -> None:
        if self._c is not None:
            self._lib.arl2_kvcache_destroy(self._c)
            self._c = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def query(self, q, k, v, out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(self.act_shape, dtype=torch.bfloat16, device=q.device)
        s = self.act_shape
        _check(self._lib.arl2_kvcache_query(self._c, _cuda(q, torch.bfloat16, s, "q"), _cuda(k, torch.bfloat16, s, "k"),
                                            _cuda(v, torch.bfloat16, s, "v"), _cuda(out, torch.bfloat16, s, "o"),
                                            _stream(stream)), "arl2_kvcache_query")
        return out

    def commit(self, k, v, stream=None) -> None:
        s = self.act_shape
        _check(self._lib.arl2_kvcache_commit(self._c, _cuda(k, torch.bfloat16, s, "k"), _cuda(v, torch.bfloat16, s, "v"),
                                             _stream(stream)), "arl2_kvcache_commit")

    def reset(self) -> None:
        _check(self._lib.arl2_kvcache_reset(self._c), "arl2_kvcache_reset")

    @property
    def frames(self) -> int:
        return self._lib.arl2_kvcache_frames(self._c)

    def status(self) -> int:
        return self._lib.arl2_kvcache_get_status(self._c)

    @property
    def memory_bytes(self) -> int:
        return self._lib.arl2_kvcache_memory_bytes(self._c)
