"""ctypes binding of ``libh2o.so`` (the C ABI in ``include/h2o.h``).

Argument marshalling only: PyTorch provides device memory and streams, and
every step of the computation runs in the library's CUDA kernels.  There is
no fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libh2o.so")

H2O_OK = 0
H2O_BF16, H2O_F32, H2O_Q8 = 0, 1, 2
POLICIES = {"h2o": 0, "lr": 1, "slr": 2}  # h2o_policy
STATUS_NAMES = {0: "H2O_OK", 1: "H2O_ERR_INVALID_ARG", 2: "H2O_ERR_SHAPE", 3: "H2O_ERR_DTYPE",
                4: "H2O_ERR_ALIGN", 5: "H2O_ERR_CUDA", 6: "H2O_ERR_TIMEOUT", 7: "H2O_ERR_STATE"}

EXPORTED = ["h2o_required_bytes", "h2o_cache_create", "h2o_chunk_step", "h2o_chunk_step_host",
            "h2o_cache_host_join", "h2o_attention", "h2o_attention_backward", "h2o_evict",
            "h2o_cache_read", "h2o_cache_write", "h2o_cache_check", "h2o_cache_info",
            "h2o_cache_set_timing", "h2o_cache_kernel_ms", "h2o_attention_static_scratch",
            "h2o_static_scratch_check", "h2o_selftest_wait_timeout", "h2o_selftest_exp2",
            "h2o_cache_destroy",
            "h2o_status_string"]


class H2OError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {STATUS_NAMES.get(status, status)}")


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("max_chunk", ctypes.c_int32),
                ("recent_window", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("policy", ctypes.c_int32),
                ("sink_tokens", ctypes.c_int32)]


class Sizes(ctypes.Structure):
    _fields_ = [("k_bytes", ctypes.c_size_t), ("v_bytes", ctypes.c_size_t),
                ("scores_bytes", ctypes.c_size_t), ("pos_bytes", ctypes.c_size_t),
                ("state_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t)]


class Buffers(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("scores", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("state", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m kv_cache_sparse_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, V = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
    lib.h2o_required_bytes.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Sizes)]
    lib.h2o_cache_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Buffers), P,
                                     ctypes.POINTER(P)]
    for name in ("h2o_chunk_step", "h2o_chunk_step_host", "h2o_attention"):
        getattr(lib, name).argtypes = [P, P, P, P, I, P, P, P]
    lib.h2o_cache_host_join.argtypes = [P, P]
    lib.h2o_attention_backward.argtypes = [P, P, P, P, I, P, P, P, P, P, P, P, P]
    lib.h2o_attention_static_scratch.argtypes = [ctypes.POINTER(Config), P, P, I, P, P, P, I, P,
                                                 P, P]
    lib.h2o_static_scratch_check.argtypes = [P]
    lib.h2o_selftest_wait_timeout.argtypes = [P, ctypes.c_uint32, P]
    lib.h2o_selftest_exp2.argtypes = [P, P, I, P]
    lib.h2o_evict.argtypes = [P, P, P, P, I, P]
    lib.h2o_cache_read.argtypes = [P, P, P, P, P, P, P]
    lib.h2o_cache_write.argtypes = [P, P, P, P, P, P, P]
    lib.h2o_cache_check.argtypes = [P, P]
    lib.h2o_cache_info.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I),
                                   ctypes.POINTER(ctypes.c_uint64)]
    lib.h2o_cache_set_timing.argtypes = [P, V]
    lib.h2o_cache_kernel_ms.argtypes = [P, ctypes.POINTER(ctypes.c_float)]
    lib.h2o_cache_destroy.argtypes = [P]
    lib.h2o_cache_destroy.restype = None
    lib.h2o_status_string.argtypes = [V]
    lib.h2o_status_string.restype = ctypes.c_char_p
    for name in EXPORTED:
        if name not in ("h2o_cache_destroy", "h2o_status_string"):
            getattr(lib, name).restype = V
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(call: str, status: int):
    if status != H2O_OK:
        raise H2OError(call, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class CacheShape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    capacity: int
    max_chunk: int
    recent_window: int
    dtype: torch.dtype = torch.bfloat16   # torch.int8: the int8 cache (Q8), bf16 activations
    softmax_scale: float = 0.0
    policy: str = "h2o"     # "h2o", "lr" or "slr"
    sink_tokens: int = 0    # "slr": the first positions that always stay

    @property
    def q8(self) -> bool:
        return self.dtype == torch.int8

    @property
    def act_dtype(self) -> torch.dtype:
        """Element type of q, k_new, v_new and out."""
        return torch.bfloat16 if self.q8 else self.dtype

    def config(self) -> Config:
        dt = {torch.bfloat16: H2O_BF16, torch.float32: H2O_F32, torch.int8: H2O_Q8}[self.dtype]
        return Config(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.capacity,
                      self.max_chunk, self.recent_window, dt, self.softmax_scale,
                      POLICIES[self.policy], self.sink_tokens)


def required_bytes(shape: CacheShape) -> Sizes:
    sz = Sizes()
    cfg = shape.config()
    _check("h2o_required_bytes", lib().h2o_required_bytes(ctypes.byref(cfg), ctypes.byref(sz)))
    return sz


class H2OCache:
    """``batch`` H2O caches on one GPU, advanced one chunk at a time.

    Device buffers are torch tensors owned by this object; the step itself is
    the library's ``h2o_chunk_step``.
    """

    def __init__(self, shape: CacheShape, device="cuda", stream=None):
        self.shape = shape
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        sz = required_bytes(shape)
        s = shape
        kw = dict(device=self.device)
        if s.q8:
            # int8 codes [B, H_kv, C, d] followed by fp32 scales [B, H_kv, C]
            self.k = torch.empty(sz.k_bytes, dtype=torch.uint8, **kw)
            self.v = torch.empty_like(self.k)
        else:
            self.k = torch.empty(s.batch, s.n_kv_heads, s.capacity, s.head_dim, dtype=s.dtype, **kw)
            self.v = torch.empty_like(self.k)
        self.scores = torch.empty(s.batch, s.n_kv_heads, s.capacity, dtype=torch.float32, **kw)
        self.pos = torch.empty(s.batch, s.n_kv_heads, s.capacity, dtype=torch.int32, **kw)
        self.state = torch.zeros(4, dtype=torch.int32, **kw)
        self.workspace = torch.empty(sz.workspace_bytes + 256, dtype=torch.uint8, **kw)
        off = (-self.workspace.data_ptr()) % 256
        self._ws_ptr = self.workspace.data_ptr() + off
        bufs = Buffers(self.k.data_ptr(), self.v.data_ptr(), self.scores.data_ptr(),
                       self.pos.data_ptr(), self.state.data_ptr(), self._ws_ptr,
                       sz.workspace_bytes)
        self._cfg = shape.config()
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check("h2o_cache_create", lib().h2o_cache_create(
                ctypes.byref(self._cfg), ctypes.byref(bufs), _stream(stream),
                ctypes.byref(handle)))
        self._h = handle

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            try:
                _lib.h2o_cache_destroy(h)
            except Exception:  # interpreter shutdown
                pass
            self._h = None

    # ----------------------------------------------------------------- shapes
    def _alloc_out(self, n_q):
        s = self.shape
        return torch.empty(s.batch, n_q, s.n_q_heads, s.head_dim, dtype=s.act_dtype,
                           device=self.device)

    def _alloc_colsum(self, n_q):
        s = self.shape
        return torch.empty(s.batch, s.n_kv_heads, s.capacity + n_q, dtype=torch.float32,
                           device=self.device)

    def _check_inputs(self, q, k_new, v_new):
        s = self.shape
        for t in (q, k_new, v_new):
            if t.device != self.device or t.dtype != s.act_dtype or not t.is_contiguous():
                raise ValueError("inputs must be contiguous tensors of the cache's dtype on its device")
        n_q = q.shape[1]
        if q.shape != (s.batch, n_q, s.n_q_heads, s.head_dim) or \
                k_new.shape != (s.batch, n_q, s.n_kv_heads, s.head_dim) or \
                v_new.shape != k_new.shape:
            raise ValueError("bad input shapes")
        return n_q

    # ----------------------------------------------------------------- calls
    def step(self, q, k_new, v_new, return_colsum=False, out=None, stream=None):
        n_q = self._check_inputs(q, k_new, v_new)
        out = self._alloc_out(n_q) if out is None else out
        colsum = self._alloc_colsum(n_q) if return_colsum else None
        _check("h2o_chunk_step", lib().h2o_chunk_step(
            self._h, _ptr(q), _ptr(k_new), _ptr(v_new), n_q, _ptr(out), _ptr(colsum),
            _stream(stream)))
        return (out, colsum) if return_colsum else out

    def step_host(self, q, k_new, v_new, out, colsum=None, stream=None, join=True):
        """The step on HOST (ideally pinned) tensors.  Uploads and downloads
        run on the cache's own copy streams and overlap neighbouring steps;
        with join=True the stream then waits for this step's download, so
        `out` is complete once the stream is synchronised.  With join=False
        call host_join() before reading `out`."""
        n_q = q.shape[1]
        _check("h2o_chunk_step_host", lib().h2o_chunk_step_host(
            self._h, _ptr(q), _ptr(k_new), _ptr(v_new), n_q, _ptr(out), _ptr(colsum),
            _stream(stream)))
        if join:
            self.host_join(stream)
        return out

    def host_join(self, stream=None):
        """Makes the stream wait for every download step_host has issued."""
        _check("h2o_cache_host_join", lib().h2o_cache_host_join(self._h, _stream(stream)))

    def attention(self, q, k_new, v_new, stream=None):
        n_q = self._check_inputs(q, k_new, v_new)
        out = self._alloc_out(n_q)
        colsum = self._alloc_colsum(n_q)
        _check("h2o_attention", lib().h2o_attention(
            self._h, _ptr(q), _ptr(k_new), _ptr(v_new), n_q, _ptr(out), _ptr(colsum),
            _stream(stream)))
        return out, colsum

    def attention_backward(self, q, k_new, v_new, out, d_out, stream=None):
        """Gradients of ``attention``'s O (call it right after ``attention``
        with the same inputs, before the cache changes): returns float32
        (dq, dk_cache, dv_cache, dk_new, dv_new)."""
        n_q = self._check_inputs(q, k_new, v_new)
        s = self.shape
        f = dict(dtype=torch.float32, device=self.device)
        dq = torch.empty(s.batch, n_q, s.n_q_heads, s.head_dim, **f)
        dkc = torch.empty(s.batch, s.n_kv_heads, s.capacity, s.head_dim, **f)
        dvc = torch.empty_like(dkc)
        dkn = torch.empty(s.batch, n_q, s.n_kv_heads, s.head_dim, **f)
        dvn = torch.empty_like(dkn)
        out = out.contiguous()
        d_out = d_out.to(device=self.device, dtype=s.act_dtype).contiguous()
        _check("h2o_attention_backward", lib().h2o_attention_backward(
            self._h, _ptr(q), _ptr(k_new), _ptr(v_new), n_q, _ptr(out), _ptr(d_out), _ptr(dq),
            _ptr(dkc), _ptr(dvc), _ptr(dkn), _ptr(dvn), _stream(stream)))
        return dq, dkc, dvc, dkn, dvn

    def evict(self, colsum, k_new, v_new, stream=None):
        n_q = k_new.shape[1]
        colsum = colsum.to(device=self.device, dtype=torch.float32).contiguous()
        _check("h2o_evict", lib().h2o_evict(self._h, _ptr(colsum), _ptr(k_new), _ptr(v_new),
                                            n_q, _stream(stream)))

    def read(self, stream=None):
        """The cache state.  For the int8 cache (Q8) k and v are the codes
        [B, H_kv, C, d] int8 and k_scale, v_scale the row scales [B, H_kv, C]."""
        s = self.shape
        k = torch.empty_like(self.k)
        v = torch.empty_like(self.v)
        scores = torch.empty_like(self.scores)
        pos = torch.empty_like(self.pos)
        nt = (ctypes.c_int32 * 2)()
        _check("h2o_cache_read", lib().h2o_cache_read(self._h, _ptr(k), _ptr(v), _ptr(scores),
                                                      _ptr(pos), nt, _stream(stream)))
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        out = dict(k=k, v=v, scores=scores, pos=pos, n=nt[0], t0=nt[1])
        if s.q8:
            for name, raw in (("k", k), ("v", v)):
                codes, scale = self.split_q8(raw)
                out[name], out[name + "_scale"] = codes, scale
        return out

    def split_q8(self, raw: torch.Tensor):
        """(codes, scales) views of a raw int8-cache K or V buffer."""
        s = self.shape
        nc = s.batch * s.n_kv_heads * s.capacity * s.head_dim
        codes = raw[:nc].view(torch.int8).view(s.batch, s.n_kv_heads, s.capacity, s.head_dim)
        scale = raw[nc:].view(torch.float32).view(s.batch, s.n_kv_heads, s.capacity)
        return codes, scale

    @staticmethod
    def join_q8(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
        """The raw int8-cache buffer from codes and scales."""
        return torch.cat([codes.contiguous().view(torch.uint8).reshape(-1),
                          scale.to(torch.float32).contiguous().view(torch.uint8).reshape(-1)])

    def write(self, k, v, scores, pos, n, t0, stream=None, k_scale=None, v_scale=None):
        """Replaces the state.  For the int8 cache pass the codes as k, v and
        the row scales as k_scale, v_scale."""
        nt = (ctypes.c_int32 * 2)(n, t0)
        if self.shape.q8:
            k, v = self.join_q8(k, k_scale), self.join_q8(v, v_scale)
        k, v = k.to(self.device).contiguous(), v.to(self.device).contiguous()
        scores = scores.to(self.device, torch.float32).contiguous()
        pos = pos.to(self.device, torch.int32).contiguous()
        _check("h2o_cache_write", lib().h2o_cache_write(self._h, _ptr(k), _ptr(v), _ptr(scores),
                                                        _ptr(pos), nt, _stream(stream)))

    def check(self, stream=None) -> int:
        """Synchronises and returns the device status (0 = ok)."""
        return lib().h2o_cache_check(self._h, _stream(stream))

    def set_timing(self, enable: bool = True):
        _check("h2o_cache_set_timing", lib().h2o_cache_set_timing(self._h, int(enable)))

    def kernel_ms(self):
        """Durations (ms) of the last step's kernels: attention forward,
        summed weights, selection, scatter."""
        ms = (ctypes.c_float * 4)()
        _check("h2o_cache_kernel_ms", lib().h2o_cache_kernel_ms(self._h, ms))
        return list(ms)

    def info(self):
        n, t0, launches = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_uint64()
        _check("h2o_cache_info", lib().h2o_cache_info(self._h, ctypes.byref(n), ctypes.byref(t0),
                                                      ctypes.byref(launches)))
        return dict(n=n.value, t0=t0.value, kernel_launches=launches.value)
