"""ctypes binding of libelsaa.so (argument marshalling only).

Every step of the operator runs in the library's CUDA kernels; this module only
allocates caller-owned buffers with PyTorch and passes raw pointers and the
current CUDA stream.  The names follow include/elsaa.h.  There is no CPU
fallback: if the library is missing or no GPU is present, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libelsaa.so")

ELSAA_OK = 0
ELSAA_ERR_INVALID_ARG = 1
ELSAA_ERR_UNSUPPORTED = 2
ELSAA_ERR_WORKSPACE = 3
ELSAA_ERR_CUDA = 4
ELSAA_ERR_TIMEOUT = 5
ELSAA_DTYPE_F32 = 0
ELSAA_DTYPE_BF16 = 1
ELSAA_SEL_TOPK_BLOCKS = 0
ELSAA_SEL_SORTLSH = 1

EXPORTED = ("elsaa_saved_bytes", "elsaa_workspace_bytes", "elsaa_forward", "elsaa_backward",
            "elsaa_debug_select", "elsaa_check_device_flags", "elsaa_status_string",
            "elsaa_last_error_message", "elsaa_profile_begin", "elsaa_profile_end", "elsaa_select_noalloc",
            "elsaa_fusion_grads", "elsaa_debug_sortlsh", "elsaa_debug_set_wait_limit", "elsaa_step_host")


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("causal", ctypes.c_int32), ("rank_r", ctypes.c_int32),
                ("hash_bits", ctypes.c_int32), ("block_size", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("scale", ctypes.c_float), ("lam", ctypes.c_float), ("eps", ctypes.c_float),
                ("tau", ctypes.c_float), ("fixed_m", ctypes.c_int32), ("selector", ctypes.c_int32),
                ("lsh_bits", ctypes.c_int32), ("lsh_planes", ctypes.c_void_p)]


class ElsaaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({message})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libelsaa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_rank_approximation_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    L.elsaa_saved_bytes.argtypes = [P]
    L.elsaa_saved_bytes.restype = sz
    L.elsaa_workspace_bytes.argtypes = [P, i32]
    L.elsaa_workspace_bytes.restype = sz
    L.elsaa_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.elsaa_forward.restype = i32
    L.elsaa_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.elsaa_backward.restype = i32
    L.elsaa_debug_select.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
    L.elsaa_debug_select.restype = i32
    L.elsaa_check_device_flags.argtypes = [vp, vp]
    L.elsaa_check_device_flags.restype = i32
    L.elsaa_status_string.argtypes = [i32]
    L.elsaa_status_string.restype = ctypes.c_char_p
    L.elsaa_last_error_message.argtypes = []
    L.elsaa_last_error_message.restype = ctypes.c_char_p
    L.elsaa_profile_begin.argtypes = []
    L.elsaa_profile_begin.restype = i32
    L.elsaa_profile_end.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int), i32]
    L.elsaa_profile_end.restype = i32
    L.elsaa_select_noalloc.argtypes = [P, vp, vp, vp, vp]
    L.elsaa_select_noalloc.restype = i32
    L.elsaa_step_host.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp, vp]
    L.elsaa_step_host.restype = i32
    L.elsaa_fusion_grads.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.elsaa_fusion_grads.restype = i32
    L.elsaa_debug_sortlsh.argtypes = [P, vp, vp, vp, vp, vp]
    L.elsaa_debug_sortlsh.restype = i32
    L.elsaa_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong, i32]
    L.elsaa_debug_set_wait_limit.restype = i32
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != ELSAA_OK:
        L = lib()
        raise ElsaaError(status, where, L.elsaa_last_error_message().decode() or
                         L.elsaa_status_string(status).decode())


def make_params(B, H, N, d, *, dtype=ELSAA_DTYPE_BF16, causal=True, rank_r=128, block_size=128, topk=16,
                scale=None, lam=1.0, eps=1e-6, tau=1.0, hash_bits=4, fixed_m=False, selector=ELSAA_SEL_TOPK_BLOCKS,
                lsh_bits=0) -> Params:
    """The plain-data parameter block.  For the sortLSH selector the hyperplanes are
    attached by ``Elsaa(..., lsh_planes=...)``, which keeps them alive."""
    return Params(B, H, N, d, dtype, int(bool(causal)), rank_r, hash_bits, block_size, topk,
                  float(1.0 / math.sqrt(d) if scale is None else scale), float(lam), float(eps), float(tau),
                  int(bool(fixed_m)), int(selector), int(lsh_bits), None)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the ELSAA library must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the ELSAA library must be contiguous")
    return t.data_ptr()


def _host_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda or not t.is_pinned():
        raise ValueError("host buffers passed to the ELSAA library must be pinned CPU tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the ELSAA library must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Elsaa:
    """One operator configuration with its caller-owned saved/workspace buffers.

    ``forward`` and ``backward`` launch asynchronously on the current (or given)
    CUDA stream; all tensors are [B, H, N, d] contiguous CUDA tensors of the
    configured dtype (W: float32 [L, d, 4]; lam_vec/g_s/g_lr: float32 [B, H, N]).
    """

    def __init__(self, params: Params, device: Optional[torch.device] = None,
                 lsh_planes: Optional[torch.Tensor] = None):
        self.p = params
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        # sortLSH hyperplanes: float32 [d, lsh_bits] on the device, kept alive with the op
        self.lsh_planes = lsh_planes
        if lsh_planes is not None:
            self.p.lsh_planes = _ptr(lsh_planes)
        L = lib()
        self.saved_bytes = L.elsaa_saved_bytes(ctypes.byref(self.p))
        self.ws_fwd_bytes = L.elsaa_workspace_bytes(ctypes.byref(self.p), 0)
        self.ws_bwd_bytes = L.elsaa_workspace_bytes(ctypes.byref(self.p), 1)
        if self.saved_bytes == 0:
            _check(ELSAA_ERR_INVALID_ARG, "elsaa_saved_bytes")
        self.saved = torch.empty(self.saved_bytes, dtype=torch.uint8, device=self.device)
        self.ws = torch.empty(max(self.ws_fwd_bytes, self.ws_bwd_bytes), dtype=torch.uint8, device=self.device)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.p.dtype == ELSAA_DTYPE_BF16 else torch.float32

    def _empty_like_io(self):
        return torch.empty(self.p.B, self.p.H, self.p.N, self.p.d, dtype=self.torch_dtype, device=self.device)

    def forward(self, q, k, v, W, lam_vec=None, g_s=None, g_lr=None, out=None, stream=None):
        O = self._empty_like_io() if out is None else out
        st = lib().elsaa_forward(ctypes.byref(self.p), _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(lam_vec),
                                 _ptr(g_s), _ptr(g_lr), _ptr(O), _ptr(self.saved), _ptr(self.ws),
                                 self.ws.numel(), _stream(stream))
        _check(st, "elsaa_forward")
        return O

    def backward(self, q, k, v, W, dO, lam_vec=None, g_s=None, g_lr=None, grads=None, stream=None):
        dQ, dK, dV = grads if grads is not None else (self._empty_like_io(), self._empty_like_io(),
                                                      self._empty_like_io())
        st = lib().elsaa_backward(ctypes.byref(self.p), _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(lam_vec),
                                  _ptr(g_s), _ptr(g_lr), _ptr(dO), _ptr(self.saved), _ptr(dQ), _ptr(dK),
                                  _ptr(dV), _ptr(self.ws), self.ws.numel(), _stream(stream))
        _check(st, "elsaa_backward")
        return dQ, dK, dV

    def step_host(self, host_in, host_out, dev_in, dev_out, events, stream, h2d_stream, d2h_stream):
        """One forward + backward step from pinned host memory (``elsaa_step_host``).

        host_in: pinned CPU tensors (Q, K, V, dO, W, planes or None); host_out: (O, dQ, dK, dV);
        dev_in / dev_out: one device set of the same shapes; events: three recorded
        ``torch.cuda.Event`` of that set (inputs landed, step computed, results left)."""
        def arr(ts, conv):
            return (ctypes.c_void_p * len(ts))(*[conv(t) for t in ts])
        ins = list(host_in) + [None] * (6 - len(host_in))
        ev = (ctypes.c_void_p * 3)(*[e.cuda_event for e in events])
        st = lib().elsaa_step_host(ctypes.byref(self.p), arr(ins, _host_ptr), arr(host_out, _host_ptr),
                                   arr(dev_in, _ptr), arr(dev_out, _ptr),
                                   _ptr(self.saved), _ptr(self.ws), self.ws.numel(), stream.cuda_stream,
                                   h2d_stream.cuda_stream, d2h_stream.cuda_stream, ev)
        _check(st, "elsaa_step_host")

    def fusion_grads(self, dO, lam_vec=None, g_s=None, g_lr=None, stream=None):
        """Per-row gradients (dlambda, dg_sparse, dg_lr), float32 [B, H, N], of sum(dO * O)
        for the last forward call."""
        shape = (self.p.B, self.p.H, self.p.N)
        out = [torch.empty(shape, dtype=torch.float32, device=self.device) for _ in range(3)]
        st = lib().elsaa_fusion_grads(ctypes.byref(self.p), _ptr(lam_vec), _ptr(g_s), _ptr(g_lr), _ptr(dO),
                                      _ptr(self.saved), _ptr(out[0]), _ptr(out[1]), _ptr(out[2]), _stream(stream))
        _check(st, "elsaa_fusion_grads")
        return tuple(out)

    def debug_sortlsh(self, q, k, stream=None):
        """sortLSH codes and sorted orders, int32 [B, H, 2, N] each (0: queries, 1: keys)."""
        shape = (self.p.B, self.p.H, 2, self.p.N)
        codes = torch.empty(shape, dtype=torch.int32, device=self.device)
        order = torch.empty(shape, dtype=torch.int32, device=self.device)
        st = lib().elsaa_debug_sortlsh(ctypes.byref(self.p), _ptr(q), _ptr(k), _ptr(codes), _ptr(order),
                                       _stream(stream))
        _check(st, "elsaa_debug_sortlsh")
        return codes, order

    def debug_select(self, q, k, stream=None):
        n_t = -(-self.p.N // self.p.block_size)
        scores = torch.empty(self.p.B, self.p.H, n_t, n_t, dtype=torch.float32, device=self.device)
        idx = torch.empty(self.p.B, self.p.H, n_t, max(self.p.topk, 1), dtype=torch.int32, device=self.device)
        st = lib().elsaa_debug_select(ctypes.byref(self.p), _ptr(q), _ptr(k), _ptr(scores), _ptr(idx),
                                      _ptr(self.ws), self.ws.numel(), _stream(stream))
        _check(st, "elsaa_debug_select")
        return scores, idx[..., :self.p.topk]

    def check_device_flags(self, stream=None) -> int:
        return lib().elsaa_check_device_flags(_ptr(self.ws), _stream(stream))


def set_wait_limit(wait_ns: int = 0, stall: bool = False) -> None:
    """Test hook: limit of the tensor-core kernels' bounded waits for calls made from now on
    (0: the default 2 s); with ``stall`` the sparse forward first waits on a barrier that
    nothing completes, so its give-up path runs."""
    _check(lib().elsaa_debug_set_wait_limit(int(wait_ns), int(bool(stall))), "elsaa_debug_set_wait_limit")


def profile_begin() -> None:
    _check(lib().elsaa_profile_begin(), "elsaa_profile_begin")


def profile_end(max_entries: int = 64) -> dict:
    """{kernel name: (total device ms, launches)} since profile_begin()."""
    names = (ctypes.c_char_p * max_entries)()
    ms = (ctypes.c_double * max_entries)()
    cnt = (ctypes.c_int * max_entries)()
    n = lib().elsaa_profile_end(names, ms, cnt, max_entries)
    if n < 0:
        _check(ELSAA_ERR_CUDA, "elsaa_profile_end")
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(n)}


class ElsaaFunction(torch.autograd.Function):
    """Autograd wrapper: gradients for q, k, v (selection, W, lambda, gates constant)."""

    @staticmethod
    def forward(ctx, q, k, v, W, op: Elsaa, lam_vec=None, g_s=None, g_lr=None):
        O = op.forward(q, k, v, W, lam_vec, g_s, g_lr)
        ctx.op = op
        ctx.save_for_backward(q, k, v, W)
        ctx.extra = (lam_vec, g_s, g_lr)
        return O

    @staticmethod
    def backward(ctx, dO):
        q, k, v, W = ctx.saved_tensors
        dO = dO.contiguous()
        dQ, dK, dV = ctx.op.backward(q, k, v, W, dO, *ctx.extra)
        lam_vec, g_s, g_lr = ctx.extra
        need = [t is not None and t.requires_grad for t in (lam_vec, g_s, g_lr)]
        dl = dgs = dgl = None
        if any(need):
            dl, dgs, dgl = ctx.op.fusion_grads(dO, lam_vec, g_s, g_lr)
        return (dQ, dK, dV, None, None, dl if need[0] else None, dgs if need[1] else None,
                dgl if need[2] else None)
