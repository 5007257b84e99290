"""ctypes binding of libcf (the C ABI in include/cf.h): argument marshalling only.

Every step of the codec runs in the CUDA kernels behind libcf.  This module
only converts torch tensors / Python values to the C structs and pointers the
ABI takes, and raises on a non-OK status.  If libcf.so is missing, loading
fails loudly; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcf.so")

CF_OK, CF_E_ARG, CF_E_SHAPE, CF_E_ALIGN, CF_E_STATE, CF_E_NOMEM, CF_E_CUDA, CF_E_NONFINITE, CF_E_TIMEOUT = range(9)
STATUS_NAMES = {0: "CF_OK", 1: "CF_E_ARG", 2: "CF_E_SHAPE", 3: "CF_E_ALIGN", 4: "CF_E_STATE", 5: "CF_E_NOMEM",
                6: "CF_E_CUDA", 7: "CF_E_NONFINITE", 8: "CF_E_TIMEOUT"}
CF_MODE_QUANT, CF_MODE_LOWRANK = 0, 1
CF_PRECISION_AUTO, CF_PRECISION_TF32, CF_PRECISION_SPLIT = 0, 1, 2

EXPORTED = ["cf_create", "cf_workspace_bytes", "cf_set_workspace", "cf_compress", "cf_decompress",
            "cf_lowrank_workspace_bytes", "cf_lowrank", "cf_check", "cf_payload_bytes", "cf_last_error",
            "cf_destroy", "cf_lowrank_noalloc", "cf_loopback", "cf_resume", "cf_trace_enable", "cf_trace_read",
            "cf_attention"]
NOALLOC_SCRATCH_BYTES = 8 << 20


class cf_config(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("bits", ctypes.c_int), ("group", ctypes.c_int),
                ("sign_scale", ctypes.c_int), ("rank", ctypes.c_int), ("iters", ctypes.c_int),
                ("state_bf16", ctypes.c_int), ("warm_start", ctypes.c_int), ("precision", ctypes.c_int)]


class cf_shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class cf_trace_entry(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char * 80), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


class cf_slot(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("base", ctypes.c_void_p), ("err", ctypes.c_void_p),
                ("cache", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("q0", ctypes.c_void_p), ("U", ctypes.c_void_p), ("R", ctypes.c_void_p), ("V", ctypes.c_void_p),
                ("recon", ctypes.c_void_p)]


class cf_kv(ctypes.Structure):
    _fields_ = [("bf16", ctypes.c_void_p), ("cache_in", ctypes.c_void_p), ("cache_out", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class CfError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libcf.so (built by ``python -m activation_residual_compression_02_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libcf.so not built ({_LIB_PATH}); run python -m "
                              "activation_residual_compression_02_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.cf_create.argtypes = [ctypes.POINTER(cf_config), I, ctypes.POINTER(cf_shape), ctypes.POINTER(P)]
        L.cf_create.restype = I
        L.cf_workspace_bytes.argtypes = [P]
        L.cf_workspace_bytes.restype = SZ
        L.cf_set_workspace.argtypes = [P, P, SZ]
        L.cf_set_workspace.restype = I
        L.cf_compress.argtypes = [P, ctypes.POINTER(cf_slot), I, P]
        L.cf_compress.restype = I
        L.cf_decompress.argtypes = [P, ctypes.POINTER(cf_slot), I, P]
        L.cf_decompress.restype = I
        L.cf_loopback.argtypes = [P, ctypes.POINTER(cf_slot), I, P]
        L.cf_loopback.restype = I
        L.cf_lowrank_workspace_bytes.argtypes = [P, I, I64, I64]
        L.cf_lowrank_workspace_bytes.restype = SZ
        PP = ctypes.POINTER(P)
        L.cf_lowrank.argtypes = [P, I, I64, I64, PP, PP, PP, PP, PP, PP, PP, P]
        L.cf_lowrank.restype = I
        L.cf_check.argtypes = [P, P]
        L.cf_check.restype = I
        L.cf_payload_bytes.argtypes = [P, I]
        L.cf_payload_bytes.restype = SZ
        L.cf_last_error.argtypes = [P]
        L.cf_last_error.restype = ctypes.c_char_p
        L.cf_destroy.argtypes = [P]
        L.cf_destroy.restype = I
        L.cf_resume.argtypes = [P, I64]
        L.cf_resume.restype = I
        L.cf_trace_enable.argtypes = [P, I]
        L.cf_trace_enable.restype = I
        L.cf_trace_read.argtypes = [P, ctypes.POINTER(cf_trace_entry), I]
        L.cf_trace_read.restype = I
        L.cf_lowrank_noalloc.argtypes = [ctypes.POINTER(cf_config), I, I64, I64, PP, PP, PP, PP, PP, PP, PP, P]
        L.cf_lowrank_noalloc.restype = I
        L.cf_attention.argtypes = [P, I64, I64, I64, P, ctypes.POINTER(cf_kv), ctypes.POINTER(cf_kv), P, P, P]
        L.cf_attention.restype = I
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcf takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libcf takes contiguous tensors")
    return t.data_ptr()


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _parr(ts: Optional[Sequence[Optional[torch.Tensor]]]):
    if ts is None:
        return None
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t)
    return arr


class Slot:
    """Per-slot tensors for one call (any may be None when a call does not use it)."""

    __slots__ = ("x", "base", "err", "cache", "codes", "scales", "q0", "U", "R", "V", "recon")

    def __init__(self, x=None, base=None, err=None, cache=None, codes=None, scales=None, q0=None, U=None, R=None,
                 V=None, recon=None):
        self.x, self.base, self.err, self.cache = x, base, err, cache
        self.codes, self.scales, self.q0, self.U, self.R, self.V = codes, scales, q0, U, R, V
        self.recon = recon

    def to_c(self) -> cf_slot:
        return cf_slot(*[_ptr(getattr(self, f)) for f in Slot.__slots__])


class KV:
    """K or V of a received shard for ``Context.attention`` (``cf_kv``): either
    ``bf16`` [lk, cols], or the receiver's ``cache_in`` [lk, cols] fp32 with
    this step's ``codes`` and ``scales`` (dequantise-on-load; ``cache_out``
    [lk, cols] fp32 receives the updated cache)."""

    __slots__ = ("bf16", "cache_in", "cache_out", "codes", "scales")

    def __init__(self, bf16=None, cache_in=None, cache_out=None, codes=None, scales=None):
        self.bf16, self.cache_in, self.cache_out, self.codes, self.scales = bf16, cache_in, cache_out, codes, scales

    def to_c(self) -> cf_kv:
        return cf_kv(*[_ptr(getattr(self, f)) for f in KV.__slots__])

    def check(self, lk: int, cols: int, bits: int, group: int, name: str):
        want = {"bf16": (torch.bfloat16, lk * cols), "cache_in": (torch.float32, lk * cols),
                "cache_out": (torch.float32, lk * cols), "codes": (torch.uint8, lk * cols * bits // 8),
                "scales": (torch.float32, lk * cols // group if group else 0)}
        for f in KV.__slots__:
            t = getattr(self, f)
            if t is None:
                continue
            dt, n = want[f]
            if t.dtype != dt or t.numel() != n:
                raise ValueError(f"{name}.{f} must be {dt} with {n} elements, not {t.dtype} with {t.numel()}")


class Context:
    """A libcf context (``cf_create`` ... ``cf_destroy``)."""

    def __init__(self, shapes: Sequence[Sequence[int]], mode: int = CF_MODE_QUANT, bits: int = 2, group: int = 128,
                 sign_scale: int = 0, rank: int = 16, iters: int = 2, state_bf16: int = 0, warm_start: int = 0,
                 precision: int = CF_PRECISION_AUTO):
        L = lib()
        self.cfg = cf_config(mode, bits, group, sign_scale, rank, iters, state_bf16, warm_start, precision)
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        arr = (cf_shape * max(1, len(self.shapes)))(*[cf_shape(r, c) for r, c in self.shapes])
        h = ctypes.c_void_p()
        st = L.cf_create(ctypes.byref(self.cfg), len(self.shapes), arr, ctypes.byref(h))
        if st != CF_OK:
            raise CfError(st, "cf_create failed")
        self._h = h
        self._ws = None

    # -- plumbing -----------------------------------------------------------
    def _raise(self, st: int, what: str):
        if st != CF_OK:
            raise CfError(st, f"{what}: {lib().cf_last_error(self._h).decode()}")

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            lib().cf_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self) -> int:
        return int(lib().cf_workspace_bytes(self._h))

    def lowrank_workspace_bytes(self, nmat: int, m: int, n: int) -> int:
        return int(lib().cf_lowrank_workspace_bytes(self._h, nmat, m, n))

    def set_workspace(self, ws: Optional[torch.Tensor]):
        self._ws = ws
        st = lib().cf_set_workspace(self._h, _ptr(ws) if ws is not None else None,
                                    ws.numel() * ws.element_size() if ws is not None else 0)
        self._raise(st, "cf_set_workspace")

    def payload_bytes(self, slot: int) -> int:
        return int(lib().cf_payload_bytes(self._h, slot))

    # -- codec calls --------------------------------------------------------
    def _slots(self, slots: Sequence[Slot]):
        arr = (cf_slot * max(1, len(slots)))()
        for i, s in enumerate(slots):
            arr[i] = s.to_c()
        return arr

    def compress(self, slots: Sequence[Slot], step: int, stream: Optional[torch.cuda.Stream] = None):
        self._raise(lib().cf_compress(self._h, self._slots(slots), step, _stream_handle(stream)), "cf_compress")

    def decompress(self, slots: Sequence[Slot], step: int, stream: Optional[torch.cuda.Stream] = None):
        self._raise(lib().cf_decompress(self._h, self._slots(slots), step, _stream_handle(stream)), "cf_decompress")

    def loopback(self, slots: Sequence[Slot], step: int, stream: Optional[torch.cuda.Stream] = None):
        self._raise(lib().cf_loopback(self._h, self._slots(slots), step, _stream_handle(stream)), "cf_loopback")

    def lowrank(self, A: List[torch.Tensor], Q0: List[torch.Tensor], U: List[torch.Tensor], R: List[torch.Tensor],
                V: List[torch.Tensor], E: Optional[List[torch.Tensor]] = None, C: Optional[List[torch.Tensor]] = None,
                stream: Optional[torch.cuda.Stream] = None):
        nmat = len(A)
        _, m, n = _check_lowrank_tensors(A, Q0, U, R, V, E, C, self.cfg.rank)
        st = lib().cf_lowrank(self._h, nmat, m, n, _parr(A), _parr(Q0), _parr(U), _parr(R), _parr(V), _parr(E),
                              _parr(C), _stream_handle(stream))
        self._raise(st, "cf_lowrank")

    def attention(self, q: torch.Tensor, k: KV, v: KV, out: torch.Tensor, lk: Optional[int] = None,
                  stream: Optional[torch.cuda.Stream] = None, lse: Optional[torch.Tensor] = None):
        """cf_attention: out = softmax(q k^T / 8) v per head of 64 channels.
        q and out are bf16 [lq, cols]; lk defaults to the rows of k's tensors;
        lse (optional) is fp32 [lq, cols // 64] and receives each row's
        log-sum-exp of the scaled scores (to merge partial results over blocks)."""
        if q.dim() != 2 or q.dtype != torch.bfloat16 or out.dtype != torch.bfloat16 or out.shape != q.shape:
            raise ValueError("q and out must be bf16 [lq, cols] of the same shape")
        lq, cols = int(q.shape[0]), int(q.shape[1])
        if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (lq, cols // 64)
                                or not lse.is_contiguous()):
            raise ValueError("lse must be a contiguous fp32 [lq, cols // 64] tensor")
        if lk is None:
            t = k.bf16 if k.bf16 is not None else k.cache_in
            lk = int(t.numel() // cols) if t is not None else 0
        for kv, name in ((k, "k"), (v, "v")):
            kv.check(lk, cols, self.cfg.bits, self.cfg.group, name)
        kc, vc = k.to_c(), v.to_c()
        st = lib().cf_attention(self._h, lq, lk, cols, _ptr(q), ctypes.byref(kc), ctypes.byref(vc), _ptr(out),
                                _ptr(lse) if lse is not None else None, _stream_handle(stream))
        self._raise(st, "cf_attention")

    def trace(self, on: bool = True):
        """Time every kernel launch of this context with CUDA events (cf_trace_enable)."""
        self._raise(lib().cf_trace_enable(self._h, int(bool(on))), "cf_trace_enable")

    def trace_read(self) -> List[dict]:
        """Per-kernel launches and summed milliseconds since the last read (cf_trace_read)."""
        cap = 64
        buf = (cf_trace_entry * cap)()
        n = lib().cf_trace_read(self._h, buf, cap)
        if n < 0:
            raise CfError(-n, f"cf_trace_read: {lib().cf_last_error(self._h).decode()}")
        return [{"kernel": buf[i].kernel.decode(), "launches": buf[i].launches, "total_ms": buf[i].total_ms}
                for i in range(min(n, cap))]

    def resume(self, steps_done: int):
        """Continue a run whose state buffers the caller restored (steps
        0..steps_done done); the next call may be step steps_done + 1."""
        self._raise(lib().cf_resume(self._h, steps_done), "cf_resume")

    def check(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        """Synchronise and return the device status (CF_OK, CF_E_NONFINITE, ...)."""
        return int(lib().cf_check(self._h, _stream_handle(stream)))


def cf_create(shapes, **kw) -> Context:
    return Context(shapes, **kw)


def cf_compress(ctx: Context, slots, step, stream=None):
    ctx.compress(slots, step, stream)


def cf_decompress(ctx: Context, slots, step, stream=None):
    ctx.decompress(slots, step, stream)


def cf_loopback(ctx: Context, slots, step, stream=None):
    ctx.loopback(slots, step, stream)


def cf_lowrank(ctx: Context, A, Q0, U, R, V, E=None, C=None, stream=None):
    ctx.lowrank(A, Q0, U, R, V, E, C, stream)


def _check_lowrank_tensors(A, Q0, U, R, V, E, C, r: int):
    """Device, dtype and shape of every tensor of a low-rank call (the C ABI
    takes raw pointers, so a wrong dtype or shape would read or write out of
    bounds).  Returns (device, m, n)."""
    nmat = len(A)
    if nmat == 0:
        return None, 0, 0
    if A[0].dim() != 2:
        raise ValueError("A[i] must be [m, n]")
    dev = A[0].device
    m, n = int(A[0].shape[0]), int(A[0].shape[1])
    want = {"A": (m, n), "Q0": (n, r), "U": (m, r), "R": (r, r), "V": (n, r), "E": (m, n), "C": (m, n)}
    for name, ts in (("A", A), ("Q0", Q0), ("U", U), ("R", R), ("V", V), ("E", E), ("C", C)):
        if ts is None:
            continue
        if len(ts) != nmat:
            raise ValueError(f"{name} must hold {nmat} tensors")
        for i, t in enumerate(ts):
            if t.device != dev:
                raise ValueError(f"{name}[{i}] is on {t.device}, A[0] on {dev}")
            if t.dtype != torch.float32:
                raise ValueError(f"{name}[{i}] must be float32, not {t.dtype}")
            if tuple(t.shape) != want[name]:
                raise ValueError(f"{name}[{i}] must have shape {list(want[name])}, not {list(t.shape)}")
    return dev, m, n


def cf_lowrank_noalloc(A, Q0, U, R, V, E=None, C=None, rank: int = 16, iters: int = 2, stream=None,
                       precision: int = CF_PRECISION_AUTO) -> int:
    """cf_lowrank without a context or workspace, for callers that cannot
    allocate device memory: the scratch is a fixed 8 MiB device array inside
    libcf.  Runs on the device of A[0] (made current for the call); every
    tensor must be a float32 tensor of that device with its call shape.
    Synchronous; returns the C status (CF_OK, CF_E_NOMEM when the call does
    not fit the scratch, ...)."""
    cfg = cf_config(CF_MODE_LOWRANK, 0, 0, 0, rank, iters, 0, 0, precision)
    nmat = len(A)
    dev, m, n = _check_lowrank_tensors(A, Q0, U, R, V, E, C, rank)
    L = lib()
    if dev is None:
        return int(L.cf_lowrank_noalloc(ctypes.byref(cfg), 0, 0, 0, None, None, None, None, None, None, None,
                                        _stream_handle(stream)))
    with torch.cuda.device(dev):
        return int(L.cf_lowrank_noalloc(ctypes.byref(cfg), nmat, m, n, _parr(A), _parr(Q0), _parr(U), _parr(R),
                                        _parr(V), _parr(E), _parr(C), _stream_handle(stream)))


def cf_check(ctx: Context, stream=None) -> int:
    return ctx.check(stream)


def cf_payload_bytes(ctx: Context, slot: int) -> int:
    return ctx.payload_bytes(slot)


def cf_resume(ctx: Context, steps_done: int):
    ctx.resume(steps_done)


def cf_destroy(ctx: Context):
    ctx.close()
