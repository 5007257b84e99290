"""CPU oracle of the residual-compression activation codec (test infrastructure).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline / reference leg may load this package; the product path never
does, and the CUDA path shares no code with it.

The arithmetic lives in ``cf_oracle.c`` (plain C, built with
``-O2 -ffp-contract=off -fno-fast-math``); this module only builds it, loads it
with ctypes and marshals numpy arrays.  ctypes releases the GIL during each
call, so independent slots can run on several host threads.

Sources: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (arXiv 2507.17511) -- abstract (residuals plus error feedback),
reproducibility table "Dataset Splits" row (1-step warmup initialises the base
tensor) and "Pseudocode" row, Algorithm 3 (subspace iteration).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cf_oracle.c")
_LIB = os.path.join(_HERE, "libcf_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
           "-fPIC", "-shared", "-Wall", "-Wextra"]

FLAG_NONFINITE = 0x1


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libcf_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # CF_ORACLE_LIB names another build of this source (the mutation test
        # runs the pins against deliberately broken copies of the oracle)
        _lib = ctypes.CDLL(os.environ.get("CF_ORACLE_LIB") or build())
        P, I64, I, U32P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)
        _lib.cfo_warmup_sender.argtypes = [I64, P, P, P]
        _lib.cfo_warmup_receiver.argtypes = [I64, P, P]
        _lib.cfo_residual.argtypes = [I64, P, P, P, P]
        _lib.cfo_compress.argtypes = [I64, I, I, I, P, P, P, P, P, U32P]
        _lib.cfo_decompress.argtypes = [I64, I, I, P, P, P]
        _lib.cfo_payload_bytes.argtypes = [I64, I, I]
        _lib.cfo_payload_bytes.restype = I64
        _lib.cfo_put_code.argtypes = [P, I64, I, ctypes.c_uint]
        _lib.cfo_get_code.argtypes = [P, I64, I, ctypes.POINTER(ctypes.c_uint)]
        _lib.cfo_cholqr.argtypes = [I64, I, P, P, P]
        _lib.cfo_subspace_iteration.argtypes = [I64, I64, I, I, P, P, P, P, P]
        _lib.cfo_lowrank_apply.argtypes = [I64, I64, I, P, P, P, P, P, P, P, P]
        _lib.cfo_warmup_sender_lean.argtypes = [I64, P, P, P]
        _lib.cfo_warmup_receiver_lean.argtypes = [I64, P, P]
        _lib.cfo_compress_lean.argtypes = [I64, I, I, I, P, P, P, P, P, U32P]
        _lib.cfo_decompress_lean.argtypes = [I64, I, I, P, P, P]
        _lib.cfo_to_bf16.argtypes = [I64, P, P]
        _lib.cfo_attention.argtypes = [I64, I64, I64, P, P, P, P, P]
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def _u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype in (np.uint16, np.int16), "bf16 data is passed as raw 16-bit patterns"
    return x.view(np.uint16)


# ------------------------------------------------------------ quantised path

def warmup_sender(x_bits: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Step 0 on the sender: returns (base bf16 bits, E = 0 fp32)."""
    x = _u16(x_bits).ravel()
    base = np.empty_like(x)
    err = np.empty(x.size, np.float32)
    _check(lib().cfo_warmup_sender(x.size, _ptr(x), _ptr(base), _ptr(err)), "warmup_sender")
    return base, err


def warmup_receiver(x_bits: np.ndarray) -> np.ndarray:
    """Step 0 on the receiver: returns the cache C = float(X_0)."""
    x = _u16(x_bits).ravel()
    cache = np.empty(x.size, np.float32)
    _check(lib().cfo_warmup_receiver(x.size, _ptr(x), _ptr(cache)), "warmup_receiver")
    return cache


def residual(x_bits: np.ndarray, base: np.ndarray, err: np.ndarray) -> np.ndarray:
    """A = (X_t - base) + E in fp32; advances ``base`` to X_t in place."""
    x = _u16(x_bits).ravel()
    assert base.dtype == np.uint16 and base.flags["C_CONTIGUOUS"] and err.dtype == np.float32
    a = np.empty(x.size, np.float32)
    _check(lib().cfo_residual(x.size, _ptr(x), _ptr(base), _ptr(err), _ptr(a)), "residual")
    return a


def payload_bytes(n: int, bits: int, group: int) -> int:
    return int(lib().cfo_payload_bytes(n, bits, group))


def compress(x_bits: np.ndarray, base: np.ndarray, err: np.ndarray, bits: int, group: int,
             sign_scale: int = 0) -> Tuple[np.ndarray, np.ndarray, int]:
    """Sender step t >= 1.  Updates ``base`` and ``err`` in place.

    Returns (codes u8 [n*bits/8], scales fp32 [n/group], flags).
    """
    x = _u16(x_bits).ravel()
    n = x.size
    assert base.dtype == np.uint16 and base.size == n and base.flags["C_CONTIGUOUS"]
    assert err.dtype == np.float32 and err.size == n and err.flags["C_CONTIGUOUS"]
    if n % group:
        raise ValueError("n must be a multiple of the group size")
    codes = np.zeros(n * bits // 8, np.uint8)
    scales = np.empty(n // group, np.float32)
    flags = ctypes.c_uint32(0)
    _check(lib().cfo_compress(n, bits, group, sign_scale, _ptr(x), _ptr(base), _ptr(err), _ptr(codes),
                              _ptr(scales), ctypes.byref(flags)), "compress")
    return codes, scales, int(flags.value)


def decompress(codes: np.ndarray, scales: np.ndarray, cache: np.ndarray, bits: int, group: int) -> None:
    """Receiver step t >= 1: C += dequant(codes, scales), in place."""
    assert cache.dtype == np.float32 and cache.flags["C_CONTIGUOUS"]
    n = cache.size
    assert codes.dtype == np.uint8 and codes.size == n * bits // 8
    assert scales.dtype == np.float32 and scales.size == n // group
    _check(lib().cfo_decompress(n, bits, group, _ptr(np.ascontiguousarray(codes)),
                                _ptr(np.ascontiguousarray(scales)), _ptr(cache)), "decompress")


def to_bf16(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (raw 16-bit patterns), round to nearest even."""
    f = np.ascontiguousarray(f, dtype=np.float32).ravel()
    out = np.empty(f.size, np.uint16)
    _check(lib().cfo_to_bf16(f.size, _ptr(f), _ptr(out)), "to_bf16")
    return out


def put_code(stream: np.ndarray, i: int, bits: int, code: int) -> None:
    _check(lib().cfo_put_code(_ptr(stream), i, bits, code), "put_code")


def get_code(stream: np.ndarray, i: int, bits: int) -> int:
    c = ctypes.c_uint(0)
    _check(lib().cfo_get_code(_ptr(stream), i, bits, ctypes.byref(c)), "get_code")
    return int(c.value)


def compress_lean(x_bits: np.ndarray, base: np.ndarray, err_bits: np.ndarray, bits: int, group: int,
                  sign_scale: int = 0) -> Tuple[np.ndarray, np.ndarray, int]:
    """Sender step with bf16 E (raw bits, updated in place)."""
    x = _u16(x_bits).ravel()
    n = x.size
    assert base.dtype == np.uint16 and err_bits.dtype == np.uint16 and err_bits.size == n
    codes = np.zeros(n * bits // 8, np.uint8)
    scales = np.empty(n // group, np.float32)
    flags = ctypes.c_uint32(0)
    _check(lib().cfo_compress_lean(n, bits, group, sign_scale, _ptr(x), _ptr(base), _ptr(err_bits), _ptr(codes),
                                   _ptr(scales), ctypes.byref(flags)), "compress_lean")
    return codes, scales, int(flags.value)


def decompress_lean(codes: np.ndarray, scales: np.ndarray, cache_bits: np.ndarray, bits: int, group: int) -> None:
    """Receiver step with a bf16 cache (raw bits, updated in place)."""
    assert cache_bits.dtype == np.uint16 and cache_bits.flags["C_CONTIGUOUS"]
    _check(lib().cfo_decompress_lean(cache_bits.size, bits, group, _ptr(np.ascontiguousarray(codes)),
                                     _ptr(np.ascontiguousarray(scales)), _ptr(cache_bits)), "decompress_lean")


class QuantSlot:
    """Sender + receiver state of one slot, stepped by the oracle.

    ``lean=True`` keeps E and C in bf16 (raw 16-bit patterns) instead of fp32.
    """

    def __init__(self, bits: int, group: int, sign_scale: int = 0, lean: bool = False):
        self.bits, self.group, self.sign_scale, self.lean = bits, group, sign_scale, lean
        self.base = self.err = self.cache = None
        self.codes = self.scales = None
        self.flags = 0

    @property
    def recon(self) -> np.ndarray:
        """The receiver's reconstruction in bf16 (raw bits): bf16(C) after the last step."""
        return self.cache.copy() if self.lean else to_bf16(self.cache)

    def step(self, t: int, x_bits: np.ndarray) -> None:
        if self.lean:
            x = _u16(x_bits).ravel()
            if t == 0:
                self.base = np.empty_like(x)
                self.err = np.empty_like(x)
                self.cache = np.empty_like(x)
                _check(lib().cfo_warmup_sender_lean(x.size, _ptr(x), _ptr(self.base), _ptr(self.err)), "warmup")
                _check(lib().cfo_warmup_receiver_lean(x.size, _ptr(x), _ptr(self.cache)), "warmup")
                return
            self.codes, self.scales, fl = compress_lean(x, self.base, self.err, self.bits, self.group,
                                                        self.sign_scale)
            self.flags |= fl
            decompress_lean(self.codes, self.scales, self.cache, self.bits, self.group)
            return
        if t == 0:
            self.base, self.err = warmup_sender(x_bits)
            self.cache = warmup_receiver(x_bits)
            return
        self.codes, self.scales, fl = compress(x_bits, self.base, self.err, self.bits, self.group,
                                               self.sign_scale)
        self.flags |= fl
        decompress(self.codes, self.scales, self.cache, self.bits, self.group)


# ----------------------------------------------------------- low-rank path

def cholqr(Z: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """CholeskyQR in fp64: returns (Q, R) with Z = Q R, R upper triangular."""
    Z = np.ascontiguousarray(Z, dtype=np.float64)
    rows, r = Z.shape
    Q = np.empty_like(Z)
    R = np.empty((r, r), np.float64)
    _check(lib().cfo_cholqr(rows, r, _ptr(Z), _ptr(Q), _ptr(R)), "cholqr")
    return Q, R


def subspace_iteration(A: np.ndarray, Q0: np.ndarray, T: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Algorithm 3 on fp32 A [m, n] from start block Q0 [n, r]: returns (U, R, V) fp64."""
    A = np.ascontiguousarray(A, dtype=np.float32)
    Q0 = np.ascontiguousarray(Q0, dtype=np.float32)
    m, n = A.shape
    r = Q0.shape[1]
    assert Q0.shape[0] == n
    U = np.empty((m, r), np.float64)
    R = np.empty((r, r), np.float64)
    V = np.empty((n, r), np.float64)
    _check(lib().cfo_subspace_iteration(m, n, r, T, _ptr(A), _ptr(Q0), _ptr(U), _ptr(R), _ptr(V)),
           "subspace_iteration")
    return U, R, V


def lowrank_apply(A: np.ndarray, U: np.ndarray, R: np.ndarray, V: np.ndarray,
                  C_in: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]:
    """D = U R V^T, E = A - D and C_out = C_in + D (fp64)."""
    A = np.ascontiguousarray(A, dtype=np.float32)
    m, n = A.shape
    r = U.shape[1]
    D = np.empty((m, n), np.float64)
    E = np.empty((m, n), np.float64)
    C_out = None
    if C_in is not None:
        C_in = np.ascontiguousarray(C_in, dtype=np.float32)
        C_out = np.empty((m, n), np.float64)
    _check(lib().cfo_lowrank_apply(m, n, r, _ptr(A), _ptr(np.ascontiguousarray(U, np.float64)),
                                   _ptr(np.ascontiguousarray(R, np.float64)),
                                   _ptr(np.ascontiguousarray(V, np.float64)), _ptr(D), _ptr(E),
                                   _ptr(C_in), _ptr(C_out)), "lowrank_apply")
    return D, E, C_out


# ----------------------------------------------------------------- attention

def attention(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, cols: int, lse: bool = False):
    """softmax(q k^T / 8) v per head of 64 channels, in fp64.

    q [lq, cols], k and v [lk, cols] as raw bf16 bit patterns (token-major);
    returns fp64 [lq, cols], and with ``lse`` also the fp64 log-sum-exp of the
    scaled scores [lq, cols // 64] (the weight of this K/V block when partial
    results over several blocks are merged)."""
    q = np.ascontiguousarray(_u16(q_bits)).reshape(-1, cols)
    k = np.ascontiguousarray(_u16(k_bits)).reshape(-1, cols)
    v = np.ascontiguousarray(_u16(v_bits)).reshape(-1, cols)
    assert k.shape == v.shape
    out = np.empty((q.shape[0], cols), np.float64)
    ls = np.empty((q.shape[0], cols // 64), np.float64) if lse else None
    _check(lib().cfo_attention(q.shape[0], k.shape[0], cols, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                               _ptr(ls) if lse else None), "attention")
    return (out, ls) if lse else out
