"""Python handle on the fp64 CPU oracle (``qlinear_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The product library never
imports this module, and this module never imports the product: the two share
only the seeded input generators, which hold none of the method's arithmetic.

Every function takes and returns numpy arrays.  bf16 and f16 values travel as
their uint16 bit patterns, e4m3 codes as uint8, so no conversion happens in
Python: the oracle's own codecs do all of it.

Functions whose result no independent pin checks say "parity unpinned"; at
present every function here is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "qlinear_oracle.c"
_LIB = _HERE / "libqlinear_oracle.so"

# The format identifiers (numeric values of the library's public enum).
I8_G128_BF16 = 1
I8_G128_F16 = 2
I8A8_G128_BF16 = 3
I4_G64_BF16 = 4
I5Z_G128_F16 = 5
FP8_B128_BF16 = 6
FP8A8_B128_BF16 = 7
HADAMARD = 1

_c_p = ctypes.c_void_p
_c_i = ctypes.c_int


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (plain C, OpenMP over output rows)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", str(tmp), str(_SRC), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        L.qo_bf16_decode.restype = ctypes.c_double
        L.qo_bf16_decode.argtypes = [ctypes.c_uint16]
        L.qo_bf16_encode.restype = ctypes.c_uint16
        L.qo_bf16_encode.argtypes = [ctypes.c_double]
        L.qo_f16_decode.restype = ctypes.c_double
        L.qo_f16_decode.argtypes = [ctypes.c_uint16]
        L.qo_f16_encode.restype = ctypes.c_uint16
        L.qo_f16_encode.argtypes = [ctypes.c_double]
        L.qo_e4m3_decode.restype = ctypes.c_double
        L.qo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.qo_e4m3_encode.restype = ctypes.c_uint8
        L.qo_e4m3_encode.argtypes = [ctypes.c_double]
        for name, args in {
            "qo_fwht128_f64": [_c_p, _c_p],
            "qo_fwht128_spec_f32": [_c_p, _c_p],
            "qo_hadamard128_rotate": [_c_p, _c_i, _c_i, _c_p],
            "qo_act_quant_i8_g128": [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p],
            "qo_act_quant_group": [_c_p, _c_p, _c_p],
            "qo_act_quant_e4m3_g128": [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p],
            "qo_act_quant_e4m3_group": [_c_p, _c_p, _c_p],
            "qo_quant_i8_g128": [_c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p],
            "qo_scale_search_group": [_c_p, _c_i, _c_p, _c_p, _c_p],
            "qo_quant_i8_g128_search": [_c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p],
            "qo_quant_i4_g64": [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p],
            "qo_quant_fp8_b128": [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p],
            "qo_pack_i4": [_c_p, _c_i, _c_i, _c_p],
            "qo_unpack_i4": [_c_p, _c_i, _c_i, _c_p],
            "qo_pack_i5": [_c_p, _c_i, _c_i, _c_p],
            "qo_unpack_i5": [_c_p, _c_i, _c_i, _c_p],
            "qo_dequant": [_c_i, _c_p, _c_p, _c_p, _c_i, _c_i, _c_p],
        }.items():
            getattr(L, name).restype = None
            getattr(L, name).argtypes = args
        L.qo_packed_sizes.restype = _c_i
        L.qo_packed_sizes.argtypes = [_c_i, _c_i, _c_i, _c_p, _c_p, _c_p]
        L.qo_forward.restype = _c_i
        L.qo_forward.argtypes = [_c_p, _c_i, _c_i, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_p, _c_p]
        L.qo_moe_permute.restype = _c_i
        L.qo_moe_permute.argtypes = [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p]
        L.qo_moe_gate_up.restype = _c_i
        L.qo_moe_gate_up.argtypes = [_c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p]
        L.qo_gelu_tanh.restype = ctypes.c_double
        L.qo_gelu_tanh.argtypes = [ctypes.c_double]
        L.qo_moe_down_combine.restype = _c_i
        L.qo_moe_down_combine.argtypes = [_c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p]
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- scalar codecs -------------------------------------------------------
def bf16_decode(bits) -> np.ndarray:
    b = _c(bits, np.uint16).ravel()
    return np.array([lib().qo_bf16_decode(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def bf16_encode(vals) -> np.ndarray:
    v = _c(vals, np.float64).ravel()
    return np.array([lib().qo_bf16_encode(float(t)) for t in v], dtype=np.uint16).reshape(np.shape(vals))


def f16_decode(bits) -> np.ndarray:
    b = _c(bits, np.uint16).ravel()
    return np.array([lib().qo_f16_decode(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def f16_encode(vals) -> np.ndarray:
    v = _c(vals, np.float64).ravel()
    return np.array([lib().qo_f16_encode(float(t)) for t in v], dtype=np.uint16).reshape(np.shape(vals))


def e4m3_decode(bits) -> np.ndarray:
    b = _c(bits, np.uint8).ravel()
    return np.array([lib().qo_e4m3_decode(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def e4m3_encode(vals) -> np.ndarray:
    v = _c(vals, np.float64).ravel()
    return np.array([lib().qo_e4m3_encode(float(t)) for t in v], dtype=np.uint8).reshape(np.shape(vals))


# ---- transforms and quantisers --------------------------------------------
def fwht128_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(128, np.float64)
    lib().qo_fwht128_f64(_p(v), _p(out))
    return out


def fwht128_spec_f32(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(128, np.float32)
    lib().qo_fwht128_spec_f32(_p(v), _p(out))
    return out


def hadamard128_rotate(x_bits: np.ndarray) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    y = np.empty_like(x)
    lib().qo_hadamard128_rotate(_p(x), M, K, _p(y))
    return y


def act_quant_i8_g128(x_bits: np.ndarray, rotate: bool):
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M, K // 128), np.float32)
    lib().qo_act_quant_i8_g128(_p(x), M, K, int(rotate), _p(q), _p(s))
    return q, s


def act_quant_e4m3_g128(x_bits: np.ndarray, rotate: bool):
    """E4M3 codes (uint8) and fp32 scales per token per 128 (format 7's activations)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((M, K // 128), np.float32)
    lib().qo_act_quant_e4m3_g128(_p(x), M, K, int(rotate), _p(q), _p(s))
    return q, s


def act_quant_e4m3_group(v) -> tuple[np.ndarray, np.float32]:
    """Quantise one fp32 group of 128 values to E4M3 (no rotation)."""
    v = _c(v, np.float32)
    q = np.empty(128, np.uint8)
    s = np.empty(1, np.float32)
    lib().qo_act_quant_e4m3_group(_p(v), _p(q), _p(s))
    return q, s[0]


def act_quant_group(v) -> tuple[np.ndarray, np.float32]:
    """Quantise one fp32 group of 128 values (no rotation)."""
    v = _c(v, np.float32)
    q = np.empty(128, np.int8)
    s = np.empty(1, np.float32)
    lib().qo_act_quant_group(_p(v), _p(q), _p(s))
    return q, s[0]


def quant_i8_g128(W: np.ndarray, hadamard: bool = False, scale_f16: bool = False):
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 128), np.uint16)
    lib().qo_quant_i8_g128(_p(W), N, K, HADAMARD if hadamard else 0, int(scale_f16), _p(q), _p(s))
    return q, s


def scale_search_group(v, scale_f16: bool = False):
    """One fp32 group of 128 through the scale search: (codes, scale bits, chosen candidate i)."""
    v = _c(v, np.float32)
    q = np.empty(128, np.int8)
    s = np.empty(1, np.uint16)
    i = np.empty(1, np.int32)
    lib().qo_scale_search_group(_p(v), int(scale_f16), _p(q), _p(s), _p(i))
    return q, s[0], int(i[0])


def quant_i8_g128_search(W: np.ndarray, hadamard: bool = False, scale_f16: bool = False):
    """int8 g128 with the scale search: (codes [N, K], scale bits [N, K/128], chosen i [N, K/128])."""
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 128), np.uint16)
    ci = np.empty((N, K // 128), np.int32)
    lib().qo_quant_i8_g128_search(_p(W), N, K, HADAMARD if hadamard else 0, int(scale_f16), _p(q), _p(s), _p(ci))
    return q, s, ci


def quant_i4_g64(W: np.ndarray, hadamard: bool = False):
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 64), np.uint16)
    lib().qo_quant_i4_g64(_p(W), N, K, HADAMARD if hadamard else 0, _p(q), _p(s))
    return q, s


def quant_fp8_b128(W: np.ndarray, hadamard: bool = False):
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty(((N + 127) // 128, K // 128), np.uint16)
    lib().qo_quant_fp8_b128(_p(W), N, K, HADAMARD if hadamard else 0, _p(q), _p(s))
    return q, s


# ---- packers ----------------------------------------------------------------
def pack_i4(q: np.ndarray) -> np.ndarray:
    q = _c(q, np.int8)
    N, K = q.shape
    out = np.empty((N, K // 2), np.uint8)
    lib().qo_pack_i4(_p(q), N, K, _p(out))
    return out


def unpack_i4(p: np.ndarray, K: int) -> np.ndarray:
    p = _c(p, np.uint8)
    N = p.shape[0]
    q = np.empty((N, K), np.int8)
    lib().qo_unpack_i4(_p(p), N, K, _p(q))
    return q


def pack_i5(q: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    N, K = q.shape
    out = np.empty((N, K * 5 // 8), np.uint8)
    lib().qo_pack_i5(_p(q), N, K, _p(out))
    return out


def unpack_i5(p: np.ndarray, K: int) -> np.ndarray:
    p = _c(p, np.uint8)
    N = p.shape[0]
    q = np.empty((N, K), np.uint8)
    lib().qo_unpack_i5(_p(p), N, K, _p(q))
    return q


def packed_sizes(fmt: int, N: int, K: int):
    c, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    rc = lib().qo_packed_sizes(fmt, N, K, ctypes.byref(c), ctypes.byref(s), ctypes.byref(z))
    if rc:
        raise ValueError(f"unknown format {fmt}")
    return c.value, s.value, z.value


def dequant(fmt: int, codes, scales, zeros, N: int, K: int) -> np.ndarray:
    codes = _c(codes, np.uint8) if np.asarray(codes).dtype != np.int8 else _c(codes, np.int8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint8)
    W = np.empty((N, K), np.float64)
    lib().qo_dequant(fmt, _p(codes), _p(scales), _p(zeros), N, K, _p(W))
    return W


def forward(x_bits, codes, scales, zeros, fmt: int, flags: int, N: int, want_acc: bool = False):
    """y = x~ . dequant(W)^T in fp64; for W8A8 also the int32 group sums."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.ascontiguousarray(codes)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint8)
    y = np.empty((M, N), np.float64)
    acc = np.empty((M, N, K // 128), np.int32) if want_acc else None
    rc = lib().qo_forward(_p(x), M, K, _p(codes), _p(scales), _p(zeros), fmt, flags, N, _p(y), _p(acc))
    if rc:
        raise ValueError(f"oracle forward rejected format {fmt}")
    return (y, acc) if want_acc else y


def moe_permute(ids: np.ndarray, E: int):
    ids = _c(ids, np.int32)
    T, topk = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.full(T * topk, -1, np.int32)
    bad = lib().qo_moe_permute(_p(ids), T, topk, E, _p(counts), _p(offsets), _p(perm))
    return counts, offsets, perm, bad


def moe_gate_up(x_bits, ids, codes, scales, fmt: int, flags: int, E: int, N: int):
    x = _c(x_bits, np.uint16)
    ids = _c(ids, np.int32)
    T, K = x.shape
    topk = ids.shape[1]
    codes = np.ascontiguousarray(codes)
    scales = _c(scales, np.uint16)
    out = np.zeros((T, topk, N), np.float64)
    rc = lib().qo_moe_gate_up(_p(x), _p(ids), T, topk, E, N, K, fmt, flags, _p(codes), _p(scales), _p(out))
    if rc:
        raise ValueError(f"oracle moe_gate_up rejected format {fmt}")
    return out


def gelu_tanh(v) -> np.ndarray:
    """The tanh form of GELU in fp64, element by element."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty_like(v)
    f = lib().qo_gelu_tanh
    for i, x in enumerate(v.ravel()):
        out.ravel()[i] = f(float(x))
    return out


def moe_down_combine(h, ids, weights, wd_bits, E: int):
    """out [T, K] fp64: per pair gelu(gate) * up of its gate_up row h [T, topk, 2I] (fp32), through its
    expert's bf16 down weight wd [E, K, I], summed over the slots with the routing weights."""
    h = _c(h, np.float32)
    ids = _c(ids, np.int32)
    w = _c(weights, np.float32)
    wd = _c(wd_bits, np.uint16)
    T, topk = ids.shape
    I = h.shape[-1] // 2
    K = wd.shape[1]
    out = np.empty((T, K), np.float64)
    lib().qo_moe_down_combine(_p(h), _p(ids), _p(w), T, topk, E, I, K, _p(wd), _p(out))
    return out
