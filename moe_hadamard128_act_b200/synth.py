"""Seeded synthetic inputs for the quantized linear layer and its MoE use.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no transform, no quantiser, no packing, no matmul).  Both
the CUDA path and the CPU oracle consume exactly the arrays it returns, so
both sides see identical inputs.

Generator: a counter-based splitmix64 (synth_rng.c, compiled with gcc on first
use).  Value i of stream `name` under seed `seed` is mix64(key + (i + 1) *
0x9E3779B97F4A7C15), with key = mix64(FNV-1a(name) ^ seed * 0x9E37...) and
mix64 the splitmix64 output function.  Uniform doubles take the top 53 bits;
normals come from the Box-Muller transform of the uniform pair (2p, 2p+1):
value 2p is the cosine branch, value 2p+1 the sine branch.  Because every
value is a function of its index, computed with scalar libm calls, any slice of
any tensor can be regenerated on its own, bit for bit (the parity tests use
this to regenerate sampled weight rows at full size).

Arrays come back as numpy: fp32 weights, and bf16 / f16 values as their
uint16 bit patterns (rounded from the fp64 draw by torch / numpy casts, which
are input plumbing, not the method).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "synth_rng.c"
_LIB = _HERE / "libsynth_rng.so"
_rng = None


def build(force: bool = False) -> Path:
    """Compile the generator (plain C, scalar libm, OpenMP over elements)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_name(f"libsynth_rng.so.tmp{os.getpid()}")
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-fPIC", "-shared", "-o", str(tmp),
                               str(_SRC), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _lib():
    global _rng
    if _rng is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        L.synth_mix64.restype = ctypes.c_uint64
        L.synth_mix64.argtypes = [ctypes.c_uint64]
        for name in ("synth_uniform01", "synth_normal"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.synth_uniform_int8.restype = None
        L.synth_uniform_int8.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p]
        L.synth_normal_f32.restype = None
        L.synth_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                       ctypes.c_void_p]
        _rng = L
    return _rng


def _key(seed: int, name: str) -> int:
    h = 0xCBF29CE484222325  # FNV-1a 64 of the stream name, mixed with the seed
    for ch in name.encode():
        h = ((h ^ ch) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return _lib().synth_mix64(h ^ ((seed * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF))


def uniform01(seed: int, name: str, start: int, count: int) -> np.ndarray:
    out = np.empty(count, np.float64)
    _lib().synth_uniform01(_key(seed, name), start, count, out.ctypes.data)
    return out


def normal(seed: int, name: str, start: int, count: int) -> np.ndarray:
    """Standard normals with indices [start, start + count) of the stream."""
    out = np.empty(count, np.float64)
    _lib().synth_normal(_key(seed, name), start, count, out.ctypes.data)
    return out


def uniform_int(seed: int, name: str, lo: int, hi: int, shape) -> np.ndarray:
    """Integers uniform in [lo, hi] (a range inside [-128, 127]) as int8:
    lo + floor(u * (hi - lo + 1)) for the stream's uniforms u."""
    assert -128 <= lo <= hi <= 127
    out = np.empty(int(np.prod(shape)), np.int8)
    _lib().synth_uniform_int8(_key(seed, name), 0, out.size, lo, hi, out.ctypes.data)
    return out.reshape(shape)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def to_f16_bits(v: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(v, np.float64).astype(np.float16).view(np.uint16)


# ---- tensors of the workloads ----------------------------------------------
def weight_rows(seed: int, name: str, K: int, row0: int, rows: int, std: float = 0.02) -> np.ndarray:
    """Rows [row0, row0 + rows) of an fp32 weight W = fp32(std * N(0, 1)) of width K."""
    out = np.empty((rows, K), np.float32)
    _lib().synth_normal_f32(_key(seed, name), row0 * K, rows * K, std, out.ctypes.data)
    return out


def activations(seed: int, name: str, M: int, K: int, outlier_frac: float = 0.0, outlier_gain: float = 20.0):
    """bf16 x ~ N(0, 1) [M, K]; with outlier_frac > 0, floor(outlier_frac * K)
    channels (a seeded choice of columns) are multiplied by outlier_gain for
    every token before the bf16 rounding."""
    x = normal(seed, name, 0, M * K).reshape(M, K)
    n_out = int(np.floor(outlier_frac * K))
    if n_out:
        keys = uniform01(seed, name + "/outlier_channels", 0, K)
        ch = np.argsort(keys, kind="stable")[:n_out]
        x[:, ch] *= outlier_gain
    return to_bf16_bits(x)


def lognormal_scales(seed: int, name: str, shape, mu: float = -4.0, sigma: float = 0.5, f16: bool = False):
    n = int(np.prod(shape))
    v = np.exp(mu + sigma * normal(seed, name, 0, n)).reshape(shape)
    return to_f16_bits(v) if f16 else to_bf16_bits(v)


def routing(seed: int, T: int, E: int = 128, topk: int = 8, sigma: float = 2.0):
    """Top-k expert ids from logits ~ N(0, sigma^2) per (token, expert): the
    k largest logits, ties to the lower id; weights are the softmax over all
    E logits taken at the chosen ids (not renormalised)."""
    logits = sigma * normal(seed, "router_logits", 0, T * E).reshape(T, E)
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -logits), axis=-1)[:, :topk]
    ids = order.astype(np.int32)
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = ex / ex.sum(axis=1, keepdims=True)
    w = np.take_along_axis(p, order, axis=1).astype(np.float32)
    return ids, w


# ---- the workload recipes ---------------------------------------------------
def tiny_w8a16(seed: int = 0, M: int = 1, K: int = 256, N: int = 512):
    """Int8 W8A16 linear: codes uniform in [-127, 127], bf16 scale per row per
    128 of K lognormal(-4, 0.5), x ~ N(0, 1) bf16."""
    codes = uniform_int(seed, "codes", -127, 127, (N, K)).astype(np.int8)
    scales = lognormal_scales(seed, "scales", (N, K // 128))
    x = activations(seed, "x", M, K)
    return dict(x=x, codes=codes, scales=scales, M=M, N=N, K=K)


def dense_w8a8_hadamard(M: int, seed: int = 0, K: int = 5376, N: int = 21504, rows=None):
    """Dense decode W8A8 with the Hadamard domain: W ~ N(0, 0.02^2) fp32 (to be
    rotated and quantised by the packer), x ~ N(0, 1) bf16 with 1% outlier
    channels x20.  `rows` = (row0, count) draws only that slice of W."""
    r0, nr = rows if rows is not None else (0, N)
    W = weight_rows(seed, "W", K, r0, nr)
    x = activations(seed, f"x_M{M}", M, K, outlier_frac=0.01)
    return dict(W=W, x=x, M=M, N=N, K=K)


def w4a16(M: int, seed: int = 0, K: int = 5376, N: int = 21504):
    codes = uniform_int(seed, "i4_codes", -8, 7, (N, K)).astype(np.int8)
    scales = lognormal_scales(seed, "i4_scales", (N, K // 64))
    x = activations(seed, f"x_M{M}", M, K)
    return dict(codes=codes, scales=scales, x=x, M=M, N=N, K=K)


def w5a16(M: int, seed: int = 0, K: int = 5376, N: int = 21504):
    codes = uniform_int(seed, "i5_codes", 0, 31, (N, K)).astype(np.uint8)
    zeros = uniform_int(seed, "i5_zeros", 0, 31, (N, K // 128)).astype(np.uint8)
    scales = lognormal_scales(seed, "i5_scales", (N, K // 128), f16=True)
    x = activations(seed, f"x_M{M}", M, K)
    return dict(codes=codes, zeros=zeros, scales=scales, x=x, M=M, N=N, K=K)


def moe_gate_up(T: int, seed: int = 0, E: int = 128, topk: int = 8, K: int = 2816, N: int = 1408,
                experts=None):
    """MoE gate_up: per-expert W ~ N(0, 0.02^2) [N, K] (expert e is stream
    "W_e<e>"), routing from softmax over N(0, 2^2) logits, x ~ N(0, 1) bf16.
    `experts` limits which experts' weights are drawn (others are None)."""
    ids, w = routing(seed, T, E, topk)
    x = activations(seed, f"x_T{T}", T, K)
    which = range(E) if experts is None else experts
    Ws = {e: weight_rows(seed, f"W_e{e}", K, 0, N) for e in which}
    return dict(ids=ids, weights=w, x=x, W=Ws, T=T, E=E, topk=topk, N=N, K=K)


def prefill(seed: int = 0, M: int = 2048, K: int = 5376, N: int = 21504, rows=None):
    r0, nr = rows if rows is not None else (0, N)
    W = weight_rows(seed, "W", K, r0, nr)
    x = activations(seed, "x_prefill", M, K)
    return dict(W=W, x=x, M=M, N=N, K=K)


def moe_down(T: int, seed: int = 0, E: int = 128, topk: int = 8, K: int = 2816, I: int = 704, experts=None):
    """The down projection's inputs: routing as moe_gate_up's workload (same seed, so the same ids and
    weights), the gate_up output h ~ N(0, 1) as fp32 [T, topk, 2I], and per expert a bf16 down weight
    [K, I] ~ N(0, 0.02^2) (expert e is stream "Wd_e<e>"; `experts` limits which are drawn)."""
    ids, w = routing(seed, T, E, topk)
    h = normal(seed, f"h_T{T}", 0, T * topk * 2 * I).astype(np.float32).reshape(T, topk, 2 * I)
    which = range(E) if experts is None else experts
    Wd = {e: to_bf16_bits(weight_rows(seed, f"Wd_e{e}", I, 0, K)) for e in which}
    return dict(ids=ids, weights=w, h=h, Wd=Wd, T=T, E=E, topk=topk, K=K, I=I)
