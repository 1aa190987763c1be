"""Python binding of libqlinear.so (C ABI in include/qlinear.h).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in the library's kernels.
There is no fallback: if the compiled library is missing or a call fails,
an exception is raised.

The functions keep the C names.  Each takes CUDA tensors and returns new
tensors (outputs and workspaces are allocated with torch), except the *_size
helpers, which return integers.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libqlinear.so"

I8_G128_BF16 = 1
I8_G128_F16 = 2
I8A8_G128_BF16 = 3
I4_G64_BF16 = 4
I5Z_G128_F16 = 5
FP8_B128_BF16 = 6
FP8A8_B128_BF16 = 7  # the fp8 weights with E4M3 activations
HADAMARD = 1
SCALE_SEARCH = 2  # qlinear_pack of an fp32 W, int8 formats: the best of 21 scales per group
FORMATS = (I8_G128_BF16, I8_G128_F16, I8A8_G128_BF16, I4_G64_BF16, I5Z_G128_F16, FP8_B128_BF16, FP8A8_B128_BF16)

DEVERR_EXPERT_ID = 1
DEVERR_CODE_RANGE = 2
DEVERR_TIMEOUT = 4
DEVERR_BOUNDS = 8

A16_MAX_K = 32768  # QL_A16_MAX_K: largest K for the formats whose activations stay 16-bit

STATUS = {0: "QL_OK", 1: "QL_EINVAL", 2: "QL_EUNSUPPORTED", 3: "QL_EALIGN", 4: "QL_EWORKSPACE", 5: "QL_ECUDA",
          6: "QL_EDEVICE"}


class QLError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = lib().ql_status_string(status).decode()
        if status == 5:
            detail += ": " + lib().ql_last_cuda_error().decode()
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({detail})")


class ql_experts(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int), ("fmt", ctypes.c_int),
                ("flags", ctypes.c_int), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class ql_down_experts(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("K", ctypes.c_int), ("I", ctypes.c_int), ("weights", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_PSZ = ctypes.POINTER(ctypes.c_size_t)

_SIGS = {
    "ql_status_string": (ctypes.c_char_p, [_I]),
    "ql_last_cuda_error": (ctypes.c_char_p, []),
    "qlinear_packed_sizes": (_I, [_I, _I, _I, _PSZ, _PSZ, _PSZ]),
    "qlinear_pack": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P]),
    "qlinear_workspace_size": (_I, [_I, _I, _I, _I, _I, _PSZ]),
    "qlinear_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "qlinear_forward_i8_acc": (_I, [_P, _P, _I, _I, _I, _P, _P]),
    "qlinear_gemm_a8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P]),
    "act_quant_i8_g128": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "act_quant_e4m3_g128": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "hadamard128_rotate": (_I, [_P, _I, _I, _P, _P]),
    "moe_permute": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "moe_workspace_size": (_I, [ctypes.POINTER(ql_experts), _I, _I, _PSZ]),
    "moe_gate_up": (_I, [_P, _P, _P, ctypes.POINTER(ql_experts), _I, _I, _P, _P, _SZ, _P]),
    "moe_down_workspace_size": (_I, [ctypes.POINTER(ql_down_experts), _I, _I, _PSZ]),
    "moe_down_combine": (_I, [_P, _P, _P, ctypes.POINTER(ql_down_experts), _I, _I, _P, _P, _SZ, _P]),
    "ql_get_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "ql_set_wait_limit": (_I, [ctypes.c_ulonglong]),
    "qlinear_forward_w8a8_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "ql_trace_enable": (_I, [_I]),
    "ql_trace_read": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float), _I,
                           ctypes.POINTER(ctypes.c_int)]),
}

KIND_NAMES = {1: "rotate", 2: "act_quant", 3: "prep_a16", 4: "skinny", 5: "moe_permute", 6: "moe_gemm", 7: "pack",
              8: "prefill", 9: "prefill_prep", 10: "moe_act", 11: "moe_down"}

_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m moe_hadamard128_act_b200.build`")
        L = ctypes.CDLL(str(_LIB_PATH))
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, st: int):
    if st != 0:
        raise QLError(fn, st)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _empty(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ---- sizes ------------------------------------------------------------------------
def qlinear_packed_sizes(fmt: int, N: int, K: int):
    c, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("qlinear_packed_sizes", lib().qlinear_packed_sizes(fmt, N, K, ctypes.byref(c), ctypes.byref(s),
                                                              ctypes.byref(z)))
    return c.value, s.value, z.value


def qlinear_workspace_size(fmt: int, flags: int, M: int, N: int, K: int) -> int:
    b = ctypes.c_size_t()
    _check("qlinear_workspace_size", lib().qlinear_workspace_size(fmt, flags, M, N, K, ctypes.byref(b)))
    return b.value


def _experts_struct(E, N, K, fmt, flags, codes, scales):
    return ql_experts(E, N, K, fmt, flags, codes.data_ptr(), scales.data_ptr())


def moe_workspace_size(E: int, N: int, K: int, fmt: int, flags: int, T: int, topk: int) -> int:
    ex = ql_experts(E, N, K, fmt, flags, 16, 16)  # placeholder aligned pointers: only sizes are read
    b = ctypes.c_size_t()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(ex), T, topk, ctypes.byref(b)))
    return b.value


# ---- packing ---------------------------------------------------------------------
def qlinear_pack(fmt: int, N: int, K: int, W: torch.Tensor | None = None, codes: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, zeros: torch.Tensor | None = None, flags: int = 0,
                 stream=None):
    """Pack a weight: RTN-quantise fp32 W [N, K], or bit-pack given codes with
    their scales (and int5 zeros).  flags: HADAMARD quantises in the rotated
    domain; SCALE_SEARCH (int8 formats, from W) takes each group's best of 21
    scales instead of round to nearest's.  Returns (codes, scales, zeros) as
    uint8 tensors of the packed byte sizes (zeros is None except for int5)."""
    dev = (W if W is not None else codes).device
    cb, sb, zb = qlinear_packed_sizes(fmt, N, K)
    c_out, s_out = _empty(cb, dev), _empty(sb, dev)
    z_out = _empty(zb, dev) if zb else None
    st = lib().qlinear_pack(_ptr(W), _ptr(codes), _ptr(scales), _ptr(zeros), fmt, flags, N, K, _ptr(c_out),
                            _ptr(s_out), _ptr(z_out), _stream(stream))
    _check("qlinear_pack", st)
    return c_out[:cb], s_out[:sb], (z_out[:zb] if z_out is not None else None)


# ---- forward -----------------------------------------------------------------------
def qlinear_forward(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor | None,
                    fmt: int, N: int, flags: int = 0, y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """y [M, N] fp32 = x~ . dequant(W)^T for bf16 x [M, K]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    need = qlinear_workspace_size(fmt, flags, M, N, K)
    if ws is None or ws.numel() < need:
        ws = _empty(need, x.device)
    st = lib().qlinear_forward(_ptr(x), _ptr(codes), _ptr(scales), _ptr(zeros), fmt, flags, M, N, K, _ptr(y),
                               _ptr(ws), ws.numel(), _stream(stream))
    _check("qlinear_forward", st)
    return y


def qlinear_forward_w8a8_noalloc(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, N: int,
                                 flags: int = 0, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W8A8 forward without a workspace, for callers that cannot allocate
    device memory (M <= 16, K <= 16384): the activation scratch lives in a fixed
    array inside the library.  Calls that may overlap on the GPU race on it."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    elif y.dtype != torch.float32 or tuple(y.shape) != (M, N):
        raise ValueError(f"y must be an fp32 tensor of shape ({M}, {N})")
    st = lib().qlinear_forward_w8a8_noalloc(_ptr(x), _ptr(codes), _ptr(scales), flags, M, N, K, _ptr(y),
                                            _stream(stream))
    _check("qlinear_forward_w8a8_noalloc", st)
    return y


def qlinear_forward_i8_acc(qx: torch.Tensor, qw: torch.Tensor, stream=None) -> torch.Tensor:
    """int32 [M, N, K/128] group sums of int8 qx [M, K] and qw [N, K]."""
    M, K = qx.shape
    N = qw.shape[0]
    acc = torch.empty((M, N, K // 128), dtype=torch.int32, device=qx.device)
    _check("qlinear_forward_i8_acc", lib().qlinear_forward_i8_acc(_ptr(qx), _ptr(qw), M, N, K, _ptr(acc),
                                                                  _stream(stream)))
    return acc


def qlinear_gemm_a8(qx: torch.Tensor, sx: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, fmt: int, N: int,
                    y: torch.Tensor | None = None, accumulate: bool = False, stream=None) -> torch.Tensor:
    """The decode GEMM on quantised activations (M <= 16): qx [M, K] int8
    (W8A8) or E4M3 bytes (format 7) with fp32 scales sx [M, K/128], as the
    act_quant_* calls make them.  y [M, N] fp32 is overwritten, or added to
    with accumulate=True."""
    if qx.dim() != 2 or qx.element_size() != 1:
        raise ValueError("qx must be a 2-D one-byte tensor")
    M, K = qx.shape
    if sx.dtype != torch.float32 or tuple(sx.shape) != (M, K // 128):
        raise ValueError(f"sx must be an fp32 tensor of shape ({M}, {K // 128})")
    if y is None:
        if accumulate:
            raise ValueError("accumulate needs y")
        y = torch.empty((M, N), dtype=torch.float32, device=qx.device)
    elif y.dtype != torch.float32 or tuple(y.shape) != (M, N):
        raise ValueError(f"y must be an fp32 tensor of shape ({M}, {N})")
    _check("qlinear_gemm_a8", lib().qlinear_gemm_a8(_ptr(qx), _ptr(sx), _ptr(codes), _ptr(scales), fmt, M, N, K,
                                                    _ptr(y), int(accumulate), _stream(stream)))
    return y


def act_quant_i8_g128(x: torch.Tensor, rotate: bool = False, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check("act_quant_i8_g128", lib().act_quant_i8_g128(_ptr(x), M, K, int(rotate), _ptr(q), _ptr(s),
                                                        _stream(stream)))
    return q, s


def act_quant_e4m3_g128(x: torch.Tensor, rotate: bool = False, stream=None):
    """E4M3 codes (uint8 [M, K]) and fp32 scales [M, K/128] per token per 128."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check("act_quant_e4m3_g128", lib().act_quant_e4m3_g128(_ptr(x), M, K, int(rotate), _ptr(q), _ptr(s),
                                                            _stream(stream)))
    return q, s


def hadamard128_rotate(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    M, K = x.shape
    y = torch.empty_like(x) if out is None else out
    _check("hadamard128_rotate", lib().hadamard128_rotate(_ptr(x), M, K, _ptr(y), _stream(stream)))
    return y


# ---- MoE ---------------------------------------------------------------------------
def moe_permute(topk_ids: torch.Tensor, E: int, stream=None):
    T, topk = topk_ids.shape
    dev = topk_ids.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1 + 3, dtype=torch.int32, device=dev)  # padded to 16 bytes
    perm = torch.empty(T * topk + 4, dtype=torch.int32, device=dev)
    _check("moe_permute", lib().moe_permute(_ptr(topk_ids), T, topk, E, _ptr(counts), _ptr(offsets), _ptr(perm),
                                            _stream(stream)))
    return counts, offsets[:E + 1], perm[:T * topk]


def moe_gate_up(x: torch.Tensor, topk_ids: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, E: int, N: int,
                fmt: int = I8_G128_BF16, flags: int = HADAMARD, topk_weights: torch.Tensor | None = None,
                y: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [T, topk, N] fp32 for stacked expert weights (codes [E*N*K], scales)."""
    T, K = x.shape
    topk = topk_ids.shape[1]
    ex = _experts_struct(E, N, K, fmt, flags, codes, scales)
    b = ctypes.c_size_t()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(ex), T, topk, ctypes.byref(b)))
    if ws is None or ws.numel() < b.value:
        ws = _empty(b.value, x.device)
    if y is None:
        y = torch.empty((T, topk, N), dtype=torch.float32, device=x.device)
    st = lib().moe_gate_up(_ptr(x), _ptr(topk_ids), _ptr(topk_weights), ctypes.byref(ex), T, topk, _ptr(y),
                           _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_gate_up", st)
    return y


def moe_down_workspace_size(E: int, K: int, I: int, T: int, topk: int) -> int:
    ex = ql_down_experts(E, K, I, 16)  # placeholder aligned pointer: only sizes are read
    b = ctypes.c_size_t()
    _check("moe_down_workspace_size", lib().moe_down_workspace_size(ctypes.byref(ex), T, topk, ctypes.byref(b)))
    return b.value


def moe_down_combine(h: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor, wd: torch.Tensor, E: int,
                     out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out [T, K] fp32: the experts' bf16 down projections of gelu(gate) * up of the gate_up output
    h [T, topk, 2I] (fp32), summed over each token's slots with the routing weights.  wd: the stacked
    bf16 weights [E, K, I] (any 2-byte dtype, viewed as bits)."""
    if h.dtype != torch.float32 or h.dim() != 3:
        raise ValueError("h must be an fp32 tensor [T, topk, 2I]")
    T, topk, I2 = h.shape
    if wd.element_size() != 2 or wd.dim() != 3 or wd.shape[0] != E or wd.shape[2] * 2 != I2:
        raise ValueError("wd must be a 2-byte tensor [E, K, I] with 2I = h.shape[-1]")
    K = wd.shape[1]
    ex = ql_down_experts(E, K, I2 // 2, wd.data_ptr())
    b = ctypes.c_size_t()
    _check("moe_down_workspace_size", lib().moe_down_workspace_size(ctypes.byref(ex), T, topk, ctypes.byref(b)))
    if ws is None or ws.numel() < b.value:
        ws = _empty(b.value, h.device)
    if out is None:
        out = torch.empty((T, K), dtype=torch.float32, device=h.device)
    st = lib().moe_down_combine(_ptr(h), _ptr(topk_ids), _ptr(topk_weights), ctypes.byref(ex), T, topk, _ptr(out),
                                _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_down_combine", st)
    return out


def ql_trace_enable(capacity: int):
    """Record CUDA events around up to `capacity` library launches (0 stops)."""
    _check("ql_trace_enable", lib().ql_trace_enable(capacity))


def ql_trace_read(max_records: int = 1 << 16):
    """[(kind_name, ms)] of the recorded launches, in launch order."""
    kinds = (ctypes.c_int * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = ctypes.c_int()
    _check("ql_trace_read", lib().ql_trace_read(kinds, ms, max_records, ctypes.byref(n)))
    m = min(n.value, max_records)
    return [(KIND_NAMES.get(kinds[i], str(kinds[i])), ms[i]) for i in range(m)]


def ql_get_device_error(stream=None):
    """(status, bits) after synchronising the stream; clears the error word."""
    bits = ctypes.c_uint()
    st = lib().ql_get_device_error(_stream(stream), ctypes.byref(bits))
    return st, bits.value


def ql_set_wait_limit(ns: int):
    """Bound the kernels' pipeline waits to ns nanoseconds on the current device (0: the default)."""
    _check("ql_set_wait_limit", lib().ql_set_wait_limit(int(ns)))
