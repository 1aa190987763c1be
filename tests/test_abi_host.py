"""Host-only checks of libqlinear.so: it loads, exports every entry point the
header declares, and rejects bad arguments with the documented status before
touching the GPU.  Every call here fails validation on purpose, so none of them
launches a kernel (they run on machines with or without a GPU)."""
import ctypes
import re
from pathlib import Path

import pytest

from moe_hadamard128_act_b200 import build as qbuild
from oracle import oracle as O

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear as Q
    return Q.lib()


def declared_functions():
    text = (ROOT / "include" / "qlinear.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert {"qlinear_pack", "qlinear_forward", "act_quant_i8_g128", "hadamard128_rotate", "moe_gate_up"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_binding_constants_match_header():
    from moe_hadamard128_act_b200 import qlinear as Q
    text = (ROOT / "include" / "qlinear.h").read_text()
    assert int(re.search(r"QL_A16_MAX_K\s*=\s*(\d+)", text).group(1)) == Q.A16_MAX_K
    assert int(re.search(r"QL_HADAMARD\s*=\s*(\d+)", text).group(1)) == Q.HADAMARD
    assert int(re.search(r"QL_SCALE_SEARCH\s*=\s*(\d+)", text).group(1)) == Q.SCALE_SEARCH
    for name in ("I8_G128_BF16", "I8_G128_F16", "I8A8_G128_BF16", "I4_G64_BF16", "I5Z_G128_F16", "FP8_B128_BF16",
                 "FP8A8_B128_BF16"):
        assert int(re.search(rf"QL_{name}\s*=\s*(\d+)", text).group(1)) == getattr(Q, name), name


def test_status_strings(L):
    for st in range(7):
        assert L.ql_status_string(st)
    assert L.ql_status_string(99) == b"unknown status"


@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6, 7])
@pytest.mark.parametrize("N,K", [(1, 128), (200, 384), (21504, 5376), (1408, 2816)])
def test_packed_sizes_match_oracle(L, fmt, N, K):
    from moe_hadamard128_act_b200 import qlinear as Q
    assert Q.qlinear_packed_sizes(fmt, N, K) == O.packed_sizes(fmt, N, K)


def test_packed_sizes_and_workspace_reject_bad_args(L):
    from moe_hadamard128_act_b200 import qlinear as Q
    for fmt, N, K in ((0, 8, 128), (8, 8, 128), (1, 0, 128), (1, 8, 64), (1, 8, 200)):
        with pytest.raises(Q.QLError) as e:
            Q.qlinear_packed_sizes(fmt, N, K)
        assert e.value.status == 1
    with pytest.raises(Q.QLError):
        Q.qlinear_workspace_size(1, 4, 1, 8, 128)  # unknown flag
    # the scale-search bit describes how W was packed, not its layout: accepted and ignored
    assert Q.qlinear_workspace_size(3, 2 | 1, 16, 21504, 5376) == Q.qlinear_workspace_size(3, 1, 16, 21504, 5376)
    assert Q.qlinear_workspace_size(1, 0, 16, 21504, 5376) >= 16 * 5376 * 2
    assert Q.qlinear_workspace_size(3, 1, 16, 21504, 5376) >= 16 * 5376 + 16 * 42 * 4
    # the 16-bit activations, their token factors and the tokens' group sums (the decode kernels take
    # the codes' offset off with them): per 128 for int8 and int5, per 64 for int4
    for fmt, per in ((1, 128), (2, 128), (5, 128), (4, 64)):
        assert Q.qlinear_workspace_size(fmt, 0, 16, 21504, 5376) >= 16 * 5376 * 2 + 16 * 4 + 16 * (5376 // per) * 4
    # format 7: E4M3 codes and their scales for the decode kernel (M <= 16); from 17 rows the tensor-core
    # GEMM also takes transposed scales and its weight-scale scratch
    assert 5376 + 42 * 4 <= Q.qlinear_workspace_size(7, 1, 1, 21504, 5376) < 42 * 21504 * 4
    assert Q.qlinear_workspace_size(7, 1, 17, 21504, 5376) >= 17 * 5376 + 42 * 128 * 4 + 42 * 21504 * 4
    # int5 switches to int8 activations at 65 rows: the workspace then holds the activation codes, their
    # transposed scales, the GEMM's weight scales and the weight converted to int8 codes (N * K bytes)
    assert Q.qlinear_workspace_size(5, 0, 64, 21504, 5376) < 21504 * 5376
    assert Q.qlinear_workspace_size(5, 0, 65, 21504, 5376) >= 65 * 5376 + 42 * 128 * 4 + 42 * 21504 * 4 + 21504 * 5376


A = 1 << 20  # an aligned fake address: every call below fails validation first


def test_forward_validation_statuses(L):
    P = ctypes.c_void_p
    f = L.qlinear_forward
    ok = dict(x=P(A), W=P(A), s=P(A), z=None, fmt=1, flags=0, M=4, N=64, K=256, y=P(A), ws=P(A), wsb=1 << 30)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["x"], a["W"], a["s"], a["z"], a["fmt"], a["flags"], a["M"], a["N"], a["K"], a["y"], a["ws"],
                 a["wsb"], None)

    assert call(fmt=0) == 1
    assert call(fmt=9) == 1
    assert call(K=200) == 1
    assert call(M=0) == 1
    assert call(flags=4) == 1
    assert call(x=None) == 1
    assert call(fmt=5) == 1  # int5 needs zeros
    assert call(K=32768 + 128) == 2  # a 16-bit activation row no longer fits in shared memory
    # byte activations have no such limit: W8A8, format 7 (decode and prefill) and int5 from 65 rows on
    # pass that check and stop at the (too small) workspace instead
    big = 32768 + 128
    assert call(fmt=3, K=big, wsb=16) == 4
    assert call(fmt=7, K=big, M=1, wsb=16) == 4
    assert call(fmt=7, K=big, M=17, wsb=16) == 4
    assert call(fmt=5, z=P(A), K=big, M=64) == 2
    assert call(fmt=5, z=P(A), K=big, M=65, wsb=16) == 4
    assert call(x=P(A + 8)) == 3
    assert call(y=P(A + 4)) == 3
    assert call(ws=None) == 4
    assert call(wsb=16) == 4


def test_pack_and_act_validation_statuses(L):
    P = ctypes.c_void_p
    p = L.qlinear_pack
    assert p(P(A), None, None, None, 5, 0, 8, 128, P(A), P(A), P(A), None) == 2  # int5 from floats
    assert p(P(A), P(A), P(A), None, 1, 0, 8, 128, P(A), P(A), None, None) == 1  # two sources
    assert p(None, None, None, None, 1, 0, 8, 128, P(A), P(A), None, None) == 1  # no source
    assert p(P(A + 4), None, None, None, 1, 0, 8, 128, P(A), P(A), None, None) == 3
    assert p(None, P(A), None, None, 4, 0, 8, 128, P(A), P(A), None, None) == 1  # codes without scales
    assert p(None, P(A), P(A), None, 5, 0, 8, 128, P(A), P(A), P(A), None) == 1  # int5 codes without zeros
    assert p(P(A), None, None, None, 4, 2, 8, 128, P(A), P(A), None, None) == 2  # scale search: int8 only
    assert p(P(A), None, None, None, 6, 3, 8, 128, P(A), P(A), None, None) == 2
    assert p(None, P(A), P(A), None, 1, 2, 8, 128, P(A), P(A), None, None) == 1  # a rule for W, not for codes
    assert p(P(A), None, None, None, 1, 4, 8, 128, P(A), P(A), None, None) == 1  # unknown flag bit
    assert L.act_quant_i8_g128(P(A), 4, 100, 0, P(A), P(A), None) == 1
    assert L.act_quant_e4m3_g128(P(A), 4, 100, 0, P(A), P(A), None) == 1
    assert L.act_quant_e4m3_g128(P(A), 4, 128, 0, P(A + 4), P(A), None) == 3
    assert L.act_quant_i8_g128(P(A + 2), 4, 128, 0, P(A), P(A), None) == 3
    assert L.hadamard128_rotate(P(A), 0, 128, P(A), None) == 1
    assert L.hadamard128_rotate(P(A), 1, 128, P(A + 1), None) == 3
    assert L.qlinear_forward_i8_acc(P(A), P(A), 1, 1, 64, P(A), None) == 1
    g = L.qlinear_gemm_a8  # (qx, sx, W, scales, fmt, M, N, K, y, accumulate, stream)
    assert g(P(A), P(A), P(A), P(A), 1, 4, 64, 256, P(A), 0, None) == 1  # weight-only formats take bf16 x
    assert g(P(A), P(A), P(A), P(A), 3, 4, 64, 200, P(A), 0, None) == 1
    assert g(P(A), None, P(A), P(A), 3, 4, 64, 256, P(A), 0, None) == 1
    assert g(P(A), P(A), P(A), P(A), 3, 17, 64, 256, P(A), 0, None) == 2  # decode shapes only
    assert g(P(A), P(A), P(A), P(A), 7, 4, 64, 256, P(A + 4), 1, None) == 3


def test_moe_validation_statuses(L):
    from moe_hadamard128_act_b200 import qlinear as Q
    P = ctypes.c_void_p
    ex = Q.ql_experts(128, 1408, 2816, 1, 1, A, A)
    g = L.moe_gate_up
    assert g(P(A), P(A), None, ctypes.byref(ex), 4, 65, P(A), P(A), 1 << 30, None) == 1  # topk > 64
    assert g(P(A), P(A), None, ctypes.byref(ex), 0, 8, P(A), P(A), 1 << 30, None) == 1
    assert g(P(A), P(A), None, ctypes.byref(ex), 4, 8, P(A), None, 0, None) == 4
    bad = Q.ql_experts(128, 1408, 2816, 4, 1, A, A)  # int4 experts are not offered
    assert g(P(A), P(A), None, ctypes.byref(bad), 4, 8, P(A), P(A), 1 << 30, None) == 2
    bad = Q.ql_experts(128, 1408, 2816, 1, 0, A + 8, A)
    assert g(P(A), P(A), None, ctypes.byref(bad), 4, 8, P(A), P(A), 1 << 30, None) == 3
    assert g(P(A), P(A), None, None, 4, 8, P(A), P(A), 1 << 30, None) == 1
    big = Q.ql_experts(8, 256, 32768 + 128, 1, 0, A, A)
    assert g(P(A), P(A), None, ctypes.byref(big), 4, 8, P(A), P(A), 1 << 40, None) == 2
    assert L.moe_permute(P(A), 4, 8, 0, P(A), P(A), P(A), None) == 1
    assert Q.moe_workspace_size(128, 1408, 2816, 1, 1, 2048, 8) > 2048 * 2816 * 2
