"""GPU parity: every C-ABI call of libqlinear.so against the fp64 CPU oracle on
the same seeded inputs.  Bit-exact for packed codes, scales, activation codes,
W8A8 int32 group sums and the MoE permutation; rel-L2 <= 1e-5 and max-abs <=
1e-3 * max|oracle| for fp32 outputs."""
import numpy as np
import pytest
import torch

from moe_hadamard128_act_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_close, dev, dev_bf16, host_u16, host_u8

pytestmark = pytest.mark.gpu

Q = None


@pytest.fixture(scope="module", autouse=True)
def qlib():
    global Q
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    Q = qlinear
    Q.lib()
    yield
    st, bits = Q.ql_get_device_error()
    assert st == 0 and bits == 0, f"device error word left set: {bits}"


def x_bits(M, K, seed=0, name="x", outliers=0.0):
    return synth.activations(seed, name, M, K, outlier_frac=outliers)


# --------------------------------------------------------------------------
# Activation kernels
# --------------------------------------------------------------------------
@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (16, 5376), (7, 2816), (33, 640)])
def test_hadamard128_rotate_bitexact(M, K):
    x = x_bits(M, K, outliers=0.01)
    ref = O.hadamard128_rotate(x)
    xd = dev_bf16(x)
    got = host_u16(Q.hadamard128_rotate(xd))
    assert np.array_equal(got, ref)
    Q.hadamard128_rotate(xd, out=xd)  # in place
    assert np.array_equal(host_u16(xd), ref)


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (4, 384), (16, 5376), (2048, 256)])
def test_act_quant_bitexact(M, K, rotate):
    x = x_bits(M, K, outliers=0.01)
    x[0, :128] = 0  # an all-zero group
    if K >= 256:
        x[-1, 128:256] = O.bf16_encode(np.r_[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, np.zeros(121)])  # ties
    q_ref, s_ref = O.act_quant_i8_g128(x, rotate)
    q, s = Q.act_quant_i8_g128(dev_bf16(x), rotate)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (4, 384), (16, 5376), (2048, 256)])
def test_act_quant_e4m3_bitexact(M, K, rotate):
    x = x_bits(M, K, outliers=0.01)
    x[0, :128] = 0  # an all-zero group
    if K >= 256:  # amax 448: ties between E4M3 neighbours, a subnormal, a value that rounds to zero
        x[-1, 128:256] = O.bf16_encode(np.r_[448.0, 1.0625, 1.1875, -2.0 ** -9, 2.0 ** -12, 240.0, np.zeros(122)])
    q_ref, s_ref = O.act_quant_e4m3_g128(x, rotate)
    q, s = Q.act_quant_e4m3_g128(dev_bf16(x), rotate)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------
def oracle_pack_rtn(fmt, W, had):
    if fmt in (Q.I8_G128_BF16, Q.I8A8_G128_BF16, Q.I8_G128_F16):
        q, s = O.quant_i8_g128(W, hadamard=had, scale_f16=fmt == Q.I8_G128_F16)
        return q.view(np.uint8), s, None
    if fmt == Q.I4_G64_BF16:
        q, s = O.quant_i4_g64(W, hadamard=had)
        return O.pack_i4(q), s, None
    if fmt in (Q.FP8_B128_BF16, Q.FP8A8_B128_BF16):
        q, s = O.quant_fp8_b128(W, hadamard=had)
        return q, s, None
    raise ValueError(fmt)


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 6, 7])
@pytest.mark.parametrize("N,K", [(64, 256), (200, 384), (130, 1024)])
def test_pack_rtn_bitexact(fmt, had, N, K):
    W = synth.weight_rows(3, f"Wp{N}", K, 0, N)
    W[1, :128] = 0.0  # a zero group
    codes, scales, _ = Q.qlinear_pack(fmt, N, K, W=dev(W), flags=had)
    c_ref, s_ref, _ = oracle_pack_rtn(fmt, W, bool(had))
    assert np.array_equal(host_u8(codes), c_ref.ravel())
    assert np.array_equal(host_u8(scales).view(np.uint16), s_ref.ravel())


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("fmt", [1, 2, 3])
@pytest.mark.parametrize("N,K", [(40, 384), (300, 1024)])
def test_pack_scale_search_bitexact(fmt, had, N, K):
    # codes, scales and (through them) every group's pick among the 21 candidates, bit for bit;
    # heavy-tailed rows make some groups pick a smaller scale, and a zero group keeps s = 0
    rng = np.random.default_rng(61 + N)
    W = synth.weight_rows(61, f"Ws{N}", K, 0, N)
    W[::3] = (rng.standard_t(3, size=W[::3].shape) * 0.01).astype(np.float32)
    W[1, :128] = 0.0
    codes, scales, _ = Q.qlinear_pack(fmt, N, K, W=dev(W), flags=had | Q.SCALE_SEARCH)
    q_ref, s_ref, picks = O.quant_i8_g128_search(W, hadamard=bool(had), scale_f16=(fmt == Q.I8_G128_F16))
    assert np.array_equal(host_u8(codes), q_ref.view(np.uint8).ravel())
    assert np.array_equal(host_u8(scales).view(np.uint16), s_ref.ravel())
    assert (picks > 0).any() and s_ref[1, 0] == 0
    # and it is a different packing from round to nearest on those groups
    c_rtn, s_rtn, _ = Q.qlinear_pack(fmt, N, K, W=dev(W), flags=had)
    assert not np.array_equal(host_u8(scales), host_u8(s_rtn))


def test_pack_scale_search_then_forward():
    # the searched weights through the W8A8 forward, decode and prefill sizes, against the oracle
    N, K = 320, 512
    W = synth.weight_rows(67, "Wsf", K, 0, N)
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=dev(W), flags=Q.HADAMARD | Q.SCALE_SEARCH)
    q_ref, s_ref, _ = O.quant_i8_g128_search(W, hadamard=True)
    for M in (3, 40):
        x = x_bits(M, K, seed=67)
        y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.I8A8_G128_BF16, N, flags=Q.HADAMARD | Q.SCALE_SEARCH)
        ref = O.forward(x, q_ref.view(np.uint8), s_ref, None, Q.I8A8_G128_BF16, Q.HADAMARD, N)
        assert_close(y.cpu().numpy(), ref, f"searched W8A8 M={M}")


def test_pack_given_codes_bitexact_and_range_flag():
    N, K = 96, 256
    rng = np.random.default_rng(7)
    q4 = rng.integers(-8, 8, (N, K)).astype(np.int8)
    s4 = O.bf16_encode(np.exp(rng.normal(-4, 0.5, (N, K // 64))))
    c, s, _ = Q.qlinear_pack(Q.I4_G64_BF16, N, K, codes=dev(q4), scales=dev(s4))
    assert np.array_equal(host_u8(c), O.pack_i4(q4).ravel())
    assert np.array_equal(host_u8(s).view(np.uint16), s4.ravel())
    q5 = rng.integers(0, 32, (N, K)).astype(np.uint8)
    z5 = rng.integers(0, 32, (N, K // 128)).astype(np.uint8)
    s5 = O.f16_encode(np.exp(rng.normal(-4, 0.5, (N, K // 128))))
    c, s, z = Q.qlinear_pack(Q.I5Z_G128_F16, N, K, codes=dev(q5), scales=dev(s5), zeros=dev(z5))
    assert np.array_equal(host_u8(c), O.pack_i5(q5).ravel())
    assert np.array_equal(host_u8(z), z5.ravel())
    q8 = rng.integers(-127, 128, (N, K)).astype(np.int8)
    c, s, _ = Q.qlinear_pack(Q.I8_G128_BF16, N, K, codes=dev(q8), scales=dev(s4[:, ::2].copy()))
    assert np.array_equal(host_u8(c), q8.view(np.uint8).ravel())
    st, bits = Q.ql_get_device_error()
    assert st == 0 and bits == 0
    q4[3, 5] = 9  # out of the int4 range: packed as 0 and flagged, no fault
    c, s, _ = Q.qlinear_pack(Q.I4_G64_BF16, N, K, codes=dev(q4), scales=dev(s4))
    st, bits = Q.ql_get_device_error()
    assert st == 6 and bits & Q.DEVERR_CODE_RANGE
    q4[3, 5] = 0
    assert np.array_equal(host_u8(c), O.pack_i4(q4).ravel())


# --------------------------------------------------------------------------
# Linear layer
# --------------------------------------------------------------------------
def make_weights(fmt, N, K, had, seed=5):
    """Packed weights on the device plus the same bytes on the host."""
    if fmt == Q.I5Z_G128_F16:
        rng = np.random.default_rng(seed)
        q5 = synth.uniform_int(seed, "i5", 0, 31, (N, K)).astype(np.uint8)
        z5 = synth.uniform_int(seed, "i5z", 0, 31, (N, K // 128)).astype(np.uint8)
        s5 = synth.lognormal_scales(seed, "i5s", (N, K // 128), f16=True)
        c, s, z = Q.qlinear_pack(fmt, N, K, codes=dev(q5), scales=dev(s5), zeros=dev(z5))
        del rng
    else:
        W = synth.weight_rows(seed, f"W{N}x{K}", K, 0, N)
        c, s, z = Q.qlinear_pack(fmt, N, K, W=dev(W), flags=had)
    return (c, s, z), (host_u8(c), host_u8(s).view(np.uint16), None if z is None else host_u8(z))


SHAPES = [(1, 512, 256), (4, 200, 384), (5, 1000, 1024), (8, 64, 128), (9, 130, 256), (16, 333, 640),
          (17, 64, 256), (33, 48, 128)]


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_forward_parity(fmt, had, M, N, K):
    (c, s, z), (ch, sh, zh) = make_weights(fmt, N, K, had)
    x = x_bits(M, K, seed=11, outliers=0.01)
    y = Q.qlinear_forward(dev_bf16(x), c, s, z, fmt, N, flags=had)
    ref = O.forward(x, ch, sh, zh, fmt, had, N)
    assert_close(y.cpu().numpy(), ref, f"fmt {fmt} had {had} {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 64, 128), (5, 200, 384), (16, 130, 1024), (20, 48, 256)])
def test_w8a8_group_sums_bitexact(M, N, K):
    x = x_bits(M, K, seed=2, outliers=0.01)
    W = synth.weight_rows(2, "Wacc", K, 0, N)
    qw, sw = O.quant_i8_g128(W, hadamard=True)
    y_ref, acc_ref = O.forward(x, qw.view(np.uint8), sw, None, Q.I8A8_G128_BF16, Q.HADAMARD, N, want_acc=True)
    qx, _ = O.act_quant_i8_g128(x, rotate=True)
    acc = Q.qlinear_forward_i8_acc(dev(qx), dev(qw))
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    # full path on the same weights, extreme group: every code +-127
    qw[0, :128] = 127
    y = Q.qlinear_forward(dev_bf16(x), dev(qw), dev(sw), None, Q.I8A8_G128_BF16, N, flags=Q.HADAMARD)
    assert_close(y.cpu().numpy(), O.forward(x, qw.view(np.uint8), sw, None, Q.I8A8_G128_BF16, Q.HADAMARD, N))


@pytest.mark.parametrize("fmt", [3, 7])
@pytest.mark.parametrize("M,N,K", [(1, 512, 256), (5, 1000, 1024), (9, 130, 256), (16, 333, 640), (16, 4000, 5376)])
def test_gemm_a8_parity(fmt, M, N, K):
    """The decode GEMM on activations quantised beforehand: the act_quant call's codes (bit-exact
    against the oracle's quantiser) into qlinear_gemm_a8, against the oracle's forward of the bf16 x,
    overwriting y and then adding to a y that already holds values."""
    had = 1
    (c, s, z), (ch, sh, zh) = make_weights(fmt, N, K, had)
    x = x_bits(M, K, seed=13, outliers=0.01)
    quant = Q.act_quant_i8_g128 if fmt == Q.I8A8_G128_BF16 else Q.act_quant_e4m3_g128
    qx, sx = quant(dev_bf16(x), rotate=True)
    ref = O.forward(x, ch, sh, zh, fmt, had, N)
    y = Q.qlinear_gemm_a8(qx, sx, c, s, fmt, N)
    assert_close(y.cpu().numpy(), ref, f"fmt {fmt} {M}x{N}x{K}")
    y0 = np.linspace(-1.0, 1.0, M * N, dtype=np.float32).reshape(M, N)
    y = dev(y0)
    Q.qlinear_gemm_a8(qx, sx, c, s, fmt, N, y=y, accumulate=True)
    assert_close(y.cpu().numpy(), ref + y0.astype(np.float64), f"fmt {fmt} {M}x{N}x{K} accumulate")


def test_forward_zero_and_constant_inputs():
    N, K = 64, 256
    (c, s, z), (ch, sh, zh) = make_weights(Q.I8_G128_BF16, N, K, 0)
    x = np.zeros((3, K), np.uint16)
    y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.I8_G128_BF16, N)
    assert not y.abs().sum().item()
    x = O.bf16_encode(np.full((2, K), 3.0e4))  # large tokens: the per-token power-of-two keeps f16 in range
    y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.I8_G128_BF16, N)
    assert_close(y.cpu().numpy(), O.forward(x, ch, sh, None, Q.I8_G128_BF16, 0, N))


# --------------------------------------------------------------------------
# MoE
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,topk", [(1, 8, 2), (16, 128, 8), (40, 16, 4), (300, 32, 8), (2048, 128, 8)])
def test_moe_permute_bitexact(T, E, topk):
    ids, _ = synth.routing(4, T, E, topk)
    counts, offsets, perm = Q.moe_permute(dev(ids), E)
    c_ref, o_ref, p_ref, bad = O.moe_permute(ids, E)
    assert bad == 0
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)


def test_moe_permute_degenerate_and_invalid():
    ids = np.zeros((5, 8), np.int32)  # every pair on expert 0
    counts, offsets, perm = Q.moe_permute(dev(ids), 4)
    assert np.array_equal(perm.cpu().numpy(), np.arange(40))
    ids[2, 3] = 77  # invalid id: dropped, flagged, no fault
    counts, offsets, perm = Q.moe_permute(dev(ids), 4)
    c_ref, o_ref, p_ref, bad = O.moe_permute(ids, 4)
    assert np.array_equal(perm.cpu().numpy()[:39], p_ref[:39]) and perm[39].item() == -1
    st, bits = Q.ql_get_device_error()
    assert st == 6 and bits & Q.DEVERR_EXPERT_ID


def moe_weights(E, N, K, fmt, seed=9):
    qs, ss = [], []
    for e in range(E):
        W = synth.weight_rows(seed, f"moeW{e}", K, 0, N)
        if fmt in (Q.FP8_B128_BF16, Q.FP8A8_B128_BF16):
            q, s = O.quant_fp8_b128(W, hadamard=True)
        else:
            q, s = O.quant_i8_g128(W, hadamard=True, scale_f16=fmt == Q.I8_G128_F16)
            q = q.view(np.uint8)
        qs.append(q)
        ss.append(s)
    return np.stack(qs), np.stack(ss)


@pytest.mark.parametrize("fmt", [1, 2, 6, 7])
@pytest.mark.parametrize("T,E,topk,N,K", [(1, 8, 2, 96, 256), (8, 16, 4, 64, 384), (16, 32, 8, 130, 256),
                                          (20, 32, 8, 130, 256), (40, 8, 3, 48, 128)])
def test_moe_gate_up_parity(fmt, T, E, topk, N, K):
    # T * topk <= 128: the expert GEMM ranks the ids itself; (20, 32, 8): 160 pairs, the
    # permute kernel's chunk table; (40, 8, 3): format 7 on the grouped tensor-core GEMM, the other
    # formats on the chunk table.
    codes, scales = moe_weights(E, N, K, fmt)
    ids, w = synth.routing(6, T, E, topk)
    x = x_bits(T, K, seed=13)
    y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N, fmt=fmt, flags=Q.HADAMARD,
                      topk_weights=dev(w))
    ref = O.moe_gate_up(x, ids, codes, scales, fmt, O.HADAMARD, E, N)
    assert_close(y.cpu().numpy(), ref, f"moe fmt {fmt} T{T}")


@pytest.mark.parametrize("fmt", [1, 2, 6, 7])
@pytest.mark.parametrize("T,E,topk,N,K", [(64, 8, 4, 130, 384), (300, 16, 8, 200, 256), (50, 64, 8, 128, 128),
                                          (600, 8, 2, 400, 256)])
def test_moe_gate_up_grouped_parity(fmt, T, E, topk, N, K):
    # T * topk >= 8 E: format 7 on the grouped tensor-core GEMM, the formats with 16-bit activations
    # on the weight-streaming kernel over the permute kernel's 16-row chunks.  (300, 16, 8): ~150
    # rows per expert; N = 200: a ragged second weight block. (50, 64, 8): some experts get no rows.
    # (600, 8, 2): ~150 rows per expert, several 128-row tiles each; N = 400: three weight tiles of the
    # E4M3 GEMM (192 rows each), the last one ragged.
    codes, scales = moe_weights(E, N, K, fmt)
    ids, w = synth.routing(7, T, E, topk)
    x = x_bits(T, K, seed=17)
    ref = O.moe_gate_up(x, ids, codes, scales, fmt, O.HADAMARD, E, N)
    for _ in range(2):
        y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N, fmt=fmt, flags=Q.HADAMARD,
                          topk_weights=dev(w))
        assert_close(y.cpu().numpy(), ref, f"moe grouped fmt {fmt} T{T} E{E}")


@pytest.mark.parametrize("T,E,topk,K,I", [(1, 8, 2, 96, 64), (4, 16, 4, 130, 128), (16, 32, 8, 64, 192),
                                          (20, 32, 8, 200, 64), (300, 16, 8, 48, 128), (400, 8, 2, 200, 192),
                                          (500, 64, 8, 256, 64), (600, 4, 2, 136, 128)])
def test_moe_down_combine_parity(T, E, topk, K, I):
    # T * topk <= 128: the weight-streaming kernel ranks the ids itself; 160 pairs: the permute
    # kernel's chunks; from 8 pairs per expert on (2400, 800 and 4000 pairs) the grouped bf16
    # tensor-core GEMM over tiles of up to 160 rows (600 x top-2 over 4 experts: two row tiles per
    # expert, the second short).  K = 130, 136, 200: ragged 16-row slabs and ragged 128-row weight
    # blocks; I = 192: three 64-wide steps per plane.
    d = synth.moe_down(T, seed=3, E=E, topk=topk, K=K, I=I)
    wd = np.stack([d["Wd"][e] for e in range(E)])
    ref = O.moe_down_combine(d["h"], d["ids"], d["weights"], wd, E)
    for _ in range(2):
        out = Q.moe_down_combine(dev(d["h"]), dev(d["ids"]), dev(d["weights"]), dev(wd.view(np.int16)), E)
        assert_close(out.cpu().numpy(), ref, f"down T{T} E{E} K{K} I{I}")


@pytest.mark.parametrize("T", [4, 20])
def test_moe_down_combine_bad_id(T):
    E, topk, K, I = 8, 8 if T == 20 else 2, 64, 64
    d = synth.moe_down(T, seed=4, E=E, topk=topk, K=K, I=I)
    wd = np.stack([d["Wd"][e] for e in range(E)])
    ids = d["ids"].copy()
    ids[1, 1] = E + 5  # adds nothing, flagged
    Q.ql_get_device_error()
    out = Q.moe_down_combine(dev(d["h"]), dev(ids), dev(d["weights"]), dev(wd.view(np.int16)), E).cpu().numpy()
    st, bits = Q.ql_get_device_error()
    assert st == 6 and bits & Q.DEVERR_EXPERT_ID
    assert_close(out, O.moe_down_combine(d["h"], ids, d["weights"], wd, E), "down with a bad id")


def test_moe_gate_up_then_down_combine():
    """The whole routed-expert MLP: gate_up (int8 experts in the rotated domain) then the bf16 down
    projection and the combine, against the oracle's two steps (its gate_up output rounded to fp32,
    the input the down step takes)."""
    T, E, topk, K, I = 12, 16, 4, 256, 128
    codes, scales = moe_weights(E, 2 * I, K, Q.I8_G128_BF16)
    dd = synth.moe_down(T, seed=5, E=E, topk=topk, K=K, I=I)
    wd = np.stack([dd["Wd"][e] for e in range(E)])
    ids, w = dd["ids"], dd["weights"]
    x = x_bits(T, K, seed=23)
    h = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, 2 * I, fmt=Q.I8_G128_BF16,
                      flags=Q.HADAMARD)
    out = Q.moe_down_combine(h, dev(ids), dev(w), dev(wd.view(np.int16)), E).cpu().numpy()
    h_ref = O.moe_gate_up(x, ids, codes, scales, Q.I8_G128_BF16, O.HADAMARD, E, 2 * I).astype(np.float32)
    assert_close(out, O.moe_down_combine(h_ref, ids, w, wd, E), "gate_up then down")


def test_moe_gate_up_grouped_bad_id():
    E, N, K, T, topk = 8, 64, 128, 40, 4
    codes, scales = moe_weights(E, N, K, Q.I8_G128_BF16)
    ids, _ = synth.routing(8, T, E, topk)
    ids[5, 2] = 99  # skipped: flagged, its output row zero, every other pair exact
    x = x_bits(T, K, seed=19)
    Q.ql_get_device_error()
    y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N).cpu().numpy()
    st, bits = Q.ql_get_device_error()
    assert st == 6 and bits & Q.DEVERR_EXPERT_ID
    assert np.all(y[5, 2] == 0.0)
    ids_ok = ids.copy()
    ids_ok[5, 2] = 0
    ref = O.moe_gate_up(x, ids_ok, codes, scales, 1, 1, E, N)
    ref[5, 2] = 0.0
    assert_close(y, ref, "moe grouped, one bad id")


@pytest.mark.parametrize("T,E,topk", [(4, 8, 2), (20, 32, 8)])  # skinny modes: in-kernel ranking, permute kernel
def test_moe_gate_up_skinny_bad_ids(T, E, topk):
    N, K = 64, 128
    codes, scales = moe_weights(E, N, K, Q.I8_G128_BF16)
    ids, _ = synth.routing(8, T, E, topk)
    ids[1, 0] = E + 5  # skipped: flagged, their output rows zero, every other pair exact
    ids[2, topk - 1] = -1
    x = x_bits(T, K, seed=19)
    Q.ql_get_device_error()
    y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N).cpu().numpy()
    st, bits = Q.ql_get_device_error()
    assert st == 6 and bits & Q.DEVERR_EXPERT_ID
    assert np.all(y[1, 0] == 0.0) and np.all(y[2, topk - 1] == 0.0)
    ids_ok = ids.copy()
    ids_ok[1, 0] = ids_ok[2, topk - 1] = 0
    ref = O.moe_gate_up(x, ids_ok, codes, scales, 1, 1, E, N)
    ref[1, 0] = ref[2, topk - 1] = 0.0
    assert_close(y, ref, "moe skinny, bad ids")


def test_moe_duplicate_expert_in_token():
    E, N, K, T = 4, 64, 128, 3
    codes, scales = moe_weights(E, N, K, Q.I8_G128_BF16)
    ids = np.array([[1, 1, 2], [1, 3, 1], [0, 0, 0]], np.int32)
    x = x_bits(T, K, seed=1)
    y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N)
    assert_close(y.cpu().numpy(), O.moe_gate_up(x, ids, codes, scales, 1, 1, E, N))


# --------------------------------------------------------------------------
# Prefill (tcgen05) path: M >= 17 for W8A8
# --------------------------------------------------------------------------
# N % 4 == 0: y is written by TMA stores (N = 388: a ragged last tile, boxes clipped or skipped);
# N = 130 / 257: plain stores
PREFILL_SHAPES = [(17, 64, 128), (128, 128, 256), (200, 384, 512), (300, 130, 1024), (129, 257, 384), (150, 388, 256)]


@pytest.mark.parametrize("M,N,K", PREFILL_SHAPES)
def test_prefill_group_sums_bitexact(M, N, K):
    x = x_bits(M, K, seed=31, outliers=0.01)
    W = synth.weight_rows(31, f"Wpf{N}x{K}", K, 0, N)
    qw, sw = O.quant_i8_g128(W, hadamard=True)
    _, acc_ref = O.forward(x, qw.view(np.uint8), sw, None, Q.I8A8_G128_BF16, Q.HADAMARD, N, want_acc=True)
    qx, _ = O.act_quant_i8_g128(x, rotate=True)
    qx[0, :128] = 127  # extreme groups: +-127 against +-127
    qw_ext = qw.copy()
    qw_ext[0, :128] = -127
    acc = Q.qlinear_forward_i8_acc(dev(qx), dev(qw_ext))
    ref = np.einsum("mgk,ngk->mng", qx.reshape(M, K // 128, 128).astype(np.int64),
                    qw_ext.reshape(N, K // 128, 128).astype(np.int64))
    assert np.array_equal(acc.cpu().numpy(), ref)
    assert ref[0, 0, 0] == -128 * 127 * 127
    del acc_ref


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("M,N,K", PREFILL_SHAPES)
def test_prefill_forward_parity(M, N, K, had):
    x = x_bits(M, K, seed=37, outliers=0.01)
    W = synth.weight_rows(37, f"Wpf{N}x{K}", K, 0, N)
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=dev(W), flags=had)
    y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.I8A8_G128_BF16, N, flags=had)
    ref = O.forward(x, host_u8(c), host_u8(s).view(np.uint16), None, Q.I8A8_G128_BF16, had, N)
    assert_close(y.cpu().numpy(), ref, f"prefill {M}x{N}x{K} had {had}")


def test_prefill_large_tile_count_and_repeat():
    # 11 x 21 = 231 output tiles of 128 x 192, more than the 148 SMs, so
    # persistent CTAs walk two tiles each; ragged in both M and N; called twice
    M, N, K = 1290, 3980, 256
    x = x_bits(M, K, seed=41)
    W = synth.weight_rows(41, "Wpf_big", K, 0, N)
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=dev(W))
    ref, acc_ref = O.forward(x, host_u8(c), host_u8(s).view(np.uint16), None, Q.I8A8_G128_BF16, 0, N,
                             want_acc=True)
    for _ in range(2):
        y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.I8A8_G128_BF16, N)
        assert_close(y.cpu().numpy(), ref, f"prefill {M}x{N}x{K}")
    qx, _ = O.act_quant_i8_g128(x, rotate=False)
    acc = Q.qlinear_forward_i8_acc(dev(qx), c.view(torch.int8).reshape(N, K))
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


# --------------------------------------------------------------------------
# Format 7: E4M3 activations x fp8 weights on the tcgen05 kind::f8f6f4 GEMM (every M)
# --------------------------------------------------------------------------
FP8A8_SHAPES = [(1, 64, 128), (5, 130, 256), (16, 333, 640), (17, 64, 256), (129, 257, 384), (200, 384, 512),
                (300, 130, 1024), (150, 388, 256)]


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("M,N,K", FP8A8_SHAPES)
def test_fp8a8_forward_parity(M, N, K, had):
    (c, s, z), (ch, sh, zh) = make_weights(Q.FP8A8_B128_BF16, N, K, had)
    x = x_bits(M, K, seed=43, outliers=0.01)
    y = Q.qlinear_forward(dev_bf16(x), c, s, z, Q.FP8A8_B128_BF16, N, flags=had)
    ref = O.forward(x, ch, sh, zh, O.FP8A8_B128_BF16, had, N)
    assert_close(y.cpu().numpy(), ref, f"fp8a8 had {had} {M}x{N}x{K}")


# --------------------------------------------------------------------------
# int5 from 65 rows on: int8 activations on the W8A8 tensor-core GEMM (W5A8)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("M,N,K", [(64, 130, 256), (65, 130, 256), (65, 64, 128), (130, 388, 512),
                                   (300, 200, 384)])
def test_w5a8_forward_parity(M, N, K, had):
    # M = 64 is the last weight-only call, M = 65 the first W5A8 one; the oracle switches alike
    (c, s, z), (ch, sh, zh) = make_weights(Q.I5Z_G128_F16, N, K, had, seed=73)
    x = x_bits(M, K, seed=73, outliers=0.01)
    y = Q.qlinear_forward(dev_bf16(x), c, s, z, Q.I5Z_G128_F16, N, flags=had)
    ref = O.forward(x, ch, sh, zh, Q.I5Z_G128_F16, had, N)
    assert_close(y.cpu().numpy(), ref, f"int5 had {had} {M}x{N}x{K}")


def test_w5a8_large_tile_count_and_repeat():
    M, N, K = 1290, 3980, 256  # more tiles than SMs, ragged in M and N, called twice
    (c, s, z), (ch, sh, zh) = make_weights(Q.I5Z_G128_F16, N, K, 0, seed=79)
    x = x_bits(M, K, seed=79)
    ref = O.forward(x, ch, sh, zh, Q.I5Z_G128_F16, 0, N)
    for _ in range(2):
        y = Q.qlinear_forward(dev_bf16(x), c, s, z, Q.I5Z_G128_F16, N)
        assert_close(y.cpu().numpy(), ref, f"w5a8 {M}x{N}x{K}")


def test_fp8a8_large_tile_count_and_repeat():
    M, N, K = 1290, 3980, 256  # more tiles than SMs, ragged in M and N, called twice
    (c, s, z), (ch, sh, zh) = make_weights(Q.FP8A8_B128_BF16, N, K, 0, seed=47)
    x = x_bits(M, K, seed=47)
    ref = O.forward(x, ch, sh, zh, O.FP8A8_B128_BF16, 0, N)
    for _ in range(2):
        y = Q.qlinear_forward(dev_bf16(x), c, s, z, Q.FP8A8_B128_BF16, N)
        assert_close(y.cpu().numpy(), ref, f"fp8a8 {M}x{N}x{K}")


# --------------------------------------------------------------------------
# Prefill (tcgen05 kind::f16) path: M >= 17 for the 16-bit-activation formats
# with one-byte codes (int8 + bf16 / f16 scales, fp8 128x128 blocks)
# --------------------------------------------------------------------------
A16_PREFILL_SHAPES = [(17, 64, 128), (191, 128, 256), (193, 129, 384), (300, 130, 1024), (400, 6500, 256)]


@pytest.mark.parametrize("had", [0, 1])
@pytest.mark.parametrize("fmt", [1, 2, 6])  # int8 g128 bf16, int8 g128 f16, fp8 128x128
@pytest.mark.parametrize("M,N,K", A16_PREFILL_SHAPES)
def test_prefill_a16_parity(fmt, had, M, N, K):
    # (400, 6500, 256): 51 x 3 = 153 tiles of 128 weight rows x 192 tokens, more than the SMs
    (c, s, z), (ch, sh, zh) = make_weights(fmt, N, K, had)
    x = x_bits(M, K, seed=53, outliers=0.01)
    for _ in range(2):
        y = Q.qlinear_forward(dev_bf16(x), c, s, z, fmt, N, flags=had)
        ref = O.forward(x, ch, sh, zh, fmt, had, N)
        assert_close(y.cpu().numpy(), ref, f"a16 prefill fmt {fmt} had {had} {M}x{N}x{K}")
