"""Parity at the full workload sizes, in the launch configuration the bench
times: the GPU computes every output; the oracle recomputes sampled weight rows
(regenerated independently from the counter-based generator) and those rows'
packed codes and outputs are compared."""
import numpy as np
import pytest
import torch

from moe_hadamard128_act_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_close, dev, dev_bf16, host_u8

pytestmark = pytest.mark.gpu

N_FULL, K_FULL = 21504, 5376


@pytest.fixture(scope="module")
def Q():
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    return qlinear


def sample_rows(N, seed=0, n_rand=24):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.r_[np.arange(16), np.arange(N - 8, N), rng.choice(N, n_rand, replace=False)])
    return rows


def test_tiny_w8a16_recipe(Q):
    d = synth.tiny_w8a16(seed=0)
    c, s, _ = Q.qlinear_pack(Q.I8_G128_BF16, d["N"], d["K"], codes=dev(d["codes"]), scales=dev(d["scales"]))
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, None, Q.I8_G128_BF16, d["N"])
    ref = O.forward(d["x"], d["codes"].view(np.uint8), d["scales"], None, Q.I8_G128_BF16, 0, d["N"])
    assert_close(y.cpu().numpy(), ref)


@pytest.fixture(scope="module")
def dense_w8a8(Q):
    """Dense decode W8A8 in the Hadamard domain, N=21504, K=5376, packed on the GPU."""
    W = synth.weight_rows(0, "W", K_FULL, 0, N_FULL)
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N_FULL, K_FULL, W=dev(W), flags=Q.HADAMARD)
    del W
    return c, s


@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_dense_w8a8_hadamard_full(Q, dense_w8a8, M):
    c, s = dense_w8a8
    d = synth.dense_w8a8_hadamard(M, rows=(0, 0))
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, None, Q.I8A8_G128_BF16, N_FULL, flags=Q.HADAMARD).cpu().numpy()
    rows = sample_rows(N_FULL, seed=M)
    Wr = np.concatenate([synth.weight_rows(0, "W", K_FULL, int(n), 1) for n in rows])
    qr, sr = O.quant_i8_g128(Wr, hadamard=True)
    G = K_FULL // 128
    ch = host_u8(c).reshape(N_FULL, K_FULL)
    sh = host_u8(s).view(np.uint16).reshape(N_FULL, G)
    assert np.array_equal(ch[rows], qr.view(np.uint8))
    assert np.array_equal(sh[rows], sr)
    ref = O.forward(d["x"], qr.view(np.uint8), sr, None, Q.I8A8_G128_BF16, Q.HADAMARD, len(rows))
    assert_close(y[:, rows], ref, f"W8A8 M={M}")


@pytest.mark.parametrize("M", [1, 4, 5, 16])
def test_w4a16_full(Q, M):
    d = synth.w4a16(M)
    c, s, _ = Q.qlinear_pack(Q.I4_G64_BF16, N_FULL, K_FULL, codes=dev(d["codes"]), scales=dev(d["scales"]))
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, None, Q.I4_G64_BF16, N_FULL).cpu().numpy()
    rows = sample_rows(N_FULL, seed=10 + M)
    cr = O.pack_i4(d["codes"][rows])
    assert np.array_equal(host_u8(c).reshape(N_FULL, -1)[rows], cr)
    ref = O.forward(d["x"], cr, d["scales"][rows], None, Q.I4_G64_BF16, 0, len(rows))
    assert_close(y[:, rows], ref, f"W4A16 M={M}")


def test_w5a8_prefill_full(Q):
    # the int5 weight at full size with 2048 tokens: int8 activations (W5A8), sampled rows
    M = 2048
    d = synth.w5a16(M)
    c, s, z = Q.qlinear_pack(Q.I5Z_G128_F16, N_FULL, K_FULL, codes=dev(d["codes"]), scales=dev(d["scales"]),
                             zeros=dev(d["zeros"]))
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, z, Q.I5Z_G128_F16, N_FULL).cpu().numpy()
    rows = sample_rows(N_FULL, seed=29)
    ref = O.forward(d["x"], O.pack_i5(d["codes"][rows]), d["scales"][rows], d["zeros"][rows], Q.I5Z_G128_F16, 0,
                    len(rows))
    assert_close(y[:, rows], ref, "W5A8 M=2048")


@pytest.mark.parametrize("M", [1, 4, 5, 16])
def test_w5a16_full(Q, M):
    d = synth.w5a16(M)
    c, s, z = Q.qlinear_pack(Q.I5Z_G128_F16, N_FULL, K_FULL, codes=dev(d["codes"]), scales=dev(d["scales"]),
                             zeros=dev(d["zeros"]))
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, z, Q.I5Z_G128_F16, N_FULL).cpu().numpy()
    rows = sample_rows(N_FULL, seed=20 + M)
    cr = O.pack_i5(d["codes"][rows])
    assert np.array_equal(host_u8(c).reshape(N_FULL, -1)[rows], cr)
    ref = O.forward(d["x"], cr, d["scales"][rows], d["zeros"][rows], Q.I5Z_G128_F16, 0, len(rows))
    assert_close(y[:, rows], ref, f"W5A16 M={M}")


@pytest.mark.parametrize("T", [1, 8, 16, 2048])
def test_moe_gate_up_full(Q, T):
    E, topk, K, N = 128, 8, 2816, 1408
    ids, w = synth.routing(0, T, E, topk)
    touched = sorted(set(ids.ravel().tolist()))
    d = synth.moe_gate_up(T, experts=touched)
    codes = dev(np.zeros((E, N, K), np.int8))
    scales = dev(np.zeros((E, N, K // 128), np.int16))
    for e in touched:
        c, s, _ = Q.qlinear_pack(Q.I8_G128_BF16, N, K, W=dev(d["W"][e]), flags=Q.HADAMARD)
        codes[e] = c.view(torch.int8).reshape(N, K)
        scales[e] = s.view(torch.int16).reshape(N, K // 128)
    y = Q.moe_gate_up(dev_bf16(d["x"]), dev(ids), codes, scales, E, N, topk_weights=dev(w)).cpu().numpy()
    rng = np.random.default_rng(T)
    pairs = rng.choice(T * topk, min(T * topk, 12), replace=False)
    for p in pairs:
        t, j = divmod(int(p), topk)
        e = ids[t, j]
        qr, sr = O.quant_i8_g128(d["W"][e], hadamard=True)
        ref = O.forward(d["x"][t:t + 1], qr.view(np.uint8), sr, None, Q.I8_G128_BF16, Q.HADAMARD, N)
        assert_close(y[t, j][None], ref, f"moe T={T} pair {p}")


@pytest.mark.parametrize("T", [1, 16, 2048])
def test_moe_gate_up_fp8a8_full(Q, T):
    """The fp8 experts ("gemma4-26b-a4b-dflash-fp8" README, table "Weights") with E4M3 activations at
    the MoE workload's sizes: 128 experts of [1408, 2816], top-8 routing, the weights packed on the GPU
    in the rotated domain.  T = 1 and 16 run the weight-streaming kernel, T = 2048 the grouped E4M3
    tensor-core GEMM.  Sampled pairs against the oracle's dense format-7 forward of their expert."""
    E, topk, K, N = 128, 8, 2816, 1408
    ids, w = synth.routing(0, T, E, topk)
    touched = sorted(set(ids.ravel().tolist()))
    d = synth.moe_gate_up(T, experts=touched)
    codes = dev(np.zeros((E, N, K), np.uint8))
    sb = (N + 127) // 128 * (K // 128)
    scales = dev(np.zeros((E, sb), np.int16))
    for e in touched:
        c, s, _ = Q.qlinear_pack(Q.FP8A8_B128_BF16, N, K, W=dev(d["W"][e]), flags=Q.HADAMARD)
        codes[e] = c.reshape(N, K)
        scales[e] = s.view(torch.int16)
    y = Q.moe_gate_up(dev_bf16(d["x"]), dev(ids), codes, scales, E, N, fmt=Q.FP8A8_B128_BF16, flags=Q.HADAMARD,
                      topk_weights=dev(w)).cpu().numpy()
    rng = np.random.default_rng(100 + T)
    pairs = rng.choice(T * topk, min(T * topk, 12), replace=False)
    for p in pairs:
        t, j = divmod(int(p), topk)
        e = ids[t, j]
        qr, sr = O.quant_fp8_b128(d["W"][e], hadamard=True)
        ref = O.forward(d["x"][t:t + 1], qr, sr, None, Q.FP8A8_B128_BF16, Q.HADAMARD, N)
        assert_close(y[t, j][None], ref, f"moe format 7 T={T} pair {p}")


@pytest.mark.parametrize("T", [1, 16, 2048])
def test_moe_down_combine_full(Q, T):
    """The experts' bf16 down projections (128 x [2816, 704], "gemma4-26b-a4b-dflash-i8" README, table
    "Weights") and the routing-weighted combine at the MoE workload's sizes, top-8 routing; sampled
    tokens against the oracle (only the experts they touch, renumbered)."""
    E, topk, K, I = 128, 8, 2816, 704
    ids, _ = synth.routing(0, T, E, topk)
    touched = sorted(set(ids.ravel().tolist()))
    d = synth.moe_down(T, experts=touched)
    wd = torch.zeros((E, K, I), dtype=torch.int16, device="cuda")
    for e in touched:
        wd[e] = dev(d["Wd"][e].view(np.int16))
    out = Q.moe_down_combine(dev(d["h"]), dev(d["ids"]), dev(d["weights"]), wd, E).cpu().numpy()
    rng = np.random.default_rng(200 + T)
    for t in rng.choice(T, min(T, 6), replace=False):
        es = sorted(set(d["ids"][t].tolist()))
        local = np.array([[es.index(e) for e in d["ids"][t]]], np.int32)
        ref = O.moe_down_combine(d["h"][t:t + 1], local, d["weights"][t:t + 1], np.stack([d["Wd"][e] for e in es]),
                                 len(es))
        assert_close(out[t:t + 1], ref, f"down T={T} token {t}")


def test_prefill_w8a8_full(Q):
    """W8A8 prefill at M=2048, N=21504, K=5376 (no Hadamard transform)."""
    d = synth.prefill()
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N_FULL, K_FULL, W=dev(d["W"]))
    del d["W"]
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, None, Q.I8A8_G128_BF16, N_FULL).cpu().numpy()
    rows = sample_rows(N_FULL, seed=55, n_rand=8)
    Wr = np.concatenate([synth.weight_rows(0, "W", K_FULL, int(n), 1) for n in rows])
    qr, sr = O.quant_i8_g128(Wr)
    assert np.array_equal(host_u8(c).reshape(N_FULL, K_FULL)[rows], qr.view(np.uint8))
    ref = O.forward(d["x"], qr.view(np.uint8), sr, None, Q.I8A8_G128_BF16, 0, len(rows))
    assert_close(y[:, rows], ref, "prefill W8A8 full")


@pytest.mark.parametrize("M", [1, 16])
def test_fp8a8_decode_full(Q, M):
    """Format 7 (fp8 weights, E4M3 activations) at decode sizes, on the weight-streaming kernel.  A
    weight block's scale depends on all of its 128 rows, so whole blocks are sampled."""
    W = dev(synth.weight_rows(0, "W", K_FULL, 0, N_FULL))
    c, s, _ = Q.qlinear_pack(Q.FP8A8_B128_BF16, N_FULL, K_FULL, W=W)
    del W
    x = synth.activations(0, f"x_M{M}", M, K_FULL)
    y = Q.qlinear_forward(dev_bf16(x), c, s, None, Q.FP8A8_B128_BF16, N_FULL).cpu().numpy()
    blocks = [0, 97, N_FULL // 128 - 1]
    rows = np.concatenate([np.arange(128 * b, 128 * b + 128) for b in blocks])
    qr, sr = O.quant_fp8_b128(np.concatenate([synth.weight_rows(0, "W", K_FULL, 128 * b, 128) for b in blocks]))
    assert np.array_equal(host_u8(c).reshape(N_FULL, K_FULL)[rows], qr)
    assert np.array_equal(host_u8(s).view(np.uint16).reshape(N_FULL // 128, K_FULL // 128)[blocks], sr)
    ref = O.forward(x, qr, sr, None, Q.FP8A8_B128_BF16, 0, len(rows))
    assert_close(y[:, rows], ref, f"format 7 decode M={M}")


def test_prefill_fp8_full(Q):
    """FP8 E4M3 weights per 128 x 128 block with bf16 block scales and bf16 activations
    ("gemma4-26b-a4b-dflash-fp8" README, table "Weights") at M=2048, N=21504, K=5376: the weight
    packed on the GPU from the seeded fp32 draw, the tensor-core prefill GEMM over all 1232
    persistent tiles.  A block scale depends on all 128 rows of its block, so whole blocks are
    sampled: their codes and scales bit-exact, their outputs against the oracle."""
    d = synth.prefill()
    c, s, _ = Q.qlinear_pack(Q.FP8_B128_BF16, N_FULL, K_FULL, W=dev(d["W"]))
    del d["W"]
    y = Q.qlinear_forward(dev_bf16(d["x"]), c, s, None, Q.FP8_B128_BF16, N_FULL).cpu().numpy()
    blocks = [0, 61, N_FULL // 128 - 1]
    rows = np.concatenate([np.arange(128 * b, 128 * b + 128) for b in blocks])
    qr, sr = O.quant_fp8_b128(np.concatenate([synth.weight_rows(0, "W", K_FULL, 128 * b, 128) for b in blocks]))
    assert np.array_equal(host_u8(c).reshape(N_FULL, K_FULL)[rows], qr)
    assert np.array_equal(host_u8(s).view(np.uint16).reshape(N_FULL // 128, K_FULL // 128)[blocks], sr)
    ref = O.forward(d["x"], qr, sr, None, Q.FP8_B128_BF16, 0, len(rows))
    assert_close(y[:, rows], ref, "prefill fp8 full")
