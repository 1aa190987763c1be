"""GPU parity at the limits the C-ABI documents: the largest K of the formats
with 16-bit activations (QL_A16_MAX_K), W8A8 at the same K, and the largest
expert count of moe_gate_up / moe_permute (E = 1024), each against the fp64
oracle on seeded inputs."""
import numpy as np
import pytest

from moe_hadamard128_act_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_close, dev, dev_bf16
from tests.test_gpu_parity import make_weights, moe_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    import tests.test_gpu_parity as tp
    tp.Q = qlinear  # the shared weight helpers read the binding from there
    yield qlinear
    st, bits = qlinear.ql_get_device_error()
    assert st == 0 and bits == 0, f"device error word left set: {bits}"


@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6])
# the decode GEMM (M <= 16; at M = 8 the staged activations fill the most shared memory, so
# K splits into the most parts) and the prefill GEMM (M >= 17)
@pytest.mark.parametrize("M", [1, 8, 20])
def test_forward_parity_at_max_k(Q, fmt, M):
    K, N = Q.A16_MAX_K, 72  # N: one 64-row block and a ragged tail
    (c, s, z), (ch, sh, zh) = make_weights(fmt, N, K, Q.HADAMARD, seed=21)
    x = synth.activations(23, "x_maxk", M, K, outlier_frac=0.01)
    y = Q.qlinear_forward(dev_bf16(x), c, s, z, fmt, N, flags=Q.HADAMARD)
    ref = O.forward(x, ch, sh, zh, fmt, O.HADAMARD, N)
    assert_close(y.cpu().numpy(), ref, f"fmt {fmt} M {M} K {K}")


@pytest.mark.parametrize("T", [16, 1024])  # in-kernel ranking, then the permute kernel's chunks
def test_moe_gate_up_max_experts(Q, T):
    E, topk, N, K = 1024, 8, 64, 128
    codes, scales = moe_weights(E, N, K, Q.I8_G128_BF16)
    ids, w = synth.routing(31, T, E, topk)
    x = synth.activations(33, "x_moe_maxe", T, K)
    ref = O.moe_gate_up(x, ids, codes, scales, Q.I8_G128_BF16, O.HADAMARD, E, N)
    y = Q.moe_gate_up(dev_bf16(x), dev(ids), dev(codes), dev(scales), E, N, topk_weights=dev(w))
    assert_close(y.cpu().numpy(), ref, f"moe E {E} T {T}")


def test_moe_permute_max_experts(Q):
    T, E, topk = 512, 1024, 8
    ids, _ = synth.routing(35, T, E, topk)
    counts, offsets, perm = Q.moe_permute(dev(ids), E)
    rc, ro, rp, bad = O.moe_permute(ids, E)
    assert bad == 0
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
