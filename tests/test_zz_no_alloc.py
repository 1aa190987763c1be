"""The workspace-free W8A8 forward, for callers that cannot allocate device
memory (for example a plugin whose host engine owns all device memory).  It
must give the same result as qlinear_forward with a caller workspace, call
after call, since every call reuses the same fixed scratch array.  This file is
collected last so that a run stopping at its first failure has already run
every other test."""
import numpy as np
import pytest

from moe_hadamard128_act_b200 import synth
from tests.gpu_util import assert_close, dev, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    return qlinear


@pytest.mark.parametrize("M,N,K,flags", [(16, 1000, 5376, 1), (5, 333, 640, 0), (1, 64, 16384, 1)])
def test_noalloc_matches_workspace_forward_twice(Q, M, N, K, flags):
    W = dev(synth.weight_rows(21, f"noalloc_W{K}", K, 0, N))
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=W, flags=flags)
    for call in range(2):  # the second call finds the first call's contents in the scratch
        x = dev_bf16(synth.activations(call, f"noalloc_x{M}", M, K, outlier_frac=0.01))
        ref = Q.qlinear_forward(x, c, s, None, Q.I8A8_G128_BF16, N, flags=flags).cpu().numpy()
        got = Q.qlinear_forward_w8a8_noalloc(x, c, s, N, flags=flags).cpu().numpy()
        assert_close(got, ref.astype(np.float64), f"call {call}")
    st, bits = Q.ql_get_device_error()
    assert st == 0 and bits == 0


def test_noalloc_rejects_sizes_beyond_the_scratch(Q):
    N = 64
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, 256, W=dev(synth.weight_rows(22, "noalloc_big", 256, 0, N)))
    with pytest.raises(Q.QLError) as e:
        Q.qlinear_forward_w8a8_noalloc(dev_bf16(synth.activations(0, "nb", 17, 256)), c, s, N)
    assert e.value.status == 2  # QL_EUNSUPPORTED: more tokens than the scratch holds
    with pytest.raises(Q.QLError) as e:
        Q.qlinear_forward_w8a8_noalloc(dev_bf16(synth.activations(0, "nb2", 1, 16512)), c, s, N)
    assert e.value.status == 2
