"""The bounded waits of the library's kernels, made to run out on purpose.

Every wait of a kernel for a copy, an MMA or another warp's work gives up after
a bound and sets QL_DEVERR_TIMEOUT instead of hanging; the kernel then lets the
copies and MMAs it already started finish and frees its tensor memory.  Here the
bound is set to 1 ns, so the decode GEMM's ring waits and the tcgen05 prefill
GEMM's pipeline waits run out at once: the calls must return, the error word
must report the timeout, and after the default bound is restored the same calls
on the same process and GPU must match the oracle (nothing was left allocated
or in flight)."""
import numpy as np
import pytest

from moe_hadamard128_act_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_close, dev, dev_bf16, host_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    yield qlinear
    qlinear.ql_set_wait_limit(0)


def test_waits_run_out_then_recover(Q):
    N, K = 4096, 1024
    W = dev(synth.weight_rows(31, "waits_W", K, 0, N))
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=W, flags=Q.HADAMARD)
    ch, sh = host_u8(c), host_u8(s).view(np.uint16)
    cases = [(16, "decode"), (256, "prefill")]  # the TMA-fed decode GEMM, the tcgen05 W8A8 GEMM
    xs = {M: synth.activations(32, f"waits_x{M}", M, K, outlier_frac=0.01) for M, _ in cases}
    assert Q.ql_get_device_error() == (0, 0)
    try:
        Q.ql_set_wait_limit(1)
        for M, what in cases:
            Q.qlinear_forward(dev_bf16(xs[M]), c, s, None, Q.I8A8_G128_BF16, N, flags=Q.HADAMARD)
            st, bits = Q.ql_get_device_error()
            assert st == 6 and bits & Q.DEVERR_TIMEOUT, (what, st, bits)
    finally:
        Q.ql_set_wait_limit(0)
    for M, what in cases:
        y = Q.qlinear_forward(dev_bf16(xs[M]), c, s, None, Q.I8A8_G128_BF16, N, flags=Q.HADAMARD).cpu().numpy()
        assert Q.ql_get_device_error() == (0, 0), what
        assert_close(y, O.forward(xs[M], ch, sh, None, Q.I8A8_G128_BF16, Q.HADAMARD, N), f"{what} after recovery")
