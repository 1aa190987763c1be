"""The bounded waits of the library's kernels, made to run out on purpose.

Every wait of a kernel for a copy, an MMA or another warp's work gives up after
a bound and sets QL_DEVERR_TIMEOUT instead of hanging; the kernel then lets the
copies and MMAs it already started finish and frees its tensor memory.  Here the
bound is set to 1 ns, which makes every pipeline wait a single probe that does
not block.  The tcgen05 prefill GEMM's first waits (for its first operand tiles,
its first MMAs) cannot be satisfied that early, so it must report the timeout,
with copies in flight to drain and tensor memory to free.  The decode GEMM's
ring runs several units ahead of its use, so its probes may all succeed; its
call must return either way.  After the default bound is restored, both calls
on the same process and GPU must match the oracle (nothing was left allocated or
in flight)."""
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
            if what == "prefill":
                assert st == 6 and bits & Q.DEVERR_TIMEOUT, (what, st, bits)
            else:  # returned, and nothing but a timeout was flagged
                assert st in (0, 6) and bits & ~Q.DEVERR_TIMEOUT == 0, (what, st, bits)
    finally:
        Q.ql_set_wait_limit(0)
    for M, what in cases:
        y = Q.qlinear_forward(dev_bf16(xs[M]), c, s, None, Q.I8A8_G128_BF16, N, flags=Q.HADAMARD).cpu().numpy()
        assert Q.ql_get_device_error() == (0, 0), what
        assert_close(y, O.forward(xs[M], ch, sh, None, Q.I8A8_G128_BF16, Q.HADAMARD, N), f"{what} after recovery")
