"""The workspace-free W8A8 forward, for callers that cannot allocate device
memory (for example a plugin whose host engine owns all device memory, or a
loop that must never meet cudaMalloc's implicit synchronisation).  Every call
reuses the same fixed scratch array inside the library, so the result must be
right call after call: it is checked against the oracle and against
qlinear_forward with a caller workspace, on two calls in a row.  A call must
also leave the device's free memory and torch's allocations untouched.  This
file is collected last so that a run stopping at its first failure has already
run every other test."""
import numpy as np
import pytest
import torch

from moe_hadamard128_act_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_close, dev, dev_bf16, host_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from moe_hadamard128_act_b200 import build as qbuild
    qbuild.build()
    from moe_hadamard128_act_b200 import qlinear
    return qlinear


@pytest.mark.parametrize("M,N,K,flags", [(16, 1000, 5376, 1), (5, 333, 640, 0), (1, 64, 16384, 1)])
def test_noalloc_matches_oracle_and_workspace_forward_twice(Q, M, N, K, flags):
    W = dev(synth.weight_rows(21, f"noalloc_W{K}", K, 0, N))
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=W, flags=flags)
    codes = host_u8(c).reshape(N, K)
    scales = host_u8(s).view(np.uint16).reshape(N, K // 128)
    for call in range(2):  # the second call finds the first call's contents in the scratch
        xb = synth.activations(call, f"noalloc_x{M}", M, K, outlier_frac=0.01)
        x = dev_bf16(xb)
        ref = Q.qlinear_forward(x, c, s, None, Q.I8A8_G128_BF16, N, flags=flags).cpu().numpy()
        got = Q.qlinear_forward_w8a8_noalloc(x, c, s, N, flags=flags).cpu().numpy()
        assert_close(got, ref.astype(np.float64), f"call {call} vs workspace forward")
        assert_close(got, O.forward(xb, codes, scales, None, Q.I8A8_G128_BF16, flags, N), f"call {call} vs oracle")
    st, bits = Q.ql_get_device_error()
    assert st == 0 and bits == 0


def test_noalloc_allocates_nothing(Q):
    M, N, K = 8, 512, 1024
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, K, W=dev(synth.weight_rows(23, "noalloc_mem", K, 0, N)), flags=1)
    x = dev_bf16(synth.activations(0, "noalloc_mem_x", M, K))
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Q.qlinear_forward_w8a8_noalloc(x, c, s, N, flags=1, y=y)  # warm-up: kernel attributes, module load
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        Q.qlinear_forward_w8a8_noalloc(x, c, s, N, flags=1, y=y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 >= free0


def test_noalloc_rejects_sizes_beyond_the_scratch(Q):
    N = 64
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N, 256, W=dev(synth.weight_rows(22, "noalloc_big", 256, 0, N)))
    with pytest.raises(Q.QLError) as e:
        Q.qlinear_forward_w8a8_noalloc(dev_bf16(synth.activations(0, "nb", 17, 256)), c, s, N)
    assert e.value.status == 2  # QL_EUNSUPPORTED: more tokens than the scratch holds
    with pytest.raises(Q.QLError) as e:
        Q.qlinear_forward_w8a8_noalloc(dev_bf16(synth.activations(0, "nb2", 1, 16512)), c, s, N)
    assert e.value.status == 2
