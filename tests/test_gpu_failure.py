"""The failure path that every kernel uses, exercised on the GPU without a fault: a bounded
wait on an mbarrier that nothing arrives on gives up after its limit, records its code in the
device error word, raises the CTA's abort flag (which releases the other waiter) and returns.
The host reads WR_ERR_TIMEOUT, and the context stays usable for the next call."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, torch_mod

WR_OK, WR_ERR_TIMEOUT = 0, 4


@pytest.fixture(scope="module")
def wr():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as lib
    return lib


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives(wr):
    torch = torch_mod()
    assert wr.wr_get_device_error() == WR_OK            # clean before
    wr.wr_selftest_wait_timeout()
    assert wr.wr_get_device_error() == WR_ERR_TIMEOUT   # the wait gave up and said so
    assert wr.wr_get_device_error() == WR_OK            # reading cleared the word
    # the context is intact: a normal call still matches the oracle
    N, K, M = 64, 512, 2
    codes, scales, packed, s_d = q_case(wr, 2, N, K, seed=77)
    x = wr_synth.activations_bf16(78, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, 2)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    wr.wr_gemv(M, N, K, dev(x), packed, s_d, 2, y, ws, nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_codes(x, codes, scales, 2)
    check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == WR_OK
