"""A bounded device wait that expires: the kernel returns, the host sees I8Q_ERR_TIMEOUT, and the
next call on the same stream is correct again.

Every mbarrier wait in the library's kernels gives up after a time limit (2 s by default), sets a
device error word, and lets the kernel finish without its result.  Here the limit is lowered to
1 ms and one accumulator-ready signal of a decode-size channel-wise GEMM is withheld (the test aid
i8q_test_skip_accumulator_signal), so that one CTA's epilogue wait runs out.  Nothing faults or
hangs: every copy and MMA already issued still completes and is waited for before the CTA exits."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return setup_library()


def test_expired_wait_reports_timeout_and_recovers(q):
    M, N, K = 16, 256, 512
    x = synth.activation_bf16(M, K, seed=61)
    w = synth.weight_bf16(N, K, seed=62)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)
    Y, A = O.gemm_w8a8_channel(xq, sx, wq, sw)
    xqd, sxd, wqd, swd = dev(xq), dev(sx), dev(wq), dev(sw)
    q.i8q_status_check()                                   # nothing pending before the test
    y = empty((M, N), torch.int16, 0x7FC0)
    try:
        q.i8q_test_set_wait_limit_ns(1_000_000)            # 1 ms
        q.i8q_test_skip_accumulator_signal(True)
        q.i8q_gemm_w8a8_channel(xqd, sxd, wqd, swd, y)
        with pytest.raises(q.I8QError) as err:
            q.i8q_status_check()
        assert err.value.status == 6, err.value           # I8Q_ERR_TIMEOUT
        assert "expired" in str(err.value)
    finally:
        q.i8q_test_skip_accumulator_signal(False)
        q.i8q_test_set_wait_limit_ns(0)
    q.i8q_status_check()                                   # the error word was cleared
    for _ in range(2):                                     # the same stream works again, bit for bit
        y2 = empty((M, N), torch.int16, 0x7FC0)
        acc = empty((M, N), torch.int32, 0x7FFFFFFF)
        q.i8q_gemm_w8a8_channel(xqd, sxd, wqd, swd, y2, debug_acc=acc)
        q.i8q_status_check()
        assert np.array_equal(host(acc), A.astype(np.int32))
        check_half(host(y2, np.uint16), Y, np.abs(Y), "bf16", "after timeout", strict=True)
