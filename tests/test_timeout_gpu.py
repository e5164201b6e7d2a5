"""The timeout path of the kernels' bounded waits, made to run out without a GPU fault.

Every wait in the library gives up after a limit, records W4A16_ERR_TIMEOUT in a device
status word and lets the kernel end normally.  W4A16_FLAG_TEST_DROP_COPY makes the row-block
matvec skip one copy (CTA 0 never requests its first group's codes), so the waits for it
cannot complete, with a 200 us limit.  Nothing traps, nothing is left in flight: the test
checks that the status word reports the timeout once and is clear afterwards, and that the
next normal calls on the same context match the oracle.
"""
import numpy as np
import pytest

import w4a16_synth as synth
from tolerance import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import decode_w4a16_g128_b200 as w4  # noqa: E402
from gpu_util import bits, oracle_y, to_device  # noqa: E402


@pytest.mark.parametrize("M,N,K,splits", [(1, 4096, 2560, 1), (8, 2560, 9728, 2), (4, 1024, 2560, 2)])
def test_dropped_copy_times_out_and_context_recovers(M, N, K, splits):
    prob = synth.make_problem(M, N, K)
    d = to_device(prob)
    assert w4.w4a16_device_status() == w4.OK
    w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC_ROWS, splits=splits,
                       flags=w4.FLAG_TEST_DROP_COPY)
    torch.cuda.synchronize()                                  # the kernel ended
    assert w4.w4a16_device_status() == w4.ERR_TIMEOUT         # ... after giving up on the dropped copy
    assert w4.w4a16_device_status() == w4.OK                  # the word was cleared
    ref = oracle_y(prob)
    for path in (w4.PATH_MATVEC_ROWS, w4.PATH_MATVEC):        # the same context computes correctly
        y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=path)
        torch.cuda.synchronize()
        assert w4.w4a16_device_status() == w4.OK
        assert_close(bits(y), ref, f"after the timeout, path {path}")


def test_drop_flag_only_for_the_row_block_kernel():
    prob = synth.make_problem(1, 256, 256)
    d = to_device(prob)
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC,
                           flags=w4.FLAG_TEST_DROP_COPY)
    assert e.value.status == w4.ERR_INVALID_ARG
    assert w4.w4a16_device_status() == w4.OK
