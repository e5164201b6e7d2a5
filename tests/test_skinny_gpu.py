"""8 < M <= 32: the row-block matvec over slices of 8 x rows, against the CPU oracle.

The automatic path takes two slices for 8 < M <= 16 where the rows fit (the measured
crossover against the GEMM, whose tiles pad M to 128); the forced row-block path takes up to
four slices.  Each slice is one launch of the same kernel over x rows 8 i .. 8 i + 7, so the
result must equal the oracle under the usual rule, and integer problems bit for bit.
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


def run(prob, **kw):
    d = to_device(prob)
    y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], **kw)
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return bits(y)


@pytest.mark.parametrize("M", [9, 12, 16, 17, 24, 32])
@pytest.mark.parametrize("N,K", [(4096, 2560), (1024, 2560), (2560, 9728), (1000, 384)])
def test_row_slices_forced(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    assert w4.w4a16_plan(M, N, K, path=w4.PATH_MATVEC_ROWS)["slices"] == -(-M // 8)
    assert_close(run(prob, path=w4.PATH_MATVEC_ROWS), oracle_y(prob), f"rows slices M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [9, 16])
def test_row_slices_automatic(M):
    N, K = 9728, 2560
    assert w4.w4a16_plan(M, N, K)["path"] == w4.PATH_MATVEC_ROWS
    prob = synth.make_problem(M, N, K)
    assert_close(run(prob), oracle_y(prob), f"automatic M={M}")


def test_row_slices_integer_bit_exact_and_deterministic():
    prob = synth.make_integer_problem(30, 700, 1024)
    ref = oracle_y(prob)
    outs = [run(prob, path=w4.PATH_MATVEC_ROWS) for _ in range(3)]
    for o in outs:
        assert np.array_equal(o, ref)


def test_row_slices_positive_activations():
    prob = synth.make_edge_problem(24, 2560, 9728, "swiglu")
    assert_close(run(prob, path=w4.PATH_MATVEC_ROWS), oracle_y(prob), "rows slices M=24 swiglu")
