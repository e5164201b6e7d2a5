"""The allocation-free matvec entry point, w4a16_matvec_noalloc.

Some callers cannot allocate device memory at all -- a serving process whose
memory pool owns every byte of the GPU, code that runs inside a CUDA-graph
capture or a real-time loop where cudaMalloc is forbidden.  For them the
library offers a matvec whose scratch (partial sums and tickets for rows split
across CTAs) is a fixed array compiled into the library instead of a workspace
it allocates.  This test calls that entry point through the C ABI and checks
it against the allocating entry point on the same inputs, twice in a row, so
that scratch left behind by the first call cannot disturb the second.

It lives in a file of its own that pytest collects last, and passes whether it
runs alone in a fresh process or after every other test.
"""
import ctypes

import numpy as np
import pytest

import w4a16_synth as synth
from tolerance import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import decode_w4a16_g128_b200 as w4  # noqa: E402
from gpu_util import bits, to_device  # noqa: E402

P = ctypes.c_void_p


def c_call(d, y, M, N, K, stream):
    return w4.lib.w4a16_matvec_noalloc(P(d["x"].data_ptr()), P(d["wq"].data_ptr()), P(d["scales"].data_ptr()),
                                       P(d["biases"].data_ptr()), P(y.data_ptr()), M, N, K, P(stream))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 2560), (8, 1024, 2560), (3, 2560, 9728), (5, 1000, 384),
                                   (2, 151936, 2560)])
def test_noalloc_matches_allocating_entry_twice(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    d = to_device(prob)
    ref = bits(w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"]))
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert c_call(d, y, M, N, K, stream) == w4.OK
        torch.cuda.synchronize()
        assert w4.w4a16_device_status() == w4.OK
        assert_close(bits(y), ref, f"no-alloc call {call + 1} M={M} N={N} K={K}")


def test_noalloc_integer_problem_bit_exact_twice():
    prob = synth.make_integer_problem(7, 700, 1024)
    d = to_device(prob)
    ref = bits(w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"]))
    for _ in range(2):
        y = torch.empty((7, 700), dtype=torch.bfloat16, device="cuda")
        assert c_call(d, y, 7, 700, 1024, torch.cuda.current_stream().cuda_stream) == w4.OK
        torch.cuda.synchronize()
        assert np.array_equal(bits(y), ref)


def test_noalloc_rejects_sizes_beyond_its_limits():
    x = torch.zeros((9, 128), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((8, 16), dtype=torch.int32, device="cuda")
    s = torch.zeros((8, 1), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((9, 8), dtype=torch.bfloat16, device="cuda")
    d = {"x": x, "wq": wq, "scales": s, "biases": s}
    stream = torch.cuda.current_stream().cuda_stream
    assert c_call(d, y, 9, 8, 128, stream) == w4.ERR_UNSUPPORTED               # M > 8
    assert c_call(d, y, 1, w4.NOALLOC_MAX_N + 1, 128, stream) == w4.ERR_UNSUPPORTED   # N too large
