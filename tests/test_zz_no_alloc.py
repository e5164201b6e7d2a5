"""The allocation-free matvec entry point, w4a16_matvec_noalloc.

Some callers cannot allocate device memory at all -- a serving process whose
memory pool owns every byte of the GPU, code that runs inside a CUDA-graph
capture or a real-time loop where cudaMalloc is forbidden.  For them the
library offers a matvec whose scratch (partial sums and tickets for rows split
across CTAs) is a fixed array compiled into the library instead of a workspace
it allocates.  These tests call that entry point through the C ABI and check it
against the CPU oracle on the same inputs, twice in a row, so that scratch left
behind by the first call cannot disturb the second; they also check that a call
allocates nothing (free device memory is unchanged, and a call captured into a
CUDA graph replays correctly), the empty-sum case and the argument checks.

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
from gpu_util import bits, oracle_y, to_device  # noqa: E402

P = ctypes.c_void_p


def c_call(d, y, M, N, K, stream, x_offset=0):
    return w4.lib.w4a16_matvec_noalloc(P(d["x"].data_ptr() + x_offset), P(d["wq"].data_ptr()),
                                       P(d["scales"].data_ptr()), P(d["biases"].data_ptr()), P(y.data_ptr()),
                                       M, N, K, P(stream))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 2560), (8, 1024, 2560), (3, 2560, 9728), (5, 1000, 384),
                                   (2, 151936, 2560)])
def test_noalloc_matches_oracle_twice(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    d = to_device(prob)
    ref = oracle_y(prob)
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
    ref = oracle_y(prob)
    for _ in range(2):
        y = torch.empty((7, 700), dtype=torch.bfloat16, device="cuda")
        assert c_call(d, y, 7, 700, 1024, torch.cuda.current_stream().cuda_stream) == w4.OK
        torch.cuda.synchronize()
        assert np.array_equal(bits(y), ref)


def test_noalloc_allocates_nothing_and_captures():
    """After one call on the device (its set-up), further calls leave the free device memory
    unchanged, and a call captured into a CUDA graph (where an allocation would break the
    capture) replays to the oracle's result."""
    M, N, K = 4, 4096, 2560
    prob = synth.make_problem(M, N, K)
    d = to_device(prob)
    ref = oracle_y(prob)
    stream = torch.cuda.Stream()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert c_call(d, y, M, N, K, stream.cuda_stream) == w4.OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert c_call(d, y, M, N, K, stream.cuda_stream) == w4.OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    y.fill_(float("nan"))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        rc = c_call(d, y, M, N, K, stream.cuda_stream)
    assert rc == w4.OK
    g.replay()
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    assert_close(bits(y), ref, "captured no-alloc call")
    del g


def test_noalloc_empty_sum_and_argument_checks():
    stream = torch.cuda.current_stream().cuda_stream
    x = torch.zeros((9, 128), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((8, 16), dtype=torch.int32, device="cuda")
    s = torch.zeros((8, 1), dtype=torch.bfloat16, device="cuda")
    y = torch.full((9, 8), 7.0, dtype=torch.bfloat16, device="cuda")
    d = {"x": x, "wq": wq, "scales": s, "biases": s}
    assert c_call(d, y, 9, 8, 128, stream) == w4.ERR_UNSUPPORTED                    # M > 8
    assert c_call(d, y, 1, w4.NOALLOC_MAX_N + 1, 128, stream) == w4.ERR_UNSUPPORTED  # N too large
    assert c_call(d, y, 1, 8, 128, stream, x_offset=2) == w4.ERR_MISALIGNED          # x not 16-byte aligned
    assert c_call(d, y, 3, 8, 0, stream) == w4.OK                                    # K = 0: an empty sum
    torch.cuda.synchronize()
    host = y.float().cpu().numpy()
    assert (host[:3] == 0).all() and (host[3:] == 7).all()
