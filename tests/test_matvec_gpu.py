"""Parity of the M <= 8 matvec path against the CPU oracle, on the device.

Covers the decode configuration (M in {1, 2, 4, 8} over the seven Qwen3-4B
projection shapes) element by element, ragged row counts, every M up to 8,
exact integer problems (bit-exact on every worker split), determinism, the
stream-K split at many worker counts, guard bands around y, and a stream
other than the default one.  These tests force the stream-K kernel
(W4A16_PATH_MATVEC) where the automatic choice would take the row-block one;
test_rows_gpu.py covers that kernel.
"""
import numpy as np
import pytest

import w4a16_synth as synth
from tolerance import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines too; skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)

import decode_w4a16_g128_b200 as w4  # noqa: E402
from gpu_util import bits, oracle_y, to_device  # noqa: E402


def run(prob, **kw):
    d = to_device(prob)
    if kw:
        y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], **kw)
    else:
        y = w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"])
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return bits(y)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("name,K,N", synth.QWEN3_4B_PROJECTIONS, ids=[p[0] for p in synth.QWEN3_4B_PROJECTIONS])
def test_decode_projection(M, name, K, N):
    prob = synth.make_problem(M, N, K)
    got = run(prob, path=w4.PATH_MATVEC)
    r = assert_close(got, oracle_y(prob), f"{name} M={M}")
    assert r["exact"] > 0.9 * r["n"]


@pytest.mark.parametrize("M", [1, 3, 5, 7, 8])
@pytest.mark.parametrize("N,K", [(8, 128), (129, 256), (1000, 2560), (1001, 384), (130, 9728), (4097, 128)])
def test_ragged_shapes(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    assert_close(run(prob, path=w4.PATH_MATVEC), oracle_y(prob), f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 24, 384), (5, 130, 640), (8, 257, 1024), (3, 1, 256), (8, 1000, 512)])
@pytest.mark.parametrize("workers", [0, 1, 3, 7, 64, 148, 1000])
def test_integer_problems_bit_exact(M, N, K, workers):
    prob = synth.make_integer_problem(M, N, K)
    got = run(prob, path=w4.PATH_MATVEC, workers=workers)
    assert np.array_equal(got, oracle_y(prob)), f"M={M} N={N} K={K} workers={workers}"


@pytest.mark.parametrize("workers", [1, 2, 5, 19, 100, 148, 5000])
def test_worker_splits(workers):
    prob = synth.make_problem(4, 2560, 9728, outliers=True)
    assert_close(run(prob, path=w4.PATH_MATVEC, workers=workers), oracle_y(prob), f"workers={workers}")


def test_deterministic_repeats():
    prob = synth.make_problem(8, 4096, 2560)
    d = to_device(prob)
    outs = []
    for _ in range(10):
        y = w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"])
        outs.append(bits(y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_pr1_problem_rows_as_matvec():
    prob = synth.make_pr1_problem()
    for rows in (slice(0, 1), slice(5, 13), slice(31, 32)):
        sub = dict(prob, x=np.ascontiguousarray(prob["x"][rows]))
        assert_close(run(sub), oracle_y(sub))


def test_guard_bands_untouched():
    prob = synth.make_problem(3, 1000, 2560)
    d = to_device(prob)
    M, N = 3, 1000
    pad = 4096
    buf = torch.full((pad + M * N + pad,), -12345, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"], y=y)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert (host[:pad] == -12345).all() and (host[pad + M * N:] == -12345).all()
    assert_close(bits(y), oracle_y(prob))


def test_side_stream_and_status():
    prob = synth.make_problem(2, 9728, 2560)
    d = to_device(prob)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"])
    s.synchronize()
    assert w4.w4a16_device_status(s) == w4.OK
    assert_close(bits(y), oracle_y(prob))


def test_k_zero_gives_zeros():
    x = torch.empty((2, 0), dtype=torch.bfloat16, device="cuda")
    wq = torch.empty((5, 0), dtype=torch.int32, device="cuda")
    s = torch.empty((5, 0), dtype=torch.bfloat16, device="cuda")
    y = torch.full((2, 5), 7.0, dtype=torch.bfloat16, device="cuda")
    w4.w4a16_matmul(x, wq, s, s, y=y)
    torch.cuda.synchronize()
    assert (y.float() == 0).all()


def test_last_rows_matvec():
    prob = synth.make_problem(6, 4096, 2560)
    d = to_device(prob)
    y = w4.w4a16_matmul_last_rows(d["x"], d["wq"], d["scales"], d["biases"], keep=1)
    torch.cuda.synchronize()
    assert y.shape == (1, 4096)
    sub = dict(prob, x=np.ascontiguousarray(prob["x"][5:6]))
    assert_close(bits(y), oracle_y(sub))


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
@pytest.mark.parametrize("M,N,K", [(4, 2560, 9728), (1, 1000, 2560), (8, 129, 384)])
def test_launch_flags(flags, M, N, K):
    prob = synth.make_integer_problem(M, N, min(K, 1024)) if K <= 1024 else synth.make_problem(M, N, K)
    got = run(prob, flags=flags)
    if K <= 1024:
        assert np.array_equal(got, oracle_y(prob))
    else:
        assert_close(got, oracle_y(prob), f"flags={flags}")


@pytest.mark.parametrize("workers", [1, 2, 3, 148])
def test_single_slab_slot_recycling(workers):
    """K = 9728 keeps one scale/bias slab slot, so CTAs spanning several row
    tiles must recycle it; a single worker walks all 20 tiles in sequence."""
    prob = synth.make_problem(2, 2560, 9728, outliers=True)
    assert_close(run(prob, path=w4.PATH_MATVEC, workers=workers, flags=w4.FLAG_STATIC_WEIGHTS),
                 oracle_y(prob), f"workers={workers}")


def test_long_k_without_slab():
    """K = 65536 (512 groups) is too long for a scale/bias slab: values come from global memory."""
    prob = synth.make_problem(3, 200, 65536)
    slab_pair = 2 * 128 * 512 * 2   # the scale and bias rows of one 128-row tile
    assert w4.w4a16_plan(3, 200, 65536)["smem_bytes"] < slab_pair
    assert_close(run(prob), oracle_y(prob), "K=65536")

