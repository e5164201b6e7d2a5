"""Parity of the row-block matvec (W4A16_PATH_MATVEC_ROWS) against the CPU oracle.

Each CTA of this kernel owns whole weight rows over all of K, so the cases
are chosen around its own edges: the decode configuration (M in {1, 2, 4, 8}
over the seven Qwen3-4B projections, which the automatic choice sends here),
row counts that end inside an octet and inside a CTA's block, an odd number
of groups (a half-empty last code box), K from 128 to 9728, every M up to 8,
integer problems that must be bit-exact, launch flags and determinism.
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


def run(prob, flags=0):
    d = to_device(prob)
    y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC_ROWS, flags=flags)
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return bits(y)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("name,K,N", synth.QWEN3_4B_PROJECTIONS, ids=[p[0] for p in synth.QWEN3_4B_PROJECTIONS])
def test_decode_projection(M, name, K, N):
    assert w4.w4a16_plan(M, N, K)["path"] == w4.PATH_MATVEC_ROWS   # the automatic choice
    prob = synth.make_problem(M, N, K)
    r = assert_close(run(prob), oracle_y(prob), f"{name} M={M}")
    assert r["exact"] > 0.9 * r["n"]


@pytest.mark.parametrize("M", [1, 3, 5, 7, 8])
@pytest.mark.parametrize("N,K", [(1, 128), (8, 128), (129, 256), (1001, 384), (1000, 2560), (130, 9728),
                                 (4097, 128), (9733, 2560), (2563, 4096)])
def test_ragged_shapes(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    assert_close(run(prob), oracle_y(prob), f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 24, 384), (5, 130, 640), (8, 257, 1024), (3, 1, 256), (8, 1000, 512),
                                   (2, 77, 128)])
def test_integer_problems_bit_exact(M, N, K):
    prob = synth.make_integer_problem(M, N, K)
    assert np.array_equal(run(prob), oracle_y(prob)), f"M={M} N={N} K={K}"


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_launch_flags(flags):
    prob = synth.make_integer_problem(8, 129, 384)
    assert np.array_equal(run(prob, flags=flags), oracle_y(prob))
    prob = synth.make_problem(4, 2560, 9728)
    assert_close(run(prob, flags=flags), oracle_y(prob), f"flags={flags}")


def test_deterministic_repeats():
    prob = synth.make_problem(8, 9728, 2560)
    d = to_device(prob)
    outs = []
    for _ in range(10):
        y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC_ROWS)
        outs.append(bits(y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_back_to_back_static_weights():
    """A graph of calls that fetch their weights before the previous call ends."""
    probs = [synth.make_problem(M, N, K) for (M, N, K) in ((1, 4096, 2560), (2, 1024, 2560), (1, 2560, 4096),
                                                            (8, 9728, 2560), (4, 2560, 9728))]
    devs = [to_device(p) for p in probs]
    ys = [torch.empty((p["x"].shape[0], p["wq"].shape[0]), dtype=torch.bfloat16, device="cuda") for p in probs]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(3):
            for d, y in zip(devs, ys):
                w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], y=y, flags=w4.FLAG_STATIC_WEIGHTS)
    stream.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    for p, y in zip(probs, ys):
        assert_close(bits(y), oracle_y(p), "back-to-back")


@pytest.mark.parametrize("splits", [1, 2, 3, 4])
@pytest.mark.parametrize("M,N,K", [(1, 24, 1024), (8, 1000, 768), (5, 2568, 1024), (3, 136, 512)])
def test_forced_splits_integer_bit_exact(splits, M, N, K):
    """Every K split of a cluster (uneven group counts for 3), odd half-block counts and
    clusters padded with CTAs that own no rows: integer problems are exact on every path."""
    prob = synth.make_integer_problem(M, N, K)
    d = to_device(prob)
    y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC_ROWS, splits=splits)
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    assert np.array_equal(bits(y), oracle_y(prob)), f"splits={splits} M={M} N={N} K={K}"


@pytest.mark.parametrize("splits,row_blocks", [(1, 1), (1, 3), (2, 2), (4, 5), (2, 5)])
def test_forced_launch_shapes(splits, row_blocks):
    """Explicit (splits, row blocks) launches of the gate and down projections at M = 8."""
    for (N, K) in ((9728, 2560), (2560, 9728)):
        try:
            w4.w4a16_plan(8, N, K, path=w4.PATH_MATVEC_ROWS, splits=splits, row_blocks=row_blocks)
        except w4.W4A16Error:
            continue   # the layout does not fit
        prob = synth.make_problem(8, N, K)
        d = to_device(prob)
        y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], path=w4.PATH_MATVEC_ROWS,
                               splits=splits, row_blocks=row_blocks)
        torch.cuda.synchronize()
        assert w4.w4a16_device_status() == w4.OK
        assert_close(bits(y), oracle_y(prob), f"splits={splits} rb={row_blocks} N={N} K={K}")
