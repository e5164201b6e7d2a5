"""Parity of the tcgen05 tensor-core GEMM (M > 8) against the CPU oracle.

Covers the small reference problem (M=32, K=256, N=64), the M=128 prefill
configuration over the seven Qwen3-4B projections, partial tiles with long K
and 1 % outliers, the M=2048 configuration on sampled rows (including the
vocabulary projection), exact integer problems, ragged M and N, the forced
GEMM path at small M, determinism, and the last-row projection.
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


def test_pr1_problem():
    prob = synth.make_pr1_problem()
    r = assert_close(run(prob), oracle_y(prob), "M=32 K=256 N=64")
    assert r["exact"] > 0.9 * r["n"]


@pytest.mark.parametrize("name,K,N", synth.QWEN3_4B_PROJECTIONS, ids=[p[0] for p in synth.QWEN3_4B_PROJECTIONS])
def test_prefill_m128(name, K, N):
    prob = synth.make_problem(128, N, K)
    r = assert_close(run(prob), oracle_y(prob), f"{name} M=128")
    assert r["exact"] > 0.9 * r["n"]


@pytest.mark.parametrize("M", [129, 509])
@pytest.mark.parametrize("N", [1000, 4096])
@pytest.mark.parametrize("K", [2560, 9728])
def test_partial_tiles_long_k(M, N, K):
    prob = synth.make_problem(M, N, K, outliers=True)
    assert_close(run(prob), oracle_y(prob), f"M={M} N={N} K={K}")


def _sample_rows(M, seed=0):
    rng = np.random.default_rng([seed, M])
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, size=30, replace=False)]))


@pytest.mark.parametrize("name,K,N", synth.QWEN3_4B_PROJECTIONS + (synth.QWEN3_4B_LM_HEAD,),
                         ids=[p[0] for p in synth.QWEN3_4B_PROJECTIONS] + ["lm_head"])
def test_prefill_m2048_sampled_rows(name, K, N):
    prob = synth.make_problem(2048, N, K)
    got = run(prob)
    rows = _sample_rows(2048)
    assert_close(got[rows], oracle_y(prob, rows), f"{name} M=2048 rows {len(rows)}")


@pytest.mark.parametrize("M,N,K", [(9, 24, 384), (16, 130, 640), (17, 257, 1024), (127, 8, 256), (129, 1000, 512),
                                   (300, 136, 128)])
def test_integer_problems_bit_exact(M, N, K):
    prob = synth.make_integer_problem(M, N, K)
    got = run(prob, path=w4.PATH_GEMM)
    assert np.array_equal(got, oracle_y(prob)), f"M={M} N={N} K={K}"


@pytest.mark.parametrize("M", [9, 15, 17, 127, 129, 255, 257])
@pytest.mark.parametrize("N", [8, 1000, 1001])
def test_ragged(M, N):
    prob = synth.make_problem(M, N, 384, outliers=True)
    assert_close(run(prob), oracle_y(prob), f"M={M} N={N}")


@pytest.mark.parametrize("M", [1, 2, 8])
def test_forced_gemm_small_m(M):
    prob = synth.make_problem(M, 4096, 2560)
    assert_close(run(prob, path=w4.PATH_GEMM), oracle_y(prob), f"forced GEMM M={M}")


def test_deterministic_repeats():
    prob = synth.make_problem(300, 2560, 4096)
    d = to_device(prob)
    outs = [bits(w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"])) for _ in range(5)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_guard_bands_untouched():
    prob = synth.make_problem(129, 1000, 2560)
    d = to_device(prob)
    M, N, pad = 129, 1000, 4096
    buf = torch.full((pad + M * N + pad,), -12345, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"], y=y)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert (host[:pad] == -12345).all() and (host[pad + M * N:] == -12345).all()
    assert_close(bits(y), oracle_y(prob))


def test_logits_to_keep_lm_head():
    """Last-row vocabulary projection (matvec) vs all rows (GEMM) of the same call."""
    K, N = 2560, 151936
    prob = synth.make_problem(64, N, K)
    d = to_device(prob)
    last = w4.w4a16_matmul_last_rows(d["x"], d["wq"], d["scales"], d["biases"], keep=1)
    full = w4.w4a16_matmul_last_rows(d["x"], d["wq"], d["scales"], d["biases"], keep=0)
    torch.cuda.synchronize()
    assert last.shape == (1, N) and full.shape == (64, N)
    ref_last = oracle_y(prob, np.array([63]))
    assert_close(bits(last), ref_last, "last row")
    assert_close(bits(full)[63:64], ref_last, "row 63 of all rows")


@pytest.mark.parametrize("splits", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("M,N,K", [(128, 1000, 1024), (300, 257, 1024), (17, 130, 768), (64, 100, 1024)])
def test_split_k_integer_bit_exact(splits, M, N, K):
    prob = synth.make_integer_problem(M, N, K)
    got = run(prob, path=w4.PATH_GEMM, splits=splits)
    assert np.array_equal(got, oracle_y(prob)), f"splits={splits} M={M} N={N} K={K}"


@pytest.mark.parametrize("splits", [2, 3, 4, 6, 8])
def test_split_k_down_proj(splits):
    prob = synth.make_problem(128, 2560, 9728, outliers=True)
    assert_close(run(prob, path=w4.PATH_GEMM, splits=splits), oracle_y(prob), f"down_proj splits={splits}")


def test_split_k_deterministic():
    prob = synth.make_problem(128, 1024, 2560)
    d = to_device(prob)
    assert w4.w4a16_plan(128, 1024, 2560)["splits"] > 1
    outs = [bits(w4.w4a16_matmul(d["x"], d["wq"], d["scales"], d["biases"])) for _ in range(10)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    assert_close(outs[0], oracle_y(prob))
