"""Parity of every kernel against the CPU oracle on inputs built to hit the corners of the
layer's definition.

Each kernel path is forced through w4a16_matmul_ex: the row-block matvec (automatic K split,
and forced 1 and 2), the stream-K matvec (automatic CTA count, 37 and 148 CTAs) and the
tensor-core GEMM (K splits 1 to 4 and 8).  Inputs:

* constant groups (the quantiser gives scale 0, so w = bias), and code blocks forced to all 15
  and all 0, with zero-mean, |N(0,1)| * 4 and silu(a) * b activations, at the 9728-deep down
  projection for M in {1, 8} (matvecs) and {128, 2048 sampled rows} (GEMM).  The kernels add
  s P' + (b - 128 s) X per group with P' = sum (128 + q) x and X = sum x; mostly positive
  activations make X large, so these cases check the cancellation between the two terms;
* activations of magnitude 2^122 with positive weights, where the plain FP32 sum overflows to
  +-inf for every output, and of magnitude 2^118 .. 2^121 with zero-mean weights, where the
  plain sum stays finite but P' and X overflow: the kernels' plain-definition path for
  non-finite results must reproduce the oracle.

The rule is the usual one (one BF16 ulp + 1e-3), with infinities equal to infinities of the
same sign, and no tolerance is widened for these inputs.
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

MATVEC_PATHS = [
    ("rows-auto", dict(path=w4.PATH_MATVEC_ROWS)),
    ("rows-s1", dict(path=w4.PATH_MATVEC_ROWS, splits=1)),
    ("rows-s2", dict(path=w4.PATH_MATVEC_ROWS, splits=2)),
    ("streamk-auto", dict(path=w4.PATH_MATVEC)),
    ("streamk-37", dict(path=w4.PATH_MATVEC, workers=37)),
    ("streamk-148", dict(path=w4.PATH_MATVEC, workers=148)),
]
GEMM_PATHS = [(f"gemm-s{s}", dict(path=w4.PATH_GEMM, splits=s)) for s in (1, 2, 3, 4, 8)]


def run(prob, **kw):
    d = to_device(prob)
    y = w4.w4a16_matmul_ex(d["x"], d["wq"], d["scales"], d["biases"], **kw)
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return bits(y)


def fits(M, N, K, kw):
    try:
        w4.w4a16_plan(M, N, K, **kw)
        return True
    except w4.W4A16Error:
        return False


@pytest.mark.parametrize("x_kind", ["normal", "abs4", "swiglu"])
@pytest.mark.parametrize("M", [1, 8])
@pytest.mark.parametrize("name,kw", MATVEC_PATHS, ids=[n for n, _ in MATVEC_PATHS])
def test_matvec_edge_weights_and_positive_x(name, kw, M, x_kind):
    N, K = 2560, 9728
    if not fits(M, N, K, kw):
        pytest.skip(f"{name} does not fit {M}x{N}x{K}")
    prob = synth.make_edge_problem(M, N, K, x_kind)
    assert prob["const_groups"] > 0
    r = assert_close(run(prob, **kw), oracle_y(prob), f"{name} M={M} x={x_kind}")
    print(f"{name} M={M} x={x_kind}: strict_fail {r['strict_fail']}/{r['n']}, max_ratio {r['max_ratio']:.3f}")


@pytest.mark.parametrize("x_kind", ["normal", "abs4", "swiglu"])
@pytest.mark.parametrize("name,kw", GEMM_PATHS, ids=[n for n, _ in GEMM_PATHS])
def test_gemm_edge_weights_and_positive_x(name, kw, x_kind):
    prob = synth.make_edge_problem(128, 2560, 9728, x_kind)
    r = assert_close(run(prob, **kw), oracle_y(prob), f"{name} M=128 x={x_kind}")
    print(f"{name} M=128 x={x_kind}: strict_fail {r['strict_fail']}/{r['n']}, max_ratio {r['max_ratio']:.3f}")


@pytest.mark.parametrize("x_kind", ["abs4", "swiglu"])
def test_gemm_m2048_positive_x_sampled_rows(x_kind):
    prob = synth.make_edge_problem(2048, 2560, 9728, x_kind)
    got = run(prob)
    rows = np.unique(np.concatenate([[0, 2047], np.random.default_rng([5, 2048]).choice(2048, 30, replace=False)]))
    assert_close(got[rows], oracle_y(prob, rows), f"M=2048 x={x_kind} rows {len(rows)}")


OVERFLOW = [("inf+", dict(sign=1.0)), ("inf-", dict(sign=-1.0)),
            ("finite-2^118", dict(exponent=118, positive_w=False)),
            ("finite-2^121", dict(exponent=121, positive_w=False))]


@pytest.mark.parametrize("case,ckw", OVERFLOW, ids=[c for c, _ in OVERFLOW])
@pytest.mark.parametrize("name,kw", MATVEC_PATHS + GEMM_PATHS, ids=[n for n, _ in MATVEC_PATHS + GEMM_PATHS])
def test_overflowing_activations(name, kw, case, ckw):
    M = 3 if name.startswith(("rows", "streamk")) else 20
    N, K = 300, 2560
    if not fits(M, N, K, kw):
        pytest.skip(f"{name} does not fit")
    prob = synth.make_overflow_problem(M, N, K, **ckw)
    ref = oracle_y(prob)
    inf_ref = np.isinf(synth.bf16_to_f32(ref))
    assert inf_ref.all() if case.startswith("inf") else not inf_ref.any()
    assert_close(run(prob, **kw), ref, f"{name} {case}")
