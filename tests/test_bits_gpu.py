"""2- and 8-bit codes (w4a16_matmul_bits): the tensor-core decode matvec against the CPU oracle.

Every comparison uses the usual rule (one BF16 ulp + 1e-3 of the oracle's sequential FP32
result); integer-valued problems, whose FP32 sums are exact, must match bit for bit and give
the same bits on every run.  Shapes cover ragged N (rows past the last 16- or 32-row block),
K of one group and fewer groups than warps, the Qwen3-4B decode projections, M from 1 to 8
and slices of 8 x rows up to M = 32; edge weights (constant groups, all codes at the top or
zero), positive activations, and activations so large that the factorised sums overflow
FP32 where the plain definition does not (the kernel then computes that output by the plain
definition).
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
import oracle  # noqa: E402
from gpu_util import bits as to_bits, to_device  # noqa: E402


def run(prob, bits):
    d = to_device(prob)
    y = w4.w4a16_matmul_bits(d["x"], d["wq"], d["scales"], d["biases"], bits)
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return to_bits(y)


def ref(prob, bits):
    return oracle.matmul_bits(prob["x"], prob["wq"], prob["scales"], prob["biases"], bits)


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(1000, 384), (17, 128), (130, 896), (4096, 2560), (2560, 9728)])
def test_bits_against_oracle(bits, M, N, K):
    prob = synth.make_problem_bits(M, N, K, bits, outliers=True)
    assert_close(run(prob, bits), ref(prob, bits), f"{bits}-bit M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("M", [9, 16, 32])
def test_bits_row_slices(bits, M):
    prob = synth.make_problem_bits(M, 1000, 2560, bits)
    assert_close(run(prob, bits), ref(prob, bits), f"{bits}-bit slices M={M}")


@pytest.mark.parametrize("bits", [2, 8])
def test_bits_integer_bit_exact_and_deterministic(bits):
    K = 1024 if bits == 2 else 256
    prob = synth.make_integer_problem_bits(8, 333, K, bits)
    want = ref(prob, bits)
    for _ in range(3):
        assert np.array_equal(run(prob, bits), want)


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("x_kind", ["normal", "swiglu"])
def test_bits_edge_weights(bits, x_kind):
    """Constant groups (scale 0), groups of all-top and all-zero codes, positive x."""
    M, N, K = 8, 700, 2560
    G = K // 128
    rng = synth.shape_rng(M, N, K, seed=31 + bits)
    x = synth.make_x(rng, M, K) if x_kind == "normal" else synth.make_x_positive(rng, M, K, x_kind)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    Wg = W.reshape(N, G, 128)
    idx = np.arange(N * G).reshape(N, G)
    const = (idx % 7) == 3
    Wg[const] = Wg[const][:, :1]
    wq, s, b = synth.quantize_affine_g128(Wg.reshape(N, K), bits)
    words = wq.reshape(N, G, 4 * bits)
    words[(idx % 5) == 1] = np.uint32(0xFFFFFFFF)
    words[(idx % 11) == 2] = np.uint32(0)
    prob = {"x": x, "wq": words.reshape(N, K * bits // 32).copy(), "scales": s, "biases": b}
    assert_close(run(prob, bits), ref(prob, bits), f"{bits}-bit edge x={x_kind}")


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("case", ["inf+", "inf-", "finite-2^121"])
def test_bits_overflow_takes_the_plain_definition(bits, case):
    """|x| ~ 2^122 of one sign with positive weights: every plain sum overflows to +-inf.
    |x| ~ 2^121 with centred weights: the plain sums stay finite while the group sums of x
    (and so the factorised terms) overflow; the kernel's plain-definition path must agree."""
    M, N, K = 3, 300, 2560
    rng = synth.shape_rng(M, N, K, seed=97 + bits)
    exponent, sign = (121, 1.0) if case.startswith("finite") else (122, 1.0 if case == "inf+" else -1.0)
    mag = np.float32(2.0 ** exponent) * (np.float32(1) + rng.random((M, K), dtype=np.float32))
    x = synth.bf16_bits(np.float32(sign) * mag)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    if case.startswith("inf"):
        W = np.abs(W) + np.float32(0.05)
    wq, s, b = synth.quantize_affine_g128(W, bits)
    prob = {"x": x, "wq": wq, "scales": s, "biases": b}
    want = ref(prob, bits)
    inf_ref = np.isinf(synth.bf16_to_f32(want))
    assert inf_ref.all() if case.startswith("inf") else not inf_ref.any()
    assert_close(run(prob, bits), want, f"{bits}-bit overflow {case}")


def test_bits_four_is_the_4bit_layer():
    prob = synth.make_problem(4, 1000, 2560, seed=3)
    assert_close(run(prob, 4), oracle.matmul(prob["x"], prob["wq"], prob["scales"], prob["biases"]), "bits=4")


@pytest.mark.parametrize("bits", [2, 8])
def test_bits_empty_and_k_zero(bits):
    dev = "cuda"
    x = torch.zeros((3, 0), dtype=torch.bfloat16, device=dev)
    wq = torch.zeros((5, 0), dtype=torch.int32, device=dev)
    s = torch.zeros((5, 0), dtype=torch.bfloat16, device=dev)
    y = torch.full((3, 5), 7.0, dtype=torch.bfloat16, device=dev)
    w4.w4a16_matmul_bits(x, wq, s, s, bits, y=y)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), torch.zeros((3, 5), dtype=torch.int16, device=dev))
    e = w4.w4a16_matmul_bits(torch.zeros((0, 128), dtype=torch.bfloat16, device=dev),
                             torch.zeros((5, 4 * bits), dtype=torch.int32, device=dev),
                             torch.zeros((5, 1), dtype=torch.bfloat16, device=dev),
                             torch.zeros((5, 1), dtype=torch.bfloat16, device=dev), bits)
    assert e.shape == (0, 5)


@pytest.mark.parametrize("bits", [2, 8])
def test_bits_unsupported_m(bits):
    prob = synth.make_problem_bits(33, 64, 128, bits)
    with pytest.raises(w4.W4A16Error) as ei:
        run(prob, bits)
    assert ei.value.status == w4.ERR_UNSUPPORTED


@pytest.mark.parametrize("bits", [2, 8])
def test_bits_full_size_sampled(bits):
    """The benchmark's largest decode projection (gate, 2560 -> 9728) at M = 8 with all rows on
    the GPU; the oracle computes every 19th row and the last 16 (about 530 rows)."""
    M, N, K = 8, 9728, 2560
    prob = synth.make_problem_bits(M, N, K, bits)
    got = run(prob, bits)
    rows = np.unique(np.concatenate([np.arange(0, N, 19), np.arange(N - 16, N)]))
    want = oracle.matmul_bits(prob["x"], prob["wq"][rows], prob["scales"][rows], prob["biases"][rows], bits)
    assert_close(got[:, rows], want, f"{bits}-bit sampled rows, full size")
