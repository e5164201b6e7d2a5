"""The fused gate/up projection (decode) against the CPU oracle.

w4a16_gate_up reads x once and the gate and up layers' rows interleaved in blocks of 8, and
writes h = bf16(silu(g) * u) with g and u the FP32 sums of the two layers.  The oracle takes
the plain FP32 dots of the same rows, silu in double.  Cases: the Qwen3-4B gate/up shape
(2560 -> 9728) for M in {1, 2, 4, 8}, a long-K shape whose rows are split over a cluster, a
ragged output count, mostly positive activations, and activations so large that the FP32
sums overflow (the plain definition then decides).  Tolerance: the usual 1 BF16 ulp + 1e-3.
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
from gpu_util import bits  # noqa: E402


def gate_up_problem(M, N2, K, seed=0, x_kind="normal", exponent=None):
    rng = synth.shape_rng(M, N2, K, seed + 31337)
    if exponent is not None:
        x = synth.bf16_bits(np.float32(2.0 ** exponent) * (np.float32(1) + rng.random((M, K), dtype=np.float32)))
    elif x_kind == "normal":
        x = synth.make_x(rng, M, K)
    else:
        x = synth.make_x_positive(rng, M, K, x_kind)
    gq, gs, gb = synth.make_weights(rng, N2, K)
    uq, us, ub = synth.make_weights(rng, N2, K)
    return {"x": x, "wq": synth.interleave_gate_up(gq, uq), "scales": synth.interleave_gate_up(gs, us),
            "biases": synth.interleave_gate_up(gb, ub), "gate": (gq, gs, gb), "up": (uq, us, ub)}


def run(prob):
    d = {"x": torch.from_numpy(prob["x"].view(np.int16)).cuda().view(torch.bfloat16),
         "wq": torch.from_numpy(prob["wq"].view(np.int32)).cuda(),
         "scales": torch.from_numpy(prob["scales"].view(np.int16)).cuda().view(torch.bfloat16),
         "biases": torch.from_numpy(prob["biases"].view(np.int16)).cuda().view(torch.bfloat16)}
    h = w4.w4a16_gate_up(d["x"], d["wq"], d["scales"], d["biases"])
    torch.cuda.synchronize()
    assert w4.w4a16_device_status() == w4.OK
    return bits(h)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_gate_up_qwen3_4b(M):
    prob = gate_up_problem(M, 9728, 2560)
    ref = oracle.gate_up(prob["x"], prob["wq"], prob["scales"], prob["biases"])
    r = assert_close(run(prob), ref, f"gate/up M={M}")
    print(f"gate/up M={M}: strict_fail {r['strict_fail']}/{r['n']}")


@pytest.mark.parametrize("M,N2,K,x_kind", [(8, 1024, 9728, "normal"), (3, 1000, 2560, "normal"),
                                           (8, 2048, 9728, "swiglu"), (5, 512, 4096, "abs4")])
def test_gate_up_shapes(M, N2, K, x_kind):
    prob = gate_up_problem(M, N2, K, x_kind=x_kind)
    ref = oracle.gate_up(prob["x"], prob["wq"], prob["scales"], prob["biases"])
    assert_close(run(prob), ref, f"gate/up {M}x{N2}x{K} {x_kind}")


@pytest.mark.parametrize("exponent", [118, 122])
def test_gate_up_overflowing_sums(exponent):
    prob = gate_up_problem(2, 256, 2560, exponent=exponent)
    ref = oracle.gate_up(prob["x"], prob["wq"], prob["scales"], prob["biases"])
    assert_close(run(prob), ref, f"gate/up 2^{exponent}")


def test_gate_up_matches_unfused_layers():
    """The same as two layer calls and silu(g) * u, up to the BF16 rounding of g and u there."""
    M, N2, K = 4, 2048, 2560
    prob = gate_up_problem(M, N2, K, seed=1)
    h = synth.bf16_to_f32(run(prob)).astype(np.float64)
    g = oracle.matmul_f32(prob["x"], *prob["gate"]).astype(np.float64)
    u = oracle.matmul_f32(prob["x"], *prob["up"]).astype(np.float64)
    want = g / (1 + np.exp(-g)) * u
    assert np.all(np.abs(h - want) <= np.abs(want) * 2.0 ** -7 + 1e-3)


def test_gate_up_arguments():
    x = torch.zeros((9, 256), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((32, 32), dtype=torch.int32, device="cuda")
    sb = torch.zeros((32, 2), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_gate_up(x, wq, sb, sb)          # M = 9: decode only
    assert e.value.status == w4.ERR_UNSUPPORTED
    P = w4.ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)
    h = torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda")
    assert w4.lib.w4a16_gate_up(P(x.data_ptr()), P(wq.data_ptr()), P(sb.data_ptr()), P(sb.data_ptr()),
                                P(h.data_ptr()), 8, 12, 256, st) == w4.ERR_UNSUPPORTED   # N2 % 8
    assert w4.lib.w4a16_gate_up(P(0), P(0), P(0), P(0), P(0), 0, 16, 256, st) == w4.OK     # M = 0
