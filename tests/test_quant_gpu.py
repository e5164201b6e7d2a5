"""The on-GPU quantiser against the CPU oracle's quantiser, bit for bit.

w4a16_quantize turns FP32 or BF16 weights into the packed format (codes, BF16 scales and
biases per 128-group) by the min/max recipe; every step is correctly rounded, so codes,
scales and biases must equal the oracle's exactly.  Inputs: N(0, 0.02) rows of the
Qwen3-4B projection shapes (FP32 and BF16), a ragged row count, the vocabulary projection
in BF16 (sampled rows), and groups built for the corners of the recipe: constant groups
(scale 0), signed zeros as minimum or maximum, groups far from zero with a narrow range
(the BF16 bias lies away from the minimum and the codes reach both clamps), ties of
(w - bias) / scale, and subnormal values.  Then the quantised weights go through the layer
and the result is compared with the oracle's layer on the oracle's quantisation.
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
from gpu_util import bits, oracle_y  # noqa: E402


def gpu_quantize(W):
    """numpy float32 values or uint16 BF16 bits -> the GPU's (wq, scales, biases) as numpy."""
    if W.dtype == np.uint16:
        t = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    wq, s, b = w4.w4a16_quantize(t)
    torch.cuda.synchronize()
    return wq.cpu().numpy().view(np.uint32), bits(s), bits(b)


def assert_same(got, ref, what):
    for g, r, name in zip(got, ref, ("codes", "scales", "biases")):
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)
            raise AssertionError(f"{what}: {name} differ at {len(bad)} places, first {bad[:4].tolist()}")


def edge_weights(rng, N=32, K=1024):
    """N(0, 0.02) rows with groups replaced by the recipe's corner cases."""
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    W[0, 0:128] = np.float32(0.3)                                     # constant: scale 0
    W[1, 128:256] = np.float32(-1.25)                                 # constant, negative
    v = np.linspace(0.0, 1.5, 128, dtype=np.float32)
    W[2, 0:128] = v; W[2, 0] = -0.0; W[2, 7] = 0.0                    # minimum -0 before +0
    W[3, 0:128] = v; W[3, 0] = 0.0; W[3, 7] = -0.0                    # +0 before -0
    W[4, 0:128] = -v[::-1]; W[4, 127] = -0.0                          # maximum -0
    W[5:13, 256:384] = np.float32(100.2) + rng.random((8, 128), dtype=np.float32)          # clamps
    W[13:21, 384:512] = np.float32(100.3) + np.float32(0.2) * rng.random((8, 128), dtype=np.float32)   # bias above the minimum
    W[25:29, 384:512] = np.float32(-37.7) + np.float32(0.25) * rng.random((4, 128), dtype=np.float32)
    t = np.full(128, 5.0, np.float32)                                 # ties: scale 1, bias 0
    t[:10] = [0.0, 15.0, 2.5, 3.5, 14.5, 0.5, 1.5, 7.49, 12.5, 9.51]
    W[21, 512:640] = t
    W[22, 640:768] = rng.standard_normal(128, dtype=np.float32) * np.float32(1e-39)   # subnormal
    W[23, 768:896] = np.float32(3e-38) + rng.random(128, dtype=np.float32) * np.float32(1e-39)
    W[24, 896:1024] = rng.standard_normal(128, dtype=np.float32) * np.float32(3e4)     # wide range
    # quotients at half-integers (ties), each scaled so that scale and bias stay exact
    for r, sc in ((29, 0.25), (30, 1.0 / 64), (31, 3.0)):
        base = np.arange(128, dtype=np.float32) % 31 * np.float32(0.5)   # 0, 0.5, ..., 15
        W[r, 0:128] = base * np.float32(sc)
    return W


@pytest.mark.parametrize("name,N,K", [("q", 4096, 2560), ("o", 2560, 4096), ("down", 2560, 9728),
                                      ("ragged", 1001, 384), ("one_row", 1, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_projections(name, N, K, dtype):
    rng = synth.shape_rng(7, N, K, seed=3)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    if dtype == "bf16":
        W = synth.bf16_bits(W)
    assert_same(gpu_quantize(W), oracle.quantize(W), f"{name} {dtype}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_edge_groups(dtype):
    W = edge_weights(np.random.default_rng([11, 5]))
    if dtype == "bf16":
        W = synth.bf16_bits(W)
    ref = oracle.quantize(W)
    assert_same(gpu_quantize(W), ref, f"edge groups {dtype}")
    # the corners were reached: scale 0, the upper clamp (BF16 bias below the minimum, large
    # codes past 15.5) and the lower one (BF16 bias above the minimum: negative quotients)
    assert (ref[1] == 0).any()
    shifts = 4 * np.arange(8, dtype=np.uint32)
    assert ((ref[0][5:13, 32:48, None] >> shifts) & 15 == 15).any()
    assert ((ref[0][13:21, 48:64, None] >> shifts) & 15 == 0).any()


def test_quantize_vocabulary_bf16_sampled_rows():
    """The vocabulary projection's weights (151936 x 2560) in BF16 on the GPU; the oracle
    quantises 200 sampled rows, first and last included."""
    N, K = 151936, 2560
    g = torch.Generator(device="cuda").manual_seed(5)
    Wt = (torch.randn((N, K), generator=g, device="cuda", dtype=torch.float32) * 0.02).to(torch.bfloat16)
    wq, s, b = w4.w4a16_quantize(Wt)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng([N, K]).choice(N, 198, replace=False)]))
    idx = torch.from_numpy(rows).cuda()
    Wr = bits(Wt.index_select(0, idx))
    ref = oracle.quantize(Wr)
    got = (wq.index_select(0, idx).cpu().numpy().view(np.uint32), bits(s.index_select(0, idx)),
           bits(b.index_select(0, idx)))
    assert_same(got, ref, "vocabulary rows")


def test_quantize_then_layer():
    """Quantise on the GPU, run the layer on the result: equal to the oracle's layer on the
    oracle's quantisation (same packed weights, so the usual layer tolerance)."""
    M, N, K = 8, 1000, 2560
    rng = synth.shape_rng(M, N, K, seed=9)
    x = synth.make_x(rng, M, K)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    wq, s, b = w4.w4a16_quantize(torch.from_numpy(W).cuda())
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y = w4.w4a16_matmul(xt, wq, s, b)
    torch.cuda.synchronize()
    owq, os_, ob = oracle.quantize(W)
    prob = {"x": x, "wq": owq, "scales": os_, "biases": ob}
    assert_close(bits(y), oracle_y(prob), "quantise then layer")


def test_quantize_arguments():
    W = torch.zeros((4, 256), device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_quantize(torch.zeros((4, 200), device="cuda"))
    assert e.value.status == w4.ERR_UNSUPPORTED
    buf = torch.zeros(4 * 256 + 1, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_quantize(buf[1:].view(4, 256))               # 4-byte offset: not 16-byte aligned
    assert e.value.status == w4.ERR_MISALIGNED
    P = w4.ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)
    assert w4.lib.w4a16_quantize(P(W.data_ptr()), 7, P(W.data_ptr()), P(W.data_ptr()), P(W.data_ptr()), 4, 256,
                                 stream) == w4.ERR_INVALID_ARG     # unknown dtype
    assert w4.lib.w4a16_quantize(P(W.data_ptr()), 0, P(W.data_ptr()), P(W.data_ptr() + 4096),
                                 P(W.data_ptr() + 4096 + 16), 4, 256, stream) == w4.ERR_INVALID_ARG   # overlap
    assert w4.lib.w4a16_quantize(P(0), 0, P(0), P(0), P(0), 0, 256, stream) == w4.OK                  # empty
