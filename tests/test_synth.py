"""The seeded input generator: packing order, quantiser properties, determinism."""
import numpy as np

import oracle_pins
import w4a16_synth as synth


def test_pack_matches_hand_words():
    words, codes = [], []
    for line in oracle_pins._golden_lines("unpack_words.txt"):
        tok = line.split()
        words.append(int(tok[0], 16))
        codes.append([int(t) for t in tok[1:9]])
    got = synth.pack_nibbles(np.array(codes, dtype=np.uint8))
    assert np.array_equal(got[:, 0], np.array(words, dtype=np.uint32))


def test_bf16_rounding_matches_golden():
    f, e = [], []
    for line in oracle_pins._golden_lines("bf16_rounding.txt"):
        tok = line.split()
        f.append(int(tok[0], 16))
        e.append(int(tok[1], 16))
    a = np.array(f, dtype=np.uint32).view(np.float32)
    assert np.array_equal(synth.bf16_bits(a), np.array(e, dtype=np.uint16))


def test_quantiser_reconstruction_error():
    rng = np.random.default_rng(5)
    N, K = 16, 512
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    wq, s_bits, b_bits = synth.quantize_w4_g128(W)
    q = np.empty((N, K), np.int64)
    for j in range(8):
        q[:, j::8] = (wq.astype(np.int64) >> (4 * j)) & 15
    s = np.repeat(synth.bf16_to_f32(s_bits).astype(np.float64), 128, axis=1)
    b = np.repeat(synth.bf16_to_f32(b_bits).astype(np.float64), 128, axis=1)
    err = np.abs(s * q + b - W)
    # half a step from the rounding of q, plus the BF16 rounding of scale and bias
    assert (err <= 0.5 * s + 16 * s * 2.0 ** -8 + np.abs(b) * 2.0 ** -8 + 1e-7).all()
    assert q.min() == 0 and q.max() == 15


def test_constant_group_gives_zero_scale():
    W = np.full((2, 256), 0.125, np.float32)
    W[1, 128:] = -3.0
    wq, s_bits, b_bits = synth.quantize_w4_g128(W)
    assert (s_bits == 0).all()
    assert (wq == 0).all()
    assert np.array_equal(synth.bf16_to_f32(b_bits), np.array([[0.125, 0.125], [0.125, -3.0]], np.float32))


def test_outliers_fraction():
    rng = np.random.default_rng(3)
    x = synth.bf16_to_f32(synth.make_x(rng, 64, 4096, outliers=True))
    big = (np.abs(x) > 6).mean()
    assert 0.004 < big < 0.02


def test_seeded_and_shape_dependent():
    a = synth.make_problem(3, 8, 256)
    b = synth.make_problem(3, 8, 256)
    c = synth.make_problem(3, 16, 256)
    for key in ("x", "wq", "scales", "biases"):
        assert np.array_equal(a[key], b[key])
    assert not np.array_equal(a["x"], c["x"])
    p = synth.make_pr1_problem()
    assert p["x"].shape == (32, 256) and p["wq"].shape == (64, 32) and p["scales"].shape == (64, 2)
