"""Pins that tie the CPU oracle to facts other than its own code.

Each function takes an ``oracle.Oracle`` (the real build, or a deliberately
broken copy in ``test_oracle_mutants.py``) and raises AssertionError when the
oracle disagrees with:

* hand-derived values stored under ``tests/golden/`` (unpacking of hand-built
  words, BF16 round-to-nearest-even ties, FP32 accumulation corner cases);
* closed forms (identity weights reproduce x; one-hot activations read single
  codes; all-ones activations give per-column sums of the dequantised weights);
* exact integer arithmetic (integer-valued inputs whose FP32 sums are exact);
* exact rational arithmetic on tiny random problems, within the FP32 error
  bound of recursive summation.

Expected values never come from the oracle or the CUDA library.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import w4a16_synth as synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def _expand(field):
    out = []
    for tok in field.split():
        if "*" in tok:
            v, r = tok.split("*")
            out += [int(v, 0)] * int(r)
        else:
            out.append(int(tok, 0))
    return out


def _bits_to_fraction(bits: int) -> Fraction:
    """Exact value of a BF16 bit pattern (finite only)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    assert e != 0xFF, "non-finite input"
    if e == 0:
        return sign * Fraction(m, 1 << 133)          # m * 2^-133
    return sign * Fraction(128 + m, 128) * Fraction(2) ** (e - 127)


def _f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32)


# ---------------------------------------------------------------- unpacking

def pin_unpack_hand_words(orc):
    words, codes = [], []
    for line in _golden_lines("unpack_words.txt"):
        tok = line.split()
        words.append(int(tok[0], 16))
        codes.append([int(t) for t in tok[1:9]])
    wq = np.array(words, dtype=np.uint32).reshape(len(words), 1)
    got = orc.unpack(wq, 8)
    assert np.array_equal(got, np.array(codes, dtype=np.uint8)), (got, codes)


def pin_onehot_reads_codes(orc):
    """x[m] = e_{k_m}, scale 1, bias 0  =>  y[m, n] = q[n, k_m] exactly."""
    rng = np.random.default_rng(11)
    M, N, K = 6, 40, 384
    q = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    ks = rng.choice(K, size=M, replace=False)
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), ks] = 1.0
    G = K // 128
    y = orc.matmul(synth.bf16_bits(x), synth.pack_nibbles(q),
                   synth.bf16_bits(np.ones((N, G))), synth.bf16_bits(np.zeros((N, G))))
    expect = synth.bf16_bits(q[:, ks].T.astype(np.float32))
    assert np.array_equal(y, expect)


# ---------------------------------------------------------------- closed forms

def pin_identity_reproduces_x(orc):
    """N = K, q = identity, scale 1, bias 0  =>  y == x bit for bit."""
    rng = np.random.default_rng(12)
    K = 256
    M = 5
    x = synth.make_x(rng, M, K, outliers=True)
    q = np.eye(K, dtype=np.uint8)
    G = K // 128
    y = orc.matmul(x, synth.pack_nibbles(q), synth.bf16_bits(np.ones((K, G))),
                   synth.bf16_bits(np.zeros((K, G))))
    assert np.array_equal(y, x)


def pin_bias_only(orc):
    """All codes 0  =>  y[m,n] = sum_g b[n,g] * sum_{k in g} x[m,k] (integers: exact)."""
    rng = np.random.default_rng(13)
    M, N, K = 4, 9, 512
    G = K // 128
    xi = rng.integers(-3, 4, size=(M, K))
    bi = rng.integers(-5, 6, size=(N, G))
    si = rng.integers(1, 4, size=(N, G))
    xsum = xi.reshape(M, G, 128).sum(-1)                # [M, G]
    expect = xsum @ bi.T                                # [M, N]
    y = orc.matmul(synth.bf16_bits(xi.astype(np.float32)),
                   synth.pack_nibbles(np.zeros((N, K), np.uint8)),
                   synth.bf16_bits(si.astype(np.float32)), synth.bf16_bits(bi.astype(np.float32)))
    assert np.array_equal(y, synth.bf16_bits(expect.astype(np.float32)))


def pin_all_ones_column_sums(orc):
    """x = 1  =>  y[m,n] = sum_g (s[n,g] * sum_{k in g} q[n,k] + 128 * b[n,g])."""
    from tolerance import compare
    rng = np.random.default_rng(14)
    M, N, K = 3, 33, 1024
    G = K // 128
    q = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    s_bits = synth.bf16_bits(rng.uniform(0.001, 0.02, size=(N, G)))
    b_bits = synth.bf16_bits(rng.uniform(-0.06, 0.0, size=(N, G)))
    s = synth.bf16_to_f32(s_bits).astype(np.float64)
    b = synth.bf16_to_f32(b_bits).astype(np.float64)
    col = (s * q.reshape(N, G, 128).sum(-1) + 128.0 * b).sum(-1)      # [N] in float64
    expect = synth.bf16_bits(np.broadcast_to(col, (M, N)).astype(np.float32))
    y = orc.matmul(synth.bf16_bits(np.ones((M, K))), synth.pack_nibbles(q), s_bits, b_bits)
    r = compare(y, expect)
    assert r["fail"] == 0, r


# ---------------------------------------------------------------- exact integers

INTEGER_SHAPES = ((5, 24, 384), (1, 8, 128), (9, 17, 1024), (3, 1, 256), (2, 130, 640))


def pin_integer_exact(orc):
    """Integer inputs with exact FP32 sums: the accumulator equals int64
    arithmetic and the output is that integer rounded once to BF16."""
    for (M, N, K) in INTEGER_SHAPES:
        p = synth.make_integer_problem(M, N, K)
        G = K // 128
        w = (p["si"][:, :, None] * p["qi"].reshape(N, G, 128) + p["bi"][:, :, None]).reshape(N, K)
        expect = p["xi"] @ w.T
        assert np.abs(expect).max() < 2 ** 24          # every FP32 partial sum is exact
        y = orc.matmul(p["x"], p["wq"], p["scales"], p["biases"])
        assert np.array_equal(y, synth.bf16_bits(expect.astype(np.float32))), (M, N, K)
        acc = orc.matmul_f32(p["x"], p["wq"], p["scales"], p["biases"])
        assert np.array_equal(acc, expect.astype(np.float32)), (M, N, K)


# ---------------------------------------------------------------- rounding and accumulation

def pin_bf16_rounding(orc):
    f, e = [], []
    for line in _golden_lines("bf16_rounding.txt"):
        tok = line.split()
        f.append(int(tok[0], 16))
        e.append(int(tok[1], 16))
    a = np.array(f, dtype=np.uint32).view(np.float32)
    assert np.array_equal(orc.round_bf16(a), np.array(e, dtype=np.uint16))


def pin_matmul_golden_cases(orc):
    for line in _golden_lines("matmul_cases.txt"):
        name, xs, qs, sb, bb, acc_bits, y_bits = [t.strip() for t in line.split("|")]
        K = 128
        x = np.zeros((1, K), np.uint16)
        xv = _expand(xs)
        x[0, :len(xv)] = xv
        q = np.zeros((1, K), np.uint8)
        qv = _expand(qs)
        q[0, :len(qv)] = qv
        s = np.array([[int(sb, 0)]], np.uint16)
        b = np.array([[int(bb, 0)]], np.uint16)
        wq = synth.pack_nibbles(q)
        acc = orc.matmul_f32(x, wq, s, b)
        y = orc.matmul(x, wq, s, b)
        assert int(_f32_bits(acc)[0, 0]) == int(acc_bits, 0), (name, hex(int(_f32_bits(acc)[0, 0])))
        assert int(y[0, 0]) == int(y_bits, 0), (name, hex(int(y[0, 0])))


def pin_rational_brute_force(orc):
    """Tiny random problems against exact rational arithmetic.

    The FP32 accumulator must lie within the recursive-summation bound
    (K + 2) * 2^-24 * sum_k |x_k w_k| of the exact value (the dequantised
    weight itself carries one rounding, the product one, each sum one), and
    the BF16 output within one BF16 ulp of the exact value.
    """
    from tolerance import ulp_bf16
    u = Fraction(1, 1 << 24)
    for (M, N, K, seed) in ((2, 3, 128, 1), (3, 2, 256, 2), (1, 4, 256, 3)):
        rng = np.random.default_rng(seed)
        x = synth.make_x(rng, M, K, outliers=True)
        wq, s_bits, b_bits = synth.make_weights(rng, N, K)
        G = K // 128
        acc = orc.matmul_f32(x, wq, s_bits, b_bits)
        y = orc.matmul(x, wq, s_bits, b_bits)
        xf = [[_bits_to_fraction(int(v)) for v in row] for row in x]
        sf = [[_bits_to_fraction(int(v)) for v in row] for row in s_bits]
        bf = [[_bits_to_fraction(int(v)) for v in row] for row in b_bits]
        for n in range(N):
            w = []
            for k in range(K):
                code = (int(wq[n, k // 8]) >> (4 * (k % 8))) & 15
                w.append(sf[n][k // 128] * code + bf[n][k // 128])
            for m in range(M):
                terms = [xf[m][k] * w[k] for k in range(K)]
                exact = sum(terms, Fraction(0))
                bound = (K + 2) * u * sum(abs(t) for t in terms)
                err = abs(Fraction(float(acc[m, n])) - exact)
                assert err <= bound, (m, n, float(err), float(bound))
                ex = float(exact)
                yv = float(synth.bf16_to_f32(y[m:m + 1, n])[0])
                assert abs(yv - ex) <= float(ulp_bf16(np.array([ex]))[0]), (m, n, yv, ex)


def pin_rejects_bad_k(orc):
    x = np.zeros((1, 136), np.uint16)
    wq = np.zeros((1, 17), np.uint32)
    s = np.zeros((1, 1), np.uint16)
    try:
        orc.matmul(x, wq, s, s)
    except ValueError:
        return
    raise AssertionError("K % 128 != 0 was accepted")


# ------------------------------------------------------------------ quantiser pins
# The recipe of the reference problem's inputs (affine min/max per 128-group: scale =
# (max - min) / 15 and bias = min, both rounded to BF16 first, q = rint((w - bias) /
# scale) clamped to 0..15, packed low nibble first).

def _pack_codes(codes):
    """The packed format's words for a list of codes (eight per word, low nibble first)."""
    words = []
    for j in range(0, len(codes), 8):
        w = 0
        for i, c in enumerate(codes[j:j + 8]):
            w |= int(c) << (4 * i)
        words.append(w)
    return words


def pin_quantize_hand_group(orc):
    """v_k = 1 + (k % 16) / 8: min 1, max 2.875, step 1.875 / 15 = 0.125 exactly, so the
    scale is 0.125 (0x3E00), the bias 1.0 (0x3F80) and code k is k % 16."""
    v = np.array([1.0 + (k % 16) / 8.0 for k in range(128)], np.float32)
    expect_words = [0x76543210, 0xFEDCBA98] * 8
    for w in (v[None, :], synth.bf16_bits(v)[None, :]):     # FP32 and BF16 inputs (exact in both)
        wq, s, b = orc.quantize(w)
        assert int(s[0, 0]) == 0x3E00 and int(b[0, 0]) == 0x3F80, (hex(s[0, 0]), hex(b[0, 0]))
        assert [int(x) for x in wq[0]] == expect_words, [hex(int(x)) for x in wq[0]]


def pin_quantize_constant_group(orc):
    """A constant group: scale 0, bias = the value rounded to BF16, every code 0.  0.3 in
    FP32 is 0x3E99999A; its BF16 rounding is 0x3E9A (the dropped half 0x999A > 0x8000)."""
    wq, s, b = orc.quantize(np.full((1, 256), 0.3, np.float32))
    assert s.tolist() == [[0, 0]] and b.tolist() == [[0x3E9A, 0x3E9A]]
    assert not wq.any()


def pin_quantize_ties_to_even(orc):
    """min 0, max 15: scale 1, bias 0, and a code is the value rounded half to even."""
    v = np.full(128, 5.0, np.float32)
    vals = [0.0, 15.0, 2.5, 3.5, 14.5, 0.5, 1.5, 7.49, 12.5, 9.51]
    codes = [0, 15, 2, 4, 14, 0, 2, 7, 12, 10]
    v[:len(vals)] = vals
    wq, s, b = orc.quantize(v[None, :])
    assert int(s[0, 0]) == 0x3F80 and int(b[0, 0]) == 0
    expect = codes + [5] * (128 - len(codes))
    assert [int(x) for x in wq[0]] == _pack_codes(expect), [hex(int(x)) for x in wq[0]]


def pin_quantize_signed_zero(orc):
    """A zero minimum or maximum is taken as +0 whatever the order of -0 and +0."""
    v = np.linspace(0.0, 1.5, 128).astype(np.float32)
    a = v.copy(); a[0] = -0.0; a[1] = 0.0      # -0 first
    c = v.copy(); c[0] = 0.0; c[1] = -0.0      # +0 first
    d = -v[::-1].copy(); d[-1] = -0.0          # maximum -0
    wq, s, b = orc.quantize(np.stack([a, c]))
    assert b.tolist() == [[0], [0]], b
    assert np.array_equal(wq[0], wq[1]) and s[0, 0] == s[1, 0]
    d2 = d.copy(); d2[-1] = 0.0                # the same group with +0 as its maximum
    for x, y in zip(orc.quantize(d[None, :]), orc.quantize(d2[None, :])):
        assert np.array_equal(x, y)


def pin_quantize_matches_numpy_recipe(orc):
    """The recipe restated with numpy's IEEE float32 operations (w4a16_synth, an independent
    implementation) on N(0, 0.02) rows and on groups built to reach the clamps: values far
    from zero with a narrow range, so that the BF16 bias lies well away from the minimum
    ((w - bias) / scale outside 0..15 before the clamp), and steps that round up or down."""
    rng = np.random.default_rng([2024, 11])
    W = rng.standard_normal((48, 512)).astype(np.float32) * np.float32(0.02)
    off = np.float32(100.2) + rng.random((8, 128), dtype=np.float32)      # lo near 100.2, range < 1
    W[:8, :128] = off
    W[8:16, 128:256] = np.float32(-37.7) + np.float32(0.25) * rng.random((8, 128), dtype=np.float32)
    W[16:24, 256:384] = np.float32(3.0e-3) * rng.standard_normal((8, 128), dtype=np.float32) + np.float32(0.7)
    got = orc.quantize(W)
    ref = synth.quantize_w4_g128(W)
    for g, r, name in zip(got, ref, ("wq", "scales", "biases")):
        assert np.array_equal(g, r), name
    # the clamps were reached: some codes 0 and 15 in the offset groups
    q = (ref[0][:8, :16, None] >> (4 * np.arange(8, dtype=np.uint32))) & 15
    assert (q == 15).any() and (q == 0).any()


def pin_quantize_rejects_bad_k(orc):
    try:
        orc.quantize(np.zeros((1, 136), np.float32))
    except ValueError:
        return
    raise AssertionError("K % 128 != 0 was accepted")


# ------------------------------------------------------------------ fused gate/up pins
# h = bf16(silu(g) * u) over gate/up rows interleaved in blocks of 8.

def _gate_up_problem(gvals, uvals, K=128):
    """One x row of ones [1, K] and per output a gate row and an up row whose dot with x
    is the given integer: codes q and scale 1, so the sum is sum(q) + K * bias (exact)."""
    n2 = len(gvals)
    assert n2 % 8 == 0
    def rows(vals):
        q = np.zeros((n2, K), np.uint8)
        bias = np.zeros((n2, K // 128), np.float32)
        for j, v in enumerate(vals):
            base = int(np.floor(v / K))            # bias per element, the rest from the codes
            rest = int(v - base * K)
            assert 0 <= rest <= 15 * K
            q[j, :rest // 15] = 15
            q[j, rest // 15] = rest % 15 if rest // 15 < K else 0
            bias[j, :] = base
        return synth.pack_nibbles(q), synth.bf16_bits(np.ones((n2, K // 128), np.float32)), synth.bf16_bits(bias)
    gq, gs, gb = rows(gvals)
    uq, us, ub = rows(uvals)
    x = synth.bf16_bits(np.ones((1, K), np.float32))
    return x, synth.interleave_gate_up(gq, uq), synth.interleave_gate_up(gs, us), synth.interleave_gate_up(gb, ub)


def pin_gate_up_closed_forms(orc):
    """silu(0) = 0, so g = 0 gives +0 for any u; u = 0 gives +0 (g >= 0); for g >= 64,
    exp(-g) < 2^-92 and silu(g) = g in double, so h = bf16(g * u) exactly; for g <= -256,
    silu(g) * u is below the smallest BF16 subnormal and h is a zero of u's sign times g's."""
    g = [0, 0, 64, 100, 700, -256, -300, 5, 0, 64, 1000, 100, -1000, 3, 0, 0]
    u = [7, -3, 2, -5, 1, 9, -4, 0, 0, 1, 3, 100, 1, 0, 1, 1000]
    x, wq, s, b = _gate_up_problem(g, u)
    h = orc.gate_up(x, wq, s, b)[0]
    want = {0: 0x0000, 1: 0x8000, 7: 0x0000, 8: 0x0000, 13: 0x0000, 14: 0x0000, 15: 0x0000}
    for j, bits in want.items():
        assert int(h[j]) in (bits, bits ^ 0x8000) and _bits_to_fraction(int(h[j])) == 0, (j, hex(h[j]))
    for j in (2, 3, 4, 9, 10, 11):
        assert int(h[j]) == int(synth.bf16_bits(np.array([g[j] * u[j]], np.float32))[0]), (j, hex(h[j]))
    for j in (5, 6, 12):
        assert _bits_to_fraction(int(h[j])) == 0, (j, hex(h[j]))


def pin_gate_up_interleave(orc):
    """The fused op reads gate j from row 16 (j / 8) + j % 8 and up j eight rows later: with
    u = 1 and g >= 64 on every output, h is the gate layer's own output, column by column."""
    rng = np.random.default_rng([77, 1])
    g = [int(v) for v in rng.integers(64, 1900, 24)]
    x, wq, s, b = _gate_up_problem(g, [1] * 24)
    h = orc.gate_up(x, wq, s, b)[0]
    assert [int(v) for v in h] == [int(v) for v in synth.bf16_bits(np.array(g, np.float32))]


def pin_gate_up_odd_part(orc):
    """silu(g) - silu(-g) = g: for u = 1 the outputs of g and -g differ by g up to the two
    BF16 roundings (half an ulp of each output)."""
    gs = [1, 2, 3, 5, 8, 13, 21, 34]
    g = gs + [-v for v in gs]
    x, wq, s, b = _gate_up_problem(g, [1] * 16)
    h = orc.gate_up(x, wq, s, b)[0]
    for j, v in enumerate(gs):
        hp, hn = _bits_to_fraction(int(h[j])), _bits_to_fraction(int(h[j + 8]))
        tol = (abs(hp) + abs(hn)) / 256 + Fraction(1, 1 << 20)
        assert abs(hp - hn - v) <= tol, (v, float(hp), float(hn))


# ---------------------------------------------------------------- other bit widths
# The affine format with b-bit codes: 32 / b codes per uint32, the lowest code in the
# lowest bits; dequantisation and accumulation as for 4 bits.

def pin_bits_unpack_hand_words(orc):
    """Hand-built words: 0xE4 holds the 2-bit codes 0, 1, 2, 3 (low first), 0x1B holds
    3, 2, 1, 0; 0x03020100 holds the bytes 0, 1, 2, 3; rows are words apart."""
    wq2 = np.array([[0xE4E4E4E4, 0x0000001B], [0xFFFFFFFF, 0x00000000]], np.uint32)
    want2 = np.array([[0, 1, 2, 3] * 4 + [3, 2, 1, 0] + [0] * 12, [3] * 16 + [0] * 16], np.uint8)
    assert np.array_equal(orc.unpack_bits(wq2, 32, 2), want2)
    wq8 = np.array([[0x03020100, 0xFF80017F], [0x00000010, 0x20000000]], np.uint32)
    want8 = np.array([[0, 1, 2, 3, 0x7F, 0x01, 0x80, 0xFF], [0x10, 0, 0, 0, 0, 0, 0, 0x20]], np.uint8)
    assert np.array_equal(orc.unpack_bits(wq8, 8, 8), want8)
    # four bits read the nibble layout of the 4-bit format
    assert np.array_equal(orc.unpack_bits(np.array([[0x76543210]], np.uint32), 8, 4), [[0, 1, 2, 3, 4, 5, 6, 7]])


def pin_bits_onehot_reads_codes(orc):
    """x = e_k, scale 1, bias 0: y[n] is the code of (n, k), for every k of two groups."""
    for bits in (2, 8):
        N, K = 3, 256
        top = (1 << bits) - 1
        q = (np.arange(N * K).reshape(N, K) * 37 + 11) % (top + 1)
        wq = synth.pack_codes(q.astype(np.uint8), bits)
        s = synth.bf16_bits(np.ones((N, 2), np.float32))
        b = np.zeros((N, 2), np.uint16)
        x = synth.bf16_bits(np.eye(K, dtype=np.float32))
        y = synth.bf16_to_f32(orc.matmul_bits(x, wq, s, b, bits))
        assert np.array_equal(y, q.T.astype(np.float32)), bits


def pin_bits_integer_exact(orc):
    """Integer inputs whose FP32 sums are exact: the output is the int64 result rounded once."""
    for bits, shapes in ((2, ((5, 24, 384), (1, 8, 1024), (3, 17, 128))), (8, ((5, 24, 256), (2, 9, 128)))):
        for (M, N, K) in shapes:
            p = synth.make_integer_problem_bits(M, N, K, bits)
            G = K // 128
            w = (p["si"][:, :, None] * p["qi"].reshape(N, G, 128) + p["bi"][:, :, None]).reshape(N, K)
            expect = p["xi"] @ w.T
            assert np.abs(expect).max() < 2 ** 24
            y = orc.matmul_bits(p["x"], p["wq"], p["scales"], p["biases"], bits)
            assert np.array_equal(y, synth.bf16_bits(expect.astype(np.float32))), (bits, M, N, K)


def pin_bits_rational_brute_force(orc):
    """Tiny random problems of both widths against exact rationals: the BF16 output within
    one BF16 ulp plus the FP32 recursive-summation bound of the exact value."""
    from tolerance import ulp_bf16
    u = Fraction(1, 1 << 24)
    for (bits, M, N, K, seed) in ((2, 2, 3, 256, 4), (8, 2, 3, 256, 5), (8, 1, 2, 128, 6)):
        p = synth.make_problem_bits(M, N, K, bits, seed=seed, outliers=True)
        y = orc.matmul_bits(p["x"], p["wq"], p["scales"], p["biases"], bits)
        xf = [[_bits_to_fraction(int(v)) for v in row] for row in p["x"]]
        sf = [[_bits_to_fraction(int(v)) for v in row] for row in p["scales"]]
        bf = [[_bits_to_fraction(int(v)) for v in row] for row in p["biases"]]
        per = 32 // bits
        for n in range(N):
            w = [sf[n][k // 128] * ((int(p["wq"][n, k // per]) >> (bits * (k % per))) & ((1 << bits) - 1))
                 + bf[n][k // 128] for k in range(K)]
            for m in range(M):
                terms = [xf[m][k] * w[k] for k in range(K)]
                exact = sum(terms, Fraction(0))
                slack = float((K + 2) * u * sum(abs(t) for t in terms))
                ex = float(exact)
                yv = float(synth.bf16_to_f32(y[m:m + 1, n])[0])
                assert abs(yv - ex) <= float(ulp_bf16(np.array([ex]))[0]) + slack, (bits, m, n, yv, ex)


def pin_bits_fp32_sequential_sum(orc):
    """Every code 1, scale 1, bias 0, x = (1, 2^-24 x 126, -1): in FP32 taken in ascending k
    each 2^-24 meets 1.0 at a tie and is lost (ties to even), so the sum is exactly 0; the
    exact sum (or one in FP64, or one taken from the top) is 126 x 2^-24."""
    K = 128
    x = np.array([[1.0] + [2.0 ** -24] * 126 + [-1.0]], np.float32)
    s = synth.bf16_bits(np.ones((1, 1), np.float32))
    b = np.zeros((1, 1), np.uint16)
    for bits in (2, 8):
        wq = synth.pack_codes(np.ones((1, K), np.uint8), bits)
        y = orc.matmul_bits(synth.bf16_bits(x), wq, s, b, bits)
        assert int(y[0, 0]) == 0x0000, (bits, hex(int(y[0, 0])))


def pin_bits_four_is_the_w4_layer(orc):
    """bits = 4 is the 4-bit layer itself (pinned above) on the same words."""
    p = synth.make_problem(3, 40, 384, seed=9)
    assert np.array_equal(orc.matmul_bits(p["x"], p["wq"], p["scales"], p["biases"], 4),
                          orc.matmul(p["x"], p["wq"], p["scales"], p["biases"]))


def pin_bits_rejects_bad_arguments(orc):
    x = np.zeros((1, 128), np.uint16)
    s = np.zeros((1, 1), np.uint16)
    for bits, words in ((3, 12), (16, 64), (1, 4)):
        try:
            orc.matmul_bits(x, np.zeros((1, words), np.uint32), s, s, bits)
        except ValueError:
            continue
        raise AssertionError(f"bits={bits} was accepted")
    try:
        orc.matmul_bits(np.zeros((1, 136), np.uint16), np.zeros((1, 34), np.uint32), s, s, 8)
    except ValueError:
        return
    raise AssertionError("K % 128 != 0 was accepted")


ALL_PINS = (
    pin_unpack_hand_words,
    pin_onehot_reads_codes,
    pin_identity_reproduces_x,
    pin_bias_only,
    pin_all_ones_column_sums,
    pin_integer_exact,
    pin_bf16_rounding,
    pin_matmul_golden_cases,
    pin_rational_brute_force,
    pin_rejects_bad_k,
    pin_quantize_hand_group,
    pin_quantize_constant_group,
    pin_quantize_ties_to_even,
    pin_quantize_signed_zero,
    pin_quantize_matches_numpy_recipe,
    pin_quantize_rejects_bad_k,
    pin_gate_up_closed_forms,
    pin_gate_up_interleave,
    pin_gate_up_odd_part,
    pin_bits_unpack_hand_words,
    pin_bits_onehot_reads_codes,
    pin_bits_integer_exact,
    pin_bits_fp32_sequential_sum,
    pin_bits_rational_brute_force,
    pin_bits_four_is_the_w4_layer,
    pin_bits_rejects_bad_arguments,
)


def run_all(orc) -> list[str]:
    """Run every pin; return the names of those that failed."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


if __name__ == "__main__":
    # used by the mutation test: run the pins against the library given on argv
    import sys
    from oracle import Oracle
    bad = run_all(Oracle(sys.argv[1]))
    print("FAILED:" + ",".join(bad))
    sys.exit(1 if bad else 0)
