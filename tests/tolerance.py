"""Element-wise acceptance rule for BF16 outputs.

Pass rule: |got - ref| <= ulp_bf16(ref) + 1e-3, with
ulp_bf16(r) = 2**(floor(log2|r|) - 7) (one unit in the last place of a BF16
value of that magnitude; 0 for r == 0, leaving the 1e-3 floor).

Infinities match infinities of the same sign; any other non-finite value fails.

The stricter "relative 2**-8 plus 1e-3" reading is half an ulp to one ulp
depending on where |r| sits in its binade; an honest one-ulp flip between two
FP32 sums that differ only in their last bits fails it, so it is reported for
information and not enforced.
"""
import os
import sys

import numpy as np

ABS_FLOOR = 1e-3

# (test module, outputs compared, outside the rule, outside the strict form) of every
# assert_close call, summarised per module at the end of a pytest session
RECORD = []


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ulp_bf16(ref) -> np.ndarray:
    r = np.abs(np.asarray(ref, dtype=np.float64))
    out = np.zeros_like(r)
    nz = r > 0
    out[nz] = np.exp2(np.floor(np.log2(r[nz])) - 7)
    return out


def compare(got_bits, ref_bits) -> dict:
    got = bf16_bits_to_f64(got_bits)
    ref = bf16_bits_to_f64(ref_bits)
    if got.shape != ref.shape:
        raise AssertionError(f"shape {got.shape} != {ref.shape}")
    finite = np.isfinite(got) & np.isfinite(ref)
    same_inf = np.isinf(got) & np.isinf(ref) & (np.sign(got) == np.sign(ref))
    with np.errstate(invalid="ignore"):   # inf - inf where both are infinite: masked below
        d = np.where(finite, np.abs(got - ref), np.where(same_inf, 0.0, np.inf))
    tol = ulp_bf16(ref) + ABS_FLOOR
    bad = d > tol
    strict = d > (np.abs(ref) * 2.0 ** -8 + ABS_FLOOR)
    exact = np.asarray(got_bits, np.uint16) == np.asarray(ref_bits, np.uint16)
    return {
        "n": int(d.size),
        "fail": int(bad.sum()),
        "strict_fail": int(strict.sum()),
        "exact": int(exact.sum()),
        "max_abs": float(d.max()) if d.size else 0.0,
        "max_ratio": float((d / tol).max()) if d.size else 0.0,
        "first_bad": (np.argwhere(bad)[:5].tolist() if bad.any() else []),
    }


def assert_close(got_bits, ref_bits, what=""):
    r = compare(got_bits, ref_bits)
    caller = os.path.basename(sys._getframe(1).f_code.co_filename)
    RECORD.append((caller, r["n"], r["fail"], r["strict_fail"]))
    assert r["fail"] == 0, f"{what}: {r['fail']}/{r['n']} outside 1 ulp + 1e-3 ({r})"
    return r
