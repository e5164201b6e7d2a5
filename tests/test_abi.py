"""Host-side checks of the C ABI that need no GPU: every symbol the header
declares is exported, argument validation returns its status before touching
memory or CUDA, and the launch planning / stream-K bookkeeping are consistent."""
import ctypes
import os
import re

import pytest

import decode_w4a16_g128_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")
lib = w4.lib
P = ctypes.c_void_p


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a16_[a-z_0-9]+)\s*\(", text)))


def test_header_symbols_exported():
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/w4a16.h but not exported"


def test_version_and_strings():
    assert w4.w4a16_version() >= 100
    for code in range(8):
        assert w4.status_string(code)
    assert w4.status_string(99) == "unknown status"


def mm(x, wq, s, b, y, M, N, K):
    return lib.w4a16_matmul(P(x), P(wq), P(s), P(b), P(y), M, N, K, P(0))


A = 0x10000  # a 16-byte aligned address that is never dereferenced: validation fails first


@pytest.mark.parametrize("M,N,K,status", [
    (-1, 8, 128, w4.ERR_INVALID_ARG),
    (1, -8, 128, w4.ERR_INVALID_ARG),
    (1, 8, -128, w4.ERR_INVALID_ARG),
    (1, 8, 100, w4.ERR_UNSUPPORTED),
    (1, 8, 136, w4.ERR_UNSUPPORTED),
    (1, 2 ** 31, 128, w4.ERR_UNSUPPORTED),
])
def test_bad_sizes(M, N, K, status):
    assert mm(A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000, M, N, K) == status


def test_empty_outputs_need_no_gpu():
    assert mm(0, 0, 0, 0, 0, 0, 8, 128) == w4.OK
    assert mm(0, 0, 0, 0, 0, 4, 0, 128) == w4.OK


def test_null_and_misaligned_pointers():
    good = [A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000]
    for i in range(5):
        args = list(good)
        args[i] = 0
        assert mm(*args, 2, 8, 256) == w4.ERR_INVALID_ARG
        args = list(good)
        args[i] += 8
        assert mm(*args, 2, 8, 256) == w4.ERR_MISALIGNED


def test_output_overlapping_input_is_rejected():
    # y placed inside x
    assert mm(A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x100, 4, 8, 256) == w4.ERR_INVALID_ARG


def test_last_rows_argument_checks():
    f = lib.w4a16_matmul_last_rows
    args = (P(A), P(A + 0x100000), P(A + 0x200000), P(A + 0x300000), P(A + 0x400000))
    assert f(*args, 4, 5, 8, 256, P(0)) == w4.ERR_INVALID_ARG     # keep > M
    assert f(*args, 4, -1, 8, 256, P(0)) == w4.ERR_INVALID_ARG    # keep < 0
    assert f(*args, 0, 0, 8, 256, P(0)) == w4.OK                  # nothing to do


def test_bad_options():
    opt = w4.make_options(path=7)
    assert lib.w4a16_matmul_ex(P(A), P(A + 0x100000), P(A + 0x200000), P(A + 0x300000),
                               P(A + 0x400000), 2, 8, 256, P(0), ctypes.byref(opt)) == w4.ERR_INVALID_ARG
    opt = w4.make_options(path=w4.PATH_MATVEC)
    assert lib.w4a16_matmul_ex(P(A), P(A + 0x100000), P(A + 0x200000), P(A + 0x300000),
                               P(A + 0x400000), 9, 8, 256, P(0), ctypes.byref(opt)) == w4.ERR_UNSUPPORTED
    for splits in (9, 17):   # above every path's K-split limit
        opt = w4.make_options(splits=splits)
        assert lib.w4a16_matmul_ex(P(A), P(A + 0x100000), P(A + 0x200000), P(A + 0x300000),
                                   P(A + 0x400000), 2, 8, 256, P(0), ctypes.byref(opt)) == w4.ERR_INVALID_ARG


def test_row_block_split_limit():
    """The row-block matvec splits K over at most 4 CTAs of a cluster (the GEMM over up to 8 pairs)."""
    for splits in range(5, 9):
        with pytest.raises(w4.W4A16Error) as e:
            w4.w4a16_plan(2, 4096, 2560, path=w4.PATH_MATVEC_ROWS, splits=splits, sm_count=148)
        assert e.value.status == w4.ERR_UNSUPPORTED


def test_dispatch_rule():
    """M <= 8 streams weights through a matvec (the row-block one where a CTA's whole rows
    fit, the stream-K one otherwise); 8 < M <= 16 takes two slices of the row-block matvec
    where it fits (the measured crossover against the GEMM), larger M the tensor-core GEMM."""
    for M in range(1, 9):
        pl = w4.w4a16_plan(M, 4096, 2560, sm_count=148)
        assert pl["path"] == w4.PATH_MATVEC_ROWS and pl["slices"] == 1
        assert w4.w4a16_plan(M, 151936, 2560, sm_count=148)["path"] == w4.PATH_MATVEC
        assert w4.w4a16_plan(M, 4096, 2560, sm_count=148, workers=64)["path"] == w4.PATH_MATVEC
    for M in range(9, 17):
        pl = w4.w4a16_plan(M, 4096, 2560, sm_count=148)
        assert pl["path"] == w4.PATH_MATVEC_ROWS and pl["slices"] == 2
        assert w4.w4a16_plan(M, 151936, 2560, sm_count=148)["path"] == w4.PATH_GEMM   # rows do not fit
        assert w4.w4a16_plan(M, 4096, 2560, sm_count=148, splits=2)["path"] == w4.PATH_GEMM
    for M in (17, 32, 33, 128):
        assert w4.w4a16_plan(M, 4096, 2560, sm_count=148)["path"] == w4.PATH_GEMM
        assert w4.w4a16_plan(M, 4096, 2560, sm_count=148)["slices"] == 0


def test_row_block_slices():
    """The row-block path runs ceil(M / 8) slices of 8 x rows, up to M = 32."""
    for M, sl in ((9, 2), (24, 3), (25, 4), (32, 4)):
        pl = w4.w4a16_plan(M, 2560, 9728, path=w4.PATH_MATVEC_ROWS, sm_count=148)
        assert pl["path"] == w4.PATH_MATVEC_ROWS and pl["slices"] == sl
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_plan(33, 2560, 9728, path=w4.PATH_MATVEC_ROWS, sm_count=148)
    assert e.value.status == w4.ERR_UNSUPPORTED


def rows_smem(hb, gcl, s):
    """Shared memory of a row-block CTA: codes of hb half blocks (8 rows) per group plus 512 B
    of slack (or the warps' partial sums if larger), scales, biases, the cluster's partial sums
    (own + ranks 1..S-1 on rank 0 when split), barriers, alignment slack."""
    rb = (hb + 1) // 2
    work = max(512 * hb * gcl + 512, 4096 * rb)
    sb = (32 * rb * gcl + 15) // 16 * 16
    part = 512 * rb * s if s > 1 else 0
    return work + 2 * sb + part + 8 * (gcl + 2) + 128


@pytest.mark.parametrize("N,K,splits", [(1024, 2560, 2), (4096, 2560, 1), (2560, 4096, 1), (9728, 2560, 1),
                                        (2560, 9728, 2), (1000, 256, 2), (8, 128, 1), (1, 128, 1)])
def test_rows_plan(N, K, splits):
    """Row-block matvec: one CTA per SM (padded with CTAs that own no rows), the 8-row half
    blocks spread evenly over the clusters of `splits` CTAs, at most 5 MMA row blocks of 16
    rows per cluster, shared memory that leaves room for a second CTA on the SM."""
    pl = w4.w4a16_plan(1, N, K, sm_count=148)
    assert pl["path"] == w4.PATH_MATVEC_ROWS
    assert pl["block"] == 256            # 8 warps, all computing
    assert pl["splits"] == pl["cluster"] == splits
    nh, G = -(-N // 8), K // 128
    assert pl["units"] == nh             # 8-row half blocks
    assert pl["tiles"] == min(148 // splits, nh)
    assert pl["grid_x"] == (148 // splits) * splits
    hb = -(-nh // pl["tiles"])
    assert pl["row_blocks"] == (hb + 1) // 2 <= 5
    assert pl["smem_bytes"] == rows_smem(hb, -(-G // splits), splits)
    assert 2 * (pl["smem_bytes"] + 1024) <= 233472
    assert pl["workspace_bytes"] == 0


def test_rows_plan_limits():
    # the vocabulary projection does not fit two CTAs per SM: stream-K there
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_plan(1, 151936, 2560, path=w4.PATH_MATVEC_ROWS, sm_count=148)
    assert e.value.status == w4.ERR_UNSUPPORTED
    with pytest.raises(w4.W4A16Error) as e:   # at most four slices of 8 x rows
        w4.w4a16_plan(33, 4096, 2560, path=w4.PATH_MATVEC_ROWS, sm_count=148)
    assert e.value.status == w4.ERR_UNSUPPORTED
    # K = 9728 without a split would need 2 row blocks x 76 groups: more than half an SM
    assert rows_smem(4, 76, 1) > 115712 >= rows_smem(5, 38, 2)
    # every plan the rule produces: one CTA per SM, the fewest splits that fit with enough
    # work per warp (at least 4 units of 16 rows x one group), else 2, else the fewest that fit
    for N in (8, 100, 1000, 2560, 4096, 9728, 20000):
        for K in (128, 256, 2560, 4096, 9728, 16384):
            try:
                pl = w4.w4a16_plan(1, N, K, path=w4.PATH_MATVEC_ROWS, sm_count=148)
            except w4.W4A16Error:
                continue
            nh, G, s = -(-N // 8), K // 128, pl["splits"]
            fits = {}
            for t in (1, 2, 4):
                if t > G:
                    continue
                cl = min(148 // t, nh)
                hb = -(-nh // cl)
                if (hb + 1) // 2 <= 5 and rows_smem(hb, -(-G // t), t) <= 115712:
                    fits[t] = ((hb + 1) // 2) * (-(-G // t)) // 8
            enough = [t for t in sorted(fits) if fits[t] >= 4]
            want = enough[0] if enough else (2 if 2 in fits else min(fits))
            assert s == want, (N, K, fits, s)
            assert pl["grid_x"] == (148 // s) * s


def test_rows_forced_launch():
    """row_blocks and splits together fix the launch (tests and sweeps use it)."""
    pl = w4.w4a16_plan(1, 9728, 2560, path=w4.PATH_MATVEC_ROWS, sm_count=148, splits=1, row_blocks=2)
    assert pl["tiles"] == -(-(9728 // 8) // 4) and pl["row_blocks"] == 2 and pl["splits"] == 1
    assert pl["grid_x"] == pl["tiles"]   # more clusters than SMs: no padding
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_plan(1, 9728, 2560, path=w4.PATH_MATVEC_ROWS, sm_count=148, row_blocks=6)
    assert e.value.status == w4.ERR_INVALID_ARG


@pytest.mark.parametrize("N,K", [(1024, 2560), (4096, 2560), (2560, 4096), (9728, 2560), (2560, 9728),
                                 (151936, 2560), (1000, 256), (8, 128)])
def test_matvec_plan(N, K):
    pl = w4.w4a16_plan(1, N, K, path=w4.PATH_MATVEC, sm_count=148)
    assert pl["block"] == 672   # producer warp, 4 x-preparation warps, 16 consumer warps
    assert pl["tiles"] == -(-N // 256)   # 16 consumer warps x 16 rows
    assert pl["units"] == pl["tiles"] * (K // 128)
    assert 1 <= pl["grid_x"] <= min(148, pl["units"])
    assert pl["smem_bytes"] <= 227 * 1024


def test_streamk_owner_matches_brute_force():
    for U in list(range(1, 40)) + [640, 1520, 23740]:
        for Pw in sorted({1, 2, 3, 7, 37, 148, U}):
            if Pw > U:
                continue
            owner = []
            for c in range(Pw):
                owner += [c] * ((c + 1) * U // Pw - c * U // Pw)
            assert len(owner) == U
            for u in range(0, U, max(1, U // 97)):
                assert w4.w4a16_streamk_owner(U, Pw, u) == owner[u], (U, Pw, u)
    assert w4.w4a16_streamk_owner(10, 11, 0) == -1
    assert w4.w4a16_streamk_owner(10, 2, 10) == -1


@pytest.mark.parametrize("M,N,K,expect_splits", [(128, 4096, 2560, 4), (128, 1024, 2560, 8), (128, 2560, 9728, 4),
                                                 (128, 9728, 2560, 1), (2048, 4096, 2560, 1), (32, 64, 256, 1),
                                                 (509, 4096, 9728, 1), (129, 1000, 9728, 4), (128, 2560, 4096, 4)])
def test_gemm_split_plan(M, N, K, expect_splits):
    """Tiles of 256 weight rows x 128 x rows, each on a CTA pair; K is split only while
    the pairs leave SMs idle (above 4 splits only while the grid stays within half of the
    SMs), and a tile's splits form one cluster of 2 x splits CTAs.
    Without a split the grid is persistent: one pair per two SMs, looping over the tiles."""
    pl = w4.w4a16_plan(M, N, K, sm_count=148)
    assert pl["path"] == w4.PATH_GEMM
    assert pl["splits"] == expect_splits and pl["cluster"] == 2 * expect_splits
    tiles = -(-M // 128) * -(-N // 256)
    assert pl["tiles"] == tiles
    if expect_splits == 1:
        assert (pl["grid_x"], pl["grid_y"], pl["grid_z"]) == (2, min(tiles, 74), 1)
    else:
        assert pl["grid_x"] * pl["grid_y"] * pl["grid_z"] == 2 * tiles * expect_splits
    assert pl["splits"] <= 8 and pl["splits"] <= K // 128
    assert pl["cluster"] <= 16


def test_gemm_forced_splits_plan():
    for s in range(1, 9):
        assert w4.w4a16_plan(300, 1000, 1024, path=w4.PATH_GEMM, splits=s, sm_count=148)["splits"] == s
    for s in (9, 16):   # a cluster holds at most 16 CTAs: 8 pairs
        with pytest.raises(w4.W4A16Error):
            w4.w4a16_plan(300, 1000, 1024, path=w4.PATH_GEMM, splits=s, sm_count=148)
    assert w4.w4a16_plan(300, 1000, 256, path=w4.PATH_GEMM, splits=4, sm_count=148)["splits"] == 2   # G = 2


def test_gemm_k_limit():
    """The tensor-core path stages each CTA's scales in shared memory: K <= 32768 there."""
    assert w4.w4a16_plan(128, 1000, 32768, sm_count=148)["path"] == w4.PATH_GEMM
    with pytest.raises(w4.W4A16Error) as e:
        w4.w4a16_plan(128, 1000, 32768 + 128, sm_count=148)
    assert e.value.status == w4.ERR_UNSUPPORTED
    assert w4.w4a16_plan(8, 1000, 32768 + 128, sm_count=148)["path"] == w4.PATH_MATVEC   # no limit there


@pytest.mark.parametrize("N,K,expect", [(1024, 2560, 40), (4096, 2560, 121), (2560, 4096, 121), (9728, 2560, 128),
                                        (2560, 9728, 128), (151936, 2560, 148), (64, 256, 1)])
def test_matvec_default_workers(N, K, expect):
    """Persistent CTAs of the matvec: fewer than the SMs for small and mid-size weights (the
    next call's CTAs start on the free SMs), every SM for the vocabulary projection."""
    pl = w4.w4a16_plan(1, N, K, path=w4.PATH_MATVEC, sm_count=148)
    assert pl["path"] == w4.PATH_MATVEC and pl["grid_x"] == expect
    assert w4.w4a16_plan(1, N, K, sm_count=148, workers=17)["grid_x"] == min(17, pl["units"])


def mmb(x, wq, s, b, y, M, N, K, bits):
    return lib.w4a16_matmul_bits(P(x), P(wq), P(s), P(b), P(y), M, N, K, bits, P(0))


def test_bits_argument_checks():
    good = [A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000]
    for bits in (2, 8):
        assert mmb(*good, -1, 8, 128, bits) == w4.ERR_INVALID_ARG
        assert mmb(*good, 1, 8, 136, bits) == w4.ERR_UNSUPPORTED
        assert mmb(*good, 33, 8, 128, bits) == w4.ERR_UNSUPPORTED       # decode only: M <= 32
        assert mmb(0, 0, 0, 0, 0, 0, 8, 128, bits) == w4.OK               # empty: no GPU needed
        assert mmb(0, 0, 0, 0, 0, 4, 0, 128, bits) == w4.OK
        for i in range(5):
            args = list(good)
            args[i] = 0
            assert mmb(*args, 2, 8, 256, bits) == w4.ERR_INVALID_ARG
            args = list(good)
            args[i] += 8
            assert mmb(*args, 2, 8, 256, bits) == w4.ERR_MISALIGNED
    for bits in (0, 1, 3, 5, 16, 32, -4):
        assert mmb(*good, 1, 8, 128, bits) == w4.ERR_UNSUPPORTED
    # y inside the codes: 8-bit codes of 64 rows x 1024 take 64 KB, 2-bit ones 16 KB
    assert mmb(A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x100000 + 0xC000, 1, 64, 1024, 8) == w4.ERR_INVALID_ARG
    # bits = 4 is the 4-bit layer's own validation
    assert mmb(*good, 1, 8, 136, 4) == w4.ERR_UNSUPPORTED
    assert mmb(0, 0, 0, 0, 0, 0, 8, 128, 4) == w4.OK
