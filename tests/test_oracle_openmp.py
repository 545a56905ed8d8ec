"""The oracle's OpenMP timing build (the CPU baseline that bench.py reports)
must give exactly the plain build's results: its pragmas only share the
independent outer loops (rows, tokens, heads) among threads."""
import numpy as np

import oracle


def _run_all(rng_seed):
    rng = np.random.default_rng(rng_seed)
    n = 30011
    k = rng.integers(-127, 128, (n, 16, 128), dtype=np.int8)
    q = rng.integers(-127, 128, (16, 128), dtype=np.int8)
    q2 = rng.integers(-127, 128, (16, 128), dtype=np.int8)
    s = rng.uniform(0.5, 1.5, n).astype(np.float32)
    x = (rng.standard_normal((700, 512)) * 3).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    qa = (rng.standard_normal((64, 512)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    full = oracle.full_layer(q, k, s, n)
    top_r, ppos, sc = oracle.reindex_layer(q2, k, s, full["pool"], n)
    packed, sf = oracle.fp4_quantize(xb)
    att = oracle.sparse_attention(qa, lambda P: xb[P], np.arange(0, 700, 2), xb[:128], 700, 0, 512 ** -0.5)
    dots = oracle.index_dots(q, k[:5000])
    return [full["tok_score"], full["blk_score"], full["pool"], full["top"], top_r, sc, packed, sf, att, dots]


def test_openmp_build_matches_plain_build():
    try:
        oracle.use_openmp(False)
        plain = _run_all(5)
        threads = oracle.use_openmp(True)
        assert threads >= 1
        omp = _run_all(5)
    finally:
        oracle.use_openmp(False)
    assert oracle.num_threads() == 1
    for a, b in zip(plain, omp):
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_openmp_build_rejects_int32_overflow_like_plain_build():
    k = np.full((3, 140000), 127, np.int8)         # |S| up to 140000 * 16384 > 2^31
    k[1] = -128
    q = np.full(140000, -128, np.int8)
    try:
        for on in (False, True):
            oracle.use_openmp(on)
            try:
                oracle.index_scores(q, k, np.ones(3, np.float32))
                raise AssertionError("overflow not rejected")
            except OverflowError:
                pass
    finally:
        oracle.use_openmp(False)
