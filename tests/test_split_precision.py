"""The index scores are three FP16 tensor-core products of the pooled means
split into hi + lo after a power-of-two scale (per query block for Q̄, per KV
head for K̄).  This checks, in NumPy, the precision that choice gives: the
split carries about 22 bits, the three-product score is within 2^-19 of
|q||k| of the exact dot product (2^-23 on these draws: far inside the 1e-4
near-tie rule), and a single hi*hi product is not (2^-13 on these draws).
It restates the arithmetic of the split, not the kernels, and imports neither
the library nor the oracle."""

import numpy as np


def pow2_scale(amax: float) -> float:
    # 2^a with max|x| 2^a in [2^13, 2^14)
    if not amax > 0:
        return 1.0
    _, e = np.frexp(amax)
    return float(2.0 ** (14 - int(e)))


def split(x32: np.ndarray, scale: float):
    xs = (x32.astype(np.float32) * np.float32(scale)).astype(np.float32)
    hi = xs.astype(np.float16)
    lo = (xs - hi.astype(np.float32)).astype(np.float16)
    return hi, lo


def three_products(qh, ql, kh, kl):
    f = lambda a, b: (a.astype(np.float32) * b.astype(np.float32)).astype(np.float32)
    s = np.float32(0)
    terms = f(qh, kh) + f(qh, kl) + f(ql, kh)
    for t in terms:          # fp32 accumulation
        s = np.float32(s + t)
    return float(s)


def pooled(rng, shape, mag):
    # means of 64 bf16-rounded values, as the pooling kernels see them
    x = (rng.standard_normal(shape + (64,)) * mag).astype(np.float32)
    xb = (x.view(np.uint32) + 0x8000 & 0xFFFF0000).view(np.float32)   # round to bf16 (ties away; fine here)
    return xb.mean(-1, dtype=np.float64).astype(np.float32)


def test_split_carries_about_22_bits():
    rng = np.random.default_rng(1)
    for mag in (1e-3, 1.0, 300.0):
        x = pooled(rng, (4, 128), mag)
        sc = pow2_scale(float(np.abs(x).max()))
        hi, lo = split(x, sc)
        back = (hi.astype(np.float64) + lo.astype(np.float64)) / sc
        rel = np.abs(back - x) / np.abs(x).max()
        assert rel.max() < 2.0 ** -21, (mag, rel.max())


def test_three_product_scores_are_fp32_accurate_and_one_product_is_not():
    rng = np.random.default_rng(2)
    worst3 = worst1 = 0.0
    for mag_q, mag_k in ((1.0, 1.0), (1e-3, 50.0), (200.0, 0.01)):
        q = pooled(rng, (16, 128), mag_q)
        k = pooled(rng, (32, 128), mag_k)
        sq = [pow2_scale(float(np.abs(row).max())) for row in q]    # per query block
        sk = pow2_scale(float(np.abs(k).max()))                     # per KV head
        for i in range(q.shape[0]):
            qh, ql = split(q[i], sq[i])
            for j in range(k.shape[0]):
                kh, kl = split(k[j], sk)
                exact = float(np.dot(q[i].astype(np.float64), k[j].astype(np.float64)))
                norm = float(np.linalg.norm(q[i]) * np.linalg.norm(k[j]))
                s3 = three_products(qh, ql, kh, kl) / (sq[i] * sk)
                s1 = float(np.dot(qh.astype(np.float64), kh.astype(np.float64))) / (sq[i] * sk)
                worst3 = max(worst3, abs(s3 - exact) / norm)
                worst1 = max(worst1, abs(s1 - exact) / norm)
    assert worst3 < 2.0 ** -19, worst3
    assert worst1 > 2.0 ** -14, worst1     # one product alone would blur scores at the 1e-4 rule's scale


def test_scale_puts_the_row_maximum_in_range():
    for amax in (3e-7, 1e-3, 0.7, 1.0, 5e3, 6e4):
        sc = pow2_scale(amax)
        assert 2.0 ** 13 <= amax * sc < 2.0 ** 14
        assert np.isfinite(np.float16(amax * sc))
