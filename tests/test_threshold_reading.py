"""The prefill quantisation kernel takes the outlier test |x| > t (t an fp32
threshold, AIInfra LLM.int8() section; tanjunchen section 1.2: a magnitude that
exceeds the threshold) as a comparison of fp16 values against h_t, the largest
fp16 value not above t. This checks that reading on every non-negative fp16
value for thresholds on, between and beyond fp16 values (no GPU needed); the GPU
parity tests check the kernel against the oracle's fp32 comparison."""
import numpy as np
import pytest


def largest_fp16_not_above(t: float) -> np.float16:
    if np.isinf(t):
        return np.float16(np.inf)
    fin = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)      # 0 .. 65504
    ok = fin.astype(np.float64) <= t
    return fin[np.nonzero(ok)[0][-1]]


ALL = np.arange(0, 0x7C01, dtype=np.uint16).view(np.float16)         # 0 .. +inf


@pytest.mark.parametrize("t", [0.0, 6.0, 6.001, 5.999, 1e-9, 2.0 ** -24, 2.0 ** -25, 0.5,
                               30.0, 65503.0, 65504.0, 65519.0, 65520.0, 70000.0, 1e30,
                               float("inf")])
def test_fp16_comparison_selects_the_fp32_set(t):
    ht = largest_fp16_not_above(t)
    by_fp32 = ALL.astype(np.float32) > np.float32(t)
    by_fp16 = ALL > ht
    assert np.array_equal(by_fp32, by_fp16)


def test_random_thresholds():
    rs = np.random.default_rng(7)
    for t in np.concatenate([rs.uniform(0, 100, 200), rs.uniform(0, 1e-4, 50),
                             rs.uniform(6e4, 7e4, 50)]).astype(np.float32):
        ht = largest_fp16_not_above(float(t))
        assert np.array_equal(ALL.astype(np.float32) > t, ALL > ht), t
