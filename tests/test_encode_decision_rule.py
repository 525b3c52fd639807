"""The bulk encoder's decision rule, checked on the CPU: a code taken from the fp32 rotation
is kept only when the fp32 value is farther from every threshold than the bound
2 (sqrt(d) (d + 1) + 8) 2^-24 (1 + |y| / sqrt(d)) + 1e-6; otherwise the fp64 value decides.
On adversarial inputs (rotated coordinates placed at 1e-7 .. 1e-3 from thresholds, large
and tiny norms, every group size) the rule must give exactly the fp64 codes, and the fp32
value must never stray from the fp64 one by more than the bound's error term."""
import math

import numpy as np
import pytest

import oracle as O


def _bound(d, y):
    return (2.0 * (math.sqrt(d) * (d + 1) + 8.0) * 2.0 ** -24 + 1e-6) * (1.0 + abs(y) / math.sqrt(d))


def _y32(rot32t, x32, i, norm):
    # the kernel's fp32 dot: two halves of the j range, each acc = fma(R[i][j], x_j, acc) in
    # j order, then added (numpy float32 rounds the product and the sum separately, a
    # looser computation than a fused multiply-add); then y = acc f with f = sqrt(d) / |x|
    # in fp32 (|x| from fp64, rounded to fp32)
    d = len(x32)
    half = []
    for j0, j1 in ((0, d // 2), (d // 2, d)):
        acc = np.float32(0.0)
        for j in range(j0, j1):
            acc = np.float32(acc + np.float32(rot32t[j, i] * x32[j]))
        half.append(acc)
    acc = np.float32(half[0] + half[1])
    f = np.float32(np.float32(math.sqrt(d)) / np.float32(norm))
    return float(np.float32(acc * f))


@pytest.mark.parametrize("d,rate", [(2, 1), (14, 3), (26, 4), (66, 1), (128, 2), (128, 4)])
def test_fp32_codes_with_fp64_fallback_equal_fp64_codes(d, rate):
    rng = np.random.default_rng(d * 10 + rate)
    rot = O.haar_rotation(11, rate, d)
    rot32t = rot.T.astype(np.float32)          # element (i, j) at [j, i]
    _, t, _ = O.lloyd_max(rate)
    fallbacks = 0
    for trial in range(60):
        # rotated target: most coordinates placed near thresholds, the norm closed by the rest
        y = rng.standard_normal(d)
        k = rng.integers(0, len(t), d)
        offs = rng.choice([1e-7, 1e-6, 5e-6, 3e-5, 1e-4, 1e-3], d) * rng.choice([-1, 1], d)
        near = rng.random(d) < 0.7
        y = np.where(near, t[k] + offs, y)
        y *= math.sqrt(d) / np.linalg.norm(y)
        scale = [1e-3, 1.0, 1e3][trial % 3]
        x = scale * (rot.T @ y) / math.sqrt(d)
        x32 = x.astype(np.float32)               # inputs are given in fp32 (or bf16 / fp16)
        x64 = x32.astype(np.float64)
        norm = float(np.sqrt(np.sum(x64 * x64)))
        ref = np.searchsorted(t, math.sqrt(d) * (x64 @ rot.T) / norm, side="right")
        for i in range(d):
            y32 = _y32(rot32t, x32, i, norm)
            y64 = math.sqrt(d) * float(rot[i] @ x64) / norm
            assert abs(y32 - y64) <= _bound(d, y32) / 2, (i, y32, y64)   # the rule's error term holds
            margin = float(np.min(np.abs(y32 - t.astype(np.float32).astype(np.float64))))
            if margin > _bound(d, y32):
                code = int(np.searchsorted(t.astype(np.float32).astype(np.float64), y32, side="right"))
            else:
                fallbacks += 1
                code = int(np.searchsorted(t, y64, side="right"))
            assert code == ref[i], (i, y32, y64)
    assert fallbacks > 0                         # the adversarial inputs did reach the fallback
