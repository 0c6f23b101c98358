"""The error bound the GPU tests use for the tensor-core block scores,
checked on the CPU against an emulation of that arithmetic.

The score kernel splits each fp32 pooled value x into tf32 parts hi = tf32(x),
lo = tf32(x - hi) (round to nearest, ties away from zero) and takes each term
as lo_k hi_q + hi_k lo_q + hi_k hi_q, in 32-wide chunks of d, each part of a
chunk as four MMA steps of eight products added to an fp32 accumulator. The
tests bound the score error by gamma * sum |q||k| with
gamma = (3 d / 8 + 3) * 2^-22. Here the steps are emulated with each step's
eight exact products summed exactly and the accumulator then truncated toward
zero (the worst rounding an fp32 accumulator could do), and the error against
the exact dot product of the fp32 inputs must stay within gamma * sum |q||k|.
"""
import numpy as np
import pytest


def tf32_rna(x):
    """fp32 -> nearest tf32 (10 explicit mantissa bits), ties away from zero."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x1000)) & np.uint32(0xFFFFE000)).view(np.float32)


def to_f32_toward_zero(v):
    """fp64 -> fp32, truncating toward zero."""
    f = np.float32(v)
    if abs(float(f)) > abs(v):
        f = np.nextafter(f, np.float32(0.0))
    return f


def emulated_score(q, k):
    """The kernel's product order over d, with a truncating accumulator."""
    qh = tf32_rna(q)
    ql = tf32_rna(q - qh)
    kh = tf32_rna(k)
    kl = tf32_rna(k - kh)
    acc = np.float32(0.0)
    d = q.size
    for c in range(d // 32):
        for a, b in ((kl, qh), (kh, ql), (kh, qh)):
            for s in range(4):
                lo = 32 * c + 8 * s
                step = float(np.sum(a[lo:lo + 8].astype(np.float64) * b[lo:lo + 8].astype(np.float64)))
                acc = to_f32_toward_zero(float(acc) + step)
    return float(acc)


def test_tf32_rounding_is_to_nearest_ties_away():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -10)
    assert tf32_rna(one + ulp * np.float32(0.49)) == one
    assert tf32_rna(one + ulp * np.float32(0.5)) == one + ulp  # tie goes away from zero
    assert tf32_rna(-(one + ulp * np.float32(0.5))) == -(one + ulp)
    x = np.float32(3.14159265)
    hi = tf32_rna(x)
    lo = tf32_rna(x - hi)
    assert abs(float(x) - float(hi) - float(lo)) <= 2.0 ** -22 * abs(float(x))


@pytest.mark.parametrize("d", [64, 128])
def test_tensor_core_score_error_within_the_stated_bound(d):
    rng = np.random.default_rng(d)
    gamma = (3 * d / 8 + 3) * 2.0 ** -22
    worst = 0.0
    for trial in range(300):
        # pooled means: mixed magnitudes and signs, some near-cancelling pairs
        scale = 10.0 ** rng.uniform(-3, 1, size=d)
        q = (rng.standard_normal(d) * scale).astype(np.float32)
        k = (rng.standard_normal(d) * scale[::-1]).astype(np.float32)
        if trial % 3 == 0:
            k = (q * np.float32(-1.0) + rng.standard_normal(d).astype(np.float32) * np.float32(1e-3)).astype(
                np.float32)
        exact = float(np.dot(q.astype(np.float64), k.astype(np.float64)))
        cond = float(np.dot(np.abs(q).astype(np.float64), np.abs(k).astype(np.float64)))
        err = abs(emulated_score(q, k) - exact)
        assert err <= gamma * cond, (trial, err, gamma * cond)
        worst = max(worst, err / (gamma * cond))
    # the bound is not vacuous: the emulated errors reach a visible part of
    # it (about an eighth with these inputs)
    assert worst > 0.02
