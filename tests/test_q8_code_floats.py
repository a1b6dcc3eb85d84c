"""The arithmetic identities the 8-bit streaming kernels rely on, checked on
the host in IEEE fp32 (numpy keeps subnormals).

The kernels turn an 8-bit code q into a float with one byte permute: q placed
in bits 16..23 of a zero word. They multiply it, in one fma, by an activation
pre-scaled by 2^33, and scale a 16-product chunk sum back by 2^100. These tests
pin that (a) the word reads as exactly q * 2^-133 for every code, across the
subnormal/normal boundary at q = 128; (b) each scaled product is exact, so the
scaled fma chain equals the plain fp32 fma chain of q * v bit for bit once
scaled back; (c) the affine form regrouped per chunk, s * sum(q v) + b * sum(v),
stays within fp32 rounding of the exact fp64 value of sum((s q + b) v) for
weights drawn like the tests' (bias about -128 * scale).
"""
import numpy as np

V_SCALE = np.float32(2.0 ** 33)
UNSCALE = np.float32(2.0 ** 100)


def _code_float(q: np.ndarray) -> np.ndarray:
    return (q.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fma32(a, b, c):
    # one rounding of the exact a*b + c: the product of two fp32 values is
    # exact in fp64, and so is the sum here (magnitudes within 2^53 of each other)
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def test_code_word_reads_as_q_times_2_pow_minus_133():
    q = np.arange(256, dtype=np.uint32)
    f = _code_float(q).astype(np.float64)
    assert np.array_equal(f, q * 2.0 ** -133)
    # below 128 the word is subnormal, from 128 up it is normal
    assert np.all(np.abs(f[1:128]) < np.finfo(np.float32).tiny)
    assert np.all(f[128:] >= np.finfo(np.float32).tiny)


def test_scaled_chain_equals_plain_chain_bit_for_bit():
    rng = np.random.default_rng(7)
    for trial in range(200):
        q = rng.integers(0, 256, 16).astype(np.uint32)
        mag = 10.0 ** rng.uniform(-6, 4)
        v = (rng.standard_normal(16) * mag).astype(np.float32)
        vs = v * V_SCALE  # exact: a power of two
        qf = _code_float(q)
        d = np.float32(0)
        ref = np.float32(0)
        for i in range(16):
            d = _fma32(qf[i], vs[i], d)
            ref = _fma32(np.float32(q[i]), v[i], ref)
        assert np.float32(d * UNSCALE) == ref, (trial, d * UNSCALE, ref)


def test_regrouped_affine_chunk_within_fp32_rounding():
    rng = np.random.default_rng(11)
    worst = 0.0
    for trial in range(500):
        sigma = 1.0 / 64.0
        q = np.clip(np.round(rng.standard_normal(16) * 40 + 128), 0, 255).astype(np.uint32)
        s = np.float32(sigma / 40 * rng.uniform(0.75, 1.25))
        b = np.float32(-128 * s + rng.standard_normal() * sigma / 16)
        v = rng.standard_normal(16).astype(np.float32)
        exact = float(np.sum((np.float64(s) * q + np.float64(b)) * v.astype(np.float64)))
        # the kernel's order: d = sum(q v) scaled, sv = sum(v), then fma(s, d, fma(b, sv, 0))
        vs = v * V_SCALE
        qf = _code_float(q)
        d = np.float32(0)
        sv = np.float32(0)
        for i in range(16):
            d = _fma32(qf[i], vs[i], d)
            sv = np.float32(sv + v[i])
        got = _fma32(s, np.float32(d * UNSCALE), _fma32(b, sv, np.float32(0)))
        scale = float(np.sum(np.abs(np.float64(s) * q) * np.abs(v)) + abs(float(b)) * float(np.sum(np.abs(v))))
        err = abs(float(got) - exact) / scale
        worst = max(worst, err)
    # a few fp32 roundings of terms no larger than `scale`
    assert worst < 8 * 2.0 ** -24, worst
