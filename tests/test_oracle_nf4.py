"""Pins of the oracle's NF4 quantiser against things other than itself (CPU only).

* the NF4 table printed in QLoRA (Dettmers et al. 2023), appendix "NormalFloat 4-bit data type";
* the normal CDF through math.erfc (the oracle builds the table with an inverse CDF);
* exact recovery of codebook values, brute-force nearest-value search, hand-packed bytes;
* the storage figures of [CODE] "Quantization: Shrink the Weights" (double quant saves ~0.4 GB
  at 8B) and [TKN] para 1 (4-bit shrinks the base about fourfold).
"""
import math
import os

import numpy as np
import pytest

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


# The 16 NF4 values as printed in the QLoRA paper's appendix (tests/golden, with the citation).
QLORA_NF4 = [float(l[0]) for l in _golden_lines("qlora_nf4_table.txt")]
# The pages' storage figures: name -> (value, lower, upper)
PAGE_FIGURES = {l[0]: tuple(float(x) for x in l[1:]) for l in _golden_lines("pages_storage_figures.txt")}


def test_codebook_matches_published_table():
    cb = nf4.codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    np.testing.assert_allclose(cb.astype(np.float64), QLORA_NF4, rtol=0, atol=2e-7)


def test_codebook_invariants():
    cb = nf4.codebook()
    assert np.all(np.diff(cb) > 0)
    assert cb[7] == 0.0 and cb[0] == -1.0 and cb[15] == 1.0


def test_codebook_is_normal_quantiles_via_cdf():
    # Phi(c * Phi^-1(delta)) must give back the quantile levels; Phi via erfc (not inv_cdf)
    cb = nf4.codebook_f64()
    # the scale Phi^-1(delta): solve Phi(z) = delta by bisection on erfc
    phi = lambda z: 0.5 * math.erfc(-z / math.sqrt(2.0))
    lo, hi = 0.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        lo, hi = (mid, hi) if phi(mid) < nf4.DELTA else (lo, mid)
    z = 0.5 * (lo + hi)
    d = nf4.DELTA
    want_pos = sorted(d - j * (d - 0.5) / 8 for j in range(8))
    want_neg = sorted(1.0 - (d - j * (d - 0.5) / 7) for j in range(7))
    got = [phi(c * z) for c in cb]
    np.testing.assert_allclose(got[8:], want_pos, atol=1e-12)
    np.testing.assert_allclose(got[:7], want_neg, atol=1e-12)
    assert got[7] == 0.5


def test_pack_order_and_zero_block():
    cb = nf4.codebook()
    a = np.float32(0.5)
    w = np.zeros(128, dtype=np.float32)
    w[0], w[1], w[2], w[3] = cb[0] * a, cb[15] * a, cb[7] * a, cb[9] * a
    t = nf4.quantize(w)
    assert t.packed[0] == 0x0F       # element 0 high nibble, element 1 low nibble
    assert t.packed[1] == 0x79
    # the second block is all zero: every code is 7 (the exact zero)
    assert np.all(t.packed[32:] == 0x77)
    deq = nf4.dequantize(t)
    assert np.all(deq[64:] == 0.0)


def test_codebook_values_recovered_exactly_uniform_absmax():
    # every block has absmax 2^-3: mean == absmax, group scale 0, so a^ == a exactly and the
    # dequantised value is bf16(c_k * a) with c_k the original code
    cb = nf4.codebook()
    rng = np.random.default_rng(0)
    k = rng.integers(0, 16, size=64 * 300)
    k[0::64] = 15                                     # each block reaches the absmax
    a = np.float32(0.125)
    w = (cb[k] * a).astype(np.float32)
    t = nf4.quantize(w)
    assert np.array_equal(nf4.unpack_codes(t.packed), k.astype(np.uint8))
    assert np.all(t.gscale == 0) and np.all(t.qabs == 0) and t.mean == a
    assert np.array_equal(nf4.dequantize(t), nf4.bf16_value(w))


def test_codes_recovered_with_random_absmax_and_error_bound():
    cb = nf4.codebook()
    rng = np.random.default_rng(1)
    nb = 1000
    k = rng.integers(0, 16, size=(nb, 64))
    k[:, 5] = 0                                       # absmax reached by -1 * a
    a = rng.uniform(0.001, 0.1, size=nb).astype(np.float32)
    w = (cb[k] * a[:, None]).astype(np.float32)
    t = nf4.quantize(w)
    assert np.array_equal(nf4.unpack_codes(t.packed).reshape(nb, 64), k.astype(np.uint8))
    a_hat = nf4.dequant_absmax(t)
    # second-level error: at most half a step of the int8 grid (s/254) plus fp32 rounding
    s = np.repeat(t.gscale, nf4.GROUP)[:nb]
    assert np.all(np.abs(a_hat - a) <= s / 254 * (1 + 1e-5) + 4 * np.finfo(np.float32).eps * a)
    deq = nf4.dequantize(t).reshape(nb, 64)
    bound = np.abs(cb[k]) * np.abs(a_hat - a)[:, None] + np.abs(deq) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(deq - w) <= bound)


def test_codes_are_nearest_value_brute_force():
    cb64 = nf4.codebook().astype(np.float64)
    rng = np.random.default_rng(2)
    w = rng.normal(0, 0.02, size=64 * 2000).astype(np.float32)
    t = nf4.quantize(w)
    codes = nf4.unpack_codes(t.packed)
    blocks = w.reshape(-1, 64)
    a = np.abs(blocks).max(axis=1)
    x = (blocks / a[:, None]).astype(np.float32).astype(np.float64).reshape(-1)
    # brute force: index of the nearest codebook value, ties to the lower index
    dist = np.abs(x[:, None] - cb64[None, :])
    best = np.argmin(dist, axis=1)
    assert np.array_equal(codes, best.astype(np.uint8))


def test_tie_goes_to_lower_code():
    cb = nf4.codebook()
    mid = nf4.midpoints(cb)
    w = np.zeros(64, dtype=np.float32)
    w[0] = 1.0                                      # absmax 1 -> x == w
    w[1] = mid[9]                                   # exactly on the midpoint between 9 and 10
    w[2] = np.nextafter(mid[9], np.float32(1))
    t = nf4.quantize(w)
    c = nf4.unpack_codes(t.packed)
    assert c[1] == 9 and c[2] == 10


def test_absmax_mean_matches_exact_sum():
    rng = np.random.default_rng(3)
    a = rng.uniform(0, 0.1, size=70000).astype(np.float32)
    exact = math.fsum(float(v) for v in a) / a.size
    assert abs(float(nf4.absmax_mean(a)) - exact) <= abs(exact) * 2 ** -23


def test_ragged_last_group():
    # 688 x 256 elements -> 2752 blocks -> 10 full groups + 192 (the tiny down projection)
    rng = np.random.default_rng(4)
    w = rng.normal(0, 0.02, size=(256, 688)).astype(np.float32)
    t = nf4.quantize(w)
    assert t.qabs.size == 2752 and t.gscale.size == 11
    a = np.abs(w.reshape(-1, 64)).max(axis=1)
    assert np.all(np.abs(nf4.dequant_absmax(t) - a) <= np.repeat(t.gscale, 256)[:2752] / 254 * 1.001)


def test_storage_size_claims():
    # [TKN] para 1: 4-bit shrinks the base about fourfold (vs 16-bit)
    bits = nf4.storage_bits_per_param(4096 * 4096)
    assert abs(bits - (4 + 8 / 64 + 32 / (64 * 256))) < 1e-5
    _, lo, hi = PAGE_FIGURES["fourfold_ratio"]
    assert lo < 16.0 / bits < hi
    # [CODE]: double quantisation saves ~0.4 GB more at 8B; single-level = 4 + 32/64 bits
    n8b = 32 * (2 * 4096 * 4096 + 2 * 1024 * 4096 + 3 * 4096 * 14336)
    saving_gb = n8b * ((4 + 32 / 64) - bits) / 8 / 1e9
    _, lo, hi = PAGE_FIGURES["double_quant_saving_gb_8b"]
    assert lo < saving_gb < hi


def test_quantize_rejects_non_multiple_of_64():
    with pytest.raises(ValueError):
        nf4.quantize(np.zeros(100, dtype=np.float32))
