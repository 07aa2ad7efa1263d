"""NF4 4-bit quantisation with double-quantised absmax: the oracle's definition.

[CODE] section "Quantization: Shrink the Weights" names 4-bit NormalFloat (NF4) with nested
("double") quantisation of the constants; [TKN] para 1 says quantising the streamed base shrinks it
about fourfold; [LACH] "Step 5" sets ``quantization: 4bit``. The pages give no construction, so
every rule here is a reading, following [QLORA] section 3 ("4-bit NormalFloat", "Double
Quantization"):

1. codebook: 8 positive normal quantiles, 7 negative, and an exact zero, scaled to [-1, 1];
2. blocks of 64 consecutive elements of the row-major flattened tensor; absmax per block;
3. code = number of codebook midpoints strictly below w / absmax (ties go to the lower code);
4. two codes per byte, element 2i in the high nibble;
5. absmax minus its tensor mean, quantised to int8 (symmetric, x127) in groups of 256 blocks
   with one fp32 scale per group;
6. dequant: a^ = (q * s) / 127 + mean, each operation one fp32 rounding (no fused multiply-add),
   then w^ = bf16_rne(codebook[code] * a^).

Parity is pinned by tests against: the published NF4 table of [QLORA] (values printed there),
the normal CDF (math.erfc, a different routine from the quantile used here), exact round trips
of codebook values, and brute-force nearest-value search on small blocks.
"""
from __future__ import annotations

from dataclasses import dataclass
from statistics import NormalDist

import numpy as np

BLOCK = 64          # elements per absmax block
GROUP = 256         # absmax values per double-quant group
# offset of the outermost quantile; [QLORA] uses the mean of 1-1/(2*15) and 1-1/(2*16)
DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))


def codebook_f64() -> np.ndarray:
    """The 16 NF4 values in fp64, ascending, index 7 == 0 exactly, ends at -1 and +1."""
    inv = NormalDist().inv_cdf
    pos = [inv(DELTA - j * (DELTA - 0.5) / 8.0) for j in range(8)]
    neg = [-inv(DELTA - j * (DELTA - 0.5) / 7.0) for j in range(7)]
    vals = np.array(sorted(pos + neg + [0.0]), dtype=np.float64)
    return vals / inv(DELTA)


def codebook() -> np.ndarray:
    """The NF4 codebook rounded once to fp32."""
    return codebook_f64().astype(np.float32)


def midpoints(cb: np.ndarray) -> np.ndarray:
    """The 15 decision thresholds (c_j + c_{j+1}) / 2, each an fp32 sum then an exact halving."""
    cb = cb.astype(np.float32)
    return ((cb[:-1] + cb[1:]) * np.float32(0.5)).astype(np.float32)


@dataclass
class NF4Tensor:
    """One quantised tensor: ``packed`` uint8 [n/2], ``qabs`` int8 [n/64], ``gscale`` fp32
    [ceil(n/64/256)], ``mean`` fp32 scalar, and the original shape."""
    packed: np.ndarray
    qabs: np.ndarray
    gscale: np.ndarray
    mean: np.float32
    shape: tuple

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape))


def absmax_mean(a: np.ndarray) -> np.float32:
    """Mean of the block absmax values: fp64 sums, first over each group of 256 blocks in index
    order, then over the group sums in index order; divided by the count in fp64; rounded to
    fp32 (reading: the pages do not fix a summation order)."""
    a = a.astype(np.float64)
    n = a.size
    ng = -(-n // GROUP)
    pad = np.zeros(ng * GROUP, dtype=np.float64)
    pad[:n] = a
    gsum = np.zeros(ng, dtype=np.float64)
    m = pad.reshape(ng, GROUP)
    for j in range(GROUP):          # sequential within each group
        gsum = gsum + m[:, j]
    total = 0.0
    for g in range(ng):             # sequential across groups
        total = total + float(gsum[g])
    return np.float32(total / float(n))


def quantize(w: np.ndarray) -> NF4Tensor:
    """Quantise an fp32 tensor (any shape, numel a multiple of 64) to NF4 with double quant."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    shape = w.shape
    flat = w.reshape(-1)
    n = flat.size
    if n % BLOCK != 0:
        raise ValueError("numel must be a multiple of 64")
    blocks = flat.reshape(-1, BLOCK)
    a = np.abs(blocks).max(axis=1).astype(np.float32)            # absmax per block

    # first level: codes against the true absmax
    mid = midpoints(codebook())
    with np.errstate(invalid="ignore", divide="ignore"):
        x = (blocks / a[:, None]).astype(np.float32)                # fp32 division per element
    code = np.searchsorted(mid, x, side="left").astype(np.uint8)   # count of midpoints < x
    code[a == 0] = 7                                                # all-zero block -> exact 0
    c = code.reshape(-1)
    packed = ((c[0::2] << 4) | c[1::2]).astype(np.uint8)

    # second level: absmax - mean, int8 per group of 256
    mean = absmax_mean(a)
    cdev = (a - mean).astype(np.float32)
    nb = a.size
    ng = -(-nb // GROUP)
    gscale = np.zeros(ng, dtype=np.float32)
    qabs = np.zeros(nb, dtype=np.int8)
    for g in range(ng):
        seg = cdev[g * GROUP:(g + 1) * GROUP]
        s = np.float32(np.abs(seg).max())
        gscale[g] = s
        if s == 0:
            continue
        t = (seg / s).astype(np.float32)
        u = (t * np.float32(127.0)).astype(np.float32)
        qabs[g * GROUP:(g + 1) * GROUP] = np.clip(np.rint(u), -127, 127).astype(np.int8)
    return NF4Tensor(packed, qabs, gscale, mean, shape)


def dequant_absmax(t: NF4Tensor) -> np.ndarray:
    """a^_b = (q_b * s_g) / 127 + mean, each op rounded to fp32."""
    s = np.repeat(t.gscale, GROUP)[: t.qabs.size]
    prod = (t.qabs.astype(np.float32) * s).astype(np.float32)
    quo = (prod / np.float32(127.0)).astype(np.float32)
    return (quo + t.mean).astype(np.float32)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    codes = np.empty(packed.size * 2, dtype=np.uint8)
    codes[0::2] = packed >> 4
    codes[1::2] = packed & 0x0F
    return codes


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    return ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_value(x: np.ndarray) -> np.ndarray:
    """x rounded to bf16 (round to nearest even), returned as fp32."""
    return (bf16_bits(x).astype(np.uint32) << np.uint32(16)).view(np.float32)


def dequantize(t: NF4Tensor) -> np.ndarray:
    """w^ = bf16_rne(codebook[code] * a^), returned as fp32 values of that bf16, in t.shape."""
    codes = unpack_codes(t.packed)
    a_hat = np.repeat(dequant_absmax(t), BLOCK)
    w = (codebook()[codes] * a_hat).astype(np.float32)
    return bf16_value(w).reshape(t.shape)


def dequantize_bits(t: NF4Tensor) -> np.ndarray:
    """Same as ``dequantize`` but as bf16 bit patterns (uint16), for bit-exact comparisons."""
    codes = unpack_codes(t.packed)
    a_hat = np.repeat(dequant_absmax(t), BLOCK)
    return bf16_bits((codebook()[codes] * a_hat).astype(np.float32)).reshape(t.shape)


def storage_bits_per_param(n: int) -> float:
    """Bits per parameter of this format for a tensor of n elements (nibbles + int8 absmax +
    fp32 group scales + one fp32 mean)."""
    nb = n // BLOCK
    ng = -(-nb // GROUP)
    return (4 * n + 8 * nb + 32 * ng + 32) / n
