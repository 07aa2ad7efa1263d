"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the benchmark.

This module holds none of the method's arithmetic. It has two parts:

* a counter-based random generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014) evaluated at counter values, turned into
  uniforms with the top 53 bits and into normals with the Box-Muller transform in fp64;
* the workload shapes (``WORKLOADS``) and the per-tensor seed/stream assignment, so that the
  oracle and the CUDA path are fed identical bytes.

Every tensor is drawn from its own stream, keyed by (seed, stream id), so a tensor does not
depend on the order in which others are drawn.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (the variant-13 finaliser), on uint64 arrays (wrapping)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _key(seed: int, stream: int) -> np.uint64:
    k = np.array([((seed & 0xFFFFFFFF) << 32) ^ (stream & 0xFFFFFFFF)], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(k * _GAMMA + _GAMMA)[0]


def raw_u64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Counter values start..start+count-1 of stream (seed, stream), SplitMix64-mixed."""
    key = _key(seed, stream)
    ctr = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + ctr * _GAMMA)


def uniform(seed: int, stream: int, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
    """n uniforms in [lo, hi) as fp64 (53-bit mantissa from the top bits)."""
    u = (raw_u64(seed, stream, 0, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return lo + (hi - lo) * u


def _normal_chunk(args) -> np.ndarray:
    seed, stream, s, m = args
    z = raw_u64(seed, stream, 2 * s, 2 * m) >> np.uint64(11)
    u = z.astype(np.float64) * (2.0 ** -53)
    u1 = 1.0 - u[0::2]          # (0, 1]
    u2 = u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


_POOL = None


def _pool():
    """Worker processes for large draws (spawned, so safe after CUDA is initialised)."""
    global _POOL
    if _POOL is None:
        import concurrent.futures as cf
        import multiprocessing as mp
        import os
        import atexit
        _POOL = cf.ProcessPoolExecutor(max_workers=min(16, os.cpu_count() or 1),
                                       mp_context=mp.get_context("spawn"))
        atexit.register(_shutdown_pool)
    return _POOL


def _shutdown_pool():
    """Stop the workers while the interpreter is still whole (avoids noise at exit)."""
    global _POOL
    if _POOL is not None:
        _POOL.shutdown(wait=True)
        _POOL = None


def normal(seed: int, stream: int, n: int, std: float = 1.0, chunk: int = 1 << 24) -> np.ndarray:
    """n standard normals x std (fp64) by Box-Muller: counters 2i, 2i+1 give one normal.
    The values do not depend on the chunking (each chunk starts at its own counter)."""
    out = np.empty(n, dtype=np.float64)
    jobs = [(seed, stream, s, min(chunk, n - s)) for s in range(0, n, chunk)]
    if len(jobs) > 2:
        for (_, _, s, m), part in zip(jobs, _pool().map(_normal_chunk, jobs)):
            out[s:s + m] = part
    else:
        for (_, _, s, m) in jobs:
            out[s:s + m] = _normal_chunk((seed, stream, s, m))
    return out * std


def integers(seed: int, stream: int, n: int, high: int) -> np.ndarray:
    """n integers uniform in [0, high) (int32), by floor(u * high)."""
    u = uniform(seed, stream, n)
    return np.minimum(np.floor(u * high), high - 1).astype(np.int32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even; NaN is not expected here."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Value of x after rounding to bf16 (returned as fp32)."""
    return bf16_bits_to_f32(to_bf16_bits(x))


# ----------------------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------------------

PROJ = ("q", "k", "v", "o", "gate", "up", "down")

# seeds
SEED_BASE_W, SEED_LORA, SEED_TOKENS, SEED_X, SEED_HEAD, SEED_G, SEED_PREF = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int            # 0: no embedding / head; the loss is sum(x_L * G) for a seeded G
    rms_eps: float
    rope_theta: float
    qkv_bias: bool
    lora_rank: int
    lora_alpha: float
    base_format: str      # "nf4" or "bf16"
    batch: int
    seq: int

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def dq(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def dkv(self) -> int:
        return self.n_kv_heads * self.head_dim

    def proj_shape(self, p: str) -> tuple[int, int]:
        """(out, in) of projection p; W is [out, in] row-major."""
        d, F = self.d_model, self.ffn
        return {"q": (self.dq, d), "k": (self.dkv, d), "v": (self.dkv, d), "o": (d, self.dq),
                "gate": (F, d), "up": (F, d), "down": (d, F)}[p]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny Llama-style stack (the small case the oracle finishes in seconds)
    "tiny": Workload("tiny", 2, 256, 4, 4, 64, 688, 1024, 1e-5, 1e4, False, 8, 16.0, "nf4", 2, 64),
    # one Llama-3.1-8B-shaped decoder layer, no head
    "llama8b_layer": Workload("llama8b_layer", 1, 4096, 32, 8, 128, 14336, 0, 1e-5, 5e5, False,
                              16, 32.0, "nf4", 4, 512),
    # the Llama-3.1-8B-shaped stack with its head
    "llama8b": Workload("llama8b", 32, 4096, 32, 8, 128, 14336, 128256, 1e-5, 5e5, False,
                        16, 32.0, "nf4", 4, 512),
    # Qwen2.5-3B-shaped stack with an unquantised bf16 base
    "qwen3b_bf16": Workload("qwen3b_bf16", 36, 2048, 16, 2, 128, 11008, 151936, 1e-6, 1e6, True,
                            16, 32.0, "bf16", 8, 512),
    # Qwen2.5-32B-shaped stack, ~252 MB of NF4 per layer
    "qwen32b": Workload("qwen32b", 64, 5120, 40, 8, 128, 27648, 152064, 1e-6, 1e6, True,
                        16, 32.0, "nf4", 1, 2048),
}


def _stream(layer: int, proj: int, which: int) -> int:
    return (layer << 8) | (proj << 4) | which


def base_weight(w: Workload, layer: int, p: str) -> np.ndarray:
    """Frozen base W of projection p of layer: N(0, 0.02), fp32 [out, in]."""
    out, inp = w.proj_shape(p)
    x = normal(SEED_BASE_W, _stream(layer, PROJ.index(p), 0), out * inp, 0.02)
    return x.astype(np.float32).reshape(out, inp)


def qkv_bias(w: Workload, layer: int, p: str) -> np.ndarray:
    """Bias of q/k/v (only when w.qkv_bias): N(0, 0.02), fp32."""
    out, _ = w.proj_shape(p)
    return normal(SEED_HEAD, _stream(layer, PROJ.index(p), 1), out, 0.02).astype(np.float32)


def lora_a(w: Workload, layer: int, p: str) -> np.ndarray:
    """LoRA A [r, in] ~ U(-1/sqrt(in), 1/sqrt(in)), fp32."""
    _, inp = w.proj_shape(p)
    b = 1.0 / np.sqrt(inp)
    a = uniform(SEED_LORA, _stream(layer, PROJ.index(p), 2), w.lora_rank * inp, -b, b)
    return a.astype(np.float32).reshape(w.lora_rank, inp)


def lora_b(w: Workload, layer: int, p: str) -> np.ndarray:
    """LoRA B [out, r] ~ N(0, 0.01), fp32."""
    out, _ = w.proj_shape(p)
    return normal(SEED_LORA, _stream(layer, PROJ.index(p), 3), out * w.lora_rank,
                  0.01).astype(np.float32).reshape(out, w.lora_rank)


def norm_gain(w: Workload) -> np.ndarray:
    """RMSNorm gains: all ones (fp32)."""
    return np.ones(w.d_model, dtype=np.float32)


def embedding(w: Workload) -> np.ndarray:
    """Frozen embedding E [V, d] ~ N(0, 0.02), rounded to bf16 (returned as fp32 values)."""
    return round_bf16(normal(SEED_HEAD, 1 << 30, w.vocab * w.d_model, 0.02)
                      .astype(np.float32)).reshape(w.vocab, w.d_model)


def lm_head(w: Workload) -> np.ndarray:
    """Frozen untied LM head H [V, d] ~ N(0, 0.02), rounded to bf16 (as fp32 values)."""
    return round_bf16(normal(SEED_HEAD, (1 << 30) + 1, w.vocab * w.d_model, 0.02)
                      .astype(np.float32)).reshape(w.vocab, w.d_model)


def tokens(w: Workload, step: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """(tokens, targets), each int32 [batch*seq], independent and uniform in [0, V)."""
    t = integers(SEED_TOKENS, 2 * step, w.tokens, w.vocab)
    y = integers(SEED_TOKENS, 2 * step + 1, w.tokens, w.vocab)
    return t, y


def preference_pairs(w: Workload, step: int = 0) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(tokens, targets, mask), int32 [batch*seq] each, for batch/2 preference pairs: sequences
    [0, P) are the chosen ones and [P, 2P) the rejected ones (P = batch/2). Chosen p and rejected p
    share their prompt (tokens and targets of the first seq/2 positions); the response positions
    are drawn independently; mask is 1 on the response positions, 0 on the prompt. Uniform ids."""
    assert w.batch % 2 == 0
    P, S = w.batch // 2, w.seq
    half = S // 2
    t = integers(SEED_PREF, 4 * step, w.tokens, w.vocab).reshape(w.batch, S)
    y = integers(SEED_PREF, 4 * step + 1, w.tokens, w.vocab).reshape(w.batch, S)
    t[P:, :half] = t[:P, :half]
    y[P:, :half] = y[:P, :half]
    m = np.zeros((w.batch, S), dtype=np.int32)
    m[:, half:] = 1
    return t.reshape(-1), y.reshape(-1), m.reshape(-1)


def hidden_input(w: Workload) -> np.ndarray:
    """Input activations X [T, d] ~ N(0, 1) rounded to bf16 (as fp32 values), headless case."""
    return round_bf16(normal(SEED_X, 0, w.tokens * w.d_model).astype(np.float32)).reshape(
        w.tokens, w.d_model)


def output_grad(w: Workload) -> np.ndarray:
    """G [T, d] ~ N(0, 1) rounded to bf16 (as fp32 values): headless loss is sum(x_L * G)."""
    return round_bf16(normal(SEED_G, 0, w.tokens * w.d_model).astype(np.float32)).reshape(
        w.tokens, w.d_model)


def layer_weights(w: Workload, layer: int) -> dict:
    """All synthetic inputs of one decoder layer, as fp32 numpy arrays."""
    d = {"W": {p: base_weight(w, layer, p) for p in PROJ},
         "A": {p: lora_a(w, layer, p) for p in PROJ},
         "B": {p: lora_b(w, layer, p) for p in PROJ},
         "attn_norm": norm_gain(w), "mlp_norm": norm_gain(w),
         "bias": ({p: qkv_bias(w, layer, p) for p in ("q", "k", "v")} if w.qkv_bias else None)}
    return d
