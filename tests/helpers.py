"""Shared helpers of the GPU parity tests: input construction and comparison metrics."""
from __future__ import annotations

import numpy as np

import synthetic as syn

# Tolerances of the parity criteria against the oracle with bf16 activations (the workloads'
# stated precision): loss relative, logits max|d| / max|ref|, gradients cosine and max-rel.
LOSS_RTOL = 1e-2
LOGITS_MAXREL = 1e-2
GRAD_COS = 0.999
GRAD_MAXREL = 2e-2
# Against the exact (unrounded fp64) oracle the difference is the rounding noise of bf16 operands
# (unit roundoff 2^-8, amplified by softmax and products); bound the logits at 3x the above.
EXACT_LOGITS_MAXREL = 3e-2
# Gradients against the exact oracle: the workloads compute with bf16 activations, and on two
# Qwen2.5-32B-shaped layers (batch 1 x 256) the oracle's own bf16-activation mode is already 2.48%
# (q dA) and 2.66% (k dA) max-rel from its exact mode -- the rounding of layer 0's forward
# activations moves the top layer's q/k adapter gradients that much. No bf16-activation
# computation can be held closer to exact arithmetic than that, so the exact-oracle bound is 3e-2
# (cosine unchanged); the parity bound of 2e-2 applies against the bf16-activation oracle.
EXACT_GRAD_MAXREL = 3e-2


def cosine(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def maxrel(got, ref) -> float:
    """max |got - ref| / max |ref| (elementwise relative error is ill-posed near zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / (np.abs(ref).max() + 1e-300))


def torch_bf16(x_f32, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(device).to(torch.bfloat16)


def torch_f32(x, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_np(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy() if t.dtype != torch.float32 else t.detach().cpu().numpy()


def build_inputs(wl, step: int = 0) -> dict:
    """All synthetic inputs of a workload (numpy, fp32 values)."""
    raw = [syn.layer_weights(wl, i) for i in range(wl.n_layers)]
    d = {"raw": raw}
    if wl.vocab:
        d["head"] = (syn.embedding(wl), syn.norm_gain(wl), syn.lm_head(wl))
        d["tokens"], d["targets"] = syn.tokens(wl, step)
    else:
        d["x"], d["G"] = syn.hidden_input(wl), syn.output_grad(wl)
    return d


def make_context(wl, inp: dict, streamed: bool, timeout_ms: int = 600000, **cfg_kw):
    """A library context with every layer registered from host (numpy) weights; cfg_kw go to
    make_config (head_chunk, reuse)."""
    import layer_streamed_qlora_streaming_b200 as lst
    cfg = lst.make_config(wl, streamed=streamed, timeout_ms=timeout_ms, **cfg_kw)
    if wl.vocab:
        E, gf, H = inp["head"]
        ctx = lst.Context(cfg, E, gf, H)
    else:
        ctx = lst.Context(cfg)
    for i, r in enumerate(inp["raw"]):
        ctx.register_layer(i, r["W"], r["A"], r["B"], r["attn_norm"], r["mlp_norm"], r["bias"])
    return ctx


def run_step(ctx, wl, inp: dict, want_logits: bool = True):
    """(loss, grads flat fp32 numpy, logits or None) of one library step on host inputs."""
    grads = np.zeros(ctx.lora_numel(), dtype=np.float32)
    if wl.vocab:
        loss = ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq, grads)
        logits = None
        if want_logits:
            logits = np.zeros((wl.tokens, wl.vocab), dtype=np.float32)
            ctx.logits(logits)
        return loss, grads, logits
    xb = syn.to_bf16_bits(inp["x"])
    gb = syn.to_bf16_bits(inp["G"])
    loss = ctx.step_hidden(xb, gb, wl.batch, wl.seq, grads)
    return loss, grads, None


def oracle_step(wl, inp: dict, schedule: str = "streamed", bf16_acts: bool = True):
    from oracle import model as M
    kw = dict(raw_layers=inp["raw"], schedule=schedule, bf16_acts=bf16_acts)
    if wl.vocab:
        kw.update(head=inp["head"], tokens=inp["tokens"], targets=inp["targets"])
    else:
        kw.update(x_in=inp["x"], G=inp["G"])
    return M.step(wl, **kw)


def split_grads(ctx, grads: np.ndarray) -> dict:
    out = {}
    for key, ((oa, sa), (ob, sb)) in ctx.grad_slices().items():
        out[key] = (grads[oa:oa + sa[0] * sa[1]].reshape(sa), grads[ob:ob + sb[0] * sb[1]].reshape(sb))
    return out


def compare_grads(ctx, grads: np.ndarray, ref: dict) -> list:
    """Per (layer, proj, which): (cosine, maxrel); ref = oracle grads list."""
    g = split_grads(ctx, grads)
    res = []
    for (l, p), (dA, dB) in g.items():
        rA, rB = ref[l][p]
        res.append((l, p, "A", cosine(dA, rA), maxrel(dA, rA)))
        res.append((l, p, "B", cosine(dB, rB), maxrel(dB, rB)))
    return res
