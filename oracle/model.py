"""Decoder stack, LoRA, head and analytic backward of layer-streamed LoRA fine-tuning, in fp64.

What the method computes, from the pages:

* the frozen base is kept off the GPU and each decoder layer is brought in only while it is
  needed ([5ID] para 2; [TKN] para 1), through a two-buffer pool, and read again for backward
  recomputation ([LACH] "What Soup layer streaming changes");
* only LoRA adapters are trained; the base stays frozen ([LACH] FAQ "Does Soup train the full 8B
  model?"; [CODE] "LoRA and QLoRA"); adapters are full precision ([CODE] "LoRA and QLoRA");
* logits stay resident and the loss is ordinary cross-entropy ([TESS] para 2);
* streaming changes no number: the forward is bit-exact against a resident run ([TKN] para 2).

The layer itself (Llama / Qwen2 pre-norm decoder: RMSNorm, q/k/v/o with RoPE and causal GQA
attention, SwiGLU MLP, residuals) is the reading of "Llama-style" / "Qwen2.5-shaped" workloads.
LoRA: y = x W^T + s (x A^T) B^T (+ bias for q/k/v where present), s = alpha / r, no dropout.

Every function is the plain definition in fp64. Gradients are returned only for LoRA A and B.

Activation precision. The workloads state bf16 activations ("bf16 acts") with full-precision
accumulation. ``step(..., bf16_acts=True)`` applies that rule literally: every operand of a matrix
product that is an activation or an activation gradient is rounded to bf16 (round to nearest even)
before the product -- the normalised inputs of the projections, q / k (after RoPE) / v, the attention
output, the SwiGLU inputs and output, the normalised input of the LM head, and in the backward the
upstream gradients entering a projection and the attention gradients -- while products, sums,
norms, softmax and the residual stream stay exact (fp64). With ``bf16_acts=False`` nothing is
rounded. The rounding points are where a bf16-activation computation must round; they are a
reading of "bf16 acts", not taken from any implementation.
"""
from __future__ import annotations

import numpy as np

from . import nf4

PROJ = ("q", "k", "v", "o", "gate", "up", "down")
F64 = np.float64


# ------------------------------------------------------------------------------------------
# building blocks
# ------------------------------------------------------------------------------------------

def rmsnorm(x, g, eps):
    """y = x / sqrt(mean(x^2) + eps) * g (row-wise); returns (y, r) with r = 1/sqrt(...)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    return x * r[:, None] * g[None, :], r


def rmsnorm_bwd(dy, x, g, r):
    """dL/dx of rmsnorm for upstream dy (gains are frozen, no dg)."""
    xh = x * r[:, None]
    dyg = dy * g[None, :]
    return r[:, None] * (dyg - xh * np.mean(dyg * xh, axis=-1, keepdims=True))


def rope_tables(seq, head_dim, theta):
    """cos/sin [seq, hd/2] of angle pos * theta^(-2j/hd) (rotate-half pairing, reading)."""
    j = np.arange(head_dim // 2, dtype=F64)
    inv = theta ** (-2.0 * j / head_dim)
    ang = np.arange(seq, dtype=F64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin, batch, seq):
    """Rotate pairs (j, j + hd/2) of x [T, H, hd] by the angle of position t mod seq."""
    h2 = x.shape[-1] // 2
    c = np.tile(cos, (batch, 1))[:, None, :]
    s = np.tile(sin, (batch, 1))[:, None, :]
    x1, x2 = x[..., :h2], x[..., h2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy, cos, sin, batch, seq):
    """Transpose of ``rope`` (rotation by the negative angle)."""
    h2 = dy.shape[-1] // 2
    c = np.tile(cos, (batch, 1))[:, None, :]
    s = np.tile(sin, (batch, 1))[:, None, :]
    d1, d2 = dy[..., :h2], dy[..., h2:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def attention(q, k, v, batch, seq):
    """Causal GQA attention. q [T, hq, hd], k/v [T, hkv, hd]; query head h reads kv head
    h // (hq/hkv); scale 1/sqrt(hd). Returns (o [T, hq, hd], P [B, hq, S, S])."""
    T, hq, hd = q.shape
    hkv = k.shape[1]
    grp = hq // hkv
    o = np.zeros_like(q)
    P = np.zeros((batch, hq, seq, seq))
    mask = np.triu(np.ones((seq, seq), dtype=bool), 1)
    for b in range(batch):
        rows = slice(b * seq, (b + 1) * seq)
        for h in range(hq):
            kh = h // grp
            s = q[rows, h, :] @ k[rows, kh, :].T / np.sqrt(hd)
            s[mask] = -np.inf
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            P[b, h] = p
            o[rows, h, :] = p @ v[rows, kh, :]
    return o, P


def attention_bwd(do, q, k, v, P, batch, seq):
    """Gradients (dq, dk, dv) of ``attention``; dk/dv sum over the query heads of a group."""
    T, hq, hd = q.shape
    hkv = k.shape[1]
    grp = hq // hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(batch):
        rows = slice(b * seq, (b + 1) * seq)
        for h in range(hq):
            kh = h // grp
            p = P[b, h]
            dov = do[rows, h, :]
            dv[rows, kh, :] += p.T @ dov
            dp = dov @ v[rows, kh, :].T
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
            dq[rows, h, :] = ds @ k[rows, kh, :] / np.sqrt(hd)
            dk[rows, kh, :] += ds.T @ q[rows, h, :] / np.sqrt(hd)
    return dq, dk, dv


def silu(g):
    return g / (1.0 + np.exp(-g))


def lora_linear(x, W, A, B, s, bias=None):
    """y = x W^T + s (x A^T) B^T (+ bias); returns (y, u) with u = x A^T."""
    u = x @ A.T
    y = x @ W.T + s * (u @ B.T)
    if bias is not None:
        y = y + bias[None, :]
    return y, u


def lora_linear_bwd(dy, x, u, W, A, B, s):
    """(dx, dA, dB) for y = x W^T + s (x A^T) B^T; W is frozen."""
    vv = dy @ B                      # [T, r]
    dx = dy @ W + s * (vv @ A)
    dB = s * (dy.T @ u)              # [out, r]
    dA = s * (vv.T @ x)              # [r, in]
    return dx, dA, dB


# ------------------------------------------------------------------------------------------
# weights
# ------------------------------------------------------------------------------------------

def base_to_bf16(w):
    """A bf16 base: W rounded once to bf16 (RNE) [LACH] FAQ "4-bit or no quantisation"."""
    return nf4.bf16_value(w)


def pack_layer(raw: dict, base_format: str) -> dict:
    """The per-layer blob the host arena holds: NF4 tensors (or bf16 values) + small tensors."""
    if base_format == "nf4":
        base = {p: nf4.quantize(raw["W"][p]) for p in PROJ}
    else:
        base = {p: base_to_bf16(raw["W"][p]) for p in PROJ}
    return {"format": base_format, "base": base, "attn_norm": raw["attn_norm"].copy(),
            "mlp_norm": raw["mlp_norm"].copy(),
            "bias": None if raw.get("bias") is None else {p: b.copy() for p, b in raw["bias"].items()}}


def copy_blob(blob: dict) -> dict:
    """A host-to-device copy of a blob (byte-for-byte), as the streaming schedule does it."""
    if blob["format"] == "nf4":
        base = {p: nf4.NF4Tensor(t.packed.copy(), t.qabs.copy(), t.gscale.copy(), np.float32(t.mean),
                                 t.shape) for p, t in blob["base"].items()}
    else:
        base = {p: t.copy() for p, t in blob["base"].items()}
    return {"format": blob["format"], "base": base, "attn_norm": blob["attn_norm"].copy(),
            "mlp_norm": blob["mlp_norm"].copy(),
            "bias": None if blob["bias"] is None else {p: b.copy() for p, b in blob["bias"].items()}}


def unpack_blob(blob: dict) -> dict:
    """The fp64 weights a layer computes with: W^ per projection, gains, biases."""
    if blob["format"] == "nf4":
        W = {p: nf4.dequantize(t).astype(F64) for p, t in blob["base"].items()}
    else:
        W = {p: t.astype(F64) for p, t in blob["base"].items()}
    return {"W": W, "attn_norm": blob["attn_norm"].astype(F64),
            "mlp_norm": blob["mlp_norm"].astype(F64),
            "bias": None if blob["bias"] is None else {p: b.astype(F64) for p, b in blob["bias"].items()}}


# ------------------------------------------------------------------------------------------
# decoder layer
# ------------------------------------------------------------------------------------------

def _identity(x):
    return x


def _round_bf16(x):
    return nf4.bf16_value(np.asarray(x, dtype=np.float32)).astype(F64)


class Shape:
    def __init__(self, wl, bf16_acts: bool = False):
        self.rb = _round_bf16 if bf16_acts else _identity
        self.batch, self.seq = wl.batch, wl.seq
        self.hq, self.hkv, self.hd = wl.n_heads, wl.n_kv_heads, wl.head_dim
        self.eps, self.theta = wl.rms_eps, wl.rope_theta
        self.s = wl.lora_alpha / wl.lora_rank
        self.cos, self.sin = rope_tables(wl.seq, wl.head_dim, wl.rope_theta)


def layer_fwd(x, Wt, lora, sh: Shape):
    """One pre-norm decoder layer. Wt: unpacked weights; lora: {proj: (A, B)} fp64.
    Returns (x_out, cache) where cache holds what the backward needs."""
    T = x.shape[0]
    rb = sh.rb
    bias = Wt["bias"] or {}
    n1, r1 = rmsnorm(x, Wt["attn_norm"], sh.eps)
    n1 = rb(n1)
    c = {"x": x, "n1": n1, "r1": r1}
    for p in ("q", "k", "v"):
        y, u = lora_linear(n1, Wt["W"][p], *lora[p], sh.s, bias.get(p))
        c[p + "_pre"], c["u_" + p] = y, u
    q = rb(rope(c["q_pre"].reshape(T, sh.hq, sh.hd), sh.cos, sh.sin, sh.batch, sh.seq))
    k = rb(rope(c["k_pre"].reshape(T, sh.hkv, sh.hd), sh.cos, sh.sin, sh.batch, sh.seq))
    v = rb(c["v_pre"].reshape(T, sh.hkv, sh.hd))
    o, P = attention(q, k, v, sh.batch, sh.seq)
    c.update(q=q, k=k, v=v, P=P, o=rb(o.reshape(T, -1)))
    ao, c["u_o"] = lora_linear(c["o"], Wt["W"]["o"], *lora["o"], sh.s)
    h = x + ao
    n2, r2 = rmsnorm(h, Wt["mlp_norm"], sh.eps)
    n2 = rb(n2)
    g, c["u_gate"] = lora_linear(n2, Wt["W"]["gate"], *lora["gate"], sh.s)
    u, c["u_up"] = lora_linear(n2, Wt["W"]["up"], *lora["up"], sh.s)
    g, u = rb(g), rb(u)
    m = rb(silu(g) * u)
    dn, c["u_down"] = lora_linear(m, Wt["W"]["down"], *lora["down"], sh.s)
    c.update(h=h, n2=n2, r2=r2, g=g, up=u, m=m)
    return h + dn, c


def layer_bwd(dout, c, Wt, lora, sh: Shape):
    """Backward of ``layer_fwd``: returns (dx, {proj: (dA, dB)})."""
    T = dout.shape[0]
    rb = sh.rb
    grads = {}
    dm, grads["down"] = _lin_bwd(rb(dout), c["m"], c["u_down"], Wt["W"]["down"], lora["down"], sh.s)
    sg = 1.0 / (1.0 + np.exp(-c["g"]))
    dg = rb(dm * c["up"] * sg * (1.0 + c["g"] * (1.0 - sg)))
    du = rb(dm * c["g"] * sg)
    dn2_g, grads["gate"] = _lin_bwd(dg, c["n2"], c["u_gate"], Wt["W"]["gate"], lora["gate"], sh.s)
    dn2_u, grads["up"] = _lin_bwd(du, c["n2"], c["u_up"], Wt["W"]["up"], lora["up"], sh.s)
    dh = dout + rmsnorm_bwd(dn2_g + dn2_u, c["h"], Wt["mlp_norm"], c["r2"])
    do, grads["o"] = _lin_bwd(rb(dh), c["o"], c["u_o"], Wt["W"]["o"], lora["o"], sh.s)
    dq, dk, dv = attention_bwd(rb(do).reshape(T, sh.hq, sh.hd), c["q"], c["k"], c["v"], c["P"],
                               sh.batch, sh.seq)
    dq = rb(rope_bwd(dq, sh.cos, sh.sin, sh.batch, sh.seq).reshape(T, -1))
    dk = rb(rope_bwd(dk, sh.cos, sh.sin, sh.batch, sh.seq).reshape(T, -1))
    dv = rb(dv.reshape(T, -1))
    dn1 = 0.0
    for p, dy in (("q", dq), ("k", dk), ("v", dv)):
        dxp, grads[p] = _lin_bwd(dy, c["n1"], c["u_" + p], Wt["W"][p], lora[p], sh.s)
        dn1 = dn1 + dxp
    dx = dh + rmsnorm_bwd(dn1, c["x"], Wt["attn_norm"], c["r1"])
    return dx, grads


def _lin_bwd(dy, x, u, W, AB, s):
    dx, dA, dB = lora_linear_bwd(dy, x, u, W, AB[0], AB[1], s)
    return dx, (dA, dB)


# ------------------------------------------------------------------------------------------
# head: final norm, resident LM head, cross-entropy
# ------------------------------------------------------------------------------------------

def head_fwd(x, gf, H, targets, eps, rb=_identity):
    """logits = rmsnorm(x) H^T; loss = mean_t(logsumexp(logits_t) - logits_t[target_t])."""
    n, r = rmsnorm(x, gf, eps)
    n = rb(n)
    logits = n @ H.T
    mx = logits.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(logits - mx).sum(axis=1, keepdims=True)))[:, 0]
    T = x.shape[0]
    loss = float(np.mean(lse - logits[np.arange(T), targets]))
    return loss, logits, (x, n, r, lse)


def head_bwd(cache, logits, gf, H, targets, rb=_identity):
    """dL/dx of ``head_fwd``: dlogits = (softmax - onehot) / T, dn = dlogits H."""
    x, n, r, lse = cache
    T = x.shape[0]
    dlog = np.exp(logits - lse[:, None])
    dlog[np.arange(T), targets] -= 1.0
    dlog /= T
    return rmsnorm_bwd(rb(dlog) @ H, x, gf, r)


# ------------------------------------------------------------------------------------------
# one training step: resident and streamed schedules
# ------------------------------------------------------------------------------------------

def _lora64(raw):
    return {p: (raw["A"][p].astype(F64), raw["B"][p].astype(F64)) for p in PROJ}


def step(wl, raw_layers, blobs=None, head=None, tokens=None, targets=None, x_in=None, G=None,
         schedule="resident", lora=None, bf16_acts=False):
    """Loss and LoRA gradients of one step.

    raw_layers: per layer the synthetic dict (only A/B are read here; base comes from ``blobs``).
    blobs: per layer ``pack_layer`` output (built here when None).
    head: (E, gf, H) fp32 arrays, or None for a headless stack with loss = sum(x_L * G).
    schedule: "resident" (all layers unpacked once, activations of every layer kept) or
      "streamed" (2L reads through two buffers: forward keeps only each layer's input, backward
      copies the layer again and recomputes it).
    bf16_acts: round matrix-product operands that are activations to bf16 (see module doc).
    Returns dict(loss, grads[layer][proj] = (dA, dB), logits or None, reads).
    """
    L = wl.n_layers
    sh = Shape(wl, bf16_acts)
    if blobs is None:
        blobs = [pack_layer(raw_layers[i], wl.base_format) for i in range(L)]
    if lora is None:
        lora = [_lora64(raw_layers[i]) for i in range(L)]
    if head is not None:
        E, gf, H = (a.astype(F64) for a in head)
        x = E[tokens]
    else:
        x = x_in.astype(F64)

    reads = []
    if schedule == "resident":
        Ws = [unpack_blob(blobs[i]) for i in range(L)]
        caches = []
        for i in range(L):
            x, c = layer_fwd(x, Ws[i], lora[i], sh)
            caches.append(c)
    elif schedule == "streamed":
        buf = [None, None]
        saved = []
        for n in range(L):                           # forward reads n = 0..L-1
            buf[n % 2] = copy_blob(blobs[n])
            reads.append(n)
            saved.append(x)
            x, _ = layer_fwd(x, unpack_blob(buf[n % 2]), lora[n], sh)
    else:
        raise ValueError(schedule)

    logits = None
    if head is not None:
        loss, logits, hc = head_fwd(x, gf, H, targets, wl.rms_eps, sh.rb)
        dx = head_bwd(hc, logits, gf, H, targets, sh.rb)
    else:
        Gf = G.astype(F64)
        loss = float(np.sum(x * Gf))
        dx = Gf

    grads = [None] * L
    if schedule == "resident":
        for i in reversed(range(L)):
            dx, grads[i] = layer_bwd(dx, caches[i], Ws[i], lora[i], sh)
    else:
        for n in range(L, 2 * L):                    # backward reads n = L..2L-1
            i = 2 * L - 1 - n
            buf[n % 2] = copy_blob(blobs[i])
            reads.append(i)
            Wt = unpack_blob(buf[n % 2])
            _, c = layer_fwd(saved[i], Wt, lora[i], sh)   # recompute from the saved input
            dx, grads[i] = layer_bwd(dx, c, Wt, lora[i], sh)
    return {"loss": loss, "grads": grads, "logits": logits, "reads": reads, "dx_in": dx}


# ------------------------------------------------------------------------------------------
# preference step: DPO against the same base with the adapters switched off
# ------------------------------------------------------------------------------------------
# [TESS] (the paragraph on the economics of layer streaming) names DPO among the preference
# losses run over the streamed base and fixes its reference model: the same streamed base with
# the adapters switched off, so the reference costs one more forward pass of reads, not weights.
# The loss is the one of Rafailov et al., "Direct Preference Optimization: Your Language Model is
# Secretly a Reward Model" (2023): for a pair (chosen w, rejected l)
#     L = -log sigmoid(beta * ((pi_w - ref_w) - (pi_l - ref_l)))
# with pi / ref the sequence log-likelihood under the policy / reference. Readings: the batch holds
# the P chosen sequences first, then the P rejected ones (row-aligned pairs); a sequence's
# log-likelihood sums log softmax(logits_t)[target_t] over its positions whose mask is 1 (all
# positions when no mask is given); the step's loss is the mean over the P pairs.

def seq_logp(logits, targets, mask, nseq, seq):
    """Per-sequence sum over the masked positions of log softmax(logits_t)[target_t]."""
    mx = logits.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(logits - mx).sum(axis=1, keepdims=True)))[:, 0]
    T = logits.shape[0]
    lp = (logits[np.arange(T), targets] - lse) * mask
    return lp.reshape(nseq, seq).sum(axis=1), lse


def dpo_loss(pi, ref, beta):
    """Mean DPO loss over pairs and dL/dpi per sequence (pi, ref: [2P], chosen first)."""
    P = pi.shape[0] // 2
    z = beta * ((pi[:P] - ref[:P]) - (pi[P:] - ref[P:]))
    loss = float(np.mean(np.logaddexp(0.0, -z)))          # -log sigmoid(z)
    g = (1.0 / (1.0 + np.exp(-z)) - 1.0) * beta / P        # dL/dz_p * dz/dpi_w
    return loss, np.concatenate([g, -g])


def dpo_dlogits(logits, targets, mask, nseq, seq, ref, beta):
    """(loss, dL/dlogits, pi) of the DPO loss as a function of the policy logits [nseq*seq, V]:
    d pi_s / d logits_t = mask_t (onehot(target_t) - softmax(logits_t)) for t in sequence s."""
    pi, lse = seq_logp(logits, targets, mask, nseq, seq)
    loss, g = dpo_loss(pi, ref, beta)
    T = logits.shape[0]
    w = -np.repeat(g, seq) * mask
    dlog = np.exp(logits - lse[:, None])
    dlog[np.arange(T), targets] -= 1.0
    return loss, dlog * w[:, None], pi


def _forward(x, Ws, lora, sh):
    caches = []
    for i in range(len(Ws)):
        x, c = layer_fwd(x, Ws[i], lora[i], sh)
        caches.append(c)
    return x, caches


def dpo_step(wl, raw_layers, head, tokens, targets, npairs, beta, mask=None, blobs=None, bf16_acts=False,
             lora=None):
    """Loss and LoRA gradients of one DPO step on 2 * npairs sequences of wl.seq tokens.

    The reference pass runs every layer with the adapters off (B = 0 makes the side path exactly
    zero); the policy pass is the ordinary forward, then the head turns the per-sequence weights
    dL/dpi into dlogits = -w (softmax - onehot) on masked rows, and the backward is the SFT one.
    Returns dict(loss, grads, pi, ref).
    """
    L = wl.n_layers
    sh = Shape(wl, bf16_acts)
    nseq, S = 2 * npairs, wl.seq
    assert nseq == wl.batch
    if blobs is None:
        blobs = [pack_layer(raw_layers[i], wl.base_format) for i in range(L)]
    if lora is None:
        lora = [_lora64(raw_layers[i]) for i in range(L)]
    off = [{p: (a, np.zeros_like(b)) for p, (a, b) in lo.items()} for lo in lora]
    E, gf, H = (a.astype(F64) for a in head)
    T = nseq * S
    m = np.ones(T) if mask is None else np.asarray(mask, dtype=F64)
    Ws = [unpack_blob(blobs[i]) for i in range(L)]

    def head_logits(xL):
        n, r = rmsnorm(xL, gf, wl.rms_eps)
        n = sh.rb(n)
        return n @ H.T, (n, r)

    x_ref, _ = _forward(E[tokens], Ws, off, sh)
    ref, _ = seq_logp(head_logits(x_ref)[0], targets, m, nseq, S)

    x0 = E[tokens]
    xL, caches = _forward(x0, Ws, lora, sh)
    logits, (n, r) = head_logits(xL)
    loss, dlog, pi = dpo_dlogits(logits, targets, m, nseq, S, ref, beta)
    dx = rmsnorm_bwd(sh.rb(dlog) @ H, xL, gf, r)
    grads = [None] * L
    for i in reversed(range(L)):
        dx, grads[i] = layer_bwd(dx, caches[i], Ws[i], lora[i], sh)
    return {"loss": loss, "grads": grads, "pi": pi, "ref": ref}


# ------------------------------------------------------------------------------------------
# reference-free preference losses named next to DPO (ORPO, SimPO)
# ------------------------------------------------------------------------------------------
# [TESS] lists ORPO and SimPO (with DPO and KTO) among the preference losses run over the streamed
# base. Neither needs a reference model, so a step is the ordinary 2L reads. Losses as published:
# SimPO (Meng, Xia and Chen, "SimPO: Simple Preference Optimization with a Reference-Free Reward",
# 2024): reward r(y) = beta / |y| * log pi(y); L = -log sigmoid(r(y_w) - r(y_l) - gamma).
# ORPO (Hong, Lee and Thorne, "ORPO: Monolithic Preference Optimization without Reference Model",
# 2024): with l(y) = log pi(y) / |y| (length-normalised) and odds(y) = e^l / (1 - e^l),
# L = -l(y_w) + lambda * -log sigmoid(log odds(y_w) - log odds(y_l)).
# |y| is the number of masked positions of a sequence. Same batch layout and masks as DPO; the
# step's loss is the mean over pairs.

def simpo_loss(pi, counts, beta, gamma):
    """Mean SimPO loss over pairs and dL/dpi per sequence (pi, counts: [2P], chosen first)."""
    P = pi.shape[0] // 2
    r = beta * pi / counts
    z = r[:P] - r[P:] - gamma
    loss = float(np.mean(np.logaddexp(0.0, -z)))
    dz = (1.0 / (1.0 + np.exp(-z)) - 1.0) / P                # dL/dz per pair
    return loss, np.concatenate([dz * beta / counts[:P], -dz * beta / counts[P:]])


def orpo_loss(pi, counts, lam):
    """Mean ORPO loss over pairs and dL/dpi per sequence (pi, counts: [2P], chosen first)."""
    P = pi.shape[0] // 2
    ell = pi / counts                                        # mean log-likelihood per token, < 0
    log_odds = ell - np.log1p(-np.exp(ell))
    z = log_odds[:P] - log_odds[P:]
    loss = float(np.mean(-ell[:P] + lam * np.logaddexp(0.0, -z)))
    dz = lam * (1.0 / (1.0 + np.exp(-z)) - 1.0) / P           # d(mean lam * L_OR)/dz per pair
    dodds = 1.0 / (1.0 - np.exp(ell))                          # d log_odds / d ell
    d_ell = np.concatenate([-1.0 / P + dz * dodds[:P], -dz * dodds[P:]])
    return loss, d_ell / counts


def pref_dlogits(logits, targets, mask, nseq, seq, kind, **kw):
    """(loss, dL/dlogits, pi) of a reference-free preference loss (kind "simpo" or "orpo") as a
    function of the policy logits, the same way as ``dpo_dlogits``."""
    pi, lse = seq_logp(logits, targets, mask, nseq, seq)
    counts = np.asarray(mask, dtype=F64).reshape(nseq, seq).sum(axis=1)
    if kind == "simpo":
        loss, g = simpo_loss(pi, counts, kw["beta"], kw["gamma"])
    elif kind == "orpo":
        loss, g = orpo_loss(pi, counts, kw["lam"])
    else:
        raise ValueError(kind)
    T = logits.shape[0]
    w = -np.repeat(g, seq) * mask
    dlog = np.exp(logits - lse[:, None])
    dlog[np.arange(T), targets] -= 1.0
    return loss, dlog * w[:, None], pi


def pref_step(wl, raw_layers, head, tokens, targets, npairs, kind, mask=None, blobs=None, bf16_acts=False,
              lora=None, **kw):
    """Loss and LoRA gradients of one SimPO or ORPO step (no reference pass)."""
    L = wl.n_layers
    sh = Shape(wl, bf16_acts)
    nseq, S = 2 * npairs, wl.seq
    assert nseq == wl.batch
    if blobs is None:
        blobs = [pack_layer(raw_layers[i], wl.base_format) for i in range(L)]
    if lora is None:
        lora = [_lora64(raw_layers[i]) for i in range(L)]
    E, gf, H = (a.astype(F64) for a in head)
    m = np.ones(nseq * S) if mask is None else np.asarray(mask, dtype=F64)
    Ws = [unpack_blob(blobs[i]) for i in range(L)]
    xL, caches = _forward(E[tokens], Ws, lora, sh)
    n, r = rmsnorm(xL, gf, wl.rms_eps)
    logits = sh.rb(n) @ H.T
    loss, dlog, pi = pref_dlogits(logits, targets, m, nseq, S, kind, **kw)
    dx = rmsnorm_bwd(sh.rb(dlog) @ H, xL, gf, r)
    grads = [None] * L
    for i in reversed(range(L)):
        dx, grads[i] = layer_bwd(dx, caches[i], Ws[i], lora[i], sh)
    return {"loss": loss, "grads": grads, "pi": pi}
