"""Independent pin of the oracle's decoder-layer composition (CPU only).

The oracle's backward is pinned to its own forward by finite differences; this file pins the
forward itself -- the order of the pre-norm layer, where the residuals are taken, which projection
is the gate and which the up projection, which tensors are rotated -- against a second model
written only from library operations (torch fp64 autograd on the CPU): ``F.rms_norm``,
``F.linear``, ``F.scaled_dot_product_attention`` (causal, grouped-query), ``F.silu`` and
``F.cross_entropy``, with rotate-half RoPE written out. The layer is the Llama / Qwen2 pre-norm
decoder the workloads name ("Llama-style", "Qwen2.5-shaped"); the LoRA form is
y = x W^T + s (x A^T) B^T ("Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU", section
"LoRA and QLoRA"). Both models compute from the same dequantised base weights (NF4 is pinned in
test_oracle_nf4.py) and the same fp32 adapters, in fp64 with no rounding.

A mistake planted in the oracle's forward (gate and up roles swapped inside SwiGLU, RoPE applied
to v, the attention residual taken from the normalised input) must make the two disagree.
"""
import inspect

import numpy as np
import pytest

import synthetic as syn
from oracle import model as M

torch = pytest.importorskip("torch")
F = torch.nn.functional

TOL = 1e-12  # fp64 on both sides; observed agreement is ~3e-15


def _t(a):
    return torch.tensor(np.asarray(a, dtype=np.float64))


def _rotate_half(x):
    h = x.shape[-1] // 2
    return torch.cat([-x[..., h:], x[..., :h]], dim=-1)


def torch_step(wl, inp):
    """Loss, logits and every adapter gradient of one step, by torch autograd."""
    B, S, d = wl.batch, wl.seq, wl.d_model
    T = B * S
    hq, hkv, hd = wl.n_heads, wl.n_kv_heads, wl.head_dim
    s = wl.lora_alpha / wl.lora_rank
    pos = torch.arange(S, dtype=torch.float64)
    inv = wl.rope_theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    ang = torch.cat([pos[:, None] * inv[None, :]] * 2, dim=-1)        # [S, hd]
    cos, sin = torch.cos(ang), torch.sin(ang)
    adapters = []
    if wl.vocab:
        E, gf, H = (_t(a) for a in inp["head"])
        x = E[torch.tensor(inp["tokens"], dtype=torch.long)]
    else:
        x = _t(inp["x_in"])
    for raw in inp["raw"]:
        Wt = M.unpack_blob(M.pack_layer(raw, wl.base_format))
        W = {p: _t(Wt["W"][p]) for p in M.PROJ}
        A = {p: _t(raw["A"][p]).requires_grad_() for p in M.PROJ}
        Bm = {p: _t(raw["B"][p]).requires_grad_() for p in M.PROJ}
        adapters.append((A, Bm))
        bias = {p: _t(raw["bias"][p]) for p in ("q", "k", "v")} if raw["bias"] is not None else {}

        def lin(z, p):
            return F.linear(z, W[p], bias.get(p)) + s * F.linear(F.linear(z, A[p]), Bm[p])

        n1 = F.rms_norm(x, (d,), weight=_t(raw["attn_norm"]), eps=wl.rms_eps)
        q = lin(n1, "q").view(B, S, hq, hd).transpose(1, 2)
        k = lin(n1, "k").view(B, S, hkv, hd).transpose(1, 2)
        v = lin(n1, "v").view(B, S, hkv, hd).transpose(1, 2)
        q = q * cos + _rotate_half(q) * sin
        k = k * cos + _rotate_half(k) * sin
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=hq != hkv)
        h = x + lin(o.transpose(1, 2).reshape(T, hq * hd), "o")
        n2 = F.rms_norm(h, (d,), weight=_t(raw["mlp_norm"]), eps=wl.rms_eps)
        x = h + lin(F.silu(lin(n2, "gate")) * lin(n2, "up"), "down")
    logits = None
    if wl.vocab:
        logits = F.linear(F.rms_norm(x, (d,), weight=gf, eps=wl.rms_eps), H)
        loss = F.cross_entropy(logits, torch.tensor(inp["targets"], dtype=torch.long))
    else:
        loss = (x * _t(inp["G"])).sum()
    loss.backward()
    grads = [{p: (A[p].grad.numpy(), Bm[p].grad.numpy()) for p in M.PROJ} for A, Bm in adapters]
    return {"loss": float(loss.detach()), "grads": grads,
            "logits": None if logits is None else logits.detach().numpy()}


def _inputs(wl):
    d = {"raw": [syn.layer_weights(wl, i) for i in range(wl.n_layers)]}
    if wl.vocab:
        d["head"] = (syn.embedding(wl), syn.norm_gain(wl), syn.lm_head(wl))
        d["tokens"], d["targets"] = syn.tokens(wl)
    else:
        d["x_in"], d["G"] = syn.hidden_input(wl), syn.output_grad(wl)
    return d


def _oracle(wl, inp):
    kw = dict(raw_layers=inp["raw"], schedule="resident", bf16_acts=False)
    if wl.vocab:
        kw.update(head=inp["head"], tokens=inp["tokens"], targets=inp["targets"])
    else:
        kw.update(x_in=inp["x_in"], G=inp["G"])
    return M.step(wl, **kw)


def _distance(a, b):
    """Largest max|got - ref| / max|ref| over the loss, the logits and every gradient tensor."""
    def mr(x, y):
        x, y = np.asarray(x, np.float64), np.asarray(y, np.float64)
        return float(np.abs(x - y).max() / (np.abs(y).max() + 1e-300))
    worst = mr(a["loss"], b["loss"])
    if b["logits"] is not None:
        worst = max(worst, mr(a["logits"], b["logits"]))
    for ga, gb in zip(a["grads"], b["grads"]):
        for p in M.PROJ:
            worst = max(worst, mr(ga[p][0], gb[p][0]), mr(ga[p][1], gb[p][1]))
    return worst


WORKLOADS = {
    # the tiny stack: NF4 base, multi-head attention, LM head + cross-entropy
    "tiny": syn.WORKLOADS["tiny"],
    # grouped-query attention, q/k/v bias, unquantised bf16 base, ragged length, with the head
    "gqa_bias_bf16": syn.WORKLOADS["tiny"].with_(n_kv_heads=2, qkv_bias=True, base_format="bf16", batch=3,
                                                 seq=37),
    # the same without a head (loss = sum(x_L * G))
    "gqa_headless": syn.WORKLOADS["tiny"].with_(n_kv_heads=1, vocab=0, batch=2, seq=24, n_layers=1),
}


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_oracle_step_equals_torch_autograd(name):
    wl = WORKLOADS[name]
    inp = _inputs(wl)
    assert _distance(_oracle(wl, inp), torch_step(wl, inp)) <= TOL


# A mistake planted in the oracle's forward, as a source edit of layer_fwd: (original, planted).
PLANTS = {
    "swiglu_gate_up_swapped": ("m = rb(silu(g) * u)", "m = rb(silu(u) * g)"),
    "rope_on_v": ('v = rb(c["v_pre"].reshape(T, sh.hkv, sh.hd))',
                  'v = rb(rope(c["v_pre"].reshape(T, sh.hkv, sh.hd), sh.cos, sh.sin, sh.batch, sh.seq))'),
    "residual_from_n1": ("h = x + ao", "h = n1 + ao"),
}


@pytest.mark.parametrize("plant", list(PLANTS))
def test_planted_forward_mistakes_are_caught(monkeypatch, plant):
    wl = WORKLOADS["gqa_bias_bf16"].with_(n_layers=1)
    inp = _inputs(wl)
    ref = torch_step(wl, inp)
    assert _distance(_oracle(wl, inp), ref) <= TOL
    orig, planted = PLANTS[plant]
    src = inspect.getsource(M.layer_fwd)
    assert src.count(orig) == 1
    ns = dict(vars(M))
    exec(compile(src.replace(orig, planted), "<planted layer_fwd>", "exec"), ns)
    monkeypatch.setattr(M, "layer_fwd", ns["layer_fwd"])
    assert _distance(_oracle(wl, inp), ref) > 1e-3
