"""Pins of the oracle's decoder stack, LoRA, head and backward (CPU only).

Each test checks the oracle against something other than itself: closed forms and special
cases, brute-force loops in pure Python, torch's cross-entropy, and central finite differences
of the oracle's own loss (the backward is derived by hand, the differences need no derivation).
"""
import math

import numpy as np
import pytest

import synthetic as syn
from oracle import model as M
from oracle import nf4


def tiny(**kw):
    return syn.WORKLOADS["tiny"].with_(**kw)


def build(wl):
    raw = [syn.layer_weights(wl, i) for i in range(wl.n_layers)]
    head = None
    toks = tgts = x_in = G = None
    if wl.vocab:
        head = (syn.embedding(wl), syn.norm_gain(wl), syn.lm_head(wl))
        toks, tgts = syn.tokens(wl)
    else:
        x_in, G = syn.hidden_input(wl), syn.output_grad(wl)
    blobs = [M.pack_layer(r, wl.base_format) for r in raw]
    return dict(raw_layers=raw, blobs=blobs, head=head, tokens=toks, targets=tgts, x_in=x_in, G=G)


# ---------------------------------------------------------------- building blocks

def test_lora_b_zero_is_base_output_exactly():
    rng = np.random.default_rng(0)
    x, W, A = rng.normal(size=(5, 64)), rng.normal(size=(32, 64)), rng.normal(size=(4, 64))
    y, _ = M.lora_linear(x, W, A, np.zeros((32, 4)), 2.0)
    assert np.array_equal(y, x @ W.T)


def test_lora_merged_weight_identity():
    rng = np.random.default_rng(1)
    x, W = rng.normal(size=(7, 48)), rng.normal(size=(24, 48))
    A, B = rng.normal(size=(8, 48)), rng.normal(size=(24, 8))
    y, _ = M.lora_linear(x, W, A, B, 2.0)
    np.testing.assert_allclose(y, x @ (W + 2.0 * B @ A).T, rtol=1e-12, atol=1e-12)


def test_rmsnorm_special_cases():
    g = np.linspace(0.5, 1.5, 16)
    y, _ = M.rmsnorm(np.full((3, 16), 3.0), g, 1e-5)
    np.testing.assert_allclose(y, np.tile(3.0 / math.sqrt(9.0 + 1e-5) * g, (3, 1)), rtol=1e-14)
    y0, _ = M.rmsnorm(np.zeros((2, 16)), g, 1e-5)
    assert np.all(y0 == 0)


def test_rope_identity_at_zero_norm_preserving_and_inverse():
    cos, sin = M.rope_tables(8, 16, 1e4)
    rng = np.random.default_rng(2)
    x = rng.normal(size=(16, 3, 16))                         # batch 2 x seq 8
    y = M.rope(x, cos, sin, 2, 8)
    assert np.array_equal(y[0], x[0]) and np.array_equal(y[8], x[8])   # position 0
    pair = lambda z: z[..., :8] ** 2 + z[..., 8:] ** 2
    np.testing.assert_allclose(pair(y), pair(x), rtol=1e-12)
    np.testing.assert_allclose(M.rope_bwd(y, cos, sin, 2, 8), x, rtol=1e-12, atol=1e-12)
    # the angle of pair j at position t is t * theta^(-2j/hd)
    t, j = 5, 3
    ang = t * 1e4 ** (-2 * j / 16)
    e = np.zeros((16, 1, 16)); e[t, 0, j] = 1.0
    r = M.rope(e, cos, sin, 2, 8)
    assert abs(r[t, 0, j] - math.cos(ang)) < 1e-14 and abs(r[t, 0, j + 8] - math.sin(ang)) < 1e-14


def _attn_bruteforce(q, k, v, batch, seq):
    T, hq, hd = q.shape
    grp = hq // k.shape[1]
    o = np.zeros_like(q)
    for b in range(batch):
        for h in range(hq):
            for i in range(seq):
                ti = b * seq + i
                sc = [sum(q[ti, h, c] * k[b * seq + j, h // grp, c] for c in range(hd)) / math.sqrt(hd)
                      for j in range(i + 1)]
                m = max(sc)
                e = [math.exp(s - m) for s in sc]
                z = sum(e)
                for c in range(hd):
                    o[ti, h, c] = sum(e[j] / z * v[b * seq + j, h // grp, c] for j in range(i + 1))
    return o


def test_attention_brute_force_gqa():
    rng = np.random.default_rng(3)
    q, k, v = rng.normal(size=(10, 4, 4)), rng.normal(size=(10, 2, 4)), rng.normal(size=(10, 2, 4))
    o, P = M.attention(q, k, v, 2, 5)
    np.testing.assert_allclose(o, _attn_bruteforce(q, k, v, 2, 5), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(P.sum(axis=-1), 1.0, rtol=1e-13)


def test_attention_seq1_is_v_and_gqa_equals_repeated_mha():
    rng = np.random.default_rng(4)
    q, k, v = rng.normal(size=(3, 4, 8)), rng.normal(size=(3, 2, 8)), rng.normal(size=(3, 2, 8))
    o, _ = M.attention(q, k, v, 3, 1)
    np.testing.assert_allclose(o, np.repeat(v, 2, axis=1), rtol=1e-14)
    q, k, v = rng.normal(size=(12, 6, 8)), rng.normal(size=(12, 2, 8)), rng.normal(size=(12, 2, 8))
    o1, _ = M.attention(q, k, v, 2, 6)
    o2, _ = M.attention(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), 2, 6)
    np.testing.assert_allclose(o1, o2, rtol=1e-13)


def test_cross_entropy_matches_torch_and_zero_logits():
    import torch
    rng = np.random.default_rng(5)
    x = rng.normal(size=(6, 16))
    H = rng.normal(size=(50, 16)) * 0.3
    gf = np.ones(16)
    y = rng.integers(0, 50, size=6)
    loss, logits, _ = M.head_fwd(x, gf, H, y, 1e-5)
    ref = torch.nn.functional.cross_entropy(torch.tensor(logits), torch.tensor(y)).item()
    assert abs(loss - ref) < 1e-12
    loss0, _, _ = M.head_fwd(x, gf, np.zeros((1024, 16)), y, 1e-5)
    assert abs(loss0 - math.log(1024)) < 1e-12


def test_swiglu_silu_closed_form():
    g = np.array([-3.0, 0.0, 2.0])
    np.testing.assert_allclose(M.silu(g), g / (1 + np.exp(-g)))
    assert M.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(M.silu(np.array([40.0])), [40.0], rtol=1e-15)


# ---------------------------------------------------------------- whole step

def test_initial_loss_near_log_vocab():
    wl = tiny()
    r = M.step(wl, **build(wl))
    assert abs(r["loss"] - math.log(wl.vocab)) < 0.2


def test_streamed_equals_resident_bitwise():
    wl = tiny(n_layers=3)
    inp = build(wl)
    a = M.step(wl, schedule="resident", **inp)
    b = M.step(wl, schedule="streamed", **inp)
    assert a["loss"] == b["loss"]
    assert b["reads"] == [0, 1, 2, 2, 1, 0]
    for la, lb in zip(a["grads"], b["grads"]):
        for p in M.PROJ:
            assert np.array_equal(la[p][0], lb[p][0]) and np.array_equal(la[p][1], lb[p][1])


def test_adapter_changes_output():
    # an adapter that silently does nothing must be caught: B != 0 changes the loss
    wl = tiny(n_layers=1)
    inp = build(wl)
    base = M.step(wl, lora=[{p: (a.astype(float), np.zeros_like(b, dtype=float))
                             for p, (a, b) in {p: (inp["raw_layers"][0]["A"][p], inp["raw_layers"][0]["B"][p])
                                                for p in M.PROJ}.items()}], **inp)["loss"]
    with_ad = M.step(wl, **inp)["loss"]
    assert base != with_ad


def _fd_check(wl, picks, h=1e-4, rtol=1e-6):
    inp = build(wl)
    ref = M.step(wl, **inp)
    lora0 = [{p: (r["A"][p].astype(np.float64), r["B"][p].astype(np.float64)) for p in M.PROJ}
             for r in inp["raw_layers"]]
    rng = np.random.default_rng(7)
    for layer, proj, which in picks:
        an = ref["grads"][layer][proj][which]
        scale = np.abs(an).max()
        for _ in range(2):
            idx = tuple(rng.integers(0, s) for s in an.shape)
            vals = []
            for sgn in (1, -1):
                lora = [{p: (A.copy(), B.copy()) for p, (A, B) in l.items()} for l in lora0]
                lora[layer][proj][which][idx] += sgn * h
                vals.append(M.step(wl, lora=lora, **inp)["loss"])
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - an[idx]) <= rtol * scale + 1e-11, (layer, proj, which, idx, fd, an[idx])


def test_backward_matches_finite_differences_tiny():
    wl = tiny()
    picks = [(l, p, w) for l in (0, 1) for p in M.PROJ for w in (0, 1)]
    _fd_check(wl, picks)


def test_backward_finite_differences_gqa_bias_bf16_headless():
    # GQA (hkv=2 of 4 heads), q/k/v bias, unquantised bf16 base, headless loss sum(x_L * G)
    wl = tiny(n_kv_heads=2, qkv_bias=True, base_format="bf16", vocab=0, n_layers=2)
    picks = [(l, p, w) for l in (0, 1) for p in ("q", "k", "v", "o", "down") for w in (0, 1)]
    _fd_check(wl, picks)


def test_input_gradient_matches_finite_differences_headless():
    wl = tiny(n_kv_heads=2, vocab=0, n_layers=1)
    inp = build(wl)
    ref = M.step(wl, **inp)
    rng = np.random.default_rng(8)
    h = 1e-4
    for _ in range(6):
        t, c = rng.integers(0, wl.tokens), rng.integers(0, wl.d_model)
        vals = []
        for sgn in (1, -1):
            x = inp["x_in"].astype(np.float64).copy()
            x[t, c] += sgn * h
            vals.append(M.step(wl, **{**inp, "x_in": x})["loss"])
        fd = (vals[0] - vals[1]) / (2 * h)
        assert abs(fd - ref["dx_in"][t, c]) <= 1e-6 * np.abs(ref["dx_in"]).max() + 1e-9


def test_bf16_rounding_matches_torch_and_bf16_mode_is_consistent():
    import torch
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.normal(size=10000), rng.normal(size=1000) * 1e-30,
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()   # library routine
    assert np.array_equal(nf4.bf16_value(x), ref)
    # bf16 mode: streamed == resident bitwise, and close to the exact mode
    wl = tiny(n_layers=2)
    inp = build(wl)
    a = M.step(wl, schedule="resident", bf16_acts=True, **inp)
    b = M.step(wl, schedule="streamed", bf16_acts=True, **inp)
    e = M.step(wl, schedule="resident", bf16_acts=False, **inp)
    assert a["loss"] == b["loss"]
    assert abs(a["loss"] - e["loss"]) < 1e-3 * abs(e["loss"])
    assert a["loss"] != e["loss"]          # the rounding is really applied


def test_adamw_matches_torch():
    import torch
    from oracle import optim
    rng = np.random.default_rng(12)
    p0 = rng.normal(size=500)
    grads = [rng.normal(size=500) * s for s in (1e-3, 1e-1, 1.0)]
    tp = torch.tensor(p0.copy(), dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=1e-2, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    p, m, v = p0.copy(), np.zeros(500), np.zeros(500)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g)
        opt.step()
        p, m, v = optim.adamw_step(p, g, m, v, t, lr=1e-2, b1=0.9, b2=0.95, eps=1e-8, wd=0.1)
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- DPO (preference step)
def _dpo_inputs(wl):
    raw = [syn.layer_weights(wl, i) for i in range(wl.n_layers)]
    head = (syn.embedding(wl), syn.norm_gain(wl), syn.lm_head(wl))
    toks, tgts, mask = syn.preference_pairs(wl)
    return raw, head, toks, tgts, mask


def test_dpo_loss_is_log2_when_policy_equals_reference():
    # B = 0 on every adapter: the policy is the reference, so z = 0 and the loss is ln 2
    wl = tiny(batch=4)
    raw, head, toks, tgts, mask = _dpo_inputs(wl)
    lora = [{p: (r["A"][p].astype(np.float64), np.zeros_like(r["B"][p], dtype=np.float64)) for p in M.PROJ}
            for r in raw]
    out = M.dpo_step(wl, raw, head, toks, tgts, 2, 0.1, mask=mask, lora=lora)
    assert np.array_equal(out["pi"], out["ref"])
    assert out["loss"] == math.log(2.0)
    # the gradient is still live: dL/dz = -1/2 at z = 0
    assert any(np.abs(dB).max() > 0 for g in out["grads"] for (_, dB) in g.values())


def test_dpo_identical_pair_has_no_gradient():
    # chosen == rejected: both sequences get opposite weights, so every gradient cancels
    wl = tiny(batch=2)
    raw, head, toks, tgts, mask = _dpo_inputs(wl)
    S = wl.seq
    toks[S:], tgts[S:], mask[S:] = toks[:S], tgts[:S], mask[:S]
    out = M.dpo_step(wl, raw, head, toks, tgts, 1, 0.5, mask=mask)
    assert abs(out["loss"] - math.log(2.0)) < 1e-15
    for g in out["grads"]:
        for dA, dB in g.values():
            assert np.abs(dA).max() < 1e-14 and np.abs(dB).max() < 1e-14


def test_dpo_logit_gradient_matches_torch_autograd():
    # the loss as a function of the logits, differentiated by torch on CPU (fp64)
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    nseq, S, V, beta = 4, 6, 11, 0.3
    logits = rng.normal(size=(nseq * S, V)) * 2
    tg = rng.integers(0, V, nseq * S)
    mask = (rng.random(nseq * S) < 0.7).astype(np.float64)
    ref = rng.normal(size=nseq) * 3
    loss, dlog, pi = M.dpo_dlogits(logits, tg, mask, nseq, S, ref, beta)
    lt = torch.tensor(logits, requires_grad=True)
    lp = torch.log_softmax(lt, dim=1).gather(1, torch.tensor(tg)[:, None])[:, 0] * torch.tensor(mask)
    pit = lp.reshape(nseq, S).sum(1)
    r = torch.tensor(ref)
    P = nseq // 2
    z = beta * ((pit[:P] - r[:P]) - (pit[P:] - r[P:]))
    lt_loss = -torch.nn.functional.logsigmoid(z).mean()
    lt_loss.backward()
    assert abs(float(lt_loss.detach()) - loss) < 1e-12
    assert np.allclose(pit.detach().numpy(), pi, rtol=0, atol=1e-12)
    assert np.allclose(lt.grad.numpy(), dlog, rtol=0, atol=1e-13)


def test_dpo_backward_matches_finite_differences():
    wl = tiny(batch=2, n_layers=1)
    raw, head, toks, tgts, mask = _dpo_inputs(wl)
    lora0 = [{p: (r["A"][p].astype(np.float64), r["B"][p].astype(np.float64)) for p in M.PROJ} for r in raw]
    ref = M.dpo_step(wl, raw, head, toks, tgts, 1, 0.5, mask=mask, lora=lora0)
    rng = np.random.default_rng(11)
    h = 1e-4
    for proj in M.PROJ:
        for which in (0, 1):
            an = ref["grads"][0][proj][which]
            idx = tuple(rng.integers(0, s) for s in an.shape)
            vals = []
            for sgn in (1, -1):
                lora = [{p: (A.copy(), B.copy()) for p, (A, B) in l.items()} for l in lora0]
                lora[0][proj][which][idx] += sgn * h
                vals.append(M.dpo_step(wl, raw, head, toks, tgts, 1, 0.5, mask=mask, lora=lora)["loss"])
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - an[idx]) <= 1e-6 * np.abs(an).max() + 1e-11, (proj, which, fd, an[idx])


def test_preference_pairs_share_prompts_and_mask_responses():
    wl = tiny(batch=6, seq=10)
    t, y, m = syn.preference_pairs(wl)
    P, S = 3, 10
    t, y, m = t.reshape(2 * P, S), y.reshape(2 * P, S), m.reshape(2 * P, S)
    assert np.array_equal(t[:P, :S // 2], t[P:, :S // 2]) and np.array_equal(y[:P, :S // 2], y[P:, :S // 2])
    assert not np.array_equal(t[:P, S // 2:], t[P:, S // 2:])          # responses differ
    assert np.all(m[:, :S // 2] == 0) and np.all(m[:, S // 2:] == 1)
    assert t.min() >= 0 and t.max() < wl.vocab and y.max() < wl.vocab
    t2, _, _ = syn.preference_pairs(wl)
    assert np.array_equal(t.reshape(-1), t2)                               # seeded


def _fd_discrepancy(wl, picks, h=1e-4):
    """max over picks of |central difference - analytic| / max|analytic| of the oracle's loss."""
    inp = build(wl)
    ref = M.step(wl, **inp)
    lora0 = [{p: (r["A"][p].astype(np.float64), r["B"][p].astype(np.float64)) for p in M.PROJ}
             for r in inp["raw_layers"]]
    rng = np.random.default_rng(5)
    worst = 0.0
    for layer, proj, which in picks:
        an = ref["grads"][layer][proj][which]
        idx = tuple(rng.integers(0, s) for s in an.shape)
        vals = []
        for sgn in (1, -1):
            lora = [{p: (A.copy(), B.copy()) for p, (A, B) in l.items()} for l in lora0]
            lora[layer][proj][which][idx] += sgn * h
            vals.append(M.step(wl, lora=lora, **inp)["loss"])
        fd = (vals[0] - vals[1]) / (2 * h)
        worst = max(worst, abs(fd - an[idx]) / np.abs(an).max())
    return worst


@pytest.mark.parametrize("plant", ["rope_sign", "rmsnorm_term", "dv_scale"])
def test_planted_backward_mistakes_fail_the_difference_check(monkeypatch, plant):
    # a mistake planted in the oracle's backward (on the CPU) must show up against central
    # differences of its own forward; the clean backward agrees to ~1e-7
    wl = tiny(n_layers=1, n_kv_heads=2)
    picks = [(0, p, w) for p in ("q", "k", "v") for w in (0, 1)]
    clean = _fd_discrepancy(wl, picks)
    assert clean < 1e-6
    if plant == "rope_sign":
        monkeypatch.setattr(M, "rope_bwd", lambda dy, cos, sin, b, s: M.rope(dy, cos, sin, b, s))
    elif plant == "rmsnorm_term":
        def no_mean_term(dy, x, g, r):
            return dy * g[None, :] * r[:, None]
        monkeypatch.setattr(M, "rmsnorm_bwd", no_mean_term)
    else:
        orig = M.attention_bwd
        monkeypatch.setattr(M, "attention_bwd", lambda *a: (lambda dq, dk, dv: (dq, dk, dv * 1.01))(*orig(*a)))
    assert _fd_discrepancy(wl, picks) > 100 * max(clean, 1e-9)


# ---------------------------------------------------------------- SimPO / ORPO (reference-free)
@pytest.mark.parametrize("kind", ["simpo", "orpo"])
def test_reference_free_losses_match_torch_autograd(kind):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(4)
    nseq, S, V = 4, 7, 13
    logits = rng.normal(size=(nseq * S, V)) * 2
    tg = rng.integers(0, V, nseq * S)
    mask = (rng.random(nseq * S) < 0.7).astype(np.float64)
    mask.reshape(nseq, S)[:, 0] = 1.0                        # every sequence counts a position
    kw = {"beta": 2.0, "gamma": 0.3} if kind == "simpo" else {"lam": 0.25}
    loss, dlog, pi = M.pref_dlogits(logits, tg, mask, nseq, S, kind, **kw)
    lt = torch.tensor(logits, requires_grad=True)
    lp = torch.log_softmax(lt, dim=1).gather(1, torch.tensor(tg)[:, None])[:, 0] * torch.tensor(mask)
    pit = lp.reshape(nseq, S).sum(1)
    cnt = torch.tensor(mask).reshape(nseq, S).sum(1)
    P = nseq // 2
    F = torch.nn.functional
    if kind == "simpo":
        r = kw["beta"] * pit / cnt
        lt_loss = -F.logsigmoid(r[:P] - r[P:] - kw["gamma"]).mean()
    else:
        ell = pit / cnt
        lo = ell - torch.log1p(-torch.exp(ell))
        lt_loss = (-ell[:P] - kw["lam"] * F.logsigmoid(lo[:P] - lo[P:])).mean()
    lt_loss.backward()
    assert abs(float(lt_loss.detach()) - loss) < 1e-12
    assert np.allclose(pit.detach().numpy(), pi, rtol=0, atol=1e-12)
    assert np.allclose(lt.grad.numpy(), dlog, rtol=0, atol=1e-13)


def test_reference_free_losses_closed_forms_on_identical_pairs():
    # chosen == rejected: SimPO's margin term alone remains and its gradient cancels; ORPO keeps
    # its SFT term on the chosen sequence
    wl = tiny(batch=2, n_layers=1)
    raw, head, toks, tgts, mask = _dpo_inputs(wl)
    S = wl.seq
    toks[S:], tgts[S:], mask[S:] = toks[:S], tgts[:S], mask[:S]
    out = M.pref_step(wl, raw, head, toks, tgts, 1, "simpo", mask=mask, beta=2.0, gamma=0.5)
    assert abs(out["loss"] - math.log1p(math.exp(0.5))) < 1e-14
    for g in out["grads"]:
        for dA, dB in g.values():
            assert np.abs(dA).max() < 1e-14 and np.abs(dB).max() < 1e-14
    out = M.pref_step(wl, raw, head, toks, tgts, 1, "orpo", mask=mask, lam=0.1)
    ell = out["pi"][0] / mask[:S].sum()
    assert abs(out["loss"] - (-ell + 0.1 * math.log(2.0))) < 1e-12
    assert any(np.abs(dB).max() > 0 for g in out["grads"] for (_, dB) in g.values())


@pytest.mark.parametrize("kind", ["simpo", "orpo"])
def test_reference_free_backward_matches_finite_differences(kind):
    wl = tiny(batch=2, n_layers=1)
    raw, head, toks, tgts, mask = _dpo_inputs(wl)
    kw = {"beta": 2.0, "gamma": 0.3} if kind == "simpo" else {"lam": 0.5}
    lora0 = [{p: (r["A"][p].astype(np.float64), r["B"][p].astype(np.float64)) for p in M.PROJ} for r in raw]
    ref = M.pref_step(wl, raw, head, toks, tgts, 1, kind, mask=mask, lora=lora0, **kw)
    rng = np.random.default_rng(12)
    h = 1e-4
    for proj in ("q", "v", "up", "down"):
        for which in (0, 1):
            an = ref["grads"][0][proj][which]
            idx = tuple(rng.integers(0, s) for s in an.shape)
            vals = []
            for sgn in (1, -1):
                lora = [{p: (A.copy(), B.copy()) for p, (A, B) in l.items()} for l in lora0]
                lora[0][proj][which][idx] += sgn * h
                vals.append(M.pref_step(wl, raw, head, toks, tgts, 1, kind, mask=mask, lora=lora, **kw)["loss"])
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - an[idx]) <= 1e-6 * np.abs(an).max() + 1e-11, (kind, proj, which, fd, an[idx])
