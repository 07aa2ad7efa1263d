"""Step-level parity (GPU): loss, logits and every LoRA gradient of the library against the oracle,
streamed == resident byte for byte, and determinism. All calls go through the C ABI (lst.h)."""
import numpy as np
import pytest

import synthetic as syn
from helpers import (EXACT_GRAD_MAXREL, EXACT_LOGITS_MAXREL, GRAD_COS, GRAD_MAXREL, LOGITS_MAXREL, LOSS_RTOL,
                     build_inputs, compare_grads, make_context, maxrel, oracle_step, run_step)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check_against_oracle(wl, inp, loss, grads, logits, ctx, exact_too=True):
    """primary: the oracle with the workload's bf16 activations, at the parity tolerances (loss and
    logits 1e-2, every gradient tensor cosine >= 0.999 and max-rel <= 2e-2); secondary: the exact
    oracle, at the bounds of bf16 noise (helpers.py). Returns the worst (tensor, cosine, max-rel)
    of each comparison."""
    ref = oracle_step(wl, inp, schedule="streamed", bf16_acts=True)
    assert abs(loss - ref["loss"]) <= LOSS_RTOL * abs(ref["loss"]), (loss, ref["loss"])
    if logits is not None:
        assert maxrel(logits, ref["logits"]) <= LOGITS_MAXREL, maxrel(logits, ref["logits"])
    res = compare_grads(ctx, grads, ref["grads"])
    for l, p, w, cs, mr in res:
        assert cs >= GRAD_COS and mr <= GRAD_MAXREL, (l, p, w, cs, mr)
    worst = {"bf16": max(res, key=lambda t: t[4])}
    if not exact_too:
        return worst
    ex = oracle_step(wl, inp, schedule="streamed", bf16_acts=False)
    assert abs(loss - ex["loss"]) <= LOSS_RTOL * abs(ex["loss"]), (loss, ex["loss"])
    if logits is not None:
        assert maxrel(logits, ex["logits"]) <= EXACT_LOGITS_MAXREL, maxrel(logits, ex["logits"])
    res = compare_grads(ctx, grads, ex["grads"])
    for l, p, w, cs, mr in res:
        assert cs >= GRAD_COS and mr <= EXACT_GRAD_MAXREL, ("exact", l, p, w, cs, mr)
    worst["exact"] = max(res, key=lambda t: t[4])
    return worst


WORKLOADS = {
    "tiny": syn.WORKLOADS["tiny"],
    # GQA, q/k/v bias, bf16 base, ragged sequence (S=100 is not a multiple of the 64-row tiles)
    "tiny_gqa_bias_bf16": syn.WORKLOADS["tiny"].with_(n_kv_heads=2, qkv_bias=True, base_format="bf16",
                                                      batch=3, seq=100),
    # one Llama-3.1-8B-shaped layer (headless), shorter sequence
    "llama8b_layer_T256": syn.WORKLOADS["llama8b_layer"].with_(batch=1, seq=256),
    # two Qwen2.5-3B-shaped layers with the bf16 base and the full head
    "qwen3b_bf16_2L": syn.WORKLOADS["qwen3b_bf16"].with_(n_layers=2, batch=2, seq=128),
}


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_step_matches_oracle_and_streamed_equals_resident(name):
    wl = WORKLOADS[name]
    inp = build_inputs(wl)
    ctx_s = make_context(wl, inp, streamed=True)
    loss_s, g_s, lg_s = run_step(ctx_s, wl, inp)
    st = ctx_s.stats()
    assert st["layer_reads_last_step"] == 2 * wl.n_layers
    ctx_s.close()
    ctx_r = make_context(wl, inp, streamed=False)
    loss_r, g_r, lg_r = run_step(ctx_r, wl, inp)
    ctx_r.close()
    # streamed and resident runs are the same bytes
    assert np.float32(loss_s).tobytes() == np.float32(loss_r).tobytes()
    assert g_s.tobytes() == g_r.tobytes()
    if lg_s is not None:
        assert lg_s.tobytes() == lg_r.tobytes()
    _check_against_oracle(wl, inp, loss_s, g_s, lg_s, ctx_s)


def test_deterministic_and_adapters_matter():
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    a = run_step(ctx, wl, inp)
    b = run_step(ctx, wl, inp)
    assert a[0] == b[0] and a[1].tobytes() == b[1].tobytes()
    # B = 0 on every projection gives a different loss (adapters are live), and then dA == 0
    for l in range(wl.n_layers):
        for j, p in enumerate(syn.PROJ):
            ctx.set_lora(l, j, inp["raw"][l]["A"][p], np.zeros_like(inp["raw"][l]["B"][p]))
    c = run_step(ctx, wl, inp)
    assert c[0] != a[0]
    from helpers import split_grads
    for (l, p), (dA, dB) in split_grads(ctx, c[1]).items():
        assert np.all(dA == 0)
        assert np.any(dB != 0)
    ctx.close()


@pytest.mark.parametrize("name", ["tiny", "qwen3b_bf16_2L"])
def test_reuse_schedule_same_bytes_fewer_reads(name):
    # keeping layers resident in the pool (turnaround, and across steps) changes the copies only
    wl = WORKLOADS[name].with_(n_layers=3) if name == "tiny" else WORKLOADS[name]
    L = wl.n_layers
    inp = build_inputs(wl)
    runs = {}
    for reuse in (False, True):
        ctx = make_context(wl, inp, streamed=True, reuse=reuse)
        out, reads = [], []
        for _ in range(3):
            out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
            reads.append(ctx.stats()["layer_reads_last_step"])
        # a re-registered layer is copied again on the next step
        r = inp["raw"][0]
        ctx.register_layer(0, r["W"], r["A"], r["B"], r["attn_norm"], r["mlp_norm"], r["bias"])
        out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
        reads.append(ctx.stats()["layer_reads_last_step"])
        ctx.close()
        runs[reuse] = (out, reads)
    for (la, ga), (lb, gb) in zip(runs[False][0], runs[True][0]):
        assert np.float32(la).tobytes() == np.float32(lb).tobytes()
        assert ga.tobytes() == gb.tobytes()
    assert runs[False][1] == [2 * L] * 4
    assert runs[True][1] == [2 * L - 2, max(2 * L - 4, 0), max(2 * L - 4, 0), 2 * L - 2]


@pytest.mark.parametrize("chunk", [48, 64])
def test_head_in_passes_same_bytes(chunk):
    # the LM head + CE in passes of `chunk` token rows (T = 128: ragged 48+48+32, even 64+64)
    import layer_streamed_qlora_streaming_b200 as lst
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    loss_a, g_a, _ = run_step(ctx, wl, inp, want_logits=False)
    ctx.close()
    ctx = make_context(wl, inp, streamed=True, head_chunk=chunk)
    loss_b, g_b, _ = run_step(ctx, wl, inp, want_logits=False)
    assert np.float32(loss_a).tobytes() == np.float32(loss_b).tobytes()
    assert g_a.tobytes() == g_b.tobytes()
    with pytest.raises(lst.LstError) as e:   # logits are not kept whole
        ctx.logits(np.zeros((wl.tokens, wl.vocab), dtype=np.float32))
    assert e.value.status == 2
    ctx.close()


def test_gradients_to_pinned_host_same_bytes():
    # a pinned host destination is filled layer by layer during the backward; same bytes as the
    # device and pageable-host destinations
    wl = WORKLOADS["qwen3b_bf16_2L"]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    n = ctx.lora_numel()
    gd = torch.full((n,), float("nan"), device="cuda")
    gp = torch.full((n,), float("nan")).pin_memory()
    gh = np.full(n, np.nan, dtype=np.float32)
    losses = [ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq, g) for g in (gd, gp, gh)]
    assert losses[0] == losses[1] == losses[2]
    assert gd.cpu().numpy().tobytes() == gp.numpy().tobytes() == gh.tobytes()
    ctx.close()


def test_guard_bytes_checked_after_steps(monkeypatch):
    # LST_CANARY=1: the guard bytes after the pool slots and weight scratches are checked after each
    # step (a write past the end of one of them would turn the step into LST_ERR_DEVICE)
    monkeypatch.setenv("LST_CANARY", "1")
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    for reuse in (False, True):
        ctx = make_context(wl, inp, streamed=True, reuse=reuse)
        for _ in range(2):
            assert np.isfinite(run_step(ctx, wl, inp, want_logits=False)[0])
        ctx.close()


def test_deferred_optimizer_matches_in_step_update():
    # data-parallel form: the step leaves its gradients, apply_optimizer takes the (here: own)
    # gradient; same adapters and losses as the update inside the step, step after step
    wl = WORKLOADS["tiny"]
    inp = build_inputs(wl)
    runs = []
    for mode in ("in_step", "deferred_device", "deferred_host"):
        ctx = make_context(wl, inp, streamed=True)
        ctx.set_optimizer(lr=1e-3, deferred=mode != "in_step")
        n = ctx.lora_numel()
        g = torch.zeros(n, device="cuda") if mode != "deferred_host" else torch.zeros(n).pin_memory()
        losses = []
        for _ in range(3):
            losses.append(ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq, g))
            if mode != "in_step":
                ctx.apply_optimizer(g)
        p = torch.zeros(n, device="cuda")
        ctx.get_lora(p)
        runs.append((losses, p.cpu().numpy()))
        ctx.close()
    for losses, p in runs[1:]:
        assert np.float32(losses).tobytes() == np.float32(runs[0][0]).tobytes()
        assert p.tobytes() == runs[0][1].tobytes()
    assert runs[0][0][2] < runs[0][0][0]


@pytest.mark.parametrize("fault,status", [("pinned_alloc:1", 3), ("device_alloc:5", 3), ("memcpy:2", 4),
                                          ("timeout", 5)])
def test_injected_host_faults_are_status_codes(monkeypatch, fault, status):
    # failures made on the host (LST_FAULT): a failed pinned or device allocation at create time,
    # a failed layer-copy enqueue in a step, a step whose wait runs out; no GPU fault involved
    import layer_streamed_qlora_streaming_b200 as lst
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    monkeypatch.setenv("LST_FAULT", fault)
    if "alloc" in fault:
        with pytest.raises(lst.LstError) as e:
            make_context(wl, inp, streamed=True)
        assert e.value.status == status
        return
    ctx = make_context(wl, inp, streamed=True)
    with pytest.raises(lst.LstError) as e:
        run_step(ctx, wl, inp, want_logits=False)
    assert e.value.status == status
    if fault.startswith("memcpy"):
        # the copy counter has moved past the failing one: the next step runs, with the clean result
        loss, g, _ = run_step(ctx, wl, inp, want_logits=False)
        monkeypatch.delenv("LST_FAULT")
        clean = make_context(wl, inp, streamed=True)
        loss_c, g_c, _ = run_step(clean, wl, inp, want_logits=False)
        clean.close()
        assert np.float32(loss).tobytes() == np.float32(loss_c).tobytes() and g.tobytes() == g_c.tobytes()
    ctx.close()


def test_errors_are_status_codes():
    import layer_streamed_qlora_streaming_b200 as lst
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    cfg = lst.make_config(wl, streamed=True)
    E, gf, H = inp["head"]
    ctx = lst.Context(cfg, E, gf, H)
    with pytest.raises(lst.LstError) as e:          # no layer registered yet
        ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq)
    assert e.value.status == 2
    for i, r in enumerate(inp["raw"]):
        ctx.register_layer(i, r["W"], r["A"], r["B"], r["attn_norm"], r["mlp_norm"], r["bias"])
    with pytest.raises(lst.LstError) as e:          # sequence beyond max_seq
        ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq * 2)
    assert e.value.status == 1
    bad = inp["tokens"].copy()
    bad[3] = wl.vocab + 5                            # token id out of range: device-side check
    with pytest.raises(lst.LstError) as e:
        ctx.step(bad, inp["targets"], wl.batch, wl.seq)
    assert e.value.status == 6
    loss = ctx.step(inp["tokens"], inp["targets"], wl.batch, wl.seq)   # context still usable
    assert np.isfinite(loss)
    with pytest.raises(lst.LstError) as e:          # apply_optimizer without a deferred optimizer
        ctx.apply_optimizer(np.zeros(ctx.lora_numel(), dtype=np.float32))
    assert e.value.status == 2
    ctx.close()


@pytest.mark.slow
def test_layer_above_165mb_nf4():
    # two Qwen2.5-32B-shaped layers: 251.6 MB of NF4 per layer, above the size at which the
    # pages report silently wrong gradients; checked directly against the oracle
    wl = syn.WORKLOADS["qwen32b"].with_(n_layers=2, batch=1, seq=256)
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    assert ctx.stats()["blob_bytes"] > 165e6
    loss, g, lg = run_step(ctx, wl, inp)
    worst = _check_against_oracle(wl, inp, loss, g, lg, ctx)
    print("layer above 165 MB: worst gradient tensors (layer, proj, A/B, cosine, max-rel):", worst)
    ctx.close()


@pytest.mark.slow
def test_full_size_llama8b_layer_against_oracle():
    # the single-layer workload at its full size (batch 4 x seq 512), streamed and resident
    wl = syn.WORKLOADS["llama8b_layer"]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    loss, g, _ = run_step(ctx, wl, inp)
    ctx.close()
    ctx_r = make_context(wl, inp, streamed=False)
    loss_r, g_r, _ = run_step(ctx_r, wl, inp)
    ctx_r.close()
    assert np.float32(loss).tobytes() == np.float32(loss_r).tobytes() and g.tobytes() == g_r.tobytes()
    worst = _check_against_oracle(wl, inp, loss, g, None, ctx)
    print("full-size 8B layer: worst gradient tensors (layer, proj, A/B, cosine, max-rel):", worst)


@pytest.mark.parametrize("name", ["tiny", "tiny_gqa_bias_bf16"])
def test_layer0_activations_match_oracle(name):
    # every stored intermediate of layer 0 (after the step it holds the recompute of layer 0)
    from oracle import model as M
    wl = WORKLOADS[name]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    run_step(ctx, wl, inp, want_logits=False)
    T, d = wl.tokens, wl.d_model

    def act(which, layer, cols, f32):
        a = np.zeros((T, cols), dtype=np.float32 if f32 else np.uint16)
        ctx.activation(which, layer, a)
        return a if f32 else syn.bf16_bits_to_f32(a)

    sh = M.Shape(wl, bf16_acts=True)
    Wt = M.unpack_blob(M.pack_layer(inp["raw"][0], wl.base_format))
    lora = {p: (inp["raw"][0]["A"][p].astype(np.float64), inp["raw"][0]["B"][p].astype(np.float64))
            for p in M.PROJ}
    E = inp["head"][0]
    x0 = E.astype(np.float64)[inp["tokens"]]
    x1, c = M.layer_fwd(x0, Wt, lora, sh)
    assert np.array_equal(act("x", 0, d, True), x0.astype(np.float32))
    qkv = act("qkv", 0, wl.dq + 2 * wl.dkv, False)
    pairs = [("n1", act("n1", 0, d, False), c["n1"]),
             ("q", qkv[:, :wl.dq], c["q"].reshape(T, -1)),
             ("k", qkv[:, wl.dq:wl.dq + wl.dkv], c["k"].reshape(T, -1)),
             ("v", qkv[:, wl.dq + wl.dkv:], c["v"].reshape(T, -1)),
             ("o", act("o", 0, wl.dq, False), c["o"]),
             ("h", act("h", 0, d, True), c["h"]),
             ("n2", act("n2", 0, d, False), c["n2"]),
             ("gate", act("gu", 0, 2 * wl.ffn, False)[:, :wl.ffn], c["g"]),
             ("up", act("gu", 0, 2 * wl.ffn, False)[:, wl.ffn:], c["up"]),
             ("m", act("m", 0, wl.ffn, False), c["m"]),
             ("x1", act("x", 1, d, True), x1)]
    ctx.close()
    for tag, got, ref in pairs:
        assert maxrel(got, ref) < 1e-2, (tag, maxrel(got, ref))


def _flat_from_oracle(ctx, ref_grads):
    out = np.zeros(ctx.lora_numel(), dtype=np.float64)
    for (l, p), ((oa, sa), (ob, sb)) in ctx.grad_slices().items():
        out[oa:oa + sa[0] * sa[1]] = ref_grads[l][p][0].ravel()
        out[ob:ob + sb[0] * sb[1]] = ref_grads[l][p][1].ravel()
    return out


def test_adamw_step_matches_oracle_and_trains():
    from oracle import optim
    from helpers import cosine
    wl = syn.WORKLOADS["tiny"]
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    lr = 1e-3
    ctx.set_optimizer(lr=lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    p0 = np.zeros(ctx.lora_numel(), dtype=np.float32)
    ctx.get_lora(p0)
    loss0, g0, _ = run_step(ctx, wl, inp, want_logits=False)
    p1 = np.zeros_like(p0)
    ctx.get_lora(p1)
    # the update rule on the step's own gradients (identical inputs): AdamW's first update is
    # close to lr * sign(g), so comparing it on independently computed gradients would only
    # measure sign flips of near-zero gradient entries
    p1_ref, _, _ = optim.adamw_step(p0, g0, np.zeros_like(g0), np.zeros_like(g0), 1, lr=lr, wd=0.01)
    assert np.abs(p1.astype(np.float64) - p1_ref).max() <= 1e-7 + 1e-6 * np.abs(p1_ref).max()
    # the gradients themselves are the oracle's (cosine; max-rel is covered by the other tests)
    ref = oracle_step(wl, inp, bf16_acts=True)
    assert cosine(g0, _flat_from_oracle(ctx, ref["grads"])) > 0.999
    # the next step computes with the updated adapters: loss matches the oracle at p1_ref
    loss1, _, _ = run_step(ctx, wl, inp, want_logits=False)
    raw1 = [dict(r) for r in inp["raw"]]
    for (l, p), ((oa, sa), (ob, sb)) in ctx.grad_slices().items():
        raw1[l] = {**raw1[l], "A": {**raw1[l]["A"], p: p1_ref[oa:oa + sa[0] * sa[1]].reshape(sa).astype(np.float32)},
                   "B": {**raw1[l]["B"], p: p1_ref[ob:ob + sb[0] * sb[1]].reshape(sb).astype(np.float32)}}
    ref1 = oracle_step(wl, {**inp, "raw": raw1}, bf16_acts=True)
    assert abs(loss1 - ref1["loss"]) <= LOSS_RTOL * abs(ref1["loss"])
    # training on one batch lowers its loss
    losses = [loss0, loss1] + [run_step(ctx, wl, inp, want_logits=False)[0] for _ in range(4)]
    assert losses[-1] < losses[0]
    assert all(b < a for a, b in zip(losses, losses[1:]))
    ctx.close()


@pytest.mark.parametrize("base", ["nf4", "bf16"])
def test_read_timeline_orders_copies_before_compute(base):
    # the per-read timeline of a profiled step: 2L reads in order, every read's compute starts after
    # its copy (and dequant) started and ends after they ended; a copy into a slot starts only once
    # the read two earlier, which used that slot, no longer needs it: with an NF4 base dequantised
    # in a separate pass, once that read's dequant has finished (its compute reads the bf16 scratch
    # and the header copied next to it, and may still be running); with a bf16 base, once its
    # compute has finished
    wl = syn.WORKLOADS["tiny"].with_(n_layers=3, base_format=base)
    inp = build_inputs(wl)
    ctx = make_context(wl, inp, streamed=True)
    ctx.set_profiling(True)
    run_step(ctx, wl, inp, want_logits=False)
    tl = ctx.read_timeline()
    ctx.close()
    L = wl.n_layers
    assert [r["layer"] for r in tl] == list(range(L)) + list(range(L - 1, -1, -1))
    assert [r["kind"] for r in tl] == ["forward"] * L + ["backward"] * L
    eps = 1e-3
    for n, r in enumerate(tl):
        c0, c1 = r["copy"]
        d0, d1 = r["dequant"]
        k0, k1 = r["compute"]
        assert None not in (c0, c1, k0, k1)
        assert 0 <= c0 <= c1 and c0 <= k0 + eps and k0 <= k1 and c1 <= k1 + eps
        if base == "nf4":
            assert None not in (d0, d1)
            assert c0 <= d0 + eps and d0 <= d1 and d1 <= k1 + eps
            if n >= 2:
                assert tl[n - 2]["dequant"][1] <= c0 + eps
        else:
            assert (d0, d1) == (None, None)
            if n >= 2:
                assert tl[n - 2]["compute"][1] <= c0 + eps


@pytest.mark.parametrize("L", [1, 3])
def test_prefetch_of_next_first_read_same_bytes(L):
    # copying the next step's first read ahead (at the end of each step) changes when layer 0 is
    # copied, not what is computed: the same loss and gradient bytes as without it, 2L reads counted
    # per step; a step after switching reuse on, and one after re-registering layer 0 (which drops
    # the prefetched copy), give the same bytes too
    wl = syn.WORKLOADS["tiny"].with_(n_layers=L)
    inp = build_inputs(wl)
    runs = {}
    for pre in (False, True):
        ctx = make_context(wl, inp, streamed=True)
        ctx.set_prefetch(pre)
        out, reads = [], []
        for _ in range(3):
            out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
            reads.append(ctx.stats()["layer_reads_last_step"])
        r = inp["raw"][0]
        ctx.register_layer(0, r["W"], r["A"], r["B"], r["attn_norm"], r["mlp_norm"], r["bias"])
        out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
        ctx.set_reuse(True)
        out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
        ctx.set_reuse(False)
        out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
        if pre:
            ctx.set_profiling(True)
            out.append(run_step(ctx, wl, inp, want_logits=False)[:2])
            tl = ctx.read_timeline()
            # the reuse-on step left nothing prefetched, the step after it did: read 0 of this
            # profiled step was copied by the previous step and starts computing without a copy
            assert tl[0]["copy"] == (None, None) and all(None not in r["copy"] for r in tl[1:])
        ctx.close()
        runs[pre] = (out, reads)
    assert runs[False][1] == runs[True][1] == [2 * L] * 3
    for (la, ga), (lb, gb) in zip(runs[False][0], runs[True][0]):
        assert np.float32(la).tobytes() == np.float32(lb).tobytes()
        assert ga.tobytes() == gb.tobytes()


@pytest.mark.parametrize("name", ["tiny", "llama8b_layer_T256"])
def test_dequant_inside_gemm_same_bytes(name):
    # NF4 dequantised inside the GEMMs (mode 1) instead of a separate pass into a bf16 scratch: the
    # same operand bits and the same GEMM order, so the same loss and gradient bytes; the tiny stack
    # mixes both (its down projection has 688-wide rows, not whole NF4 blocks, and keeps the pass)
    wl = WORKLOADS[name]
    inp = build_inputs(wl)
    out = []
    for mode in (0, 1, 0):
        ctx = make_context(wl, inp, streamed=True, reuse=True)
        ctx.set_dequant_mode(mode)
        res = [run_step(ctx, wl, inp, want_logits=False)[:2] for _ in range(2)]
        ctx.close()
        out.append(res)
    for res in out[1:]:
        for (la, ga), (lb, gb) in zip(out[0], res):
            assert np.float32(la).tobytes() == np.float32(lb).tobytes()
            assert ga.tobytes() == gb.tobytes()


def test_split_copy_one_rank_same_bytes():
    # the split-copy path with a one-rank NCCL communicator: the rank's slice is the whole blob and
    # the all-gather runs on the copy stream; every step gives the bytes of plain copies
    import layer_streamed_qlora_streaming_b200 as lst
    try:
        uid = lst.nccl_unique_id()
    except lst.LstError:
        pytest.skip("NCCL is not available")
    wl = WORKLOADS["tiny_gqa_bias_bf16"]
    inp = build_inputs(wl)
    out = []
    for split in (False, True):
        ctx = make_context(wl, inp, streamed=True)
        if split:
            ctx.set_split_copy(0, 1, uid)
            with pytest.raises(lst.LstError):      # once per context
                ctx.set_split_copy(0, 1, uid)
        out.append([run_step(ctx, wl, inp, want_logits=False)[:2] for _ in range(2)])
        assert ctx.stats()["h2d_bytes_last_step"] == 2 * wl.n_layers * ctx.stats()["blob_bytes"]
        ctx.close()
    for (la, ga), (lb, gb) in zip(*out):
        assert np.float32(la).tobytes() == np.float32(lb).tobytes() and ga.tobytes() == gb.tobytes()
    ctx = make_context(wl, inp, streamed=False)
    with pytest.raises(lst.LstError) as e:        # resident contexts copy nothing
        ctx.set_split_copy(0, 1, uid)
    assert e.value.status == 2
    ctx.close()
