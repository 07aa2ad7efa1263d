"""DPO preference step on the GPU against the oracle's DPO step (reference model = the same base
with the adapters off), and its schedule invariants (streamed == resident, reuse, head passes)."""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as M
from helpers import (GRAD_COS, GRAD_MAXREL, LOSS_RTOL, build_inputs, compare_grads, make_context)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


WORKLOADS = {
    "tiny_2pairs": syn.WORKLOADS["tiny"].with_(batch=4),
    # GQA, q/k/v bias, bf16 base, ragged sequence
    "tiny_gqa_bias_bf16": syn.WORKLOADS["tiny"].with_(n_kv_heads=2, qkv_bias=True, base_format="bf16",
                                                      batch=2, seq=100),
}
BETA = 0.5


def _run(ctx, wl, toks, tgts, mask, beta=BETA):
    grads = np.zeros(ctx.lora_numel(), dtype=np.float32)
    loss = ctx.step_dpo(toks, tgts, mask, wl.batch // 2, wl.seq, beta, grads)
    return loss, grads


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_dpo_step_matches_oracle(name):
    wl = WORKLOADS[name]
    inp = build_inputs(wl)
    toks, tgts, mask = syn.preference_pairs(wl)
    ctx = make_context(wl, inp, streamed=True)
    loss, grads = _run(ctx, wl, toks, tgts, mask)
    assert ctx.stats()["layer_reads_last_step"] == 3 * wl.n_layers
    ref = M.dpo_step(wl, inp["raw"], inp["head"], toks, tgts, wl.batch // 2, BETA, mask=mask, bf16_acts=True)
    assert abs(loss - ref["loss"]) <= LOSS_RTOL * abs(ref["loss"]), (loss, ref["loss"])
    for l, p, w, cs, mr in compare_grads(ctx, grads, ref["grads"]):
        assert cs >= GRAD_COS and mr <= GRAD_MAXREL, (l, p, w, cs, mr)
    ctx.close()


def test_dpo_schedules_give_the_same_bytes():
    wl = WORKLOADS["tiny_2pairs"].with_(n_layers=3)
    L = wl.n_layers
    inp = build_inputs(wl)
    toks, tgts, mask = syn.preference_pairs(wl)
    runs = {}
    for key, kw in {"streamed": dict(streamed=True), "resident": dict(streamed=False),
                    "reuse": dict(streamed=True, reuse=True), "head_passes": dict(streamed=True, head_chunk=96)}.items():
        ctx = make_context(wl, inp, **kw)
        out = [_run(ctx, wl, toks, tgts, mask) for _ in range(2)]
        runs[key] = (out, ctx.stats()["layer_reads_last_step"])
        ctx.close()
    (l0, g0), (l1, g1) = runs["streamed"][0]
    assert l0 == l1 and g0.tobytes() == g1.tobytes()         # deterministic
    for key in ("resident", "reuse", "head_passes"):
        for (la, ga), (lb, gb) in zip(runs["streamed"][0], runs[key][0]):
            assert np.float32(la).tobytes() == np.float32(lb).tobytes(), key
            assert ga.tobytes() == gb.tobytes(), key
    assert runs["streamed"][1] == 3 * L
    assert runs["reuse"][1] == 3 * L - 4                       # steady state: turn + across steps


def test_dpo_policy_equal_to_reference_gives_log2():
    # B = 0: the policy is the reference, so the loss is ln 2 up to rounding of identical passes
    wl = WORKLOADS["tiny_2pairs"]
    inp = build_inputs(wl)
    toks, tgts, mask = syn.preference_pairs(wl)
    ctx = make_context(wl, inp, streamed=True)
    for l in range(wl.n_layers):
        for j, p in enumerate(syn.PROJ):
            ctx.set_lora(l, j, inp["raw"][l]["A"][p], np.zeros_like(inp["raw"][l]["B"][p]))
    loss, grads = _run(ctx, wl, toks, tgts, mask)
    assert loss == pytest.approx(np.log(2.0), abs=1e-6)
    assert np.any(grads != 0)
    # all-ones mask equals no mask
    la, ga = _run(ctx, wl, toks, tgts, np.ones_like(mask))
    lb, gb = _run(ctx, wl, toks, tgts, None)
    assert la == lb and ga.tobytes() == gb.tobytes()
    ctx.close()
