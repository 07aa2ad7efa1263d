"""Run one kernel of the library on a fixed case and time it with CUDA events.

    python kernel_cases.py CASE [--iters N] [--warmup W]

Cases are the shapes of the Llama-3.1-8B-shaped layer at batch 4 x seq 512 (T = 2048 tokens):
  gemm_*       every GEMM shape of a step (GEMM_SHAPES): the q/k/v, o, gate/up and down
               projections with their LoRA block, their dX, and the LM head's two GEMMs
  gemm_{qkv,gu,dx_gu,dx_down}_nf4
               four of them with W dequantised from NF4 inside the GEMM (3 weight copies rotated
               so every launch reads its codes from HBM)
  dequant_gu   NF4 -> bf16 of the gate/up group alone (2 x 14336 x 4096 elements)
  dequant      NF4 -> bf16 of one 8B layer (218 M elements, 7 tensors)
  attn_fwd     causal GQA attention forward, 4 x 512, 32/8 heads, hd 128
  attn_bwd     its backward (D, dK/dV, dQ kernels)
  lora_u_qkv   LoRA projection U = s X Acat^T, X [2048, 4096], Acat [64, 4096]
  lora_u_down  the same for the down projection's input, X [2048, 14336]
  lora_v_gu    V = s dY Bexp, dY [2048, 28672], Bexp [28672, 64] (MN-major)
  lora_grads_qkv  dA = Vs^T X and dB = dY^T Us of the q/k/v group (dY [2048, 6144])
  lora_grads_gu   the same for gate/up (dY [2048, 28672])
  lora_grads_layer      dA and dB of the four groups of a layer (q/k/v, o, gate/up, down) in one
                        launch, as a backward read issues them
  lora_grads_layer_sep  the same four groups as four launches
  ce           cross-entropy rows + dlogits over fp32 logits [2048, 128256]
  rmsnorm_fwd / rmsnorm_bwd   RMSNorm of the fp32 residual stream [2048, 4096] (bf16 output; the
               backward with the residual gradient added and a bf16 copy, as a layer uses it)
  swiglu_fwd / swiglu_bwd     SwiGLU of gate/up [2048, 2 x 14336] (the backward from fp32 dL/dm)
The LoRA cases rotate over enough input copies to exceed the 126 MB L2, so every launch reads
its operands from HBM.
Prints one JSON line with the per-launch device time (launches queued back to back) and the
achieved rate. Inputs are seeded random
tensors on the device (values do not matter for timing). Used for the ncu captures in profiles/.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from layer_streamed_qlora_streaming_b200 import (k_attention_bwd, k_attention_fwd, k_cross_entropy, k_gemm, k_gemm_nf4,
                                                 k_rmsnorm_bwd, k_rmsnorm_fwd, k_swiglu_bwd, k_swiglu_fwd,
                                                 k_lora_grads, k_lora_grads_multi, k_lora_skinny, k_nf4_dequant,
               k_nf4_quantize)

T, D, F, HQ, HKV, HD, S = 2048, 4096, 14336, 32, 8, 128, 512
VOCAB = 128256

# Every GEMM of a training step of the 8B-shaped stack: (M, N, K, B MN-major, extra K of the LoRA
# block, fp32 output, fp32 residual added), and how many times one step launches it.
GEMM_SHAPES = {
    "gemm_qkv": (T, 6144, D, 0, 192, 0, 0),        # q/k/v forward (bias, RoPE in the step)
    "gemm_o": (T, D, D, 0, 64, 1, 1),              # o forward + residual
    "gemm_gu": (T, 2 * F, D, 0, 128, 0, 0),        # gate/up forward
    "gemm_down": (T, D, F, 0, 64, 1, 1),           # down forward + residual
    "gemm_dx_down": (T, F, D, 1, 64, 1, 0),        # dX of down
    "gemm_dx_gu": (T, D, 2 * F, 1, 128, 1, 0),     # dX of gate/up
    "gemm_dx_o": (T, D, D, 1, 64, 0, 0),           # dX of o (bf16 output)
    "gemm_dx_qkv": (T, D, 6144, 1, 192, 1, 0),     # dX of q/k/v
    "gemm_head": (T, VOCAB, D, 0, 0, 1, 0),        # logits
    "gemm_dx_head": (T, D, VOCAB, 1, 0, 1, 0),     # dlogits H
}
# per step of the 32-layer stack: forward reads run 4 projection GEMMs, backward reads recompute 3
# (the down projection's output is not needed) and run 4 dX GEMMs, and the head runs 2
GEMM_LAUNCHES_PER_STEP = {"gemm_qkv": 64, "gemm_o": 64, "gemm_gu": 64, "gemm_down": 32, "gemm_dx_down": 32,
                          "gemm_dx_gu": 32, "gemm_dx_o": 32, "gemm_dx_qkv": 32, "gemm_head": 1, "gemm_dx_head": 1}


def _bf(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g, device="cuda") * scale).to(torch.bfloat16)


def _nf4(rows_list, cols, g):
    """NF4 tensors [rows, cols] quantised on the device: the parts of a stacked weight matrix."""
    parts = []
    for rows in rows_list:
        n = rows * cols
        w = torch.randn(n, generator=g, device="cuda") * 0.02
        packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        qabs = torch.empty(n // 64, dtype=torch.int8, device="cuda")
        gs = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device="cuda")
        mean = torch.empty(1, dtype=torch.float32, device="cuda")
        k_nf4_quantize(w, packed, qabs, gs, mean)
        parts.append((packed, qabs, gs, mean, rows))
    return parts


def build(case: str):
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    if case.startswith("gemm") and case.endswith("_nf4"):
        base = case[:-4]
        M, N, K, bmn, K2, f32, _ = GEMM_SHAPES[base]
        rows = {"gemm_qkv": [4096, 1024, 1024], "gemm_gu": [F, F], "gemm_dx_gu": [F, F], "gemm_dx_down": [D]}[base]
        cols = K if bmn == 0 else N
        copies = [_nf4(rows, cols, g) for _ in range(3)]
        A = _bf((M, K), g)
        A2 = _bf((M, K2), g)
        B2 = _bf((K2, N) if bmn else (N, K2), g, 0.01)
        C = torch.empty(M, N, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
        state = {"i": 0}

        def run():
            parts = copies[state["i"] % len(copies)]
            state["i"] += 1
            k_gemm_nf4(M, N, K, A, K, parts, bmn, C, N, int(f32), A2=A2, lda2=K2, B2=B2,
                       ldb2=N if bmn else K2, K2=K2)
        return run, {"flop": 2.0 * M * N * (K + K2), "bytes": None}
    if case == "dequant_gu":
        n = 2 * F * D
        w = torch.randn(n, generator=g, device="cuda") * 0.02
        packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        qabs = torch.empty(n // 64, dtype=torch.int8, device="cuda")
        gs = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device="cuda")
        mean = torch.empty(1, dtype=torch.float32, device="cuda")
        k_nf4_quantize(w, packed, qabs, gs, mean)
        del w
        out = torch.empty(n, dtype=torch.bfloat16, device="cuda")

        def run():
            k_nf4_dequant(packed, qabs, gs, mean, n, out)
        return run, {"flop": None, "bytes": n * (0.5 + 1 / 64 + 2)}
    if case.startswith("gemm"):
        M, N, K, bmn, K2, f32, resid = GEMM_SHAPES[case]
        A = _bf((M, K), g)
        B = _bf((K, N) if bmn else (N, K), g, 0.02)
        A2 = _bf((M, K2), g) if K2 else None
        B2 = (_bf((K2, N) if bmn else (N, K2), g, 0.01)) if K2 else None
        C = torch.empty(M, N, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
        R = torch.randn(M, N, generator=g, device="cuda") if resid else None

        def run():
            k_gemm(M, N, K, A, K, B, N if bmn else K, bmn, C, N, int(f32), A2=A2, lda2=K2, B2=B2,
                   ldb2=(N if bmn else K2), K2=K2, R=R, ldr=N if resid else 0)
        return run, {"flop": 2.0 * M * N * (K + K2), "bytes": None}
    if case == "dequant":
        n = 4096 * 4096 * 2 + 1024 * 4096 * 2 + 14336 * 4096 * 3
        w = torch.randn(n, generator=g, device="cuda") * 0.02
        packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        qabs = torch.empty(n // 64, dtype=torch.int8, device="cuda")
        gs = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device="cuda")
        mean = torch.empty(1, dtype=torch.float32, device="cuda")
        k_nf4_quantize(w, packed, qabs, gs, mean)
        del w
        out = torch.empty(n, dtype=torch.bfloat16, device="cuda")

        def run():
            k_nf4_dequant(packed, qabs, gs, mean, n, out)
        return run, {"flop": None, "bytes": n * 0.5 + n / 64 + n * 2}
    if case.startswith("attn"):
        ld = (HQ + 2 * HKV) * HD
        qkv = _bf((T, ld), g)
        q, k, v = qkv, qkv[:, HQ * HD:], qkv[:, (HQ + HKV) * HD:]
        o = torch.empty(T, HQ * HD, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(T, HQ, device="cuda")
        k_attention_fwd(q, ld, k, ld, v, ld, o, HQ * HD, lse, T, S, HQ, HKV, HD)
        flop_fwd = 4.0 * (T // S) * HQ * S * S * HD / 2
        if case == "attn_fwd":
            def run():
                k_attention_fwd(q, ld, k, ld, v, ld, o, HQ * HD, lse, T, S, HQ, HKV, HD)
            return run, {"flop": flop_fwd, "bytes": None}
        do = _bf((T, HQ * HD), g)
        Dd = torch.empty(T, HQ, device="cuda")
        dqkv = torch.empty(T, ld, dtype=torch.bfloat16, device="cuda")

        def run():
            k_attention_bwd(q, ld, k, ld, v, ld, o, HQ * HD, do, HQ * HD, lse, Dd, dqkv, ld, dqkv[:, HQ * HD:], ld,
                            dqkv[:, (HQ + HKV) * HD:], ld, T, S, HQ, HKV, HD)
        return run, {"flop": 2.5 * flop_fwd, "bytes": None}
    if case.startswith("lora_"):
        return _lora_case(case, g)
    if case.startswith("rmsnorm"):
        x = torch.randn(T, D, generator=g, device="cuda")
        gam = torch.rand(D, generator=g, device="cuda") + 0.5
        rstd = torch.empty(T, device="cuda")
        if case == "rmsnorm_fwd":
            y = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")

            def run():
                k_rmsnorm_fwd(x, gam, T, D, 1e-5, y, rstd)
            return run, {"flop": None, "bytes": T * D * (4 + 2)}
        k_rmsnorm_fwd(x, gam, T, D, 1e-5, torch.empty(T, D, dtype=torch.bfloat16, device="cuda"), rstd)
        dy, dres = torch.randn(T, D, generator=g, device="cuda"), torch.randn(T, D, generator=g, device="cuda")
        dx = torch.empty(T, D, device="cuda")
        dxb = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")

        def run():
            k_rmsnorm_bwd(dy, x, gam, rstd, dres, T, D, dx, dxb)
        return run, {"flop": None, "bytes": T * D * (4 * 4 + 2)}
    if case.startswith("swiglu"):
        gu = _bf((T, 2 * F), g)
        if case == "swiglu_fwd":
            m = torch.empty(T, F, dtype=torch.bfloat16, device="cuda")

            def run():
                k_swiglu_fwd(gu, T, F, m)
            return run, {"flop": None, "bytes": T * F * (4 + 2)}
        dm = torch.randn(T, F, generator=g, device="cuda")
        dgu = torch.empty(T, 2 * F, dtype=torch.bfloat16, device="cuda")

        def run():
            k_swiglu_bwd(dm, gu, T, F, dgu)
        return run, {"flop": None, "bytes": T * F * (4 + 4 + 4)}
    if case == "ce":
        V = 128256
        logits = torch.randn(T, V, generator=g, device="cuda") * 2.0
        tg = torch.randint(0, V, (T,), generator=g, device="cuda", dtype=torch.int32)
        loss_rows = torch.empty(T, device="cuda")
        dlog = torch.empty(T, V, dtype=torch.bfloat16, device="cuda")

        def run():
            k_cross_entropy(logits, T, V, tg, 1.0 / T, loss_rows, dlog)
        return run, {"flop": None, "bytes": T * V * 4 + T * V * 2}
    raise SystemExit(f"unknown case {case}")


def _copies(nbytes: int) -> int:
    return max(2, -(-256 * 2**20 // max(nbytes, 1)))


def _lora_case(case: str, g):
    KP = 64
    if case.startswith("lora_u") or case.startswith("lora_v"):
        K, bmn = {"lora_u_qkv": (D, 0), "lora_u_down": (F, 0), "lora_v_gu": (2 * F, 1)}[case]
        nb = _copies(T * K * 2)
        Xs = [_bf((T, K), g) for _ in range(nb)]
        Bop = _bf((K, KP) if bmn else (KP, K), g, 0.02)
        Us = torch.empty(T, KP, dtype=torch.bfloat16, device="cuda")
        it = [0]

        def run():
            X = Xs[it[0] % nb]
            it[0] += 1
            k_lora_skinny(X, K, T, K, Bop, KP if bmn else K, bmn, KP, 2.0, Us)
        return run, {"flop": 2.0 * T * K * KP, "bytes": T * K * 2 + K * KP * 2 + T * KP * 2}
    if case.startswith("lora_grads_layer"):
        return _lora_layer_case(case, g)
    in_f, bounds, r = {"lora_grads_qkv": (D, [0, 4096, 5120, 6144], 16),
                       "lora_grads_gu": (D, [0, F, 2 * F], 16)}[case]
    out_f = bounds[-1]
    nb = _copies(T * (in_f + out_f) * 2)
    Xs = [_bf((T, in_f), g) for _ in range(nb)]
    dYs = [_bf((T, out_f), g) for _ in range(nb)]
    Us, Vs = _bf((T, KP), g), _bf((T, KP), g)
    nseg = len(bounds) - 1
    dA = [torch.empty(r, in_f, device="cuda") for _ in range(nseg)]
    dB = [torch.empty(bounds[p + 1] - bounds[p], r, device="cuda") for p in range(nseg)]
    it = [0]

    def run():
        i = it[0] % nb
        it[0] += 1
        k_lora_grads(Xs[i], in_f, in_f, dYs[i], out_f, out_f, T, Us, Vs, KP, r, bounds, dA, dB)
    return run, {"flop": 2.0 * T * KP * (in_f + out_f),
                 "bytes": T * (in_f + out_f) * 2 + 2 * T * KP * 2 + nseg * r * (in_f + out_f) * 4}


def _lora_layer_case(case: str, g):
    # (in, segment bounds of dY, KP) of the q/k/v, o, gate/up and down groups at r = 16
    r = 16
    specs = [(D, [0, 4096, 5120, 6144], 192), (D, [0, D], 64), (D, [0, F, 2 * F], 128), (F, [0, D], 64)]
    per_copy = sum(T * (i + b[-1]) * 2 for i, b, _ in specs)
    nb = _copies(per_copy)
    sets = []
    for _ in range(nb):
        groups = []
        for in_f, bounds, KP in specs:
            nseg, out_f = len(bounds) - 1, bounds[-1]
            groups.append(dict(X=_bf((T, in_f), g), ldx=in_f, in_f=in_f, dY=_bf((T, out_f), g), ldy=out_f,
                               out_f=out_f, Us=_bf((T, KP), g), Vs=_bf((T, KP), g), KP=KP, r=r, bounds=bounds,
                               dA=[torch.empty(r, in_f, device="cuda") for _ in range(nseg)],
                               dB=[torch.empty(bounds[p + 1] - bounds[p], r, device="cuda") for p in range(nseg)]))
        sets.append(groups)
    it = [0]

    def run():
        groups = sets[it[0] % nb]
        it[0] += 1
        if case == "lora_grads_layer":
            k_lora_grads_multi(groups, T)
        else:
            for q in groups:
                k_lora_grads(q["X"], q["ldx"], q["in_f"], q["dY"], q["ldy"], q["out_f"], T, q["Us"], q["Vs"], q["KP"],
                             q["r"], q["bounds"], q["dA"], q["dB"])
    nbytes = sum(T * (i + b[-1]) * 2 + 2 * T * kp * 2 + (len(b) - 1) * r * (i + b[-1]) * 4 for i, b, kp in specs)
    flop = sum(2.0 * T * (len(b) - 1) * r * (i + b[-1]) for i, b, _ in specs)
    return run, {"flop": flop, "bytes": nbytes}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args()
    run, work = build(a.case)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # hold the stream with a spin kernel while the host enqueues every launch, so the timed
    # region is back-to-back device time even for launches shorter than their host overhead
    torch.cuda._sleep(200_000_000)
    e0.record()
    for _ in range(a.iters):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    res = {"case": a.case, "ms_per_launch": ms}
    if work["flop"]:
        res["tflops"] = work["flop"] / (ms * 1e-3) / 1e12
    if work["bytes"]:
        res["gbs"] = work["bytes"] / (ms * 1e-3) / 1e9
    print(json.dumps(res))


if __name__ == "__main__":
    main()
