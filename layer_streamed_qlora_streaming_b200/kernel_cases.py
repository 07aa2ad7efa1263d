"""Run one kernel of the library on a fixed case and time it with CUDA events.

    python -m layer_streamed_qlora_streaming_b200.kernel_cases CASE [--iters N] [--warmup W]

Cases are the shapes of the Llama-3.1-8B-shaped layer at batch 4 x seq 512 (T = 2048 tokens):
  gemm_qkv     fused q/k/v projection: [2048, 4096] x [6144, 4096]^T + LoRA block (K + 64)
  gemm_gu      fused gate/up projection: [2048, 4096] x [28672, 4096]^T + LoRA block
  gemm_dx_gu   dX of gate/up: [2048, 28672] x [28672, 4096] (MN-major W) + LoRA block
  gemm_dx_down dX of down: [2048, 4096] x [4096, 14336] (MN-major W) + LoRA block
  dequant      NF4 -> bf16 of one 8B layer (218 M elements, 7 tensors)
  attn_fwd     causal GQA attention forward, 4 x 512, 32/8 heads, hd 128
  attn_bwd     its backward (D, dK/dV, dQ kernels)
Prints one JSON line with the per-launch time and the achieved rate. Inputs are seeded random
tensors on the device (values do not matter for timing). Used for the ncu captures in profiles/.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import k_attention_bwd, k_attention_fwd, k_gemm, k_nf4_dequant, k_nf4_quantize

T, D, F, HQ, HKV, HD, S = 2048, 4096, 14336, 32, 8, 128, 512


def _bf(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g, device="cuda") * scale).to(torch.bfloat16)


def build(case: str):
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    if case.startswith("gemm"):
        spec = {"gemm_qkv": (T, 6144, D, 0), "gemm_gu": (T, 2 * F, D, 0),
                "gemm_dx_gu": (T, D, 2 * F, 1), "gemm_dx_down": (T, F, D, 1)}[case]
        M, N, K, bmn = spec
        A = _bf((M, K), g)
        B = _bf((K, N) if bmn else (N, K), g, 0.02)
        A2 = _bf((M, 64), g)
        B2 = _bf((64, N) if bmn else (N, 64), g, 0.01)
        C = torch.empty(M, N, dtype=torch.float32 if bmn else torch.bfloat16, device="cuda")

        def run():
            k_gemm(M, N, K, A, K, B, N if bmn else K, bmn, C, N, int(bmn), A2=A2, lda2=64, B2=B2,
                   ldb2=N if bmn else 64, K2=64)
        return run, {"flop": 2.0 * M * N * (K + 64), "bytes": None}
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
    raise SystemExit(f"unknown case {case}")


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
