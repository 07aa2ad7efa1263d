"""Kernel-level parity of the CUDA library against the oracle (GPU). Every call goes through the
C ABI (include/lst_kernels.h)."""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as M
from oracle import nf4
from helpers import cosine, maxrel, to_np, torch_bf16, torch_f32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf(x):
    return syn.round_bf16(np.asarray(x, dtype=np.float32))


# ------------------------------------------------------------------------------------ NF4
@pytest.mark.parametrize("shape", [(256, 256), (688, 256), (256, 688), (1024, 4096), (14336, 4096),
                                   (27648, 5120)])
def test_nf4_quantize_and_dequant_bit_exact(shape):
    n = shape[0] * shape[1]
    w = syn.normal(11, shape[0], n, 0.02).astype(np.float32).reshape(shape)
    if shape == (256, 256):
        w[3, :64] = 0.0                      # an all-zero block
        w[5, 64:128] = 1e-3                  # a constant block
    ref = nf4.quantize(w)
    wd = torch_f32(w)
    packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    qabs = torch.empty(n // 64, dtype=torch.int8, device="cuda")
    gsc = torch.empty(ref.gscale.size, dtype=torch.float32, device="cuda")
    mean = torch.empty(1, dtype=torch.float32, device="cuda")
    lst.k_nf4_quantize(wd, packed, qabs, gsc, mean)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), ref.packed)
    assert np.array_equal(qabs.cpu().numpy(), ref.qabs)
    assert np.array_equal(gsc.cpu().numpy().view(np.uint32), ref.gscale.view(np.uint32))
    assert mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref.mean).view(np.uint32)
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    lst.k_nf4_dequant(packed, qabs, gsc, mean, n, out)
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, nf4.dequantize_bits(ref).reshape(-1))


# ------------------------------------------------------------------------------------ GEMM
GEMM_CASES = [
    # M, N, K, b_mn, ext, out_f32, bias, resid
    (128, 256, 64, 0, False, True, False, False),
    (300, 520, 200, 0, False, True, False, False),      # ragged M / N / K tails
    (256, 1000, 688, 1, False, True, False, False),     # MN-major B, ragged
    (128, 64, 128, 0, False, True, False, False),       # BN = 64
    (384, 768, 256, 0, True, False, True, True),        # LoRA extension + bias + residual, bf16 out
    (256, 1536, 512, 1, True, True, False, False),      # MN-major with extension
    (2048, 6144, 4096, 0, True, False, False, False),   # fused q/k/v of an 8B layer
    (2048, 4096, 14336, 1, True, True, False, False),   # dX of the 8B down projection
    (2048, 4096, 512, 0, True, True, False, True),      # o-like output with residual (1.7 rounds)
    (1024, 4000, 256, 0, False, True, True, False),     # ragged last N-tile, bias
]


@pytest.mark.parametrize("M,N,K,b_mn,ext,f32,bias,resid", GEMM_CASES)
def test_gemm(M, N, K, b_mn, ext, f32, bias, resid):
    r = _rng(M + N + K)
    A = _bf(r.normal(size=(M, K)))
    B = _bf(r.normal(size=(K, N) if b_mn else (N, K)) * 0.05)
    ref = A.astype(np.float64) @ (B if b_mn else B.T).astype(np.float64)
    kw = {}
    if ext:
        A2 = np.zeros((M, 64), np.float32)
        A2[:, :48] = _bf(r.normal(size=(M, 48)))
        B2 = np.zeros((64, N) if b_mn else (N, 64), np.float32)
        if b_mn:
            B2[:48] = _bf(r.normal(size=(48, N)) * 0.1)
        else:
            B2[:, :48] = _bf(r.normal(size=(N, 48)) * 0.1)
        ref = ref + A2.astype(np.float64) @ (B2 if b_mn else B2.T).astype(np.float64)
        kw.update(A2=torch_bf16(A2), lda2=64, B2=torch_bf16(B2), ldb2=N if b_mn else 64, K2=64)
    if bias:
        bv = r.normal(size=N).astype(np.float32)
        ref = ref + bv
        kw["bias"] = torch_f32(bv)
    if resid:
        Rv = r.normal(size=(M, N)).astype(np.float32)
        ref = ref + Rv
        kw.update(R=torch_f32(Rv), ldr=N)
    C = torch.zeros(M, N, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
    lst.k_gemm(M, N, K, torch_bf16(A), K, torch_bf16(B), N if b_mn else K, b_mn, C, N, int(f32), **kw)
    torch.cuda.synchronize()
    got = to_np(C)
    tol = 1e-4 if f32 else 8e-3
    assert maxrel(got, ref) < tol, maxrel(got, ref)


def _nf4_parts(rows_list, cols, seed):
    """Quantise len(rows_list) random tensors [rows, cols] on the GPU; returns (parts for
    lst_k_gemm_nf4, the stacked dequantised bf16 matrix on the GPU, keep-alive list)."""
    parts, deq, keep = [], [], []
    for i, rows in enumerate(rows_list):
        n = rows * cols
        w = syn.normal(seed, i, n, 0.02).astype(np.float32)
        packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        qabs = torch.empty(n // 64, dtype=torch.int8, device="cuda")
        gsc = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device="cuda")
        mean = torch.empty(1, dtype=torch.float32, device="cuda")
        lst.k_nf4_quantize(torch_f32(w), packed, qabs, gsc, mean)
        out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        lst.k_nf4_dequant(packed, qabs, gsc, mean, n, out)
        parts.append((packed, qabs, gsc, mean, rows))
        deq.append(out.view(rows, cols))
        keep += [packed, qabs, gsc, mean]
    return parts, torch.cat(deq, 0).contiguous(), keep


NF4_GEMM_CASES = [
    # M, parts (rows of W), cols of W, b_mn, LoRA pair, out_f32, bias, resid
    (256, [256, 64, 64], 256, 0, False, False, True, False),   # q/k/v-like, BN=128 K-major, bias
    (300, [384, 384], 128, 0, True, True, False, False),       # gate/up-like, ragged M, LoRA pair
    (128, [64], 512, 0, False, True, False, True),             # BN = 64, residual
    (256, [256, 128, 128], 320, 1, True, True, False, False),  # dX of q/k/v: W [K, N] MN-major
    (384, [1024, 1024], 256, 1, False, True, False, False),    # dX of gate/up
    (128, [688, 688], 256, 1, True, True, False, False),       # dX of the tiny gate/up: K = 1376 rows, ragged
    (2048, [4096, 1024, 1024], 4096, 0, True, False, False, False),  # 8B q/k/v forward
    (2048, [14336, 14336], 4096, 1, True, True, False, False),       # 8B gate/up dX
]


@pytest.mark.parametrize("M,rows,cols,b_mn,ext,f32,bias,resid", NF4_GEMM_CASES)
def test_gemm_nf4_equals_dequant_then_gemm(M, rows, cols, b_mn, ext, f32, bias, resid):
    # the GEMM that dequantises its NF4 operand in shared memory gives the same bytes as the
    # separate dequantisation followed by the bf16 GEMM (same operand bits, same K order)
    r = _rng(M + sum(rows) + cols + b_mn)
    parts, Wd, keep = _nf4_parts(rows, cols, 900 + len(rows) + b_mn)
    W_rows = sum(rows)
    if b_mn:
        K, N = W_rows, cols
    else:
        N, K = W_rows, cols
    A = torch_bf16(r.normal(size=(M, K)))
    kw = {}
    if ext:
        A2 = np.zeros((M, 64), np.float32)
        A2[:, :48] = _bf(r.normal(size=(M, 48)))
        B2 = np.zeros((64, N) if b_mn else (N, 64), np.float32)
        if b_mn:
            B2[:48] = _bf(r.normal(size=(48, N)) * 0.1)
        else:
            B2[:, :48] = _bf(r.normal(size=(N, 48)) * 0.1)
        kw.update(A2=torch_bf16(A2), lda2=64, B2=torch_bf16(B2), ldb2=N if b_mn else 64, K2=64)
    if bias:
        kw["bias"] = torch_f32(r.normal(size=N).astype(np.float32))
    if resid:
        kw.update(R=torch_f32(r.normal(size=(M, N)).astype(np.float32)), ldr=N)
    dt = torch.float32 if f32 else torch.bfloat16
    C1 = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    C2 = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    lst.k_gemm(M, N, K, A, K, Wd, cols, b_mn, C1, N, int(f32), **kw)
    for _ in range(2):  # twice: the same bytes again
        lst.k_gemm_nf4(M, N, K, A, K, parts, b_mn, C2, N, int(f32), **kw)
        torch.cuda.synchronize()
        assert torch.equal(C1.view(torch.int16 if not f32 else torch.int32),
                           C2.view(torch.int16 if not f32 else torch.int32))
    # and against the oracle's arithmetic on the same operand values
    Wn = to_np(Wd).astype(np.float64)
    ref = to_np(A).astype(np.float64) @ (Wn if b_mn else Wn.T)
    if ext:
        ref = ref + to_np(kw["A2"]).astype(np.float64) @ (to_np(kw["B2"]) if b_mn else to_np(kw["B2"]).T)
    if bias:
        ref = ref + to_np(kw["bias"])
    if resid:
        ref = ref + to_np(kw["R"])
    assert maxrel(to_np(C2), ref) < (1e-4 if f32 else 8e-3)
    del keep


def test_gemm_nf4_rejects_rows_not_whole_blocks():
    # a W row length that is not a multiple of 64 cannot be dequantised block by block in the tile
    parts, _, keep = _nf4_parts([64], 64, 5)
    A = torch.zeros(128, 688, dtype=torch.bfloat16, device="cuda")
    p = list(parts[0])
    p[4] = 64
    with pytest.raises(lst.LstError):
        lst.k_gemm_nf4(128, 64, 688, A, 688, [tuple(p)], 0, torch.zeros(128, 64, device="cuda"), 64, 1)
    del keep


def test_gemm_rejects_misaligned_stride():
    A = torch.zeros(128, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lst.LstError):
        lst.k_gemm(128, 128, 100, A, 100, A, 100, 0, torch.zeros(128, 128, device="cuda"), 128, 1)


# ------------------------------------------------------------------------------------ attention
@pytest.mark.parametrize("B,S,hq,hkv,hd", [(2, 64, 4, 4, 64), (2, 100, 4, 2, 64), (1, 200, 4, 1, 128),
                                           (2, 128, 8, 2, 128), (1, 160, 16, 2, 128), (2, 96, 10, 2, 64)])
def test_attention_fwd_bwd(B, S, hq, hkv, hd):
    r = _rng(S * hq + hd)
    T = B * S
    ldq = (hq + 2 * hkv) * hd
    qkv = _bf(r.normal(size=(T, ldq)))
    q = qkv[:, :hq * hd].reshape(T, hq, hd)
    k = qkv[:, hq * hd:(hq + hkv) * hd].reshape(T, hkv, hd)
    v = qkv[:, (hq + hkv) * hd:].reshape(T, hkv, hd)
    o_ref, P = M.attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), B, S)
    tq = torch_bf16(qkv)
    o = torch.empty(T, hq * hd, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, hq, dtype=torch.float32, device="cuda")
    lst.k_attention_fwd(tq, ldq, tq[:, hq * hd:], ldq, tq[:, (hq + hkv) * hd:], ldq, o, hq * hd, lse,
                        T, S, hq, hkv, hd)
    torch.cuda.synchronize()
    og = to_np(o).reshape(T, hq, hd)
    assert maxrel(og, o_ref) < 1e-2
    assert cosine(og, o_ref) > 0.9999
    # backward, upstream gradient dO ~ N(0,1)
    do = _bf(r.normal(size=(T, hq * hd)))
    dq_r, dk_r, dv_r = M.attention_bwd(do.reshape(T, hq, hd).astype(np.float64), q.astype(np.float64),
                                       k.astype(np.float64), v.astype(np.float64), P, B, S)
    dqkv = torch.zeros(T, ldq, dtype=torch.bfloat16, device="cuda")
    Dscr = torch.empty(T, hq, dtype=torch.float32, device="cuda")
    lst.k_attention_bwd(tq, ldq, tq[:, hq * hd:], ldq, tq[:, (hq + hkv) * hd:], ldq, o, hq * hd,
                        torch_bf16(do), hq * hd, lse, Dscr, dqkv, ldq, dqkv[:, hq * hd:], ldq,
                        dqkv[:, (hq + hkv) * hd:], ldq, T, S, hq, hkv, hd)
    torch.cuda.synchronize()
    g = to_np(dqkv)
    for got, ref in ((g[:, :hq * hd], dq_r), (g[:, hq * hd:(hq + hkv) * hd], dk_r), (g[:, (hq + hkv) * hd:], dv_r)):
        ref = ref.reshape(T, -1)
        assert cosine(got, ref) > 0.999, cosine(got, ref)
        assert maxrel(got, ref) < 2e-2, maxrel(got, ref)


def test_attention_deterministic():
    r = _rng(5)
    B, S, hq, hkv, hd = 2, 256, 8, 2, 128
    T, ldq = B * S, (hq + 2 * hkv) * hd
    tq = torch_bf16(_bf(r.normal(size=(T, ldq))))
    outs = []
    for _ in range(2):
        o = torch.empty(T, hq * hd, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(T, hq, dtype=torch.float32, device="cuda")
        lst.k_attention_fwd(tq, ldq, tq[:, hq * hd:], ldq, tq[:, (hq + hkv) * hd:], ldq, o, hq * hd, lse,
                            T, S, hq, hkv, hd)
        dqkv = torch.zeros(T, ldq, dtype=torch.bfloat16, device="cuda")
        Dscr = torch.empty(T, hq, dtype=torch.float32, device="cuda")
        lst.k_attention_bwd(tq, ldq, tq[:, hq * hd:], ldq, tq[:, (hq + hkv) * hd:], ldq, o, hq * hd,
                            o, hq * hd, lse, Dscr, dqkv, ldq, dqkv[:, hq * hd:], ldq,
                            dqkv[:, (hq + hkv) * hd:], ldq, T, S, hq, hkv, hd)
        torch.cuda.synchronize()
        outs.append(dqkv.view(torch.int16).cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


# ------------------------------------------------------------------------------------ small ops
def test_rmsnorm_fwd_bwd():
    r = _rng(6)
    T, d = 37, 4096
    x = r.normal(size=(T, d)).astype(np.float32)
    g = r.uniform(0.5, 1.5, size=d).astype(np.float32)
    y_ref, rs = M.rmsnorm(x.astype(np.float64), g.astype(np.float64), 1e-5)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(T, dtype=torch.float32, device="cuda")
    lst.k_rmsnorm_fwd(torch_f32(x), torch_f32(g), T, d, 1e-5, y, rstd)
    dy = r.normal(size=(T, d)).astype(np.float32)
    dres = r.normal(size=(T, d)).astype(np.float32)
    dx = torch.empty(T, d, dtype=torch.float32, device="cuda")
    lst.k_rmsnorm_bwd(torch_f32(dy), torch_f32(x), torch_f32(g), rstd, torch_f32(dres), T, d, dx)
    torch.cuda.synchronize()
    assert maxrel(to_np(y), y_ref) < 8e-3
    dx_ref = dres + M.rmsnorm_bwd(dy.astype(np.float64), x.astype(np.float64), g.astype(np.float64), rs)
    assert maxrel(to_np(dx), dx_ref) < 1e-5


def test_rope_fwd_inverse():
    r = _rng(7)
    B, S, nh, hd = 2, 48, 3, 128
    T = B * S
    x = _bf(r.normal(size=(T, nh * hd)))
    cos_t = torch.empty(S, hd // 2, device="cuda")
    sin_t = torch.empty(S, hd // 2, device="cuda")
    lst.k_rope_tables(S, hd, 5e5, cos_t, sin_t)
    buf = torch_bf16(x)
    lst.k_rope(buf, nh * hd, T, S, 0, nh, hd, cos_t, sin_t, 0)
    torch.cuda.synchronize()
    c, s = M.rope_tables(S, hd, 5e5)
    ref = M.rope(x.reshape(T, nh, hd).astype(np.float64), c, s, B, S).reshape(T, -1)
    assert maxrel(to_np(buf), ref) < 8e-3
    dy = r.normal(size=(T, nh * hd)).astype(np.float32)
    dbuf = torch_bf16(_bf(dy))
    lst.k_rope(dbuf, nh * hd, T, S, 0, nh, hd, cos_t, sin_t, 1)
    torch.cuda.synchronize()
    ref_b = M.rope_bwd(_bf(dy).reshape(T, nh, hd).astype(np.float64), c, s, B, S).reshape(T, -1)
    assert maxrel(to_np(dbuf), ref_b) < 8e-3


def test_swiglu_fwd_bwd():
    r = _rng(8)
    T, F = 64, 688
    gu = _bf(r.normal(size=(T, 2 * F)) * 2)
    m = torch.empty(T, F, dtype=torch.bfloat16, device="cuda")
    lst.k_swiglu_fwd(torch_bf16(gu), T, F, m)
    g, u = gu[:, :F].astype(np.float64), gu[:, F:].astype(np.float64)
    dm = r.normal(size=(T, F)).astype(np.float32)
    dgu = torch.empty(T, 2 * F, dtype=torch.bfloat16, device="cuda")
    lst.k_swiglu_bwd(torch_f32(dm), torch_bf16(gu), T, F, dgu)
    torch.cuda.synchronize()
    assert maxrel(to_np(m), M.silu(g) * u) < 8e-3
    sg = 1 / (1 + np.exp(-g))
    ref = np.concatenate([dm * u * sg * (1 + g * (1 - sg)), dm * g * sg], axis=1)
    assert maxrel(to_np(dgu), ref) < 8e-3


@pytest.mark.parametrize("T,V", [(40, 50000), (24, 128256), (16, 152064), (12, 60001), (20, 1001), (10, 1000),
                                 (6, 262144)])
def test_cross_entropy_rows(T, V):
    # V % 4 == 0: a cluster of 1-8 CTAs holds the row in shared memory (1000: one CTA, its four
    # copies 63/63/63/61 float4s; 50000: 4 slices; 128256 and 152064: 8; 262144: 8 slices of 128 KB);
    # otherwise (60001, 1001) the two-pass kernel. Row 0 has one logit far above the rest, row 1
    # only large negative logits, row 2 its maximum in the last slice.
    r = _rng(9 + V)
    logits = r.normal(size=(T, V)).astype(np.float32) * 2
    y = r.integers(0, V, size=T).astype(np.int32)
    logits[0, y[0]] += 60.0
    logits[1] -= 120.0
    logits[2, V - 3] = 30.0
    loss = torch.empty(T, device="cuda")
    dl = torch.empty(T, V, dtype=torch.bfloat16, device="cuda")
    lst.k_cross_entropy(torch_f32(logits), T, V, torch.from_numpy(y).cuda(), 1.0 / T, loss, dl)
    torch.cuda.synchronize()
    L = logits.astype(np.float64)
    mx = L.max(1, keepdims=True)
    lse = (mx + np.log(np.exp(L - mx).sum(1, keepdims=True)))[:, 0]
    ref = lse - L[np.arange(T), y]
    assert maxrel(to_np(loss), ref) < 1e-5
    p = np.exp(L - lse[:, None])
    p[np.arange(T), y] -= 1
    assert maxrel(to_np(dl), p / T) < 8e-3


@pytest.mark.parametrize("T,K,b_mn", [(300, 688, 0), (2048, 4096, 0), (2048, 6144, 1), (128, 256, 1)])
def test_lora_skinny(T, K, b_mn):
    r = _rng(T + K + b_mn)
    R = 48
    X = _bf(r.normal(size=(T, K)))
    if b_mn:
        Bop = np.zeros((K, 64), np.float32)
        Bop[:, :R] = _bf(r.normal(size=(K, R)) * 0.05)
        ref = 2.0 * X.astype(np.float64) @ Bop.astype(np.float64)
    else:
        Bop = np.zeros((64, K), np.float32)
        Bop[:R] = _bf(r.normal(size=(R, K)) * 0.05)
        ref = 2.0 * X.astype(np.float64) @ Bop.T.astype(np.float64)
    Us = torch.full((T, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    outs = []
    for _ in range(2):  # twice: identical bytes (fixed-order reduction over the K slices)
        lst.k_lora_skinny(torch_bf16(X), K, T, K, torch_bf16(Bop), 64 if b_mn else K, b_mn, 64, 2.0, Us)
        torch.cuda.synchronize()
        outs.append(Us.view(torch.int16).cpu().numpy().copy())
        assert maxrel(to_np(Us), ref) < 8e-3, (len(outs), maxrel(to_np(Us), ref))
    assert np.array_equal(outs[0], outs[1])
    got = to_np(Us)
    assert maxrel(got, ref) < 8e-3
    assert np.all(got[:, R:] == 0)


def _split_pair(a):
    """(hi, lo) bf16 parts of fp32 values: hi = bf16(a), lo = bf16(a - hi)."""
    hi = _bf(a)
    return hi, _bf(a.astype(np.float32) - hi)


@pytest.mark.parametrize("T,K,R,b_mn", [(300, 688, 24, 0), (2048, 4096, 48, 0), (2048, 6144, 48, 1),
                                        (128, 256, 8, 1), (256, 5120, 16, 0)])
def test_lora_skinny_split(T, K, R, b_mn):
    # U = s X (hi + lo) for an fp32 adapter held as bf16 pairs: fp32-level accuracy, stored as pairs
    rng = _rng(T * 3 + K + R + b_mn)
    RS = (R + 7) // 8 * 8
    KP = (3 * RS + 63) // 64 * 64
    X = _bf(rng.normal(size=(T, K)))
    A = (rng.uniform(-1, 1, size=(R, K)) / np.sqrt(K)).astype(np.float32)   # fp32 adapter [R, K]
    hi, lo = _split_pair(A)
    if b_mn:                                   # operand [K, KP]: sections along columns
        Bop = np.zeros((K, KP), np.float32)
        Bop[:, :R], Bop[:, RS:RS + R], Bop[:, 2 * RS:2 * RS + R] = hi.T, hi.T, lo.T
        ldb = KP
    else:                                      # operand [KP, K]: sections along rows
        Bop = np.zeros((KP, K), np.float32)
        Bop[:R], Bop[RS:RS + R], Bop[2 * RS:2 * RS + R] = hi, hi, lo
        ldb = K
    ref = 2.0 * X.astype(np.float64) @ A.astype(np.float64).T           # [T, R], exact fp32 adapter
    Us = torch.full((T, KP), float("nan"), dtype=torch.bfloat16, device="cuda")
    outs = []
    for _ in range(2):
        lst.k_lora_skinny_split(torch_bf16(X), K, T, K, torch_bf16(Bop), ldb, b_mn, R, RS, KP, 2.0, Us)
        torch.cuda.synchronize()
        outs.append(Us.view(torch.int16).cpu().numpy().copy())
    assert np.array_equal(outs[0], outs[1])
    got = to_np(Us)
    u_hi, u_lo, u_hi2 = got[:, :R], got[:, RS:RS + R], got[:, 2 * RS:2 * RS + R]
    assert np.array_equal(u_hi, u_hi2)
    assert np.array_equal(u_hi, _bf(u_hi))                             # hi is a bf16 value
    u = u_hi.astype(np.float64) + u_lo.astype(np.float64)
    # fp32 accumulation of exact bf16 products: far below bf16's 2^-8 (the lo part is live)
    assert maxrel(u, ref) < 2e-5, maxrel(u, ref)
    assert maxrel(u_hi, ref) > 1e-4 or np.allclose(u_lo, 0)
    # lo is the bf16 rounding of the remainder of the fp32 sum: |lo| <= half an ulp of hi
    assert np.all(np.abs(u_lo) <= np.abs(u_hi) * 2.0 ** -8 + 1e-30)
    # columns outside the three sections are not written
    untouched = np.ones(KP, bool)
    for s0 in (0, RS, 2 * RS):
        untouched[s0:s0 + R] = False
    assert np.all(np.isnan(got[:, untouched]))


@pytest.mark.parametrize("T,in_f,bounds,r", [
    (2048, 4096, [0, 4096, 5120, 6144], 16),   # q/k/v of an 8B layer
    (2048, 14336, [0, 4096], 16),              # down of an 8B layer
    (300, 688, [0, 688, 1376], 8),             # gate/up of the tiny stack, ragged token count
    (128, 256, [0, 256], 8),
])
def test_lora_grads(T, in_f, bounds, r):
    # dA_p = Vs_p^T X and dB_p = dY_p^T Us_p over the T tokens, every element written, same bytes twice
    rng = _rng(T + in_f + r)
    nseg, out_f, KP = len(bounds) - 1, bounds[-1], 64
    R = nseg * r
    X = _bf(rng.normal(size=(T, in_f)))
    dY = _bf(rng.normal(size=(T, out_f)) * 0.1)
    Us = np.zeros((T, KP), np.float32)
    Us[:, :R] = _bf(rng.normal(size=(T, R)))
    Vs = np.zeros((T, KP), np.float32)
    Vs[:, :R] = _bf(rng.normal(size=(T, R)))
    dA = [torch.full((r, in_f), float("nan"), device="cuda") for _ in range(nseg)]
    dB = [torch.full((bounds[p + 1] - bounds[p], r), float("nan"), device="cuda") for p in range(nseg)]
    outs = []
    for _ in range(2):
        lst.k_lora_grads(torch_bf16(X), in_f, in_f, torch_bf16(dY), out_f, out_f, T, torch_bf16(Us), torch_bf16(Vs),
                         KP, r, bounds, dA, dB)
        torch.cuda.synchronize()
        outs.append([t.cpu().numpy().copy() for t in dA + dB])
    for a, b in zip(*outs):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)
    for p in range(nseg):
        refA = Vs[:, p * r:(p + 1) * r].astype(np.float64).T @ X64
        refB = dY64[:, bounds[p]:bounds[p + 1]].T @ Us[:, p * r:(p + 1) * r].astype(np.float64)
        assert maxrel(to_np(dA[p]), refA) < 1e-4, (p, maxrel(to_np(dA[p]), refA))
        assert maxrel(to_np(dB[p]), refB) < 1e-4, (p, maxrel(to_np(dB[p]), refB))


@pytest.mark.parametrize("T", [384, 200])
def test_lora_grads_of_four_groups_in_one_launch(T):
    # the four groups of a layer (q/k/v with three segments, o, gate/up with two, down) in one launch:
    # every dA / dB against fp64, and against the same group launched alone (the K split may differ,
    # so equal up to fp32 rounding); the same bytes twice
    rng = _rng(T + 11)
    r, KP = 8, 64
    specs = [(256, [0, 256, 320, 384]), (256, [0, 256]), (256, [0, 688, 1376]), (688, [0, 256])]
    groups, refs, alone = [], [], []
    for in_f, bounds in specs:
        nseg, out_f = len(bounds) - 1, bounds[-1]
        R = nseg * r
        X = _bf(rng.normal(size=(T, in_f)))
        dY = _bf(rng.normal(size=(T, out_f)) * 0.1)
        Us = np.zeros((T, KP), np.float32)
        Us[:, :R] = _bf(rng.normal(size=(T, R)))
        Vs = np.zeros((T, KP), np.float32)
        Vs[:, :R] = _bf(rng.normal(size=(T, R)))
        mk = lambda: ([torch.full((r, in_f), float("nan"), device="cuda") for _ in range(nseg)],
                      [torch.full((bounds[p + 1] - bounds[p], r), float("nan"), device="cuda") for p in range(nseg)])
        dA, dB = mk()
        g = dict(X=torch_bf16(X), ldx=in_f, in_f=in_f, dY=torch_bf16(dY), ldy=out_f, out_f=out_f, Us=torch_bf16(Us),
                 Vs=torch_bf16(Vs), KP=KP, r=r, bounds=bounds, dA=dA, dB=dB)
        groups.append(g)
        X64, dY64 = X.astype(np.float64), dY.astype(np.float64)
        refs.append([Vs[:, p * r:(p + 1) * r].astype(np.float64).T @ X64 for p in range(nseg)] +
                    [dY64[:, bounds[p]:bounds[p + 1]].T @ Us[:, p * r:(p + 1) * r].astype(np.float64)
                     for p in range(nseg)])
        aA, aB = mk()
        lst.k_lora_grads(g["X"], in_f, in_f, g["dY"], out_f, out_f, T, g["Us"], g["Vs"], KP, r, bounds, aA, aB)
        alone.append(aA + aB)
    outs = []
    for _ in range(2):
        lst.k_lora_grads_multi(groups, T)
        torch.cuda.synchronize()
        outs.append([[t.cpu().numpy().copy() for t in g["dA"] + g["dB"]] for g in groups])
    for ga, gb in zip(*outs):
        for a, b in zip(ga, gb):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    for got, ref, al in zip(outs[0], refs, alone):
        for a, rf, b in zip(got, ref, al):
            assert maxrel(a, rf) < 1e-4
            assert maxrel(a, to_np(b)) < 1e-6


@pytest.mark.parametrize("M,N,K", [(4096, 64, 2048), (304, 64, 200), (6144, 64, 512)])
def test_gemm_transposed_a(M, N, K):
    # C = A^T B with A [K, M] and B [K, N] both MN-major: the token reductions of dA / dB
    r = _rng(M * 7 + K)
    A = _bf(r.normal(size=(K, M)))
    B = _bf(r.normal(size=(K, N)))
    ref = A.T.astype(np.float64) @ B.astype(np.float64)
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    lst.k_gemm(M, N, K, torch_bf16(A), M, torch_bf16(B), N, 1, C, N, 1, a_mn=1)
    torch.cuda.synchronize()
    assert maxrel(to_np(C), ref) < 1e-4
