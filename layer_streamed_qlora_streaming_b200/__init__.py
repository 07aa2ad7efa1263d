"""Python binding of liblst.so (include/lst.h, include/lst_kernels.h): argument marshalling only.

Every step of the path runs in the CUDA library; this module converts torch tensors / numpy arrays
to pointers and status codes to exceptions. There is no fallback: if liblst.so is missing or
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblst.so")

PROJ = ("q", "k", "v", "o", "gate", "up", "down")
BASE_NF4, BASE_BF16 = 0, 1
STATUS = {0: "LST_OK", 1: "LST_ERR_ARG", 2: "LST_ERR_STATE", 3: "LST_ERR_OOM", 4: "LST_ERR_CUDA",
          5: "LST_ERR_TIMEOUT", 6: "LST_ERR_DEVICE"}


class LstError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("d_model", C.c_int32), ("n_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("ffn", C.c_int32),
                ("vocab", C.c_int32), ("rms_eps", C.c_float), ("rope_theta", C.c_float),
                ("qkv_bias", C.c_int32), ("lora_rank", C.c_int32), ("lora_alpha", C.c_float),
                ("base_format", C.c_int32), ("max_batch", C.c_int32), ("max_seq", C.c_int32),
                ("streamed", C.c_int32), ("timeout_ms", C.c_int32), ("head_chunk", C.c_int32),
                ("reuse", C.c_int32)]


class LayerWeights(C.Structure):
    _fields_ = [("w", C.c_void_p * 7), ("bias", C.c_void_p * 3), ("attn_norm", C.c_void_p),
                ("mlp_norm", C.c_void_p), ("lora_a", C.c_void_p * 7), ("lora_b", C.c_void_p * 7)]


class AdamW(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float), ("deferred", C.c_int32)]


class Stats(C.Structure):
    _fields_ = [("steps", C.c_int64), ("launches_last_step", C.c_int64),
                ("layer_reads_last_step", C.c_int64), ("h2d_bytes_last_step", C.c_int64),
                ("blob_bytes", C.c_int64), ("arena_bytes", C.c_int64), ("device_bytes", C.c_int64),
                ("gemm_ms", C.c_double), ("attention_ms", C.c_double), ("dequant_ms", C.c_double),
                ("other_ms", C.c_double), ("copy_ms", C.c_double), ("step_ms", C.c_double),
                ("gemm_launches", C.c_int64), ("attention_launches", C.c_int64),
                ("dequant_launches", C.c_int64), ("copy_count", C.c_int64), ("gemm_flops", C.c_double),
                ("lora_ms", C.c_double), ("lora_launches", C.c_int64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


_lib = None
_P, _I32, _I64, _F32, _F64 = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_double
_SIGS = {
    "lst_create": (_I32, [C.POINTER(Config), _P, _P, _P, _P, C.POINTER(_P)]),
    "lst_register_layer": (_I32, [_P, _I32, C.POINTER(LayerWeights)]),
    "lst_set_lora": (_I32, [_P, _I32, _I32, _P, _P]),
    "lst_lora_numel": (_I64, [_P]),
    "lst_set_optimizer": (_I32, [_P, _P]),
    "lst_get_lora": (_I32, [_P, _P]),
    "lst_step": (_I32, [_P, _P, _P, _I32, _I32, C.POINTER(C.c_float), _P]),
    "lst_step_hidden": (_I32, [_P, _P, _P, _I32, _I32, C.POINTER(C.c_float), _P]),
    "lst_get_logits": (_I32, [_P, _P]),
    "lst_get_activation": (_I32, [_P, _I32, _I32, _P]),
    "lst_set_profiling": (_I32, [_P, _I32]),
    "lst_apply_optimizer": (_I32, [_P, _P]),
    "lst_step_dpo": (_I32, [_P, _P, _P, _P, _I32, _I32, _F32, C.POINTER(C.c_float), _P]),
    "lst_set_reuse": (_I32, [_P, _I32]),
    "lst_set_prefetch": (_I32, [_P, _I32]),
    "lst_plan_reads": (_I32, [_P, _I32, _I32, _I32, _P, _P, _P, _P]),
    "lst_get_stats": (_I32, [_P, C.POINTER(Stats)]),
    "lst_get_read_timeline": (_I32, [_P, _P, _I32, C.POINTER(_I32)]),
    "lst_set_split_copy": (_I32, [_P, _I32, _I32, _P]),
    "lst_set_dequant_mode": (_I32, [_P, _I32]),
    "lst_nccl_unique_id": (_I32, [_P]),
    "lst_split_plan": (_I32, [_I64, _I32, _I32, C.POINTER(_I64), C.POINTER(_I64), C.POINTER(_I64)]),
    "lst_last_error": (C.c_char_p, [_P]),
    "lst_destroy": (None, [_P]),
    "lst_nf4_codebook": (_I32, [C.POINTER(C.c_float)]),
    "lst_blob_bytes": (_I64, [C.POINTER(Config)]),
    "lst_k_nf4_quantize": (_I32, [_P, _I64, _P, _P, _P, _P, _P]),
    "lst_k_nf4_quantize_noalloc": (_I32, [_P, _I64, _P, _P, _P, _P, _P]),
    "lst_k_lora_grads_multi": (_I32, [_P, _I32, _I64, _P]),
    "lst_k_nf4_dequant": (_I32, [_P, _P, _P, _P, _I64, _P, _P]),
    "lst_k_gemm_nf4": (_I32, [_I32, _I32, _I32, _P, _I64, _P, _I32, _I32, _P, _I64, _P, _I64, _I32, _P, _I64, _I32,
                              _F32, _P, _P, _I64, _P]),
    "lst_k_gemm": (_I32, [_I32, _I32, _I32, _P, _I64, _I32, _P, _I64, _I32, _P, _I64, _P, _I64, _I32,
                          _P, _I64, _I32, _F32, _P, _P, _I64, _P]),
    "lst_k_attention_fwd": (_I32, [_P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _I64, _I32, _I32,
                                   _I32, _I32, _P]),
    "lst_k_attention_bwd": (_I32, [_P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _P, _P,
                                   _I64, _P, _I64, _P, _I64, _I64, _I32, _I32, _I32, _I32, _P]),
    "lst_k_rmsnorm_fwd": (_I32, [_P, _P, _I64, _I32, _F32, _P, _P, _P]),
    "lst_k_rmsnorm_bwd": (_I32, [_P, _P, _P, _P, _P, _I64, _I32, _P, _P, _P]),
    "lst_k_rope_tables": (_I32, [_I32, _I32, _F64, _P, _P, _P]),
    "lst_k_rope": (_I32, [_P, _I64, _I64, _I32, _I32, _I32, _I32, _P, _P, _I32, _P]),
    "lst_k_swiglu_fwd": (_I32, [_P, _I64, _I32, _P, _P]),
    "lst_k_swiglu_bwd": (_I32, [_P, _P, _I64, _I32, _P, _P]),
    "lst_k_cross_entropy": (_I32, [_P, _I64, _I32, _P, _F32, _P, _P, _P]),
    "lst_k_lora_skinny": (_I32, [_P, _I64, _I64, _I32, _P, _I64, _I32, _I32, _F32, _P, _P]),
    "lst_k_lora_skinny_split": (_I32, [_P, _I64, _I64, _I32, _P, _I64, _I32, _I32, _I32, _I32, _F32, _P, _P]),
    "lst_k_lora_grads": (_I32, [_P, _I64, _I32, _P, _I64, _I32, _I64, _P, _P, _I32, _I32, _I32, _P, _P, _P, _P]),
    "lst_k_launch_count": (_I64, []),
    "lst_k_device_error": (_I32, []),
}


def lib() -> C.CDLL:
    """The loaded liblst.so; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m layer_streamed_qlora_streaming_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _ptr(x) -> int | None:
    """Pointer of a torch tensor, numpy array, int address or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        # row-strided views are fine: every entry point takes explicit leading dimensions
        if x.dim() > 0 and x.stride(-1) != 1:
            raise ValueError("innermost dimension must be contiguous")
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return x.ctypes.data
    raise TypeError(type(x))


def _stream(s) -> int | None:
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _check(st: int, ctx=None, what: str = "") -> None:
    if st != 0:
        msg = what
        if ctx is not None:
            msg = (lib().lst_last_error(ctx) or b"").decode() or what
        raise LstError(st, msg)


def nf4_codebook():
    import numpy as np
    out = (C.c_float * 16)()
    _check(lib().lst_nf4_codebook(out), what="lst_nf4_codebook")
    return np.array(list(out), dtype=np.float32)


def make_config(wl, streamed: bool = True, max_batch=None, max_seq=None, timeout_ms: int = 600000,
                head_chunk: int = 0, reuse: bool = False) -> Config:
    """lst_config of a synthetic.Workload-like object."""
    return Config(wl.n_layers, wl.d_model, wl.n_heads, wl.n_kv_heads, wl.head_dim, wl.ffn, wl.vocab,
                  wl.rms_eps, wl.rope_theta, int(wl.qkv_bias), wl.lora_rank, wl.lora_alpha,
                  BASE_NF4 if wl.base_format == "nf4" else BASE_BF16,
                  max_batch or wl.batch, max_seq or wl.seq, int(streamed), timeout_ms, int(head_chunk),
                  int(bool(reuse)))


def plan_reads(reads, reuse: bool, nf4: bool, held=(-1, -1), wheld=(-1, -1), prefetch=None):
    """The step's copy / dequant plan (host only): (rows [n, 8] int32 of slot, copy, wait_free,
    loaded_by, wslot, dequant, wwait, wfilled_by; held after; wheld after). With prefetch given (the
    slot a previous step copied this step's first read into, -1 none) the plan copies the next
    step's first read ahead, and a fourth item (slot, read it waits for) describes that copy."""
    import numpy as np
    r = np.ascontiguousarray(reads, dtype=np.int32)
    h = np.array(held, dtype=np.int32)
    w = np.array(wheld, dtype=np.int32)
    pre = None if prefetch is None else np.array([prefetch, -1], dtype=np.int32)
    out = np.zeros((len(r), 8), dtype=np.int32)
    _check(lib().lst_plan_reads(_ptr(r), len(r), int(bool(reuse)), int(bool(nf4)), _ptr(h), _ptr(w),
                                None if pre is None else _ptr(pre), _ptr(out)),
           what="lst_plan_reads")
    res = (out, tuple(int(x) for x in h), tuple(int(x) for x in w))
    return res if pre is None else res + ((int(pre[0]), int(pre[1])),)


def split_plan(blob: int, world: int, rank: int):
    """(offset, bytes, count) of rank's slice in split-copy mode (host only)."""
    o, b, c = C.c_int64(0), C.c_int64(0), C.c_int64(0)
    _check(lib().lst_split_plan(blob, world, rank, C.byref(o), C.byref(b), C.byref(c)), what="lst_split_plan")
    return o.value, b.value, c.value


def nccl_unique_id() -> bytes:
    buf = (C.c_char * 128)()
    _check(lib().lst_nccl_unique_id(buf), what="lst_nccl_unique_id")
    return bytes(buf)


def blob_bytes(cfg: Config) -> int:
    return int(lib().lst_blob_bytes(C.byref(cfg)))


class Context:
    """One lst_ctx: frozen base (streamed or resident), resident adapters, step buffers."""

    def __init__(self, cfg: Config, embed=None, final_norm=None, lm_head=None, stream=None):
        self._keep = []
        h = C.c_void_p()
        st = lib().lst_create(C.byref(cfg), _ptr(embed), _ptr(final_norm), _ptr(lm_head),
                              _stream(stream), C.byref(h))
        _check(st, None, "lst_create")
        self.h = h
        self.cfg = cfg

    def close(self):
        if getattr(self, "h", None):
            lib().lst_destroy(self.h)
            self.h = None

    __del__ = close

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def register_layer(self, layer: int, W: dict, A: dict, B: dict, attn_norm, mlp_norm, bias=None):
        lw = LayerWeights()
        for i, p in enumerate(PROJ):
            lw.w[i] = _ptr(W[p])
            lw.lora_a[i] = _ptr(A[p])
            lw.lora_b[i] = _ptr(B[p])
        if bias is not None:
            for i, p in enumerate(("q", "k", "v")):
                lw.bias[i] = _ptr(bias[p])
        lw.attn_norm = _ptr(attn_norm)
        lw.mlp_norm = _ptr(mlp_norm)
        _check(lib().lst_register_layer(self.h, layer, C.byref(lw)), self.h, "lst_register_layer")

    def set_lora(self, layer: int, proj: int, A, B):
        _check(lib().lst_set_lora(self.h, layer, proj, _ptr(A), _ptr(B)), self.h, "lst_set_lora")

    def lora_numel(self) -> int:
        return int(lib().lst_lora_numel(self.h))

    def set_optimizer(self, lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, off=False,
                      deferred=False):
        """AdamW on the adapters at the end of every step (off=True disables it); deferred=True
        leaves the update to apply_optimizer (data-parallel: apply the replicas' mean gradient)."""
        if off:
            _check(lib().lst_set_optimizer(self.h, None), self.h, "lst_set_optimizer")
            return
        cfg = AdamW(lr, beta1, beta2, eps, weight_decay, int(bool(deferred)))
        _check(lib().lst_set_optimizer(self.h, C.byref(cfg)), self.h, "lst_set_optimizer")

    def apply_optimizer(self, grads) -> None:
        """One AdamW update with the given gradient (host or device, gradient layout)."""
        _check(lib().lst_apply_optimizer(self.h, _ptr(grads)), self.h, "lst_apply_optimizer")

    def get_lora(self, dst) -> None:
        _check(lib().lst_get_lora(self.h, _ptr(dst)), self.h, "lst_get_lora")

    def step(self, tokens, targets, batch: int, seq: int, grads=None) -> float:
        loss = C.c_float()
        _check(lib().lst_step(self.h, _ptr(tokens), _ptr(targets), batch, seq, C.byref(loss), _ptr(grads)),
               self.h, "lst_step")
        return loss.value

    def step_hidden(self, x_bits, g_bits, batch: int, seq: int, grads=None) -> float:
        loss = C.c_float()
        _check(lib().lst_step_hidden(self.h, _ptr(x_bits), _ptr(g_bits), batch, seq, C.byref(loss),
                                     _ptr(grads)), self.h, "lst_step_hidden")
        return loss.value

    def step_dpo(self, tokens, targets, mask, n_pairs: int, seq: int, beta: float, grads=None) -> float:
        """DPO step on 2 * n_pairs sequences (chosen first); mask may be None (all positions)."""
        loss = C.c_float()
        _check(lib().lst_step_dpo(self.h, _ptr(tokens), _ptr(targets), _ptr(mask), n_pairs, seq, beta,
                                  C.byref(loss), _ptr(grads)), self.h, "lst_step_dpo")
        return loss.value

    def logits(self, dst) -> None:
        _check(lib().lst_get_logits(self.h, _ptr(dst)), self.h, "lst_get_logits")

    ACT = {"x": 0, "n1": 1, "qkv": 2, "o": 3, "h": 4, "n2": 5, "gu": 6, "m": 7}

    def activation(self, which: str, layer: int, dst) -> None:
        _check(lib().lst_get_activation(self.h, self.ACT[which], layer, _ptr(dst)), self.h,
               "lst_get_activation")

    def set_profiling(self, on: bool) -> None:
        _check(lib().lst_set_profiling(self.h, int(on)), self.h, "lst_set_profiling")

    def set_reuse(self, on: bool) -> None:
        _check(lib().lst_set_reuse(self.h, int(on)), self.h, "lst_set_reuse")

    def set_prefetch(self, on: bool) -> None:
        _check(lib().lst_set_prefetch(self.h, int(on)), self.h, "lst_set_prefetch")

    def stats(self) -> dict:
        s = Stats()
        _check(lib().lst_get_stats(self.h, C.byref(s)), self.h, "lst_get_stats")
        return s.as_dict()

    def set_dequant_mode(self, mode: int) -> None:
        """0: separate NF4 dequantisation pass (default); 1: inside the GEMMs (lst_set_dequant_mode)."""
        _check(lib().lst_set_dequant_mode(self.h, int(mode)), self.h, "lst_set_dequant_mode")

    def set_split_copy(self, rank: int, world: int, unique_id: bytes) -> None:
        """Split copies over `world` GPUs (lst_set_split_copy); unique_id from nccl_unique_id()."""
        buf = (C.c_char * 128).from_buffer_copy(unique_id) if unique_id else None
        _check(lib().lst_set_split_copy(self.h, rank, world, buf), self.h, "lst_set_split_copy")

    def read_timeline(self) -> list:
        """Per-read timeline of the last profiled step: dicts with layer, kind and the copy, dequant
        and compute start / end in ms from the step's start (None where the read had none)."""
        n = C.c_int32(0)
        lib().lst_get_read_timeline(self.h, None, 0, C.byref(n))
        buf = (C.c_float * (8 * max(n.value, 1)))()
        _check(lib().lst_get_read_timeline(self.h, buf, n.value, C.byref(n)), self.h, "lst_get_read_timeline")
        kinds = ("reference", "forward", "backward")
        rows = []
        for i in range(n.value):
            r = buf[8 * i:8 * i + 8]
            t = [None if v < 0 else float(v) for v in r[2:]]
            rows.append({"layer": int(r[0]), "kind": kinds[int(r[1])], "copy": (t[0], t[1]), "dequant": (t[2], t[3]),
                         "compute": (t[4], t[5])})
        return rows

    def grad_slices(self) -> dict:
        """{(layer, proj): ((offA, shapeA), (offB, shapeB))} of the gradient layout."""
        c = self.cfg
        d, F = c.d_model, c.ffn
        dq, dkv = c.n_heads * c.head_dim, c.n_kv_heads * c.head_dim
        outs = {"q": dq, "k": dkv, "v": dkv, "o": d, "gate": F, "up": F, "down": d}
        ins = {"q": d, "k": d, "v": d, "o": dq, "gate": d, "up": d, "down": F}
        r = c.lora_rank
        off, res = 0, {}
        for l in range(c.n_layers):
            for p in PROJ:
                a = (off, (r, ins[p]))
                off += r * ins[p]
                b = (off, (outs[p], r))
                off += outs[p] * r
                res[(l, p)] = (a, b)
        return res


# ------------------------------------------------------------------------------ kernel-level calls

def k_nf4_quantize(w, packed, qabs, gscale, mean, stream=None):
    _check(lib().lst_k_nf4_quantize(_ptr(w), w.numel(), _ptr(packed), _ptr(qabs), _ptr(gscale),
                                    _ptr(mean), _stream(stream)), what="lst_k_nf4_quantize")


def k_nf4_quantize_noalloc(w, packed, qabs, gscale, mean, n=None, stream=None):
    """NF4 quantisation with the library's fixed scratch array (no device allocation)."""
    _check(lib().lst_k_nf4_quantize_noalloc(_ptr(w), w.numel() if n is None else n, _ptr(packed), _ptr(qabs),
                                            _ptr(gscale), _ptr(mean), _stream(stream)),
           what="lst_k_nf4_quantize_noalloc")


def k_nf4_dequant(packed, qabs, gscale, mean, n, out, stream=None):
    _check(lib().lst_k_nf4_dequant(_ptr(packed), _ptr(qabs), _ptr(gscale), _ptr(mean), n, _ptr(out),
                                   _stream(stream)), what="lst_k_nf4_dequant")


def k_gemm(M, N, K, A, lda, B, ldb, b_mn, C_, ldc, c_f32, alpha=1.0, A2=None, lda2=0, B2=None, ldb2=0,
           K2=0, bias=None, R=None, ldr=0, a_mn=0, stream=None):
    _check(lib().lst_k_gemm(M, N, K, _ptr(A), lda, a_mn, _ptr(B), ldb, b_mn, _ptr(A2), lda2, _ptr(B2), ldb2,
                            K2, _ptr(C_), ldc, c_f32, alpha, _ptr(bias), _ptr(R), ldr, _stream(stream)),
           what="lst_k_gemm")


class Nf4Part(C.Structure):
    _fields_ = [("packed", C.c_void_p), ("qabs", C.c_void_p), ("gscale", C.c_void_p), ("mean", C.c_void_p),
                ("rows", C.c_int32)]


def k_gemm_nf4(M, N, K, A, lda, parts, b_mn, C_, ldc, c_f32, alpha=1.0, A2=None, lda2=0, B2=None, ldb2=0, K2=0,
               bias=None, R=None, ldr=0, stream=None):
    """parts: up to 3 (packed, qabs, gscale, mean, rows) NF4 tensors stacked along W's rows."""
    arr = (Nf4Part * len(parts))(*[Nf4Part(_ptr(p), _ptr(q), _ptr(g), _ptr(m), int(r)) for p, q, g, m, r in parts])
    _check(lib().lst_k_gemm_nf4(M, N, K, _ptr(A), lda, arr, len(parts), b_mn, _ptr(A2), lda2, _ptr(B2), ldb2, K2,
                                _ptr(C_), ldc, c_f32, alpha, _ptr(bias), _ptr(R), ldr, _stream(stream)),
           what="lst_k_gemm_nf4")


def k_attention_fwd(q, ldq, k, ldk, v, ldv, o, ldo, lse, T, S, hq, hkv, hd, stream=None):
    _check(lib().lst_k_attention_fwd(_ptr(q), ldq, _ptr(k), ldk, _ptr(v), ldv, _ptr(o), ldo, _ptr(lse),
                                     T, S, hq, hkv, hd, _stream(stream)), what="lst_k_attention_fwd")


def k_attention_bwd(q, ldq, k, ldk, v, ldv, o, ldo, dout, lddo, lse, D, dq, lddq, dk, lddk, dv, lddv,
                    T, S, hq, hkv, hd, stream=None):
    _check(lib().lst_k_attention_bwd(_ptr(q), ldq, _ptr(k), ldk, _ptr(v), ldv, _ptr(o), ldo, _ptr(dout),
                                     lddo, _ptr(lse), _ptr(D), _ptr(dq), lddq, _ptr(dk), lddk, _ptr(dv),
                                     lddv, T, S, hq, hkv, hd, _stream(stream)), what="lst_k_attention_bwd")


def k_rmsnorm_fwd(x, g, T, d, eps, y, rstd, stream=None):
    _check(lib().lst_k_rmsnorm_fwd(_ptr(x), _ptr(g), T, d, eps, _ptr(y), _ptr(rstd), _stream(stream)),
           what="lst_k_rmsnorm_fwd")


def k_rmsnorm_bwd(dy, x, g, rstd, dres, T, d, dx, dxb=None, stream=None):
    _check(lib().lst_k_rmsnorm_bwd(_ptr(dy), _ptr(x), _ptr(g), _ptr(rstd), _ptr(dres), T, d, _ptr(dx),
                                   _ptr(dxb), _stream(stream)), what="lst_k_rmsnorm_bwd")


def k_rope_tables(S, hd, theta, cos_t, sin_t, stream=None):
    _check(lib().lst_k_rope_tables(S, hd, theta, _ptr(cos_t), _ptr(sin_t), _stream(stream)),
           what="lst_k_rope_tables")


def k_rope(buf, ld, T, S, col0, nh, hd, cos_t, sin_t, inverse=0, stream=None):
    _check(lib().lst_k_rope(_ptr(buf), ld, T, S, col0, nh, hd, _ptr(cos_t), _ptr(sin_t), inverse,
                            _stream(stream)), what="lst_k_rope")


def k_swiglu_fwd(gu, T, F, m, stream=None):
    _check(lib().lst_k_swiglu_fwd(_ptr(gu), T, F, _ptr(m), _stream(stream)), what="lst_k_swiglu_fwd")


def k_swiglu_bwd(dm, gu, T, F, dgu, stream=None):
    _check(lib().lst_k_swiglu_bwd(_ptr(dm), _ptr(gu), T, F, _ptr(dgu), _stream(stream)),
           what="lst_k_swiglu_bwd")


def k_cross_entropy(logits, T, V, targets, inv_T, loss_rows, dlogits, stream=None):
    _check(lib().lst_k_cross_entropy(_ptr(logits), T, V, _ptr(targets), inv_T, _ptr(loss_rows),
                                     _ptr(dlogits), _stream(stream)), what="lst_k_cross_entropy")


def k_lora_skinny(X, ldx, T, K, Bop, ldb, b_mn, KP, s, Us, stream=None):
    _check(lib().lst_k_lora_skinny(_ptr(X), ldx, T, K, _ptr(Bop), ldb, b_mn, KP, s, _ptr(Us), _stream(stream)),
           what="lst_k_lora_skinny")


def k_lora_skinny_split(X, ldx, T, K, Bop, ldb, b_mn, R, RS, KP, s, Us, stream=None):
    _check(lib().lst_k_lora_skinny_split(_ptr(X), ldx, T, K, _ptr(Bop), ldb, b_mn, R, RS, KP, s, _ptr(Us),
                                         _stream(stream)), what="lst_k_lora_skinny_split")


def k_lora_grads(X, ldx, in_f, dY, ldy, out_f, T, Us, Vs, KP, r, bounds, dA, dB, stream=None):
    """dA[p] [r, in] and dB[p] [out_p, r] (fp32 device tensors) of one fused group; bounds: the
    nseg + 1 column bounds of the segments in dY."""
    nseg = len(dA)
    b = (C.c_int32 * 4)(*([int(v) for v in bounds] + [0] * (4 - len(bounds))))
    pa = (C.c_void_p * 3)(*([_ptr(t) for t in dA] + [None] * (3 - nseg)))
    pb = (C.c_void_p * 3)(*([_ptr(t) for t in dB] + [None] * (3 - nseg)))
    _check(lib().lst_k_lora_grads(_ptr(X), ldx, in_f, _ptr(dY), ldy, out_f, T, _ptr(Us), _ptr(Vs), KP, nseg, r,
                                  b, pa, pb, _stream(stream)), what="lst_k_lora_grads")


class LoraGradGroup(C.Structure):
    _fields_ = [("X", _P), ("ldx", _I64), ("in_f", _I32), ("dY", _P), ("ldy", _I64), ("out_f", _I32),
                ("Us", _P), ("Vs", _P), ("KP", _I32), ("nseg", _I32), ("r", _I32), ("bounds", _I32 * 4),
                ("dA", _P * 3), ("dB", _P * 3)]


def k_lora_grads_multi(groups, T, stream=None):
    """The adapter gradients of up to four fused groups in one launch; groups: dicts with the
    arguments of k_lora_grads (X, ldx, in_f, dY, ldy, out_f, Us, Vs, KP, r, bounds, dA, dB)."""
    arr = (LoraGradGroup * len(groups))()
    for g, a in zip(groups, arr):
        nseg = len(g["dA"])
        a.X, a.ldx, a.in_f = _ptr(g["X"]), g["ldx"], g["in_f"]
        a.dY, a.ldy, a.out_f = _ptr(g["dY"]), g["ldy"], g["out_f"]
        a.Us, a.Vs, a.KP, a.nseg, a.r = _ptr(g["Us"]), _ptr(g["Vs"]), g["KP"], nseg, g["r"]
        for k, v in enumerate(g["bounds"]):
            a.bounds[k] = int(v)
        for k in range(nseg):
            a.dA[k] = _ptr(g["dA"][k])
            a.dB[k] = _ptr(g["dB"][k])
    _check(lib().lst_k_lora_grads_multi(C.cast(arr, C.c_void_p), len(groups), T, _stream(stream)),
           what="lst_k_lora_grads_multi")


def device_error() -> int:
    """Read and clear the device error word (0 = none)."""
    return int(lib().lst_k_device_error())


def launch_count() -> int:
    return int(lib().lst_k_launch_count())
