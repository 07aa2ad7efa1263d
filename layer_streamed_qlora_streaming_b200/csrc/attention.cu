// Causal grouped-query attention, forward and deterministic backward, on the warp-level tensor-core
// path (mma.sync m16n8k16 bf16 -> fp32) with online softmax, never materialising the S x S scores.
//
//   o = softmax(q k^T / sqrt(hd) + causal mask) v ; query head h reads kv head h / (hq / hkv)
//
// Layouts: q/k/v/o are rows of token-major matrices (token t = b * S + s); head h of a row starts
// at column h * hd; row strides are arguments so q, k, v can live side by side in one fused qkv
// buffer. lse and D are [T, hq] fp32. The backward is split in two kernels so that nothing is
// accumulated with atomics: dK/dV (a thread-block cluster per kv block, one CTA per query head of
// the group, whose partial sums are added in head order through distributed shared memory) and dQ
// (one CTA per query block). Tiles stream through double-buffered cp.async loads, and the causal
// blocks with the most work are scheduled first.
#include "attention.cuh"
#include "common.cuh"

#include <cuda_fp16.h>

namespace lst {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxGroup = 8;  // query heads per kv head: the dK/dV cluster size (portable limit)

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// The same shape with fp16 operands: the forward's P V product, where P in [0, 1] keeps 3 more
// mantissa bits in fp16 than in bf16 and V converts to fp16 without loss (see k_attn_fwd).
__device__ __forceinline__ void mma16816_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}


// Shared tile of `rows` x HD bf16 with a 16-byte row pad (conflict-free ldmatrix).
template <int HD>
struct Tile {
  static constexpr int LD = HD + 8;
};

// Cooperative load of rows [r0, r0+nrows) of one head into a shared tile; rows outside [0, S)
// of the sequence are zero.
template <int HD>
__device__ __forceinline__ void load_tile(__nv_bfloat16* sm, const __nv_bfloat16* g, int64_t ld, int64_t tok0,
                                          int r0, int nrows, int S, int col) {
  constexpr int V = HD / 8;  // 16-byte vectors per row
  for (int i = threadIdx.x; i < nrows * V; i += blockDim.x) {
    const int r = i / V, c = (i % V) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r0 + r < S) val = *reinterpret_cast<const uint4*>(g + (tok0 + r0 + r) * ld + col + c);
    *reinterpret_cast<uint4*>(sm + r * Tile<HD>::LD + c) = val;
  }
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(pred ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool pred) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(pred ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Asynchronous form of load_tile (rows outside [0, S) are zero-filled); completes at the next
// cp_async_wait_all of the issuing thread.
template <int HD>
__device__ __forceinline__ void load_tile_async(__nv_bfloat16* sm, const __nv_bfloat16* g, int64_t ld, int64_t tok0,
                                                int r0, int nrows, int S, int col) {
  constexpr int V = HD / 8;
  for (int i = threadIdx.x; i < nrows * V; i += blockDim.x) {
    const int r = i / V, c = (i % V) * 8;
    const bool in = r0 + r < S;
    cp_async16(sm + r * Tile<HD>::LD + c, in ? g + (tok0 + r0 + r) * ld + col + c : g, in);
  }
}

// Rewrite, in place, the 16-byte chunks of a shared bf16 tile that this thread loaded with
// load_tile_async (same chunk assignment) as fp16. Every bf16 value of magnitude in
// [2^-14, 65504] is an fp16 value, so the attention's V (|v| of order 1) converts exactly; smaller
// ones lose at most 2^-25 in absolute terms. Call after the thread's cp_async_wait_all and before
// the barrier that publishes the tile.
template <int HD>
__device__ __forceinline__ void tile_to_f16(__nv_bfloat16* sm, int nrows) {
  constexpr int V = HD / 8;
  for (int i = threadIdx.x; i < nrows * V; i += blockDim.x) {
    uint4* p = reinterpret_cast<uint4*>(sm + (i / V) * Tile<HD>::LD + (i % V) * 8);
    uint4 u = *p;
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      w[j] = pack_f16(f.x, f.y);
    }
    *p = u;
  }
}

// A fragment (16 rows x 16 k) at (row0, k0) of a shared tile.
template <int HD>
__device__ __forceinline__ void lda_frag(uint32_t (&a)[4], const __nv_bfloat16* sm, int row0, int k0) {
  const int l = threadIdx.x & 31;
  const int r = row0 + (l & 7) + ((l >> 3) & 1) * 8;
  const int c = k0 + (l >> 4) * 8;
  ldsm4(a, smem_u32(sm + r * Tile<HD>::LD + c));
}
// B fragments for two n-tiles (n0, n0+8) x k-step k0 where B(k, n) = tile[n][k] (rows are n).
template <int HD>
__device__ __forceinline__ void ldb_rows(uint32_t (&b)[4], const __nv_bfloat16* sm, int n0, int k0) {
  const int l = threadIdx.x & 31;
  const int r = n0 + (l & 7) + (l >> 4) * 8;
  const int c = k0 + ((l >> 3) & 1) * 8;
  ldsm4(b, smem_u32(sm + r * Tile<HD>::LD + c));
}
// B fragments for two n-tiles (n0, n0+8) x k-step k0 where B(k, n) = tile[k][n] (rows are k).
template <int HD>
__device__ __forceinline__ void ldb_trans(uint32_t (&b)[4], const __nv_bfloat16* sm, int k0, int n0) {
  const int l = threadIdx.x & 31;
  const int r = k0 + (l & 7) + ((l >> 3) & 1) * 8;
  const int c = n0 + (l >> 4) * 8;
  ldsm4t(b, smem_u32(sm + r * Tile<HD>::LD + c));
}

// Store one accumulator row (C-fragment row r of this thread) of dq or dk scaled by `scale`; with
// tables given, first apply the inverse rotary embedding of position pos (the transpose of the
// forward rotation: pairs j, j + hd/2 rotated by minus the angle), so the gradient is rounded once.
template <int HD>
__device__ __forceinline__ void store_grad_rows(__nv_bfloat16* dst, const float (&acc)[HD / 8][4], int r, int t4,
                                                int pos, float scale, const float* cos_t, const float* sin_t) {
  constexpr int HALF = HD / 2;
  if (!cos_t) {
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      const int c = i * 8 + 2 * t4;
      *reinterpret_cast<__nv_bfloat162*>(dst + c) =
          __floats2bfloat162_rn(acc[i][2 * r] * scale, acc[i][2 * r + 1] * scale);
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < HD / 16; ++i) {
    const int c = i * 8 + 2 * t4;  // first-half dimension; its partner is c + HALF (n-tile i + HD/16)
    float y1[2], y2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float x1 = acc[i][2 * r + u] * scale, x2 = acc[i + HD / 16][2 * r + u] * scale;
      const float cs = cos_t[pos * HALF + c + u], sn = sin_t[pos * HALF + c + u];
      y1[u] = x1 * cs + x2 * sn;
      y2[u] = x2 * cs - x1 * sn;
    }
    *reinterpret_cast<__nv_bfloat162*>(dst + c) = __floats2bfloat162_rn(y1[0], y1[1]);
    *reinterpret_cast<__nv_bfloat162*>(dst + c + HALF) = __floats2bfloat162_rn(y2[0], y2[1]);
  }
}

// ------------------------------------------------------------------------------------ forward
// grid (hq, B, ceil(S/64)), 128 threads; the last query block (most keys) is scheduled first;
// warp w owns query rows 16w..16w+15 of the block. K/V tiles of 64 keys, double-buffered. The
// unnormalised probabilities enter the P V product as fp16 (V tiles converted exactly to fp16 once
// they land), which keeps the rounding of P 8x below bf16's.
template <int HD>
__global__ void __launch_bounds__(128) k_attn_fwd(AttnArgs p) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  constexpr int TL = 64 * Tile<HD>::LD;
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm_raw);
  __nv_bfloat16* Kbuf = Qs + TL;       // [2] K tiles
  __nv_bfloat16* Vbuf = Kbuf + 2 * TL;  // [2] V tiles
  const int h = blockIdx.x, b = blockIdx.y, qb = (int)gridDim.z - 1 - (int)blockIdx.z;
  const int kvh = h / (p.hq / p.hkv);
  const int64_t tok0 = (int64_t)b * p.S;
  const int q0 = qb * 64;
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31, g = l >> 2, t4 = l & 3;
  const float sl2 = p.scale * kLog2e;

  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int qr0 = q0 + warp * 16 + g, qr1 = qr0 + 8;  // this thread's two query rows
  const int nkb = min(qb, (p.S - 1) / 64) + 1;

  load_tile_async<HD>(Qs, p.q, p.ldq, tok0, q0, 64, p.S, h * HD);
  load_tile_async<HD>(Kbuf, p.k, p.ldk, tok0, 0, 64, p.S, kvh * HD);
  load_tile_async<HD>(Vbuf, p.v, p.ldv, tok0, 0, 64, p.S, kvh * HD);
  cp_async_commit();
  for (int kb = 0; kb < nkb; ++kb) {
    cp_async_wait_all();
    tile_to_f16<HD>(Vbuf + (kb & 1) * TL, 64);  // this thread's chunks of V tile kb
    __syncthreads();  // tile kb is in; every warp is done with tile kb-1, whose buffer is refilled now
    if (kb + 1 < nkb) {
      const int nb = (kb + 1) & 1;
      load_tile_async<HD>(Kbuf + nb * TL, p.k, p.ldk, tok0, (kb + 1) * 64, 64, p.S, kvh * HD);
      load_tile_async<HD>(Vbuf + nb * TL, p.v, p.ldv, tok0, (kb + 1) * 64, 64, p.S, kvh * HD);
      cp_async_commit();
    }
    const __nv_bfloat16* Ks = Kbuf + (kb & 1) * TL;
    const __nv_bfloat16* Vs = Vbuf + (kb & 1) * TL;
    const bool diag = kb == nkb - 1;  // only the last block holds keys past a query or past S
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD; kk += 16) {
      uint32_t a[4];
      lda_frag<HD>(a, Qs, warp * 16, kk);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t bb[4];
        ldb_rows<HD>(bb, Ks, j * 8, kk);
        mma16816(s[j], a, bb[0], bb[1]);
        mma16816(s[j + 1], a, bb[2], bb[3]);
      }
    }
    // mask + online softmax (base-2 domain of the scaled scores)
    float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb * 64 + j * 8 + 2 * t4 + (e & 1);
        const int qr = (e < 2) ? qr0 : qr1;
        float v = s[j][e] * sl2;
        if (diag && (key > qr || key >= p.S)) v = -INFINITY;
        s[j][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mref = mx[r] == -INFINITY ? 0.f : mx[r];
      corr[r] = exp2f(mrow[r] - mref);
      mrow[r] = mx[r];
      mx[r] = mref;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = exp2f(s[j][e] - mx[e >> 1]);
        s[j][e] = pv;
        rs[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      lrow[r] = lrow[r] * corr[r] + rs[r];
    }
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      o[i][0] *= corr[0];
      o[i][1] *= corr[0];
      o[i][2] *= corr[1];
      o[i][3] *= corr[1];
    }
    // o += P v (fp16 operands)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 keys per k-step
      uint32_t a[4];
      a[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int i = 0; i < HD / 8; i += 2) {
        uint32_t bb[4];
        ldb_trans<HD>(bb, Vs, kk * 16, i * 8);
        mma16816_f16(o[i], a, bb[0], bb[1]);
        mma16816_f16(o[i + 1], a, bb[2], bb[3]);
      }
    }
  }
  // normalise and write o, lse
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qr = r ? qr1 : qr0;
    if (qr >= p.S) continue;
    const float inv = 1.0f / lrow[r];
    __nv_bfloat16* op = p.o + (tok0 + qr) * p.ldo + h * HD;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      const int c = i * 8 + 2 * t4;
      *reinterpret_cast<__nv_bfloat162*>(op + c) = __floats2bfloat162_rn(o[i][2 * r] * inv, o[i][2 * r + 1] * inv);
    }
    if (p.o32) {  // unrounded output for the backward's D = rowsum(dO * O)
      float* o32 = p.o32 + (tok0 + qr) * (int64_t)p.hq * HD + h * HD;
#pragma unroll
      for (int i = 0; i < HD / 8; ++i)
        *reinterpret_cast<float2*>(o32 + i * 8 + 2 * t4) = make_float2(o[i][2 * r] * inv, o[i][2 * r + 1] * inv);
    }
    if (t4 == 0) p.lse[(tok0 + qr) * p.hq + h] = (mrow[r] + log2f(lrow[r])) / kLog2e;
  }
}

// --------------------------------------------------------------------------- backward: D = rowsum(dO o)
__global__ void k_attn_D(AttnBwdArgs p) {
  const int64_t idx = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // (t, h)
  const int l = threadIdx.x & 31;
  if (idx >= p.T * (int64_t)p.hq) return;
  const int64_t t = idx / p.hq;
  const int h = (int)(idx % p.hq);
  const __nv_bfloat16* a = p.dout + t * p.lddo + (int64_t)h * p.hd;
  float s = 0.f;
  if (p.o32) {  // the forward's unrounded output: D then matches the normalisation of P exactly
    const float* o = p.o32 + t * (int64_t)p.hq * p.hd + (int64_t)h * p.hd;
    for (int c = l; c < p.hd; c += 32) s += __bfloat162float(a[c]) * o[c];
  } else {
    const __nv_bfloat16* o = p.o + t * p.ldo + (int64_t)h * p.hd;
    for (int c = l; c < p.hd; c += 32) s += __bfloat162float(a[c]) * __bfloat162float(o[c]);
  }
  s = warp_sum(s);
  if (l == 0) p.D[idx] = s;
}

// --------------------------------------------------------------------------- backward: dK, dV
// grid (grp, B * hkv, ceil(S/64)), cluster (grp, 1, 1), 128 threads. The cluster owns one block of
// 64 keys of kv head kvh; its CTA of rank hh sums the contributions of query head kvh * grp + hh
// over query tiles of 32 rows (double-buffered); warp w owns keys 16w..16w+15. The grp partial dK /
// dV tiles are then parked in shared memory and CTA hh adds rows [hh * 64/grp, ...) over the heads
// in order 0 .. grp-1 (distributed shared memory), scales dK, undoes the rotary embedding and
// stores both. kv block 0 (the most queries) is scheduled first.
template <int HD>
__global__ void __launch_bounds__(128) k_attn_dkdv(AttnBwdArgs p) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  constexpr int LD = Tile<HD>::LD;
  constexpr int QT = 32 * LD;  // one 32-row tile
  constexpr int RLD = HD + 4;   // fp32 row stride of a parked partial tile
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(sm_raw);
  __nv_bfloat16* Vs = Ks + 64 * LD;
  __nv_bfloat16* Qbuf = Vs + 64 * LD;  // [2] q tiles
  __nv_bfloat16* Obuf = Qbuf + 2 * QT;  // [2] dO tiles
  float* Lbuf = reinterpret_cast<float*>(Obuf + 2 * QT);  // [2][32]
  float* Dbuf = Lbuf + 64;                                 // [2][32]
  float* redK = reinterpret_cast<float*>(sm_raw);  // [64][RLD], after the main loop
  float* redV = redK + 64 * RLD;                   // [64][RLD]

  const int grp = (int)gridDim.x;
  const int hh = (int)cluster_rank();
  const int kvh = (int)blockIdx.y % p.hkv, b = (int)blockIdx.y / p.hkv, kb = (int)blockIdx.z;
  const int h = kvh * grp + hh;
  const int64_t tok0 = (int64_t)b * p.S;
  const int k0 = kb * 64;
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31, g = l >> 2, t4 = l & 3;
  const float sl2 = p.scale * kLog2e;

  auto load_q = [&](int buf, int qs0) {
    load_tile_async<HD>(Qbuf + buf * QT, p.q, p.ldq, tok0, qs0, 32, p.S, h * HD);
    load_tile_async<HD>(Obuf + buf * QT, p.dout, p.lddo, tok0, qs0, 32, p.S, h * HD);
    if (threadIdx.x < 32) {
      const int qr = qs0 + threadIdx.x;
      const bool in = qr < p.S;
      const int64_t idx = in ? (tok0 + qr) * p.hq + h : 0;
      cp_async4(Lbuf + buf * 32 + threadIdx.x, p.lse + idx, in);
      cp_async4(Dbuf + buf * 32 + threadIdx.x, p.D + idx, in);
    }
  };
  load_tile_async<HD>(Ks, p.k, p.ldk, tok0, k0, 64, p.S, kvh * HD);
  load_tile_async<HD>(Vs, p.v, p.ldv, tok0, k0, 64, p.S, kvh * HD);
  if (k0 < p.S) load_q(0, k0);
  cp_async_commit();

  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const int kr0 = k0 + warp * 16 + g, kr1 = kr0 + 8;  // this thread's key rows

  for (int qs0 = k0, it = 0; qs0 < p.S; qs0 += 32, ++it) {
    cp_async_wait_all();
    __syncthreads();  // tile `it` is in; the other buffer is free again
    if (qs0 + 32 < p.S) {
      load_q((it + 1) & 1, qs0 + 32);
      cp_async_commit();
    }
    const __nv_bfloat16* Qs = Qbuf + (it & 1) * QT;
    const __nv_bfloat16* Os = Obuf + (it & 1) * QT;
    const float* Ls = Lbuf + (it & 1) * 32;
    const float* Ds = Dbuf + (it & 1) * 32;
    const bool diag = qs0 < k0 + 64 || qs0 + 32 > p.S;  // queries before a key or past S possible
    // S^T (16 keys x 32 queries) and dP^T
    float st[4][4], dp[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[j][e] = dp[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD; kk += 16) {
      uint32_t ak[4], av[4];
      lda_frag<HD>(ak, Ks, warp * 16, kk);
      lda_frag<HD>(av, Vs, warp * 16, kk);
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        uint32_t bq[4], bo[4];
        ldb_rows<HD>(bq, Qs, j * 8, kk);
        ldb_rows<HD>(bo, Os, j * 8, kk);
        mma16816(st[j], ak, bq[0], bq[1]);
        mma16816(st[j + 1], ak, bq[2], bq[3]);
        mma16816(dp[j], av, bo[0], bo[1]);
        mma16816(dp[j + 1], av, bo[2], bo[3]);
      }
    }
    // P^T and dS^T
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = j * 8 + 2 * t4 + (e & 1);
        const int qr = qs0 + qi;
        const int kr = (e < 2) ? kr0 : kr1;
        float pv = exp2f(st[j][e] * sl2 - Ls[qi] * kLog2e);
        if (kr >= p.S || (diag && (qr < kr || qr >= p.S))) pv = 0.f;
        st[j][e] = pv;
        dp[j][e] = pv * (dp[j][e] - Ds[qi]);
      }
    }
    // dV += P^T dO ; dK += dS^T Q
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t ap[4], as[4];
      ap[0] = pack_bf16(st[2 * kk][0], st[2 * kk][1]);
      ap[1] = pack_bf16(st[2 * kk][2], st[2 * kk][3]);
      ap[2] = pack_bf16(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      ap[3] = pack_bf16(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      as[0] = pack_bf16(dp[2 * kk][0], dp[2 * kk][1]);
      as[1] = pack_bf16(dp[2 * kk][2], dp[2 * kk][3]);
      as[2] = pack_bf16(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
      as[3] = pack_bf16(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
#pragma unroll
      for (int i = 0; i < HD / 8; i += 2) {
        uint32_t bo[4], bq[4];
        ldb_trans<HD>(bo, Os, kk * 16, i * 8);
        ldb_trans<HD>(bq, Qs, kk * 16, i * 8);
        mma16816(dv[i], ap, bo[0], bo[1]);
        mma16816(dv[i + 1], ap, bo[2], bo[3]);
        mma16816(dk[i], as, bq[0], bq[1]);
        mma16816(dk[i + 1], as, bq[2], bq[3]);
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();  // every warp is done with the tiles: their space takes the partial sums
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp * 16 + g + 8 * r;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      const int c = i * 8 + 2 * t4;
      *reinterpret_cast<float2*>(redK + row * RLD + c) = make_float2(dk[i][2 * r], dk[i][2 * r + 1]);
      *reinterpret_cast<float2*>(redV + row * RLD + c) = make_float2(dv[i][2 * r], dv[i][2 * r + 1]);
    }
  }
  __syncwarp();
  cluster_sync_all();  // every head's partial tile is parked

  constexpr int HALF = HD / 2;
  const int rows = (64 + grp - 1) / grp;
  const int rbeg = hh * rows, rend = min(64, rbeg + rows);
  const uint32_t rk0 = smem_u32(redK), rv0 = smem_u32(redV);
  for (int item = threadIdx.x; item < (rend - rbeg) * (HALF / 2); item += blockDim.x) {
    const int row = rbeg + item / (HALF / 2);
    const int c = (item % (HALF / 2)) * 2;  // columns c, c+1 and their rotary partners c+HALF, c+HALF+1
    const int kr = k0 + row;
    const uint32_t o1 = (uint32_t)((row * RLD + c) * 4), o2 = (uint32_t)((row * RLD + c + HALF) * 4);
    // every head's values in flight first, then the sums in head order
    float2 a1[kMaxGroup], a2[kMaxGroup], b1[kMaxGroup], b2[kMaxGroup];
#pragma unroll
    for (int q = 0; q < kMaxGroup; ++q) {
      if (q < grp) {
        a1[q] = ld_cluster_f2(cluster_map(rk0 + o1, (uint32_t)q));
        a2[q] = ld_cluster_f2(cluster_map(rk0 + o2, (uint32_t)q));
        b1[q] = ld_cluster_f2(cluster_map(rv0 + o1, (uint32_t)q));
        b2[q] = ld_cluster_f2(cluster_map(rv0 + o2, (uint32_t)q));
      }
    }
    float2 k1 = a1[0], k2 = a2[0], v1 = b1[0], v2 = b2[0];
#pragma unroll
    for (int q = 1; q < kMaxGroup; ++q) {
      if (q < grp) {
        k1.x += a1[q].x; k1.y += a1[q].y; k2.x += a2[q].x; k2.y += a2[q].y;
        v1.x += b1[q].x; v1.y += b1[q].y; v2.x += b2[q].x; v2.y += b2[q].y;
      }
    }
    if (kr >= p.S) continue;
    __nv_bfloat16* vp = p.dv + (tok0 + kr) * p.lddv + kvh * HD;
    *reinterpret_cast<__nv_bfloat162*>(vp + c) = __floats2bfloat162_rn(v1.x, v1.y);
    *reinterpret_cast<__nv_bfloat162*>(vp + c + HALF) = __floats2bfloat162_rn(v2.x, v2.y);
    float y1[2] = {k1.x * p.scale, k1.y * p.scale}, y2[2] = {k2.x * p.scale, k2.y * p.scale};
    if (p.rope_cos) {  // inverse rotation of key position kr: pairs (c + u, c + u + HALF)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float x1 = y1[u], x2 = y2[u];
        const float cs = p.rope_cos[kr * HALF + c + u], sn = p.rope_sin[kr * HALF + c + u];
        y1[u] = x1 * cs + x2 * sn;
        y2[u] = x2 * cs - x1 * sn;
      }
    }
    __nv_bfloat16* kp = p.dk + (tok0 + kr) * p.lddk + kvh * HD;
    *reinterpret_cast<__nv_bfloat162*>(kp + c) = __floats2bfloat162_rn(y1[0], y1[1]);
    *reinterpret_cast<__nv_bfloat162*>(kp + c + HALF) = __floats2bfloat162_rn(y2[0], y2[1]);
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while another still reads its shared memory
}

// --------------------------------------------------------------------------- backward: dQ
// grid (hq, B, ceil(S/64)), 128 threads, the last query block (most keys) first; warp w owns
// queries 16w..16w+15; key tiles of 32, double-buffered.
template <int HD>
__global__ void __launch_bounds__(128) k_attn_dq(AttnBwdArgs p) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  constexpr int TL = 32 * Tile<HD>::LD;
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm_raw);
  __nv_bfloat16* Os = Qs + 64 * Tile<HD>::LD;  // dO
  __nv_bfloat16* Kbuf = Os + 64 * Tile<HD>::LD;  // [2] K tiles
  __nv_bfloat16* Vbuf = Kbuf + 2 * TL;            // [2] V tiles
  const int h = blockIdx.x, b = blockIdx.y, qb = (int)gridDim.z - 1 - (int)blockIdx.z;
  const int kvh = h / (p.hq / p.hkv);
  const int64_t tok0 = (int64_t)b * p.S;
  const int q0 = qb * 64;
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31, g = l >> 2, t4 = l & 3;
  const float sl2 = p.scale * kLog2e;

  load_tile_async<HD>(Qs, p.q, p.ldq, tok0, q0, 64, p.S, h * HD);
  load_tile_async<HD>(Os, p.dout, p.lddo, tok0, q0, 64, p.S, h * HD);
  load_tile_async<HD>(Kbuf, p.k, p.ldk, tok0, 0, 32, p.S, kvh * HD);
  load_tile_async<HD>(Vbuf, p.v, p.ldv, tok0, 0, 32, p.S, kvh * HD);
  cp_async_commit();
  const int qr0 = q0 + warp * 16 + g, qr1 = qr0 + 8;
  float lse2[2], dd[2];
  lse2[0] = qr0 < p.S ? p.lse[(tok0 + qr0) * p.hq + h] * kLog2e : 0.f;
  lse2[1] = qr1 < p.S ? p.lse[(tok0 + qr1) * p.hq + h] * kLog2e : 0.f;
  dd[0] = qr0 < p.S ? p.D[(tok0 + qr0) * p.hq + h] : 0.f;
  dd[1] = qr1 < p.S ? p.D[(tok0 + qr1) * p.hq + h] : 0.f;

  float dq[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  const int kend = min(q0 + 64, p.S);
  for (int ks0 = 0, it = 0; ks0 < kend; ks0 += 32, ++it) {
    cp_async_wait_all();
    __syncthreads();  // tile `it` is in; the other buffer is free again
    if (ks0 + 32 < kend) {
      const int nb = (it + 1) & 1;
      load_tile_async<HD>(Kbuf + nb * TL, p.k, p.ldk, tok0, ks0 + 32, 32, p.S, kvh * HD);
      load_tile_async<HD>(Vbuf + nb * TL, p.v, p.ldv, tok0, ks0 + 32, 32, p.S, kvh * HD);
      cp_async_commit();
    }
    const __nv_bfloat16* Ks = Kbuf + (it & 1) * TL;
    const __nv_bfloat16* Vs = Vbuf + (it & 1) * TL;
    const bool diag = ks0 + 31 > q0 || ks0 + 32 > p.S;  // keys past a query or past S possible
    float s[4][4], dp[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] = dp[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD; kk += 16) {
      uint32_t aq[4], ao[4];
      lda_frag<HD>(aq, Qs, warp * 16, kk);
      lda_frag<HD>(ao, Os, warp * 16, kk);
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        uint32_t bk[4], bv[4];
        ldb_rows<HD>(bk, Ks, j * 8, kk);
        ldb_rows<HD>(bv, Vs, j * 8, kk);
        mma16816(s[j], aq, bk[0], bk[1]);
        mma16816(s[j + 1], aq, bk[2], bk[3]);
        mma16816(dp[j], ao, bv[0], bv[1]);
        mma16816(dp[j + 1], ao, bv[2], bv[3]);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = ks0 + j * 8 + 2 * t4 + (e & 1);
        const int r = e >> 1;
        const int qr = r ? qr1 : qr0;
        float pv = exp2f(s[j][e] * sl2 - lse2[r]);
        if (qr >= p.S || (diag && (key > qr || key >= p.S))) pv = 0.f;
        s[j][e] = pv * (dp[j][e] - dd[r]);  // dS
      }
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int i = 0; i < HD / 8; i += 2) {
        uint32_t bk[4];
        ldb_trans<HD>(bk, Ks, kk * 16, i * 8);
        mma16816(dq[i], a, bk[0], bk[1]);
        mma16816(dq[i + 1], a, bk[2], bk[3]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qr = r ? qr1 : qr0;
    if (qr >= p.S) continue;
    __nv_bfloat16* qp = p.dq + (tok0 + qr) * p.lddq + h * HD;
    store_grad_rows<HD>(qp, dq, r, t4, qr, p.scale, p.rope_cos, p.rope_sin);
  }
}

template <typename K>
cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

bool check_common(int hd, int hq, int hkv, int S, int64_t T) {
  if (hd != 64 && hd != 128) return false;
  if (hq <= 0 || hkv <= 0 || hq % hkv) return false;
  if (S <= 0 || T <= 0 || T % S) return false;
  return true;
}

}  // namespace

cudaError_t attention_fwd(const AttnArgs& a, cudaStream_t s) {
  if (!check_common(a.hd, a.hq, a.hkv, a.S, a.T)) return cudaErrorInvalidValue;
  const int B = (int)(a.T / a.S);
  dim3 grid(a.hq, B, (a.S + 63) / 64);
  if (a.hd == 128) {
    const int sm = 5 * 64 * Tile<128>::LD * 2;
    cudaError_t e = set_smem(k_attn_fwd<128>, sm);
    if (e != cudaSuccess) return e;
    k_attn_fwd<128><<<grid, 128, sm, s>>>(a);
  } else {
    const int sm = 5 * 64 * Tile<64>::LD * 2;
    cudaError_t e = set_smem(k_attn_fwd<64>, sm);
    if (e != cudaSuccess) return e;
    k_attn_fwd<64><<<grid, 128, sm, s>>>(a);
  }
  note_launch(1);
  return cudaGetLastError();
}

template <int HD>
cudaError_t launch_dkdv(const AttnBwdArgs& a, int B, cudaStream_t s) {
  const int grp = a.hq / a.hkv;
  const int sm = 256 * Tile<HD>::LD * 2 + 4 * 32 * 4;
  static_assert(2 * 64 * (HD + 4) * 4 <= 256 * Tile<HD>::LD * 2, "partial tiles reuse the tile space");
  cudaError_t e = set_smem(k_attn_dkdv<HD>, sm);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grp, (unsigned)(B * a.hkv), (unsigned)((a.S + 63) / 64));
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)grp;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_attn_dkdv<HD>, a);
}

cudaError_t attention_bwd(const AttnBwdArgs& a, cudaStream_t s) {
  if (!check_common(a.hd, a.hq, a.hkv, a.S, a.T)) return cudaErrorInvalidValue;
  if (a.hq / a.hkv > kMaxGroup) return cudaErrorInvalidValue;
  const int B = (int)(a.T / a.S);
  {
    const int64_t n = a.T * (int64_t)a.hq;
    k_attn_D<<<(unsigned)((n + 7) / 8), 256, 0, s>>>(a);
  }
  dim3 gq(a.hq, B, (a.S + 63) / 64);
  cudaError_t e;
  if (a.hd == 128) {
    e = launch_dkdv<128>(a, B, s);
    const int smq = (64 + 64 + 4 * 32) * Tile<128>::LD * 2;
    if (e == cudaSuccess) e = set_smem(k_attn_dq<128>, smq);
    if (e == cudaSuccess) k_attn_dq<128><<<gq, 128, smq, s>>>(a);
  } else {
    e = launch_dkdv<64>(a, B, s);
    const int smq = (64 + 64 + 4 * 32) * Tile<64>::LD * 2;
    if (e == cudaSuccess) e = set_smem(k_attn_dq<64>, smq);
    if (e == cudaSuccess) k_attn_dq<64><<<gq, 128, smq, s>>>(a);
  }
  note_launch(3);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lst
