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
#include "pdl.cuh"
#include "ex2.cuh"
#include "gemm.cuh"

#include <cuda_fp16.h>

#include <atomic>
#include <cstdlib>
#include <cstring>

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

// ------------------------------------------------------------------------------------ forward, tcgen05
// One CTA per 128 queries of one head (the last query blocks, with the most keys, first); 320
// threads: warp 0 TMA producer (Q once; K and V tiles of 128 keys, double-buffered), warp 1 MMA
// issuer, warps 2-9 softmax (two threads per query row, TMEM lane = row, each half of the keys).
//   S = Q K^T           tcgen05, bf16 operands, fp32 in one of two TMEM buffers (so the next block's
//                       Q K^T runs while this block's softmax reads its scores);
//   P = exp2(S' - m)    softmax threads, written as fp16 to a 128-byte-swizzled shared tile (the
//                       MMA's A operand) -- the V tile is converted to fp16 in place meanwhile;
//   O += P V            tcgen05, fp16 operands (V MN-major), fp32 accumulator in TMEM.
// The reference max m of a row only moves when the block's max exceeds it by more than 2^8 (then O
// is rescaled in TMEM), so P <= 256 and every value of P is exact to fp16's precision; the final
// O / l and lse use the same m and l. Every wait is bounded.
template <int HD>
struct AttnTc {
  static constexpr int QB = 128, KB = 128;
  static constexpr uint32_t CH = 128 * 128;               // bytes of one [128 rows x 64] bf16 chunk
  static constexpr uint32_t Q_BYTES = (HD / 64) * CH;
  static constexpr uint32_t KV_BYTES = 2 * (HD / 64) * CH; // K then V of one stage
  static constexpr uint32_t P_BYTES = 2 * CH;              // 128 queries x 128 keys fp16
  // + barriers (128 B) and the row threads' max / sum exchange (3 KB)
  static constexpr uint32_t SMEM = Q_BYTES + 2 * KV_BYTES + P_BYTES + 1024 + 128 + 3 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;              // S[2] at columns 0 / 128, O at 256
};

template <int HD>
__global__ void __launch_bounds__(320, 1)
k_attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const AttnArgs p) {
  using C = AttnTc<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + C::Q_BYTES;        // [2] stages: K chunks, then V chunks
  uint8_t* sP = sKV + 2 * C::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + C::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);

  const int h = blockIdx.x, b = blockIdx.y, qb = (int)gridDim.z - 1 - (int)blockIdx.z;
  const int kvh = h / (p.hq / p.hkv);
  const int64_t tok0 = (int64_t)b * p.S;
  const int q0 = qb * C::QB;
  const int nkb = qb + 1;  // key blocks 0 .. qb (the causal mask ends inside block qb)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);
    }
    mbar_init(p_full, 256);
    mbar_init(pv_done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c)
        tma_load_2d(sQ + c * C::CH, &tmQ, q_full, h * HD + c * 64, (int32_t)(tok0 + q0));
      for (int j = 0; j < nkb; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&kv_empty[st], ((j - 2) >> 1) & 1)) break;
        uint8_t* sk = sKV + st * C::KV_BYTES;
        mbar_arrive_expect_tx(&kv_full[st], C::KV_BYTES);
        const int32_t y = (int32_t)(tok0 + j * C::KB);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          tma_load_2d(sk + c * C::CH, &tmK, &kv_full[st], kvh * HD + c * 64, y);
          tma_load_2d(sk + (HD / 64 + c) * C::CH, &tmV, &kv_full[st], kvh * HD + c * 64, y);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_bf16(128, C::KB, 0, 0);
      constexpr uint32_t idO = umma_idesc_f16(128, HD, 0, 1);
      bool ok = mbar_wait(q_full, 0);
      for (int j = 0; j <= nkb && ok; ++j) {
        if (j < nkb) {  // S_j = Q K_j^T into buffer j & 1
          const int st = j & 1;
          if (!mbar_wait(&kv_full[st], (j >> 1) & 1)) break;
          if (j >= 2 && !mbar_wait(&s_free[st], ((j - 2) >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t q = smem_u32(sQ), k = smem_u32(sKV + st * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::CH + (kk & 3) * 32;
            umma_bf16(tmem + st * C::KB, umma_desc(q + off, 16, 1024), umma_desc(k + off, 16, 1024), idS, kk != 0);
          }
          umma_commit(&s_full[st]);
        }
        if (j >= 1) {  // O += P_{j-1} V_{j-1}
          const int i = j - 1, st = i & 1;
          if (!mbar_wait(p_full, i & 1)) break;
          tc_fence_after();
          const uint32_t pa = smem_u32(sP), v = smem_u32(sKV + st * C::KV_BYTES + (HD / 64) * C::CH);
#pragma unroll
          for (int kk = 0; kk < C::KB / 16; ++kk) {
            const uint64_t da = umma_desc(pa + (kk >> 2) * C::CH + (kk & 3) * 32, 16, 1024);
            const uint64_t db = umma_desc(v + kk * 16 * 128, C::CH, 1024);  // 16 key rows per step
            umma_bf16(tmem + 256, da, db, idO, (i | kk) != 0);
          }
          umma_commit(&kv_empty[st]);
          umma_commit(pv_done);
        }
      }
    }
  } else {
    // Two threads per query row (warps 2-5: half 0, warps 6-9: half 1, the same TMEM lanes): half
    // h takes keys [64h, 64h + 64) of each block and O columns [h HD/2, (h + 1) HD/2). The block
    // max is exchanged through shared memory (double-buffered over blocks); the row sums are kept
    // per half and added once at the end.
    const int ts = (int)threadIdx.x - 64;  // 0 .. 255
    const int half = ts >> 7;
    const int r = (warp & 3) * 32 + lane;  // query row = TMEM lane
    const int qrow = q0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale * kLog2e;
    constexpr int NK = C::KB / 2, NO = HD / 2;
    float* smax = reinterpret_cast<float*>(bars + 12);  // [2 blocks][2 halves][128 rows]
    float* ssum = smax + 512;                            // [2 halves][128 rows]
    float mref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {  // every iteration reaches the named barrier, also after a failed wait
      const int st = j & 1;
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&kv_full[st], (j >> 1) & 1))) ok = false;
      if (ok) {  // V_j to fp16 in place, once its TMA has landed
        uint4* vt = reinterpret_cast<uint4*>(sKV + st * C::KV_BYTES + (HD / 64) * C::CH);
        for (int i = ts; i < (int)((HD / 64) * C::CH / 16); i += 256) {
          uint4 u = vt[i];
          uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            w[e] = pack_f16(f.x, f.y);
          }
          vt[i] = u;
        }
      }
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1))) ok = false;
      float x[NK];
      float pmax = -INFINITY;
      if (ok) {
        tc_fence_after();
        {
          uint32_t u[32], w[32];
          tmem_ld32(tmem + st * C::KB + half * NK + lane_off, u);
          tmem_ld32(tmem + st * C::KB + half * NK + 32 + lane_off, w);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            x[e] = __uint_as_float(u[e]) * sl2;
            x[32 + e] = __uint_as_float(w[e]) * sl2;
          }
        }
        tc_fence_before();
        mbar_arrive(&s_free[st]);
        if (j == nkb - 1) {  // only the diagonal block holds keys past a query or past S
#pragma unroll
          for (int e = 0; e < NK; ++e) {
            const int key = j * C::KB + half * NK + e;
            if (key > qrow || key >= p.S) x[e] = -INFINITY;
          }
        }
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = x[i];
#pragma unroll
        for (int e = 8; e < NK; ++e) pm[e & 7] = fmaxf(pm[e & 7], x[e]);
        pmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      smax[(j & 1) * 256 + half * 128 + r] = pmax;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (!ok) continue;
      const float bm = fmaxf(pmax, smax[(j & 1) * 256 + (1 - half) * 128 + r]);
      float corr = 1.f;
      if (j == 0) {
        mref = bm;  // block 0 always holds key 0 <= query
      } else if (bm > mref + 8.f) {
        corr = ex2_approx(mref - bm);
        mref = bm;
      }
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < NK; ++e) {
        x[e] = ex2_approx(x[e] - mref);
        ps[e & 7] += x[e];
      }
      l = l * corr + (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7])));
      if (j >= 1) {  // P_{j-1} V_{j-1} done: the P tile is free and O holds the blocks so far
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1))) {
          ok = false;
          continue;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
          for (int c = 0; c < NO; c += 32) {
            uint32_t u[32];
            tmem_ld32(tmem + 256 + half * NO + c + lane_off, u);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * corr);
            tmem_st32(tmem + 256 + half * NO + c + lane_off, u);
          }
          tmem_st_wait();
        }
      }
      // this half's 64 keys are chunk `half` of P row r; 16-byte piece i at i ^ (r & 7)
      uint8_t* prow = sP + half * C::CH + r * 128;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float* v = x + i * 8;
        *reinterpret_cast<uint4*>(prow + ((i ^ (r & 7)) * 16)) =
            make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]), pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
      }
      fence_proxy_async();  // P and the converted V are read by the tensor core
      tc_fence_before();
      mbar_arrive(p_full);
    }
    ssum[half * 128 + r] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const float lt = l + ssum[(1 - half) * 128 + r];
    // O / l (this half's columns), lse
    if (ok && __all_sync(0xffffffffu, mbar_wait(pv_done, (nkb - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.f / lt;
      const bool live = qrow < p.S;
      __nv_bfloat16* op = p.o + (tok0 + qrow) * p.ldo + h * HD + half * NO;
      float* o32 = p.o32 ? p.o32 + (tok0 + qrow) * (int64_t)p.hq * HD + h * HD + half * NO : nullptr;
#pragma unroll
      for (int c = 0; c < NO; c += 32) {
        uint32_t u[32];
        tmem_ld32(tmem + 256 + half * NO + c + lane_off, u);
        tmem_ld_wait();
        if (live) {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(u[e]) * inv;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w = make_uint4(pack_bf16(v[e], v[e + 1]), pack_bf16(v[e + 2], v[e + 3]),
                                 pack_bf16(v[e + 4], v[e + 5]), pack_bf16(v[e + 6], v[e + 7]));
            *reinterpret_cast<uint4*>(op + c + e) = w;
            if (o32) {
              *reinterpret_cast<float4*>(o32 + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
              *reinterpret_cast<float4*>(o32 + c + e + 4) = make_float4(v[e + 4], v[e + 5], v[e + 6], v[e + 7]);
            }
          }
        }
      }
      if (live && half == 0) p.lse[(tok0 + qrow) * p.hq + h] = (mref + log2f(lt)) / kLog2e;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// --------------------------------------------------------------------------- backward: dQ, tcgen05
// One CTA per 128 queries of one head (heaviest first), 320 threads: warp 0 TMA (Q and dO once; K
// and V tiles of 64 keys, three in flight), warp 1 MMA issuer, warps 2-9 two threads per query row.
// The row's threads first form D = rowsum(dO o O) and store it: this kernel runs before the dK / dV
// kernel, which reads D.
//   S = Q K^T, dP = dO V^T   tcgen05 (bf16), into one of two TMEM buffer pairs;
//   dS = P (dP - D)          the row's threads, P = exp2(S' - lse'), written bf16 to one of two
//                            swizzled tiles (so block j+1's dS is written while dQ reads block j's);
//   dQ += dS K               tcgen05 (K read MN-major from the same tile), fp32 in TMEM;
// then dQ * scale with the rotary embedding undone is stored once as bf16.
template <int HD>
struct DqTc {
  static constexpr int QB = 128, KB = 64;
  static constexpr uint32_t CH = 128 * 128;                  // [128 rows x 64] bf16 chunk
  static constexpr uint32_t KCH = 64 * 128;                  // [64 rows x 64] bf16 chunk
  static constexpr uint32_t Q_BYTES = (HD / 64) * CH;
  static constexpr uint32_t KV_BYTES = 2 * (HD / 64) * KCH;  // K then V of one stage
  static constexpr uint32_t DS_BYTES = CH;                   // 128 queries x 64 keys bf16
  static constexpr int KV_STAGES = 3;                        // K / V tiles in flight
  static constexpr uint32_t SMEM = 2 * Q_BYTES + KV_STAGES * KV_BYTES + 2 * DS_BYTES + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = 512;                 // S[2] at 0/64, dP[2] at 128/192, dQ at 256
};

template <int HD>
__global__ void __launch_bounds__(320, 1)
k_attn_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
             const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const AttnBwdArgs p) {
  using C = DqTc<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sO = sQ + C::Q_BYTES;          // dO
  constexpr int NS = C::KV_STAGES;
  uint8_t* sKV = sO + C::Q_BYTES;          // [NS] stages: K chunks, then V chunks
  uint8_t* sDS = sKV + NS * C::KV_BYTES;  // [2] dS tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + 2 * C::DS_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;        // [NS]
  uint64_t* kv_empty = bars + 1 + NS;  // [NS]
  uint64_t* s_full = bars + 1 + 2 * NS;   // [2]
  uint64_t* s_free = s_full + 2;          // [2]
  uint64_t* ds_full = s_full + 4;         // [2]
  uint64_t* ds_free = s_full + 6;         // [2] the dQ MMAs of the tile's block are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 8);

  const int h = blockIdx.x, b = blockIdx.y, qb = (int)gridDim.z - 1 - (int)blockIdx.z;
  const int kvh = h / (p.hq / p.hkv);
  const int64_t tok0 = (int64_t)b * p.S;
  const int q0 = qb * C::QB;
  const int nkb = min((q0 + C::QB + C::KB - 1) / C::KB, (p.S + C::KB - 1) / C::KB);  // keys < q0 + 128 and < S
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);
      mbar_init(&ds_full[i], 256);
      mbar_init(&ds_free[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        tma_load_2d(sQ + c * C::CH, &tmQ, q_full, h * HD + c * 64, (int32_t)(tok0 + q0));
        tma_load_2d(sO + c * C::CH, &tmO, q_full, h * HD + c * 64, (int32_t)(tok0 + q0));
      }
      for (int j = 0; j < nkb; ++j) {
        const int ks = j % NS;
        if (j >= NS && !mbar_wait(&kv_empty[ks], ((j - NS) / NS) & 1)) break;
        uint8_t* sk = sKV + ks * C::KV_BYTES;
        mbar_arrive_expect_tx(&kv_full[ks], C::KV_BYTES);
        const int32_t y = (int32_t)(tok0 + j * C::KB);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          tma_load_2d(sk + c * C::KCH, &tmK, &kv_full[ks], kvh * HD + c * 64, y);
          tma_load_2d(sk + (HD / 64 + c) * C::KCH, &tmV, &kv_full[ks], kvh * HD + c * 64, y);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_bf16(128, C::KB, 0, 0);
      constexpr uint32_t idQ = umma_idesc_bf16(128, HD, 0, 1);
      bool ok = mbar_wait(q_full, 0);
      for (int j = 0; j <= nkb && ok; ++j) {
        if (j < nkb) {  // S_j = Q K_j^T and dP_j = dO V_j^T into buffer pair j & 1
          const int st = j & 1, ks = j % NS;
          if (!mbar_wait(&kv_full[ks], (j / NS) & 1)) break;
          if (j >= 2 && !mbar_wait(&s_free[st], ((j - 2) >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t q = smem_u32(sQ), o = smem_u32(sO);
          const uint32_t k = smem_u32(sKV + ks * C::KV_BYTES), v = k + (HD / 64) * C::KCH;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t offq = (kk >> 2) * C::CH + (kk & 3) * 32, offk = (kk >> 2) * C::KCH + (kk & 3) * 32;
            umma_bf16(tmem + st * C::KB, umma_desc(q + offq, 16, 1024), umma_desc(k + offk, 16, 1024), idS, kk != 0);
            umma_bf16(tmem + 128 + st * C::KB, umma_desc(o + offq, 16, 1024), umma_desc(v + offk, 16, 1024), idS,
                      kk != 0);
          }
          umma_commit(&s_full[st]);
        }
        if (j >= 1) {  // dQ += dS_{j-1} K_{j-1}
          const int i = j - 1, st = i & 1, ks = i % NS;
          if (!mbar_wait(&ds_full[st], (i >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t ds = smem_u32(sDS + st * C::DS_BYTES), k = smem_u32(sKV + ks * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::KB / 16; ++kk) {
            const uint64_t da = umma_desc(ds + kk * 32, 16, 1024);
            const uint64_t db = umma_desc(k + kk * 16 * 128, C::KCH, 1024);  // K rows = keys: MN-major
            umma_bf16(tmem + 256, da, db, idQ, (i | kk) != 0);
          }
          umma_commit(&kv_empty[ks]);
          umma_commit(&ds_free[st]);
        }
      }
    }
  } else {
    // two threads per query row (warps 2-5 and 6-9, the same TMEM lanes): half h takes keys
    // [32h, 32h + 32) of each block, and a quarter of the rotation pairs of the dQ row at the end
    const int ts = (int)threadIdx.x - 64;
    const int half = ts >> 7;
    const int r = (warp & 3) * 32 + lane;
    const int qrow = q0 + r;
    const bool live = qrow < p.S;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale * kLog2e;
    const float lse2 = live ? p.lse[(tok0 + qrow) * p.hq + h] * kLog2e : 0.f;
    // D = rowsum(dO o O) of this row, with the forward's unrounded O when it was kept; both threads
    // of the row add the same products in the same order, and half 0 stores it for the dK / dV kernel
    float dd = 0.f;
    if (live) {
      const __nv_bfloat16* ap = p.dout + (tok0 + qrow) * p.lddo + (int64_t)h * HD;
#pragma unroll 4
      for (int c = 0; c < HD; c += 8) {
        const uint4 au = *reinterpret_cast<const uint4*>(ap + c);
        const __nv_bfloat16* a8 = reinterpret_cast<const __nv_bfloat16*>(&au);
        float o8[8];
        if (p.o32) {
          const float* op = p.o32 + (tok0 + qrow) * (int64_t)p.hq * HD + (int64_t)h * HD + c;
          const float4 u0 = *reinterpret_cast<const float4*>(op), u1 = *reinterpret_cast<const float4*>(op + 4);
          o8[0] = u0.x;
          o8[1] = u0.y;
          o8[2] = u0.z;
          o8[3] = u0.w;
          o8[4] = u1.x;
          o8[5] = u1.y;
          o8[6] = u1.z;
          o8[7] = u1.w;
        } else {
          const uint4 ou = *reinterpret_cast<const uint4*>(p.o + (tok0 + qrow) * p.ldo + (int64_t)h * HD + c);
          const __nv_bfloat16* b8 = reinterpret_cast<const __nv_bfloat16*>(&ou);
#pragma unroll
          for (int e = 0; e < 8; ++e) o8[e] = __bfloat162float(b8[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) dd += __bfloat162float(a8[e]) * o8[e];
      }
      if (half == 0) p.D[(tok0 + qrow) * p.hq + h] = dd;
    }
    bool ok = true;
    for (int j = 0; j < nkb && ok; ++j) {
      const int st = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float ds[32];
      {
        uint32_t us[32], ud[32];
        tmem_ld32(tmem + st * C::KB + half * 32 + lane_off, us);
        tmem_ld32(tmem + 128 + st * C::KB + half * 32 + lane_off, ud);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = j * C::KB + half * 32 + e;
          float pv = ex2_approx(__uint_as_float(us[e]) * sl2 - lse2);
          if (!live || key > qrow || key >= p.S) pv = 0.f;
          ds[e] = pv * (__uint_as_float(ud[e]) - dd);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[st]);
      // dS tile st is free once the dQ MMAs of block j - 2 are done
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&ds_free[st], ((j - 2) >> 1) & 1))) {
        ok = false;
        break;
      }
      uint8_t* row = sDS + st * C::DS_BYTES + r * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // pieces 4 half .. 4 half + 3 of the row
        const float* v = ds + i * 8;
        const int piece = half * 4 + i;
        *reinterpret_cast<uint4*>(row + ((piece ^ (r & 7)) * 16)) =
            make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&ds_full[st]);
    }
    // the commit after the last block's dQ MMAs: every MMA of this CTA is done
    if (ok && __all_sync(0xffffffffu, mbar_wait(&ds_free[(nkb - 1) & 1], ((nkb - 1) >> 1) & 1))) {
      tc_fence_after();
      float acc[HD];  // the whole dQ row, scaled
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t u[32];
        tmem_ld32(tmem + 256 + c + lane_off, u);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[c + e] = __uint_as_float(u[e]) * p.scale;
      }
      if (live) {  // this half's rotation pairs (c, c + hd/2), c in [half hd/4, (half + 1) hd/4)
        constexpr int HALF = HD / 2, Q4 = HD / 4;
        __nv_bfloat16* dst = p.dq + (tok0 + qrow) * p.lddq + h * HD;
#pragma unroll
        for (int c0 = 0; c0 < Q4; c0 += 8) {
          const int c = half * Q4 + c0;
          float y1[8], y2[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x1 = half ? acc[Q4 + c0 + e] : acc[c0 + e];
            const float x2 = half ? acc[Q4 + c0 + e + HALF] : acc[c0 + e + HALF];
            if (p.rope_cos) {
              const float cs = p.rope_cos[qrow * HALF + c + e], sn = p.rope_sin[qrow * HALF + c + e];
              y1[e] = x1 * cs + x2 * sn;
              y2[e] = x2 * cs - x1 * sn;
            } else {
              y1[e] = x1;
              y2[e] = x2;
            }
          }
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(pack_bf16(y1[0], y1[1]), pack_bf16(y1[2], y1[3]),
                                                          pack_bf16(y1[4], y1[5]), pack_bf16(y1[6], y1[7]));
          *reinterpret_cast<uint4*>(dst + c + HALF) = make_uint4(pack_bf16(y2[0], y2[1]), pack_bf16(y2[2], y2[3]),
                                                                 pack_bf16(y2[4], y2[5]), pack_bf16(y2[6], y2[7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// --------------------------------------------------------------------------- backward: dK, dV, tcgen05
// grid (grp, B * hkv, ceil(S/128)), cluster (grp, 1, 1), 320 threads. The cluster owns 128 keys of
// kv head kvh; its CTA of rank hh sums the contributions of query head kvh * grp + hh over query
// blocks of 64 (three Q / dO tiles in flight): warp 0 TMA, warp 1 MMA issuer, warps 2-9 two threads
// per key row.
//   S^T = K Q^T, dP^T = V dO^T      tcgen05 (bf16), into one of two TMEM buffer pairs;
//   P^T, dS^T = P^T (dP^T - D)      the key row's threads (lse and D of the block's queries from
//                                    shared memory), written bf16 to one of two pairs of swizzled
//                                    tiles (block j+1's while the MMAs read block j's);
//   dV += P^T dO, dK += dS^T Q       tcgen05, with Q / dO read MN-major from the tiles used K-major above.
// The grp partial dK / dV tiles are then parked in shared memory and CTA hh adds rows
// [hh * 128/grp, ...) over the heads in order 0 .. grp-1 (distributed shared memory), scales dK,
// undoes the rotary embedding and stores both. Deterministic, no atomics.
template <int HD>
struct DkvTc {
  static constexpr int KB = 128, QB = 64;
  static constexpr uint32_t CH = 128 * 128;                  // [128 rows x 64] bf16
  static constexpr uint32_t QCH = 64 * 128;                  // [64 rows x 64] bf16
  static constexpr uint32_t K_BYTES = (HD / 64) * CH;
  static constexpr uint32_t QO_BYTES = 2 * (HD / 64) * QCH;  // Q then dO of one stage
  static constexpr uint32_t T_BYTES = 128 * 128;             // one [128 keys x 64 queries] bf16 tile
  static constexpr int RLD = HD + 4;                         // fp32 row stride of a parked tile
  static constexpr int QO_STAGES = 3;                        // Q / dO tiles in flight
  static constexpr uint32_t MAIN = 2 * K_BYTES + QO_STAGES * QO_BYTES + 4 * T_BYTES + 2 * 2 * QB * 4;
  static constexpr uint32_t PARK = 2 * 128 * RLD * 4;
  static constexpr uint32_t SMEM = (MAIN > PARK ? MAIN : PARK) + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = 2 * 128 + 2 * HD <= 256 ? 256 : 512;
};

template <int HD>
__global__ void __launch_bounds__(320, 1)
k_attn_dkdv_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const AttnBwdArgs p) {
  using C = DkvTc<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::K_BYTES;
  constexpr int NS = C::QO_STAGES;
  uint8_t* sQO = sV + C::K_BYTES;               // [NS] stages: Q chunks, then dO chunks
  uint8_t* sP = sQO + NS * C::QO_BYTES;         // [2] P^T tiles
  uint8_t* sS = sP + 2 * C::T_BYTES;            // [2] dS^T tiles
  float* sLse = reinterpret_cast<float*>(sS + 2 * C::T_BYTES);  // [2][64]
  float* sD = sLse + 2 * C::QB;                             // [2][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (C::MAIN > C::PARK ? C::MAIN : C::PARK));
  uint64_t* kv_full = bars;
  uint64_t* qo_full = bars + 1;        // [NS]
  uint64_t* qo_empty = bars + 1 + NS;  // [NS]
  uint64_t* s_full = bars + 1 + 2 * NS;  // [2]
  uint64_t* s_free = s_full + 2;         // [2]
  uint64_t* p_full = s_full + 4;         // [2] P^T / dS^T tile pair written
  uint64_t* t_free = s_full + 6;         // [2] the dV / dK MMAs of the pair's block are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 8);
  float* redK = reinterpret_cast<float*>(smem);  // after the main loop: [128][RLD] each
  float* redV = redK + 128 * C::RLD;

  const int grp = (int)gridDim.x;
  const int hh = (int)cluster_rank();
  const int kvh = (int)blockIdx.y % p.hkv, b = (int)blockIdx.y / p.hkv, kb = (int)blockIdx.z;
  const int h = kvh * grp + hh;
  const int64_t tok0 = (int64_t)b * p.S;
  const int k0 = kb * C::KB;
  const int i0 = k0 / C::QB;                        // first query block with a query >= k0
  const int nqb = (p.S + C::QB - 1) / C::QB - i0;   // query blocks of this CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&qo_full[i], 1);
      mbar_init(&qo_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);
      mbar_init(&p_full[i], 256);
      mbar_init(&t_free[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  pdl_trigger();
  const uint32_t tV = tmem + 256, tK = tmem + 256 + HD;  // dV, dK accumulators

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * C::K_BYTES);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        tma_load_2d(sK + c * C::CH, &tmK, kv_full, kvh * HD + c * 64, (int32_t)(tok0 + k0));
        tma_load_2d(sV + c * C::CH, &tmV, kv_full, kvh * HD + c * 64, (int32_t)(tok0 + k0));
      }
      for (int j = 0; j < nqb; ++j) {
        const int qs = j % NS;
        if (j >= NS && !mbar_wait(&qo_empty[qs], ((j - NS) / NS) & 1)) break;
        uint8_t* sq = sQO + qs * C::QO_BYTES;
        mbar_arrive_expect_tx(&qo_full[qs], C::QO_BYTES);
        const int32_t y = (int32_t)(tok0 + (i0 + j) * C::QB);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          tma_load_2d(sq + c * C::QCH, &tmQ, &qo_full[qs], h * HD + c * 64, y);
          tma_load_2d(sq + (HD / 64 + c) * C::QCH, &tmO, &qo_full[qs], h * HD + c * 64, y);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_bf16(128, C::QB, 0, 0);
      constexpr uint32_t idG = umma_idesc_bf16(128, HD, 0, 1);
      bool okm = mbar_wait(kv_full, 0);
      for (int j = 0; j <= nqb && okm; ++j) {
        if (j < nqb) {  // S^T_j = K Q_j^T, dP^T_j = V dO_j^T into buffer pair j & 1
          const int st = j & 1, qs = j % NS;
          if (!mbar_wait(&qo_full[qs], (j / NS) & 1)) break;
          if (j >= 2 && !mbar_wait(&s_free[st], ((j - 2) >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t k = smem_u32(sK), v = smem_u32(sV);
          const uint32_t q = smem_u32(sQO + qs * C::QO_BYTES), o = q + (HD / 64) * C::QCH;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t offk = (kk >> 2) * C::CH + (kk & 3) * 32, offq = (kk >> 2) * C::QCH + (kk & 3) * 32;
            umma_bf16(tmem + st * C::QB, umma_desc(k + offk, 16, 1024), umma_desc(q + offq, 16, 1024), idS, kk != 0);
            umma_bf16(tmem + 128 + st * C::QB, umma_desc(v + offk, 16, 1024), umma_desc(o + offq, 16, 1024), idS,
                      kk != 0);
          }
          umma_commit(&s_full[st]);
        }
        if (j >= 1) {  // dV += P^T dO, dK += dS^T Q of block j-1
          const int i = j - 1, st = i & 1, qs = i % NS;
          if (!mbar_wait(&p_full[st], (i >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t pt = smem_u32(sP + st * C::T_BYTES), ds = smem_u32(sS + st * C::T_BYTES);
          const uint32_t q = smem_u32(sQO + qs * C::QO_BYTES), o = q + (HD / 64) * C::QCH;
#pragma unroll
          for (int kk = 0; kk < C::QB / 16; ++kk) {
            umma_bf16(tV, umma_desc(pt + kk * 32, 16, 1024), umma_desc(o + kk * 16 * 128, C::QCH, 1024), idG,
                      (i | kk) != 0);
            umma_bf16(tK, umma_desc(ds + kk * 32, 16, 1024), umma_desc(q + kk * 16 * 128, C::QCH, 1024), idG,
                      (i | kk) != 0);
          }
          umma_commit(&qo_empty[qs]);
          umma_commit(&t_free[st]);
        }
      }
    }
  } else {
    // two threads per key row (warps 2-5 and 6-9, the same TMEM lanes): half h takes queries
    // [32h, 32h + 32) of each block and parks columns [h hd/2, (h + 1) hd/2) of the row at the end
    const int t = (int)threadIdx.x - 64;   // 0 .. 255
    const int half = t >> 7;
    const int r = (warp & 3) * 32 + lane;  // key row = TMEM lane
    const int kr = k0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale * kLog2e;
    // the lse (log2 domain) and D of a block's queries, loaded by threads t < 64 one block ahead
    auto load_ld = [&](int jb, float& lv, float& dvv) {
      const int qr = (i0 + jb) * C::QB + t;
      const bool in = t < C::QB && jb < nqb && qr < p.S;
      lv = in ? p.lse[(tok0 + qr) * p.hq + h] * kLog2e : 0.f;
      dvv = in ? p.D[(tok0 + qr) * p.hq + h] : 0.f;
    };
    float nl = 0.f, nd = 0.f;
    load_ld(0, nl, nd);
    // every iteration reaches the named barrier (the eight warps together), also after a failed wait
    for (int j = 0; j < nqb; ++j) {
      const int st = j & 1;
      const int q0 = (i0 + j) * C::QB;
      if (t < C::QB) {  // the block's values, shared by every key row
        sLse[st * C::QB + t] = nl;
        sD[st * C::QB + t] = nd;
      }
      load_ld(j + 1, nl, nd);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (!ok) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1))) {
        ok = false;
        continue;
      }
      tc_fence_after();
      float pv[32], dv[32];
      {
        uint32_t us[32], ud[32];
        tmem_ld32(tmem + st * C::QB + half * 32 + lane_off, us);
        tmem_ld32(tmem + 128 + st * C::QB + half * 32 + lane_off, ud);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int qi = half * 32 + e;
          const int q = q0 + qi;
          float pe = ex2_approx(__uint_as_float(us[e]) * sl2 - sLse[st * C::QB + qi]);
          if (q < kr || q >= p.S || kr >= p.S) pe = 0.f;
          pv[e] = pe;
          dv[e] = pe * (__uint_as_float(ud[e]) - sD[st * C::QB + qi]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[st]);
      // tile pair st is free once the dV / dK MMAs of block j - 2 are done
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&t_free[st], ((j - 2) >> 1) & 1))) {
        ok = false;
        continue;
      }
      uint8_t* prow = sP + st * C::T_BYTES + r * 128;
      uint8_t* srow = sS + st * C::T_BYTES + r * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float* a = pv + i * 8;
        const float* d = dv + i * 8;
        const int pos = ((half * 4 + i) ^ (r & 7)) * 16;
        *reinterpret_cast<uint4*>(prow + pos) =
            make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]), pack_bf16(a[6], a[7]));
        *reinterpret_cast<uint4*>(srow + pos) =
            make_uint4(pack_bf16(d[0], d[1]), pack_bf16(d[2], d[3]), pack_bf16(d[4], d[5]), pack_bf16(d[6], d[7]));
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&p_full[st]);
    }
    // park this head's dK, dV rows (fp32, this half's columns) once the last block's MMAs are done
    // (the commit after them covers every earlier MMA of this CTA)
    if (ok && __all_sync(0xffffffffu, mbar_wait(&t_free[(nqb - 1) & 1], ((nqb - 1) >> 1) & 1))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = half * (HD / 2); c < (half + 1) * (HD / 2); c += 32) {
        uint32_t uk[32], uv[32];
        tmem_ld32(tK + c + lane_off, uk);
        tmem_ld32(tV + c + lane_off, uv);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          *reinterpret_cast<float4*>(redK + r * C::RLD + c + e) =
              make_float4(__uint_as_float(uk[e]), __uint_as_float(uk[e + 1]), __uint_as_float(uk[e + 2]),
                          __uint_as_float(uk[e + 3]));
          *reinterpret_cast<float4*>(redV + r * C::RLD + c + e) =
              make_float4(__uint_as_float(uv[e]), __uint_as_float(uv[e + 1]), __uint_as_float(uv[e + 2]),
                          __uint_as_float(uv[e + 3]));
        }
      }
    } else {
      ok = false;
    }
  }
  // (the tiles the parked rows overwrite are no longer read: every MMA completed before that commit)
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // every head's partial tile is parked

  constexpr int HALF = HD / 2;
  const int rows = (C::KB + grp - 1) / grp;
  const int rbeg = hh * rows, rend = min(C::KB, rbeg + rows);
  const uint32_t rk0 = smem_u32(redK), rv0 = smem_u32(redV);
  for (int item = threadIdx.x; item < (rend - rbeg) * (HALF / 2); item += blockDim.x) {
    const int row = rbeg + item / (HALF / 2);
    const int c = (item % (HALF / 2)) * 2;  // columns c, c+1 and their rotary partners c+HALF, c+HALF+1
    const int kr = k0 + row;
    const uint32_t o1 = (uint32_t)((row * C::RLD + c) * 4), o2 = (uint32_t)((row * C::RLD + c + HALF) * 4);
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// --------------------------------------------------------------------------- backward: D = rowsum(dO o)
__global__ void k_attn_D(AttnBwdArgs p) {
  pdl_wait();
  pdl_trigger();
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

template <int HD>
cudaError_t launch_fwd_tc(const AttnArgs& a, int B, cudaStream_t s) {
  using C = AttnTc<HD>;
  CUtensorMap tQ, tK, tV;
  if ((a.ldq % 8) || (a.ldk % 8) || (a.ldv % 8)) return cudaErrorInvalidValue;
  if (!make_map(&tQ, a.q, a.T, (int64_t)a.hq * HD, a.ldq, C::QB)) return cudaErrorInvalidValue;
  if (!make_map(&tK, a.k, a.T, (int64_t)a.hkv * HD, a.ldk, C::KB)) return cudaErrorInvalidValue;
  if (!make_map(&tV, a.v, a.T, (int64_t)a.hkv * HD, a.ldv, C::KB)) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr_done{0};
  if (!done_on_device(attr_done)) {
    const cudaError_t e = set_smem(k_attn_fwd_tc<HD>, C::SMEM);
    if (e != cudaSuccess) return e;
    mark_done_on_device(attr_done);
  }
  dim3 grid(a.hq, B, (a.S + C::QB - 1) / C::QB);
  return launch_k(k_attn_fwd_tc<HD>, grid, dim3(320), C::SMEM, s, 0, tQ, tK, tV, a);
}

// LST_ATTN_FWD=mma selects the warp-level mma.sync forward (for comparing the two); the tcgen05
// kernel is the default.
bool use_mma_fwd() {
  static const bool v = [] {
    const char* e = std::getenv("LST_ATTN_FWD");
    return e && std::strcmp(e, "mma") == 0;
  }();
  return v;
}

}  // namespace

cudaError_t attention_fwd(const AttnArgs& a, cudaStream_t s) {
  if (!check_common(a.hd, a.hq, a.hkv, a.S, a.T)) return cudaErrorInvalidValue;
  const int B = (int)(a.T / a.S);
  if (!use_mma_fwd()) {
    const cudaError_t e = a.hd == 128 ? launch_fwd_tc<128>(a, B, s) : launch_fwd_tc<64>(a, B, s);
    note_launch(1);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
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

namespace {

template <int HD>
cudaError_t launch_bwd_tc(const AttnBwdArgs& a, int B, cudaStream_t s) {
  using Q = DqTc<HD>;
  using K = DkvTc<HD>;
  if ((a.ldq % 8) || (a.ldk % 8) || (a.ldv % 8) || (a.lddo % 8)) return cudaErrorInvalidValue;
  CUtensorMap q64, o64, k128, v128, q128, o128, k64, v64;
  const int64_t cq = (int64_t)a.hq * HD, ck = (int64_t)a.hkv * HD;
  if (!make_map(&q64, a.q, a.T, cq, a.ldq, 64) || !make_map(&o64, a.dout, a.T, cq, a.lddo, 64) ||
      !make_map(&k128, a.k, a.T, ck, a.ldk, 128) || !make_map(&v128, a.v, a.T, ck, a.ldv, 128) ||
      !make_map(&q128, a.q, a.T, cq, a.ldq, 128) || !make_map(&o128, a.dout, a.T, cq, a.lddo, 128) ||
      !make_map(&k64, a.k, a.T, ck, a.ldk, 64) || !make_map(&v64, a.v, a.T, ck, a.ldv, 64))
    return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> attr_done{0};
  if (!done_on_device(attr_done)) {
    cudaError_t e = set_smem(k_attn_dkdv_tc<HD>, K::SMEM);
    if (e == cudaSuccess) e = set_smem(k_attn_dq_tc<HD>, Q::SMEM);
    if (e != cudaSuccess) return e;
    mark_done_on_device(attr_done);
  }
  const int grp = a.hq / a.hkv;
  dim3 gq(a.hq, B, (a.S + Q::QB - 1) / Q::QB);
  cudaError_t e = launch_k(k_attn_dq_tc<HD>, gq, dim3(320), Q::SMEM, s, 0, q128, o128, k64, v64, a);
  if (e != cudaSuccess) return e;
  const dim3 gkv((unsigned)grp, (unsigned)(B * a.hkv), (unsigned)((a.S + K::KB - 1) / K::KB));
  return launch_k(k_attn_dkdv_tc<HD>, gkv, dim3(320), K::SMEM, s, (unsigned)grp, q64, o64, k128, v128, a);
}

// LST_ATTN_BWD=mma selects the warp-level mma.sync backward (for comparing the two).
bool use_mma_bwd() {
  static const bool v = [] {
    const char* e = std::getenv("LST_ATTN_BWD");
    return e && std::strcmp(e, "mma") == 0;
  }();
  return v;
}

}  // namespace

cudaError_t attention_bwd(const AttnBwdArgs& a, cudaStream_t s) {
  if (!check_common(a.hd, a.hq, a.hkv, a.S, a.T)) return cudaErrorInvalidValue;
  if (a.hq / a.hkv > kMaxGroup) return cudaErrorInvalidValue;
  const int B = (int)(a.T / a.S);
  if (!use_mma_bwd()) {  // dQ (which forms D) then dK / dV
    const cudaError_t e = a.hd == 128 ? launch_bwd_tc<128>(a, B, s) : launch_bwd_tc<64>(a, B, s);
    note_launch(2);
    return e;
  }
  {
    const int64_t n = a.T * (int64_t)a.hq;
    const cudaError_t e = launch_k(k_attn_D, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, s, 0, a);
    if (e != cudaSuccess) return e;
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
