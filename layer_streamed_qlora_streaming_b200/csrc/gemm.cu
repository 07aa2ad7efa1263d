// bf16 GEMM on the 5th-generation tensor cores (tcgen05.mma kind::f16, fp32 accumulate in TMEM).
//
// One CTA computes a 128 x BN tile (BN = 64, 128 or 256) with three warp roles:
//   warp 0  : TMA producer (one thread) -- A and B tiles, 64 K-elements per stage, 128-byte
//             swizzle, into a ring of shared-memory stages guarded by full/empty mbarriers;
//   warp 1  : TMEM allocator and MMA issuer (one thread) -- 4 x tcgen05.mma (K = 16) per stage,
//             tcgen05.commit frees the stage when the tensor core has read it;
//   warps 2-5: epilogue -- tcgen05.ld of 32 fp32 columns per thread (one accumulator row per
//             thread), scale / bias / residual, store bf16 or fp32.
// The optional second operand pair (A2, B2) is streamed as extra K-blocks after the main ones.
#include "common.cuh"
#include "pdl.cuh"
#include "gemm.cuh"

#include <cudaTypedefs.h>

namespace lst {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

struct Epi {
  void* C;
  int64_t ldc;
  const float* bias;
  const float* R;
  int64_t ldr;
  float alpha;
  int c_f32;
  int M, N;
  // rotary embedding of output columns [0, rope_end) (whole heads of rope_hd columns)
  const float* rope_cos;
  const float* rope_sin;
  int rope_end, rope_hd, rope_S;
};

// Rotate the pair of 32-column chunks (na .. na+31) and (nb .. nb+31), nb = na + hd/2, of one row
// by the angle of position pos (pairs j, j + hd/2 with j = j0 + i), after scale and bias; store
// bf16. Used for q and k straight out of the projection GEMM, so they are rounded once.
__device__ __forceinline__ void epi_store_rope(const Epi& e, int row, int na, int nb, int j0,
                                               const uint32_t (&ra)[32], const uint32_t (&rb)[32]) {
  if (row >= e.M) return;
  const int half = e.rope_hd / 2;
  const int pos = row % e.rope_S;
  const float* cs = e.rope_cos + (int64_t)pos * half + j0;
  const float* sn = e.rope_sin + (int64_t)pos * half + j0;
  __nv_bfloat16* ca = reinterpret_cast<__nv_bfloat16*>(e.C) + (int64_t)row * e.ldc + na;
  __nv_bfloat16* cb = reinterpret_cast<__nv_bfloat16*>(e.C) + (int64_t)row * e.ldc + nb;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 ua, ub;
    __nv_bfloat162* ha = reinterpret_cast<__nv_bfloat162*>(&ua);
    __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&ub);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float ya[2], yb[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int k = q * 8 + i + u;
        float a = __uint_as_float(ra[k]) * e.alpha, b = __uint_as_float(rb[k]) * e.alpha;
        if (e.bias) {
          a += e.bias[na + k];
          b += e.bias[nb + k];
        }
        const float c = cs[k], s = sn[k];
        ya[u] = a * c - b * s;
        yb[u] = b * c + a * s;
      }
      ha[i / 2] = __floats2bfloat162_rn(ya[0], ya[1]);
      hb[i / 2] = __floats2bfloat162_rn(yb[0], yb[1]);
    }
    *reinterpret_cast<uint4*>(ca + q * 8) = ua;
    *reinterpret_cast<uint4*>(cb + q * 8) = ub;
  }
}

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t SMEM = STAGES * (A_BYTES + B_BYTES) + 1024 /*align*/ + 256 /*bars*/;
  static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;  // one accumulator; two are allocated
};

__device__ __forceinline__ void epi_store(const Epi& e, int row, int col0, const uint32_t (&r)[32]) {
  if (row >= e.M || col0 >= e.N) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * e.alpha;
  const bool full = col0 + 32 <= e.N;
  if (e.bias) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (full || col0 + i < e.N) v[i] += e.bias[col0 + i];
  }
  if (e.R) {
    const float* rp = e.R + (int64_t)row * e.ldr + col0;
    if (full && ((reinterpret_cast<uintptr_t>(rp) & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 u = *reinterpret_cast<const float4*>(rp + q * 4);
        v[q * 4] += u.x;
        v[q * 4 + 1] += u.y;
        v[q * 4 + 2] += u.z;
        v[q * 4 + 3] += u.w;
      }
    } else {
      for (int i = 0; i < 32; ++i)
        if (col0 + i < e.N) v[i] += rp[i];
    }
  }
  if (e.c_f32) {
    float* cp = reinterpret_cast<float*>(e.C) + (int64_t)row * e.ldc + col0;
    if (full && ((reinterpret_cast<uintptr_t>(cp) & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(cp + q * 4) = make_float4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
    } else {
      for (int i = 0; i < 32; ++i)
        if (col0 + i < e.N) cp[i] = v[i];
    }
  } else {
    __nv_bfloat16* cp = reinterpret_cast<__nv_bfloat16*>(e.C) + (int64_t)row * e.ldc + col0;
    if (full && ((reinterpret_cast<uintptr_t>(cp) & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
        *reinterpret_cast<uint4*>(cp + q * 8) = u;
      }
    } else {
      for (int i = 0; i < 32; ++i)
        if (col0 + i < e.N) cp[i] = __float2bfloat16_rn(v[i]);
    }
  }
}

// Tile order: groups of kGroupM M-tiles; inside a group the M-tile index runs fastest, so the
// CTAs working at the same time share a few weight (B) tiles and the group's activation rows in
// L2.
constexpr int kGroupM = 16;

struct TileSched {
  int mt, nt;
  __device__ __forceinline__ void get(int t, int& m, int& n) const {
    const int r = t;
    const int per_group = kGroupM * nt;
    const int g = r / per_group;
    const int first = g * kGroupM;
    const int gsz = min(kGroupM, mt - first);
    const int q = r - g * per_group;
    m = first + q % gsz;
    n = q / gsz;
  }
};

// Persistent tcgen05 GEMM. Each CTA loops over tiles t = blockIdx.x, + gridDim.x, ... and keeps
// two fp32 accumulators in TMEM, so the epilogue of one tile overlaps the main loop of the next.
// AMN / BMN: A / B operand MN-major (row-major [K, M] / [K, N] in global memory), else K-major.
template <int BN, int AMN, int BMN>
__global__ void __launch_bounds__(192, 1)
k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
       const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
       const Epi ep, const TileSched sched, const int total_tiles, const int nk1, const int nk2) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2] accumulator ready for the epilogue
  uint64_t* acc_empty = acc_full + 2;       // [2] accumulator drained by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (nk2) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * C::TMEM_COLS);
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
      uint32_t it = 0;  // stage counter across tiles
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        int mi, ni;
        sched.get(t, mi, ni);
        const int m0 = mi * BM, n0 = ni * BN;
        const int nk = nk1 + nk2;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
          const bool second = kb >= nk1;
          const CUtensorMap* ma = second ? &tmA2 : &tmA;
          const CUtensorMap* mb = second ? &tmB2 : &tmB;
          const int kk = (second ? kb - nk1 : kb) * BK;
          if (AMN == 0) {
            tma_load_2d(sA + s * C::A_BYTES, ma, &full[s], kk, m0);
          } else {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(sA + s * C::A_BYTES + c * (64 * BK * 2), ma, &full[s], m0 + c * 64, kk);
          }
          if (BMN == 0) {
            tma_load_2d(sB + s * C::B_BYTES, mb, &full[s], kk, n0);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(sB + s * C::B_BYTES + c * (64 * BK * 2), mb, &full[s], n0 + c * 64, kk);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN, AMN, BMN);
      uint32_t it = 0;
      bool ok = true;
      int local = 0;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++local) {
        const int nk = nk1 + nk2;
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        // the epilogue must have drained this accumulator (its use two tiles ago)
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + (uint32_t)(buf * C::TMEM_COLS);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&full[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = AMN ? umma_desc(a0 + k * 16 * 128, 64 * BK * 2, 1024)
                                    : umma_desc(a0 + k * 32, 16, 1024);
            const uint64_t db = BMN ? umma_desc(b0 + k * 16 * 128, 64 * BK * 2, 1024)
                                    : umma_desc(b0 + k * 32, 16, 1024);
            umma_bf16(dacc, da, db, idesc, (kb | k) != 0);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[buf]);
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int local = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++local) {
      int mi, ni;
      sched.get(t, mi, ni);
      const int m0 = mi * BM, n0 = ni * BN;
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&acc_full[buf], use & 1)) break;
      tc_fence_after();
      const int row = m0 + q * 32 + lane;
      const uint32_t tq = tmem + (uint32_t)(buf * C::TMEM_COLS) + ((uint32_t)(q * 32) << 16);
      if (n0 < ep.rope_end) {
        const int half = ep.rope_hd / 2;
#pragma unroll 1
        for (int h0 = 0; h0 < BN; h0 += ep.rope_hd) {
#pragma unroll 1
          for (int j0 = 0; j0 < half; j0 += 32) {
            uint32_t ra[32], rb[32];
            tmem_ld32(tq + h0 + j0, ra);
            tmem_ld32(tq + h0 + half + j0, rb);
            tmem_ld_wait();
            epi_store_rope(ep, row, n0 + h0 + j0, n0 + h0 + half + j0, j0, ra, rb);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tq + c, r);
          tmem_ld_wait();
          epi_store(ep, row, n0 + c, r);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);  // all 128 epilogue threads arrive once per tile
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// NF4-dequantising variant: the B operand is built in shared memory by dequantiser warps.
//
// Warp roles (320 threads): 0 TMA producer of A (and of the LoRA pair's A2 / B2), 1 MMA issuer,
// 2-5 epilogue (as k_gemm), 6-9 dequantisers. For each K stage below nk1 the dequantisers read the
// stage's NF4 blocks straight from global memory -- BN blocks of 64 codes, one per 128-byte row of
// the stage's B tile -- and write bf16(code value x absmax) in the same 128-byte-swizzled layout a
// TMA load of the bf16 matrix would produce, so the MMA descriptors are those of k_gemm. The
// absmax is dequantised with the same fp32 operations as nf4.cu ((q * s) / 127 + mean), so the
// operand equals the dequantised matrix bit for bit. Every generic-proxy write is fenced for the
// async proxy before the writer arrives on the stage's bfull barrier (one arrival per thread).
constexpr int kDqWarps = 4;
constexpr int kDqThreads = kDqWarps * 32;

template <int BN, int BMN>
__device__ __forceinline__ void dq_stage(const Nf4Mat& q, const float* cbs, uint8_t* sBs, int n0, int kb, int N,
                                         int K) {
  constexpr int HPT = 2 * BN / kDqThreads;  // half blocks (32 codes) per thread and stage
  const int dt = (int)threadIdx.x - 192;
  const int kk = kb * 64;
  uint4 raw[HPT];
  float ahat[HPT];
#pragma unroll
  for (int j = 0; j < HPT; ++j) {
    const int h = dt + kDqThreads * j;
    const int bi = h >> 1, half = h & 1;
    int wrow, wcol;  // W element (row, column) of the block's first code
    bool ok;
    if (BMN == 0) {  // B(n, k) = W[n][k]: tile row bi is W row n0 + bi, columns kk .. kk + 63
      wrow = n0 + bi;
      wcol = kk;
      ok = wrow < N;
    } else {         // B(k, n) = W[k][n]: sub-tile bi / 64, row bi % 64 is W row kk + bi % 64
      wrow = kk + (bi & 63);
      wcol = n0 + (bi >> 6) * 64;
      ok = wrow < K && wcol < N;
    }
    raw[j] = make_uint4(0, 0, 0, 0);
    ahat[j] = 0.f;
    if (ok) {
      int g = 0;
      while (g + 1 < q.nseg && wrow >= q.row_end[g]) ++g;
      const int r0 = g ? q.row_end[g - 1] : 0;
      const int64_t b = (int64_t)(wrow - r0) * (q.cols >> 6) + (wcol >> 6);
      raw[j] = __ldg(reinterpret_cast<const uint4*>(q.packed[g] + b * 32 + half * 16));
      const float qs = __fmul_rn((float)q.qabs[g][b], q.gscale[g][b >> 8]);
      ahat[j] = __fadd_rn(__fdiv_rn(qs, 127.0f), *q.mean[g]);
    }
  }
  // (the caller has waited until the stage is free)
#pragma unroll
  for (int j = 0; j < HPT; ++j) {
    const int h = dt + kDqThreads * j;
    const int bi = h >> 1, half = h & 1;
    const int row = BMN == 0 ? bi : (bi & 63);
    uint8_t* rowp = sBs + (BMN == 0 ? bi * 128 : (bi >> 6) * (64 * 128) + (bi & 63) * 128);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[j]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {  // 16-byte chunk 4 * half + c of the row: codes 8c .. 8c + 7 of the half
      uint4 o;
      uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int by = 0; by < 4; ++by) {
        const uint32_t v = (w[c] >> (8 * by)) & 0xffu;  // element 2 by in the high nibble
        const float hi = __fmul_rn(cbs[v >> 4], ahat[j]);
        const float lo = __fmul_rn(cbs[v & 15u], ahat[j]);
        __nv_bfloat162 pr = __floats2bfloat162_rn(hi, lo);
        op[by] = *reinterpret_cast<uint32_t*>(&pr);
      }
      const int chunk = (4 * half + c) ^ (row & 7);  // 128-byte swizzle
      *reinterpret_cast<uint4*>(rowp + chunk * 16) = o;
    }
  }
}

template <int BN, int BMN>
__global__ void __launch_bounds__(192 + kDqThreads, 1)
k_gemm_nf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
           const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ Nf4Mat q, const Epi ep,
           const TileSched sched, const int total_tiles, const int nk1, const int nk2, const int N, const int K) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* bfull = empty + C::STAGES;      // [STAGES] dequantised B tile written
  uint64_t* acc_full = bfull + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* cbs = reinterpret_cast<float*>(tmem_slot + 4);  // codebook [16]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&bfull[s], kDqThreads);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    fence_mbar_init();
  }
  if (threadIdx.x < 16) cbs[threadIdx.x] = q.cb[threadIdx.x];
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    if (nk2) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * C::TMEM_COLS);
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
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        int mi, ni;
        sched.get(t, mi, ni);
        const int m0 = mi * BM, n0 = ni * BN;
        const int nk = nk1 + nk2;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            ok = false;
            break;
          }
          if (kb < nk1) {  // A only; the dequantisers fill B
            mbar_arrive_expect_tx(&full[s], C::A_BYTES);
            tma_load_2d(sA + s * C::A_BYTES, &tmA, &full[s], kb * BK, m0);
          } else {         // the LoRA pair, both by TMA
            const int kk = (kb - nk1) * BK;
            mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
            tma_load_2d(sA + s * C::A_BYTES, &tmA2, &full[s], kk, m0);
            if (BMN == 0) {
              tma_load_2d(sB + s * C::B_BYTES, &tmB2, &full[s], kk, n0);
            } else {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c)
                tma_load_2d(sB + s * C::B_BYTES + c * (64 * BK * 2), &tmB2, &full[s], n0 + c * 64, kk);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN, 0, BMN);
      uint32_t it = 0, bph = 0;  // bph: bit s = parity of the next bfull[s] phase
      bool ok = true;
      int local = 0;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++local) {
        const int nk = nk1 + nk2;
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + (uint32_t)(buf * C::TMEM_COLS);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&full[s], ph)) {
            ok = false;
            break;
          }
          if (kb < nk1) {
            if (!mbar_wait(&bfull[s], (bph >> s) & 1)) {
              ok = false;
              break;
            }
            bph ^= 1u << s;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = umma_desc(a0 + k * 32, 16, 1024);
            const uint64_t db = BMN ? umma_desc(b0 + k * 16 * 128, 64 * BK * 2, 1024) : umma_desc(b0 + k * 32, 16, 1024);
            umma_bf16(dacc, da, db, idesc, (kb | k) != 0);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[buf]);
      }
    }
  } else if (warp < 6) {
    const int qd = warp & 3;
    int local = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++local) {
      int mi, ni;
      sched.get(t, mi, ni);
      const int m0 = mi * BM, n0 = ni * BN;
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&acc_full[buf], use & 1)) break;
      tc_fence_after();
      const int row = m0 + qd * 32 + lane;
      const uint32_t tq = tmem + (uint32_t)(buf * C::TMEM_COLS) + ((uint32_t)(qd * 32) << 16);
      if (n0 < ep.rope_end) {
        const int half = ep.rope_hd / 2;
#pragma unroll 1
        for (int h0 = 0; h0 < BN; h0 += ep.rope_hd) {
#pragma unroll 1
          for (int j0 = 0; j0 < half; j0 += 32) {
            uint32_t ra[32], rb[32];
            tmem_ld32(tq + h0 + j0, ra);
            tmem_ld32(tq + h0 + half + j0, rb);
            tmem_ld_wait();
            epi_store_rope(ep, row, n0 + h0 + j0, n0 + h0 + half + j0, j0, ra, rb);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tq + c, r);
          tmem_ld_wait();
          epi_store(ep, row, n0 + c, r);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  } else {
    uint32_t it = 0, bph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      int mi, ni;
      sched.get(t, mi, ni);
      const int n0 = ni * BN;
      const int nk = nk1 + nk2;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        if (kb >= nk1) continue;
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          ok = false;
          break;
        }
        dq_stage<BN, BMN>(q, cbs, sB + s * C::B_BYTES, n0, kb, N, K);
        fence_proxy_async();  // the tensor core reads this stage through the async proxy
        mbar_arrive(&bfull[s]);
        bph ^= 1u << s;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * C::TMEM_COLS);
  }
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <int BN, int BMN>
cudaError_t launch_nf4(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<BN>;
  constexpr uint32_t kSmemQ = C::STAGES * (C::A_BYTES + C::B_BYTES) + 1024 /*align*/ + 512 /*barriers, codebook*/;
  CUtensorMap tA, tA2, tB2;
  if (!make_map(&tA, a.A, a.M, a.K, a.lda, BM)) return cudaErrorInvalidValue;
  int nk2 = 0;
  if (a.A2 && a.B2 && a.K2 > 0) {
    if (!make_map(&tA2, a.A2, a.M, a.K2, a.lda2, BM)) return cudaErrorInvalidValue;
    if (BMN) {
      if (!make_map(&tB2, a.B2, a.K2, a.N, a.ldb2, BK)) return cudaErrorInvalidValue;
    } else {
      if (!make_map(&tB2, a.B2, a.N, a.K2, a.ldb2, BN)) return cudaErrorInvalidValue;
    }
    nk2 = (a.K2 + BK - 1) / BK;
  } else {
    tA2 = tA;
    tB2 = tA;
  }
  Epi e{a.C, a.ldc, a.bias, a.R, a.ldr, a.alpha, a.c_f32, a.M, a.N,
        a.rope_cos, a.rope_sin, a.rope_cos ? a.rope_end : 0, a.rope_hd, a.rope_S};
  static std::atomic<unsigned long long> attr_done{0};
  if (!done_on_device(attr_done)) {
    const cudaError_t err = cudaFuncSetAttribute(k_gemm_nf4<BN, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemQ);
    if (err != cudaSuccess) return err;
    mark_done_on_device(attr_done);
  }
  const int nk1 = (a.K + BK - 1) / BK;  // MN-major W: K = W's rows, any count (the tail rows are zero)
  TileSched sched;
  sched.mt = (a.M + BM - 1) / BM;
  sched.nt = (a.N + BN - 1) / BN;
  const int total = sched.mt * sched.nt;
  const int num_sms = device_sm_count();
  const int grid = total < num_sms ? total : num_sms;
  const cudaError_t err = launch_k(k_gemm_nf4<BN, BMN>, dim3(grid), dim3(192 + kDqThreads), kSmemQ, s, 0, tA, tA2, tB2,
                                   *a.Bq, e, sched, total, nk1, nk2, a.N, a.K);
  note_launch(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <int BN, int AMN, int BMN>
cudaError_t launch(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<BN>;
  CUtensorMap tA, tB, tA2, tB2;
  const int box_b = BMN ? BK : BN;  // K-major B: box [BN rows, 64 k]; MN-major: [64 k rows, 64 n]
  if (AMN) {
    if (!make_map(&tA, a.A, a.K, a.M, a.lda, BK)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tA, a.A, a.M, a.K, a.lda, BM)) return cudaErrorInvalidValue;
  }
  if (BMN) {
    if (!make_map(&tB, a.B, a.K, a.N, a.ldb, box_b)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tB, a.B, a.N, a.K, a.ldb, box_b)) return cudaErrorInvalidValue;
  }
  int nk2 = 0;
  if (a.A2 && a.B2 && a.K2 > 0) {
    if (AMN) return cudaErrorInvalidValue;
    if (!make_map(&tA2, a.A2, a.M, a.K2, a.lda2, BM)) return cudaErrorInvalidValue;
    if (BMN) {
      if (!make_map(&tB2, a.B2, a.K2, a.N, a.ldb2, box_b)) return cudaErrorInvalidValue;
    } else {
      if (!make_map(&tB2, a.B2, a.N, a.K2, a.ldb2, box_b)) return cudaErrorInvalidValue;
    }
    nk2 = (a.K2 + BK - 1) / BK;
  } else {
    tA2 = tA;
    tB2 = tB;
  }
  Epi e{a.C, a.ldc, a.bias, a.R, a.ldr, a.alpha, a.c_f32, a.M, a.N,
        a.rope_cos, a.rope_sin, a.rope_cos ? a.rope_end : 0, a.rope_hd, a.rope_S};
  static std::atomic<unsigned long long> attr_done{0};  // devices whose function attribute is set
  if (!done_on_device(attr_done)) {
    const cudaError_t err = cudaFuncSetAttribute(k_gemm<BN, AMN, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    mark_done_on_device(attr_done);
  }
  const int nk1 = (a.K + BK - 1) / BK;
  TileSched sched;
  sched.mt = (a.M + BM - 1) / BM;
  sched.nt = (a.N + BN - 1) / BN;
  const int total = sched.mt * sched.nt;
  const int num_sms = device_sm_count();
  const int grid = total < num_sms ? total : num_sms;
  const cudaError_t err = launch_k(k_gemm<BN, AMN, BMN>, dim3(grid), dim3(192), C::SMEM, s, 0, tA, tB, tA2, tB2, e,
                                   sched, total, nk1, nk2);
  note_launch(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t gemm_bf16(const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0 || !a.A || (!a.B && !a.Bq) || !a.C) return cudaErrorInvalidValue;
  // TMA: 16-byte aligned bases and row strides
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(a.A) || (a.lda % 8)) return cudaErrorInvalidValue;
  if (!a.Bq && (!al16(a.B) || (a.ldb % 8))) return cudaErrorInvalidValue;
  if (a.Bq) {
    // W's rows are whole NF4 blocks; packed tensors 16-byte aligned; rows covered by the tensors
    const Nf4Mat& q = *a.Bq;
    const int wrows = a.b_mn ? a.K : a.N, wcols = a.b_mn ? a.N : a.K;
    if (a.a_mn || q.nseg < 1 || q.nseg > 3 || q.cols != wcols || (wcols % 64) || q.row_end[q.nseg - 1] < wrows)
      return cudaErrorInvalidValue;
    for (int g = 0; g < q.nseg; ++g)
      if (!q.packed[g] || !q.qabs[g] || !q.gscale[g] || !q.mean[g] || !al16(q.packed[g]) ||
          (g && q.row_end[g] <= q.row_end[g - 1]))
        return cudaErrorInvalidValue;
  }
  if (a.A2 && (!al16(a.A2) || !al16(a.B2) || (a.lda2 % 8) || (a.ldb2 % 8))) return cudaErrorInvalidValue;
  const int64_t tiles256 = (int64_t)((a.M + BM - 1) / BM) * ((a.N + 255) / 256);
  int bn;
  if (a.N <= 64) bn = 64;
  else if (a.N <= 128 || tiles256 < 120) bn = 128;
  else bn = 256;
  if (a.rope_cos) {
    // rotated columns: whole tiles of whole heads, bf16 output, no residual / split / MN-major A
    if (!a.rope_sin || (a.rope_hd != 64 && a.rope_hd != 128) || a.rope_S <= 0 || a.c_f32 || a.R ||
        a.a_mn || (a.ldc % 8) || (reinterpret_cast<uintptr_t>(a.C) & 15))
      return cudaErrorInvalidValue;
    if (bn == 256 && (a.rope_end % 256)) bn = 128;
    if (bn < 128 || (a.rope_end % bn) || a.rope_end > a.N) return cudaErrorInvalidValue;
  }
  if (a.Bq) {
    switch (bn * 2 + (a.b_mn ? 1 : 0)) {
      case 64 * 2 + 0: return launch_nf4<64, 0>(a, s);
      case 64 * 2 + 1: return launch_nf4<64, 1>(a, s);
      case 128 * 2 + 0: return launch_nf4<128, 0>(a, s);
      case 128 * 2 + 1: return launch_nf4<128, 1>(a, s);
      case 256 * 2 + 0: return launch_nf4<256, 0>(a, s);
      default: return launch_nf4<256, 1>(a, s);
    }
  }
  const int code = bn * 4 + (a.a_mn ? 2 : 0) + (a.b_mn ? 1 : 0);
  switch (code) {
    case 64 * 4 + 0: return launch<64, 0, 0>(a, s);
    case 64 * 4 + 1: return launch<64, 0, 1>(a, s);
    case 64 * 4 + 3: return launch<64, 1, 1>(a, s);
    case 128 * 4 + 0: return launch<128, 0, 0>(a, s);
    case 128 * 4 + 1: return launch<128, 0, 1>(a, s);
    case 128 * 4 + 3: return launch<128, 1, 1>(a, s);
    case 256 * 4 + 0: return launch<256, 0, 0>(a, s);
    case 256 * 4 + 1: return launch<256, 0, 1>(a, s);
    case 256 * 4 + 3: return launch<256, 1, 1>(a, s);
    default: return cudaErrorInvalidValue;  // MN-major A with K-major B is not instantiated
  }
}

}  // namespace lst
