// LoRA side path on the tensor cores ("Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU",
// section "LoRA and QLoRA": trainable low-rank matrices next to the frozen base).
//
// For a projection y = x W^T + s (x A^T) B^T the side path needs, per fused group of projections
// sharing an input (q/k/v, o, gate/up, down):
//   forward   U  = x Acat^T          [T, nseg*r]   (then s*U enters the base GEMM as extra K columns)
//   backward  V  = dy Bexp            [T, nseg*r]  (s*V enters the dX GEMM the same way)
//             dA = s V^T x,  dB = s dy^T U          (reductions over the T tokens)
// Each of the four has one short side (nseg*r <= 64) and a long contraction (the in / out features,
// or the T tokens), so one output tile holds little work and a plain tiling leaves most SMs idle.
// The adapters are kept in full precision, so the projections run on a split operand: each adapter
// value is the bf16 pair (hi, lo), both parts are contracted against the same tile of x or dy into
// one fp32 accumulator, and U / V are stored as bf16 pairs again (lora.cuh, lora_skinny_split).
// One kernel serves all four: a 128 x 64 output tile is computed by a thread-block cluster of cs
// CTAs, CTA z contracting K-slice z with bf16 tcgen05 MMAs into TMEM (fp32); the cs partial tiles
// are then parked in shared memory and summed through distributed shared memory, each CTA summing
// 128/cs rows in slice order 0, 1, ..., cs-1, and stored by the mode's epilogue. No atomics and no
// global scratch: the result depends only on the shapes, so it is deterministic.
#include "common.cuh"
#include "pdl.cuh"
#include "gemm.cuh"
#include "lora.cuh"

namespace lst {
namespace {

constexpr int kBM = 128, kBN = 64, kBK = 64, kMaxCluster = 8;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr int kRedLd = kBN + 4;  // fp32 row stride of a parked partial tile (conflict-free float4 rows)
// DUAL: two B tiles per K step (the hi and lo parts of a split operand), one stage fewer so that
// two CTAs still fit on an SM.
template <int DUAL>
struct SideCfg {
  static constexpr int kStages = DUAL ? 3 : 4;
  static constexpr uint32_t kStageB = (1 + DUAL) * kBBytes;
  static constexpr uint32_t kSmem = kStages * (kABytes + kStageB) + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kBM * kRedLd * 4 <= kStages * kABytes, "the partial tile reuses the A stages");
};

// Destination of the summed tile C [M, N] (times scale).
struct SideOut {
  // 0: out16[row * ld + col] = bf16(c)                                      (U or V, [T, KP])
  // 1: row p*r + j (< nseg*r) -> dst[p][j * N + col]                       (dA, [r, in] each)
  // 2: row o of segment p, column p*r + j -> dst[p][(o - bounds[p]) * r + j] (dB, [out_p, r] each)
  // 3: column j < R: hi = bf16(c) to out16[row * ld + j] and [.. + 2 RS + j], lo = bf16(c - hi)
  //    to [.. + RS + j]                                                     (split U or V, [T, KP])
  int mode;
  int M, N;
  float scale;
  __nv_bfloat16* out16;
  int64_t ld;
  float* dst[3];
  int r, nseg;
  int bounds[4];
  int R, RS;  // mode 3
};

__device__ __forceinline__ void side_store(const SideOut& o, int row, int col, float4 v) {
  if (row >= o.M || col >= o.N) return;
  const float a[4] = {o.scale * v.x, o.scale * v.y, o.scale * v.z, o.scale * v.w};
  const bool full = col + 4 <= o.N;
  if (o.mode == 3) {
    __nv_bfloat16* p = o.out16 + (int64_t)row * o.ld;
    for (int i = 0; i < 4; ++i) {
      const int j = col + i;
      if (j >= o.R) break;
      const __nv_bfloat16 hi = __float2bfloat16_rn(a[i]);
      p[j] = hi;
      p[o.RS + j] = __float2bfloat16_rn(a[i] - __bfloat162float(hi));
      p[2 * o.RS + j] = hi;
    }
  } else if (o.mode == 0) {
    __nv_bfloat16* p = o.out16 + (int64_t)row * o.ld + col;
    if (full && (reinterpret_cast<uintptr_t>(p) & 7) == 0) {
      const __nv_bfloat162 h[2] = {__floats2bfloat162_rn(a[0], a[1]), __floats2bfloat162_rn(a[2], a[3])};
      *reinterpret_cast<uint2*>(p) = *reinterpret_cast<const uint2*>(h);
    } else {
      for (int i = 0; i < 4; ++i)
        if (col + i < o.N) p[i] = __float2bfloat16_rn(a[i]);
    }
  } else if (o.mode == 1) {
    if (row >= o.nseg * o.r) return;
    const int p = row / o.r;
    float* d = o.dst[p] + (int64_t)(row - p * o.r) * o.N + col;
    if (full && (reinterpret_cast<uintptr_t>(d) & 15) == 0) {
      *reinterpret_cast<float4*>(d) = make_float4(a[0], a[1], a[2], a[3]);
    } else {
      for (int i = 0; i < 4; ++i)
        if (col + i < o.N) d[i] = a[i];
    }
  } else {
    int p = 0;
    while (p + 1 < o.nseg && row >= o.bounds[p + 1]) ++p;
    float* d = o.dst[p] + (int64_t)(row - o.bounds[p]) * o.r;
    for (int i = 0; i < 4; ++i) {
      const int j = col + i - p * o.r;
      if (col + i < o.N && j >= 0 && j < o.r) d[j] = a[i];
    }
  }
}

// One problem of a launch: C [M, N] = A B^T over the launch's K, its operands' tensor maps, its
// destination, the first output tile (cluster row) it owns and its number of M-tiles.
constexpr int kMaxProbs = 8;
struct SideProb {
  CUtensorMap tA, tB;
  SideOut o;
  int tile0, mt;
};
struct SideProbs {
  SideProb p[kMaxProbs];
  int np;
};

// grid (cs, tiles), cluster (cs, 1, 1), 192 threads: warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2-5 park the accumulator; then all threads sum and store.
// AMN / BMN: A / B MN-major ([K, M] / [K, N] row-major in memory), else K-major.
// DUAL: every K step also loads the B tile b_off further along N (rows of a K-major B, columns of
// an MN-major B) and accumulates its product with the same A tile.
// A launch carries up to kMaxProbs problems of the same K (e.g. the dA and dB reductions of every
// group of a layer): cluster row y belongs to the last problem whose tile0 <= y and takes that
// problem's tile y - tile0, in M-fastest order over its M-tiles.
template <int AMN, int BMN, int DUAL>
__global__ void __launch_bounds__(192, 2)
k_side(const __grid_constant__ SideProbs P, const int nk, const int kps, const int b_off) {
  constexpr int kStages = SideCfg<DUAL>::kStages;
  constexpr uint32_t kStageB = SideCfg<DUAL>::kStageB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kStageB);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  float* red = reinterpret_cast<float*>(smem);  // parked partial tile, once the last MMA has read sA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cs = (int)gridDim.x;  // one cluster = the K slices of one output tile
  const int z = (int)cluster_rank();
  int pi = 0;
  while (pi + 1 < P.np && (int)blockIdx.y >= P.p[pi + 1].tile0) ++pi;
  const SideProb& pr = P.p[pi];
  const int tt = (int)blockIdx.y - pr.tile0;
  const int m0 = (tt % pr.mt) * kBM, n0 = (tt / pr.mt) * kBN;
  const CUtensorMap* ma = &pr.tA;
  const CUtensorMap* mb = &pr.tB;
  const SideOut& oo = pr.o;
  const int kb0 = z * kps;
  const int nkb = max(0, min(nk - kb0, kps));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(ma);
    tma_prefetch_desc(mb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kBN);
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
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        mbar_arrive_expect_tx(&full[s], kABytes + kStageB);
        const int kk = (kb0 + kb) * kBK;
        if (AMN == 0) {
          tma_load_2d(sA + s * kABytes, ma, &full[s], kk, m0);
        } else {
          tma_load_2d(sA + s * kABytes, ma, &full[s], m0, kk);
          tma_load_2d(sA + s * kABytes + 64 * kBK * 2, ma, &full[s], m0 + 64, kk);
        }
        if (BMN == 0) {
          tma_load_2d(sB + s * kStageB, mb, &full[s], kk, n0);
          if (DUAL) tma_load_2d(sB + s * kStageB + kBBytes, mb, &full[s], kk, n0 + b_off);
        } else {
          tma_load_2d(sB + s * kStageB, mb, &full[s], n0, kk);
          if (DUAL) tma_load_2d(sB + s * kStageB + kBBytes, mb, &full[s], n0 + b_off, kk);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nkb > 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, kBN, AMN, BMN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        if (!mbar_wait(&full[s], ph)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kABytes);
        const uint32_t b0 = smem_u32(sB + s * kStageB);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t da = AMN ? umma_desc(a0 + k * 16 * 128, 64 * kBK * 2, 1024) : umma_desc(a0 + k * 32, 16, 1024);
          const uint64_t db = BMN ? umma_desc(b0 + k * 16 * 128, 64 * kBK * 2, 1024) : umma_desc(b0 + k * 32, 16, 1024);
          umma_bf16(tmem, da, db, idesc, (kb | k) != 0);
          if (DUAL) {
            const uint32_t b1 = b0 + kBBytes;
            const uint64_t db1 = BMN ? umma_desc(b1 + k * 16 * 128, 64 * kBK * 2, 1024) : umma_desc(b1 + k * 32, 16, 1024);
            umma_bf16(tmem, da, db1, idesc, 1);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);  // arrives once every MMA issued above has completed
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    float* rr = red + (q * 32 + lane) * kRedLd;
    if (nkb > 0) {
      mbar_wait(acc_full, 0);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (uint32_t)c + ((uint32_t)(q * 32) << 16), r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(rr + c + i) = make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                                               __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
      }
    } else {
      for (int c = 0; c < kBN; c += 4) *reinterpret_cast<float4*>(rr + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // every slice's partial tile is parked

  // CTA z sums rows [z * 128/cs, (z + 1) * 128/cs) over the slices in order 0 .. cs-1
  const int rows = kBM / cs;
  const int r0 = z * rows;
  const uint32_t red0 = smem_u32(red);
  for (int f = threadIdx.x; f < rows * (kBN / 4); f += blockDim.x) {
    const int rl = r0 + f / (kBN / 4);
    const int c = (f % (kBN / 4)) * 4;
    const uint32_t a = red0 + (uint32_t)((rl * kRedLd + c) * 4);
    // all slices' loads in flight first, then the sum in slice order
    float4 v[kMaxCluster];
#pragma unroll
    for (int p = 0; p < kMaxCluster; ++p)
      if (p < cs) v[p] = ld_cluster_f4(cluster_map(a, (uint32_t)p));
    float4 acc = v[0];
#pragma unroll
    for (int p = 1; p < kMaxCluster; ++p) {
      if (p < cs) {
        acc.x += v[p].x;
        acc.y += v[p].y;
        acc.z += v[p].z;
        acc.w += v[p].w;
      }
    }
    side_store(oo, m0 + rl, n0 + c, acc);
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while another still reads its shared memory
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBN);
  }
}

// The problems of P (np >= 1, each with tA, tB, o set and o.M, o.N its output size) in one launch
// over the common K; fills in their tile0 / mt.
template <int AMN, int BMN, int DUAL = 0>
cudaError_t launch_side(SideProbs& P, int K, cudaStream_t st, int b_off = 0) {
  constexpr uint32_t kSmem = SideCfg<DUAL>::kSmem;
  static std::atomic<unsigned long long> attr_done{0};  // devices whose function attribute is set
  if (!done_on_device(attr_done)) {
    const cudaError_t err = cudaFuncSetAttribute(k_side<AMN, BMN, DUAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (err != cudaSuccess) return err;
    mark_done_on_device(attr_done);
  }
  if (P.np < 1 || P.np > kMaxProbs || K <= 0) return cudaErrorInvalidValue;
  int64_t tiles = 0;
  for (int i = 0; i < P.np; ++i) {
    SideProb& q = P.p[i];
    if (q.o.M <= 0 || q.o.N <= 0) return cudaErrorInvalidValue;
    q.mt = (q.o.M + kBM - 1) / kBM;
    q.tile0 = (int)tiles;
    tiles += (int64_t)q.mt * ((q.o.N + kBN - 1) / kBN);
    if (tiles > 65535) return cudaErrorInvalidValue;
  }
  const int nk = (K + kBK - 1) / kBK;
  // widest cluster (K split) that keeps every CTA resident at two per SM
  const int64_t slots = 2 * (int64_t)device_sm_count();
  int cs = 1;
  while (cs < kMaxCluster && tiles * cs * 2 <= slots && cs * 2 <= nk) cs *= 2;
  const int kps = (nk + cs - 1) / cs;
  const cudaError_t e = launch_k(k_side<AMN, BMN, DUAL>, dim3((unsigned)cs, (unsigned)tiles, 1), dim3(192), kSmem, st,
                                 (unsigned)cs, P, nk, kps, b_off);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Part `sec` of the split value of v: 0 and 1 hi = bf16(v), 2 lo = bf16(v - hi).
__device__ __forceinline__ __nv_bfloat16 split_part(float v, int sec) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  return sec == 2 ? __float2bfloat16_rn(v - __bfloat162float(hi)) : hi;
}

__global__ void k_lora_prep(const LoraPrepArgs a) {
  pdl_wait();
  pdl_trigger();
  const int R = a.nseg * a.r;
  const int out = a.bounds[a.nseg];
  const int64_t n1 = (int64_t)a.KP * a.in;
  const int64_t n2 = (int64_t)out * a.KP;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n1; i += stride) {
    const int row = (int)(i / a.in), c = (int)(i % a.in);
    const int sec = row / a.RS, j = row % a.RS;  // section 3 and beyond: padding
    float v = 0.f;
    if (sec < 3 && j < R) v = a.A[j / a.r][(int64_t)(j % a.r) * a.in + c];
    a.Acat16[i] = split_part(v, sec);
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += stride) {
    const int o = (int)(i / a.KP), col = (int)(i % a.KP);
    const int sec = col / a.RS, j = col % a.RS;
    int p = 0;
    while (p + 1 < a.nseg && o >= a.bounds[p + 1]) ++p;
    float v = 0.f;
    if (sec < 3 && j < R && j / a.r == p) v = a.B[p][(int64_t)(o - a.bounds[p]) * a.r + (j % a.r)];
    a.Bexp16[i] = split_part(v, sec);
  }
}

}  // namespace

cudaError_t lora_skinny(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                        int64_t ldb, int b_mn, int KP, float s, __nv_bfloat16* Us, cudaStream_t st) {
  if (T <= 0 || T > INT32_MAX || K <= 0 || KP <= 0 || KP % 8 || !X || !Bop || !Us) return cudaErrorInvalidValue;
  if (!al16(X) || !al16(Bop) || (ldx % 8) || (ldb % 8)) return cudaErrorInvalidValue;
  SideProbs P{};
  P.np = 1;
  SideProb& q = P.p[0];
  if (!make_map(&q.tA, X, T, K, ldx, kBM)) return cudaErrorInvalidValue;
  if (b_mn) {
    if (!make_map(&q.tB, Bop, K, KP, ldb, kBK)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&q.tB, Bop, KP, K, ldb, kBN)) return cudaErrorInvalidValue;
  }
  SideOut& o = q.o;
  o.mode = 0;
  o.M = (int)T;
  o.N = KP;
  o.scale = s;
  o.out16 = Us;
  o.ld = KP;
  return b_mn ? launch_side<0, 1>(P, K, st) : launch_side<0, 0>(P, K, st);
}

cudaError_t lora_skinny_split(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                              int64_t ldb, int b_mn, int R, int RS, int KP, float s, __nv_bfloat16* Us,
                              cudaStream_t st) {
  if (T <= 0 || T > INT32_MAX || K <= 0 || R <= 0 || R > RS || RS % 8 || RS > kBN || 3 * RS > KP || KP % 8 || !X ||
      !Bop || !Us)
    return cudaErrorInvalidValue;
  if (!al16(X) || !al16(Bop) || (ldx % 8) || (ldb % 8)) return cudaErrorInvalidValue;
  SideProbs P{};
  P.np = 1;
  SideProb& q = P.p[0];
  if (!make_map(&q.tA, X, T, K, ldx, kBM)) return cudaErrorInvalidValue;
  if (b_mn) {
    if (!make_map(&q.tB, Bop, K, KP, ldb, kBK)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&q.tB, Bop, KP, K, ldb, kBN)) return cudaErrorInvalidValue;
  }
  SideOut& o = q.o;
  o.mode = 3;
  o.M = (int)T;
  o.N = R;
  o.scale = s;
  o.out16 = Us;
  o.ld = KP;
  o.R = R;
  o.RS = RS;
  // the lo part of the operand starts 2 RS further along N: a multiple of 16 elements, so the TMA
  // x coordinate of the MN-major case stays 16-byte aligned
  return b_mn ? launch_side<0, 1, 1>(P, K, st, 2 * RS) : launch_side<0, 0, 1>(P, K, st, 2 * RS);
}

cudaError_t lora_grads_multi(const LoraGradProb* g, int n, int64_t T, cudaStream_t st) {
  if (!g || n < 1 || 2 * n > kMaxProbs || T <= 0 || T > INT32_MAX) return cudaErrorInvalidValue;
  SideProbs P{};
  P.np = 2 * n;
  for (int i = 0; i < n; ++i) {
    const LoraGradProb& q = g[i];
    if (q.nseg < 1 || q.nseg > 3 || q.r <= 0 || q.nseg * q.r > q.KP || q.KP % 8 || q.in <= 0 || q.out <= 0)
      return cudaErrorInvalidValue;
    if (!al16(q.X) || !al16(q.Vs) || !al16(q.dY) || !al16(q.Us) || (q.ldx % 8) || (q.ldy % 8) || q.bounds[0] != 0 ||
        q.bounds[q.nseg] != q.out)
      return cudaErrorInvalidValue;
    // dA: C [nseg*r, in] = Vs^T X; dB: C [out, nseg*r] = dY^T Us (both contract the T tokens)
    SideProb& pa = P.p[2 * i];
    SideProb& pb = P.p[2 * i + 1];
    if (!make_map(&pa.tA, q.Vs, T, q.KP, q.KP, kBK) || !make_map(&pa.tB, q.X, T, q.in, q.ldx, kBK) ||
        !make_map(&pb.tA, q.dY, T, q.out, q.ldy, kBK) || !make_map(&pb.tB, q.Us, T, q.KP, q.KP, kBK))
      return cudaErrorInvalidValue;
    SideOut& oa = pa.o;
    SideOut& ob = pb.o;
    oa.mode = 1;
    oa.M = q.nseg * q.r;
    oa.N = q.in;
    oa.scale = 1.0f;
    ob.mode = 2;
    ob.M = q.out;
    ob.N = q.nseg * q.r;
    ob.scale = 1.0f;
    for (int k = 0; k < q.nseg; ++k) {
      oa.dst[k] = q.dA[k];
      ob.dst[k] = q.dB[k];
    }
    for (int k = 0; k <= q.nseg; ++k) ob.bounds[k] = q.bounds[k];
    oa.r = ob.r = q.r;
    oa.nseg = ob.nseg = q.nseg;
  }
  return launch_side<1, 1>(P, (int)T, st);
}

cudaError_t lora_grads(const __nv_bfloat16* X, int64_t ldx, int in, const __nv_bfloat16* dY, int64_t ldy, int out,
                       int64_t T, const __nv_bfloat16* Us, const __nv_bfloat16* Vs, int KP, int nseg, int r,
                       const int* bounds, float* const* dA, float* const* dB, cudaStream_t st) {
  if (nseg < 1 || nseg > 3 || !bounds || !dA || !dB) return cudaErrorInvalidValue;
  LoraGradProb q{};
  q.X = X;
  q.ldx = ldx;
  q.in = in;
  q.dY = dY;
  q.ldy = ldy;
  q.out = out;
  q.Us = Us;
  q.Vs = Vs;
  q.KP = KP;
  q.nseg = nseg;
  q.r = r;
  for (int k = 0; k <= nseg; ++k) q.bounds[k] = bounds[k];
  for (int k = 0; k < nseg; ++k) {
    q.dA[k] = dA[k];
    q.dB[k] = dB[k];
  }
  return lora_grads_multi(&q, 1, T, st);
}

cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st) {
  if (a.nseg < 1 || a.nseg > 3 || a.nseg * a.r > a.RS || a.RS % 8 || 3 * a.RS > a.KP) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_lora_prep, dim3(1024), dim3(256), 0, st, 0, a);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lst
