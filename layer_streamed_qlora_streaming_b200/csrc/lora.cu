// LoRA side path on the tensor cores ("Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU",
// section "LoRA and QLoRA": trainable low-rank matrices next to the frozen base).
//
// For a projection y = x W^T + s (x A^T) B^T the side path needs, per fused group of projections
// sharing an input (q/k/v, o, gate/up, down):
//   forward   U  = x Acat^T          [T, nseg*r]   (then s*U enters the base GEMM as extra K columns)
//   backward  V  = dy Bexp            [T, nseg*r]  (s*V enters the dX GEMM the same way)
//             dA = s V^T x,  dB = s dy^T U          (reductions over the T tokens)
// All four are bf16 tcgen05 GEMMs with fp32 accumulation. U and V have only nseg*r <= 64 columns,
// so they are split along K over many CTAs and the fp32 partials are summed in a fixed order; dA and
// dB contract over tokens, with x / dy read as MN-major operands. Nothing uses atomics, so results
// are deterministic.
#include "common.cuh"
#include "gemm.cuh"
#include "lora.cuh"

namespace lst {
namespace {

constexpr int kMaxSplits = 16;

int skinny_splits(int64_t T, int K) {
  const int mtiles = (int)((T + 127) / 128);
  int splits = (148 + mtiles - 1) / mtiles;
  if (splits > kMaxSplits) splits = kMaxSplits;
  const int nk = (K + 63) / 64;
  if (splits > nk) splits = nk;
  if (splits < 1) splits = 1;
  const int kps = (nk + splits - 1) / splits;
  return (nk + kps - 1) / kps;  // the same count the GEMM launch settles on (no empty split)
}

__global__ void k_splitk_reduce(const float* __restrict__ part, int splits, int64_t stride, int64_t n, float s,
                                __nv_bfloat16* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = 0.f;
  for (int z = 0; z < splits; ++z) acc += part[z * stride + i];
  out[i] = __float2bfloat16_rn(s * acc);
}

__global__ void k_scatter_a(const float* __restrict__ C, int in, int KP, int R, int r, float* d0, float* d1,
                            float* d2) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)in * R) return;
  const int i = (int)(idx / R), jj = (int)(idx % R);
  const int p = jj / r, j = jj % r;
  float* d = p == 0 ? d0 : (p == 1 ? d1 : d2);
  d[(int64_t)j * in + i] = C[(int64_t)i * KP + jj];
}

__global__ void k_scatter_b(const float* __restrict__ C, int out, int KP, int nseg, int r, int b1, int b2,
                            float* d0, float* d1, float* d2) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)out * r) return;
  const int o = (int)(idx / r), j = (int)(idx % r);
  int p = 0, lo = 0;
  float* d = d0;
  if (nseg > 1 && o >= b1) {
    p = 1;
    lo = b1;
    d = d1;
  }
  if (nseg > 2 && o >= b2) {
    p = 2;
    lo = b2;
    d = d2;
  }
  d[(int64_t)(o - lo) * r + j] = C[(int64_t)o * KP + p * r + j];
}

__global__ void k_lora_prep(const LoraPrepArgs a) {
  const int R = a.nseg * a.r;
  const int out = a.bounds[a.nseg];
  const int64_t n1 = (int64_t)a.KP * a.in;
  const int64_t n2 = (int64_t)out * a.KP;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n1; i += stride) {
    const int j = (int)(i / a.in), c = (int)(i % a.in);
    const float v = j < R ? a.A[j / a.r][(int64_t)(j % a.r) * a.in + c] : 0.f;
    a.Acat16[i] = __float2bfloat16_rn(v);
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += stride) {
    const int o = (int)(i / a.KP), j = (int)(i % a.KP);
    int p = 0;
    while (p + 1 < a.nseg && o >= a.bounds[p + 1]) ++p;
    float v = 0.f;
    if (j < R && j / a.r == p) v = a.B[p][(int64_t)(o - a.bounds[p]) * a.r + (j % a.r)];
    a.Bexp16[i] = __float2bfloat16_rn(v);
  }
}

inline unsigned nblk(int64_t n) { return (unsigned)((n + 255) / 256); }

}  // namespace

int64_t lora_skinny_scratch(int64_t T, int KP) { return (int64_t)kMaxSplits * T * KP; }

cudaError_t lora_skinny(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                        int64_t ldb, int b_mn, int KP, float s, float* part, __nv_bfloat16* Us, cudaStream_t st) {
  if (T <= 0 || K <= 0 || KP <= 0 || KP > 256) return cudaErrorInvalidValue;
  const int splits = skinny_splits(T, K);
  GemmArgs a;
  a.M = (int)T;
  a.N = KP;
  a.K = K;
  a.A = X;
  a.lda = ldx;
  a.B = Bop;
  a.ldb = ldb;
  a.b_mn = b_mn;
  a.C = part;
  a.ldc = KP;
  a.c_f32 = 1;
  a.splits = splits;
  a.split_stride = T * KP;
  cudaError_t e = gemm_bf16(a, st);
  if (e != cudaSuccess) return e;
  k_splitk_reduce<<<nblk(T * KP), 256, 0, st>>>(part, splits, T * KP, T * KP, s, Us);
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t lora_grad_a(const __nv_bfloat16* X, int64_t ldx, int64_t T, int in, const __nv_bfloat16* Vs, int KP,
                        int nseg, int r, float* const* dst, float* part, cudaStream_t st) {
  if (nseg < 1 || nseg > 3 || nseg * r > KP) return cudaErrorInvalidValue;
  GemmArgs a;
  a.M = in;
  a.N = KP;
  a.K = (int)T;
  a.A = X;
  a.lda = ldx;
  a.a_mn = 1;
  a.B = Vs;
  a.ldb = KP;
  a.b_mn = 1;
  a.C = part;
  a.ldc = KP;
  a.c_f32 = 1;
  cudaError_t e = gemm_bf16(a, st);
  if (e != cudaSuccess) return e;
  const int R = nseg * r;
  k_scatter_a<<<nblk((int64_t)in * R), 256, 0, st>>>(part, in, KP, R, r, dst[0], nseg > 1 ? dst[1] : nullptr,
                                                     nseg > 2 ? dst[2] : nullptr);
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t lora_grad_b(const __nv_bfloat16* dY, int64_t ldy, int64_t T, int out, const __nv_bfloat16* Us, int KP,
                        int nseg, int r, const int* bounds, float* const* dst, float* part, cudaStream_t st) {
  if (nseg < 1 || nseg > 3 || nseg * r > KP) return cudaErrorInvalidValue;
  GemmArgs a;
  a.M = out;
  a.N = KP;
  a.K = (int)T;
  a.A = dY;
  a.lda = ldy;
  a.a_mn = 1;
  a.B = Us;
  a.ldb = KP;
  a.b_mn = 1;
  a.C = part;
  a.ldc = KP;
  a.c_f32 = 1;
  cudaError_t e = gemm_bf16(a, st);
  if (e != cudaSuccess) return e;
  k_scatter_b<<<nblk((int64_t)out * r), 256, 0, st>>>(part, out, KP, nseg, r, nseg > 1 ? bounds[1] : out,
                                                      nseg > 2 ? bounds[2] : out, dst[0],
                                                      nseg > 1 ? dst[1] : nullptr, nseg > 2 ? dst[2] : nullptr);
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st) {
  if (a.nseg < 1 || a.nseg > 3 || a.nseg * a.r > a.KP) return cudaErrorInvalidValue;
  k_lora_prep<<<1024, 256, 0, st>>>(a);
  note_launch(1);
  return cudaGetLastError();
}

}  // namespace lst
