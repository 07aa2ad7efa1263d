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

// fp32 partials of up to kMaxSplits splits, then one int semaphore per 128-row tile
int64_t lora_skinny_scratch(int64_t T, int KP) { return (int64_t)kMaxSplits * T * KP + (T + 127) / 128 + 4; }

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
  a.kout = Us;  // reduced in the kernel by the last split of each tile, in split order
  a.ldk = KP;
  a.kscale = s;
  a.sem = reinterpret_cast<int*>(part + (int64_t)kMaxSplits * T * KP);
  return gemm_bf16(a, st);
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
  a.C = dst[0];  // not written: the epilogue scatters straight into the per-segment dA
  a.ldc = KP;
  a.c_f32 = 1;
  a.epi_mode = 1;
  for (int k = 0; k < nseg; ++k) a.sdst[k] = dst[k];
  a.sr = r;
  a.snseg = nseg;
  (void)part;
  return gemm_bf16(a, st);
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
  a.C = dst[0];  // not written: the epilogue keeps each row's own segment and stores it as dB
  a.ldc = KP;
  a.c_f32 = 1;
  a.epi_mode = 2;
  for (int k = 0; k < nseg; ++k) a.sdst[k] = dst[k];
  for (int k = 0; k <= nseg; ++k) a.sbounds[k] = bounds[k];
  a.sr = r;
  a.snseg = nseg;
  (void)part;
  return gemm_bf16(a, st);
}

cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st) {
  if (a.nseg < 1 || a.nseg > 3 || a.nseg * a.r > a.KP) return cudaErrorInvalidValue;
  k_lora_prep<<<1024, 256, 0, st>>>(a);
  note_launch(1);
  return cudaGetLastError();
}

}  // namespace lst
