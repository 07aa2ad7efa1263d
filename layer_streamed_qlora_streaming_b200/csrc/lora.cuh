// LoRA side path on the tensor cores (host interface). See lora.cu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

// Skinny projection Us = bf16(s * X Bop) with X bf16 [T, K] (row stride ldx) and Bop the bf16
// operand of N = KP columns: K-major [KP, K] (b_mn = 0, i.e. X Bop^T) or MN-major [K, KP]
// (b_mn = 1). Split-K over the tcgen05 GEMM; the last split of each tile sums the partials in
// split order (deterministic) and writes Us. part: scratch of lora_skinny_scratch(T, KP) floats
// whose tail holds tile semaphores: zero before the first call, left zero by every call.
// Us: [T, KP] contiguous.
int64_t lora_skinny_scratch(int64_t T, int KP);
cudaError_t lora_skinny(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                        int64_t ldb, int b_mn, int KP, float s, float* part, __nv_bfloat16* Us, cudaStream_t st);

// dA of every segment of a fused group: C = X^T Vs (X bf16 [T, in], Vs = bf16(s V) [T, KP]) on the
// tensor cores, stored straight as dA_p[j][i] = C[i][p*r + j] (dst[p] fp32 [r, in]). part: unused.
cudaError_t lora_grad_a(const __nv_bfloat16* X, int64_t ldx, int64_t T, int in, const __nv_bfloat16* Vs, int KP,
                        int nseg, int r, float* const* dst, float* part, cudaStream_t st);

// dB of every segment: C = dY^T Us (dY bf16 [T, out], Us = bf16(s U) [T, KP]), then
// dB_p[o - bounds[p]][j] = C[o][p*r + j] for o in segment p (dst[p] fp32 [out_p, r]), stored by
// the GEMM epilogue. part: unused.
cudaError_t lora_grad_b(const __nv_bfloat16* dY, int64_t ldy, int64_t T, int out, const __nv_bfloat16* Us, int KP,
                        int nseg, int r, const int* bounds, float* const* dst, float* part, cudaStream_t st);

// Derived bf16 operands of one fused projection group from its fp32 adapters (nseg segments,
// A_p [r, in], B_p [out_p, r]):
//   Acat16 [KP, in]: rows p*r + j = A_p[j] (rows >= nseg*r zero);
//   Bexp16 [out, KP]: row o of segment p holds B_p[o - bounds[p]] in columns p*r .. p*r + r - 1,
//   zero elsewhere.
struct LoraPrepArgs {
  const float* A[3];
  const float* B[3];
  int nseg, r, in;
  int bounds[4];  // out-row bounds of the segments
  int KP;
  __nv_bfloat16* Acat16;
  __nv_bfloat16* Bexp16;
};
cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st);

}  // namespace lst
