// LoRA side path on the tensor cores (host interface). See lora.cu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

// Skinny projection Us = bf16(s * X Bop) with X bf16 [T, K] (row stride ldx) and Bop the bf16
// operand of N = KP columns: K-major [KP, K] (b_mn = 0, i.e. X Bop^T) or MN-major [K, KP]
// (b_mn = 1). Us: [T, KP] contiguous. The K range is split over the CTAs of a thread-block
// cluster whose fp32 partial tiles are summed in slice order through distributed shared memory
// (deterministic, no global scratch).
cudaError_t lora_skinny(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                        int64_t ldb, int b_mn, int KP, float s, __nv_bfloat16* Us, cudaStream_t st);

// dA of every segment of a fused group: dA_p[j][i] = sum_t Vs[t][p*r + j] X[t][i] with X bf16
// [T, in] and Vs = bf16(s V) [T, KP]; dst[p] fp32 [r, in]. Computed as the [KP, in] product
// Vs^T X, each row stored straight into its segment.
cudaError_t lora_grad_a(const __nv_bfloat16* X, int64_t ldx, int64_t T, int in, const __nv_bfloat16* Vs, int KP,
                        int nseg, int r, float* const* dst, cudaStream_t st);

// dB of every segment: C = dY^T Us (dY bf16 [T, out], Us = bf16(s U) [T, KP]), then
// dB_p[o - bounds[p]][j] = C[o][p*r + j] for o in segment p (dst[p] fp32 [out_p, r]).
cudaError_t lora_grad_b(const __nv_bfloat16* dY, int64_t ldy, int64_t T, int out, const __nv_bfloat16* Us, int KP,
                        int nseg, int r, const int* bounds, float* const* dst, cudaStream_t st);

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
