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

// The same projection at fp32-level precision from a split operand, for adapters kept in full
// precision: Bop holds the adapter as two bf16 parts, hi = bf16(a) in sections [0, RS) and
// lo = bf16(a - hi) in [2 RS, 3 RS) of its KP-wide dimension (rows when K-major, columns when
// MN-major), and U = s X (hi + lo) is accumulated in fp32 in one pass over X. U (columns j < R) is
// stored split as well: Us[t][j] = Us[t][2 RS + j] = bf16(U), Us[t][RS + j] = bf16(U - bf16(U)),
// so that the pair (Us, operand) sections [hi | lo | hi] x [hi | hi | lo] form the three products
// whose sum is U W'^T up to the lo x lo term. RS is a multiple of 8, R <= RS, 3 RS <= KP.
cudaError_t lora_skinny_split(const __nv_bfloat16* X, int64_t ldx, int64_t T, int K, const __nv_bfloat16* Bop,
                              int64_t ldb, int b_mn, int R, int RS, int KP, float s, __nv_bfloat16* Us,
                              cudaStream_t st);

// The adapter gradients of one fused group, in one launch (the clusters of dB follow those of dA),
// both reductions over the T tokens:
//   dA_p[j][i] = sum_t Vs[t][p*r + j] X[t][i]        with X bf16 [T, in] and Vs [T, KP]; dA[p] fp32 [r, in],
//                computed as the rows of Vs^T X that belong to the adapters;
//   dB_p[o][j] = sum_t dY[t][bounds[p] + o] Us[t][p*r + j]   with dY bf16 [T, out] and Us [T, KP];
//                dB[p] fp32 [out_p, r], the adapter columns of dY^T Us.
// Only columns < nseg * r of Us / Vs are read (the hi section of the split operands).
cudaError_t lora_grads(const __nv_bfloat16* X, int64_t ldx, int in, const __nv_bfloat16* dY, int64_t ldy, int out,
                       int64_t T, const __nv_bfloat16* Us, const __nv_bfloat16* Vs, int KP, int nseg, int r,
                       const int* bounds, float* const* dA, float* const* dB, cudaStream_t st);

// The adapter gradients of n <= 4 fused groups (the same T), in one launch: group i's dA and dB
// reductions as above, with its own operands. How far the T contraction is split over a cluster
// follows the launch's total number of output tiles, so the fp32 sums of one group can round
// differently alone and in company; a given set of groups always gives the same bytes.
struct LoraGradProb {
  const __nv_bfloat16* X;
  int64_t ldx;
  int in;
  const __nv_bfloat16* dY;
  int64_t ldy;
  int out;
  const __nv_bfloat16* Us;
  const __nv_bfloat16* Vs;
  int KP, nseg, r;
  int bounds[4];
  float* dA[3];
  float* dB[3];
};
cudaError_t lora_grads_multi(const LoraGradProb* g, int n, int64_t T, cudaStream_t st);

// Derived bf16 operands of one fused projection group from its fp32 adapters (nseg segments,
// A_p [r, in], B_p [out_p, r]), each adapter value a stored as the pair hi = bf16(a),
// lo = bf16(a - hi) in three sections of RS rows (Acat) or columns (Bexp):
//   Acat16 [KP, in]: row p*r + j holds hi(A_p[j]), row RS + p*r + j hi(A_p[j]) again and row
//   2 RS + p*r + j lo(A_p[j]);
//   Bexp16 [out, KP]: row o of segment p holds hi(B_p[o - bounds[p]]) in columns p*r .. p*r + r - 1
//   and RS + p*r .., and lo(...) in columns 2 RS + p*r ..;
// every other element zero. With the split Us / Vs of the projections this keeps the side path at
// fp32-level precision on the bf16 tensor cores.
struct LoraPrepArgs {
  const float* A[3];
  const float* B[3];
  int nseg, r, in;
  int bounds[4];  // out-row bounds of the segments
  int RS, KP;
  __nv_bfloat16* Acat16;
  __nv_bfloat16* Bexp16;
};
cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st);

}  // namespace lst
