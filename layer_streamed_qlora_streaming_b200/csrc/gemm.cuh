// bf16 tensor-core GEMM for sm_100a (tcgen05 + TMEM + TMA), host interface.
//
//   C[m, n] = alpha * ( sum_k A[m, k] B(n, k)  +  sum_j A2[m, j] B2(n, j) ) + bias[n] + R[m, n]
//
// A, A2 are row-major [M, K] / [M, K2] (K-major), or A is row-major [K, M] (a_mn = 1, "X^T ...").
// B is either row-major [N, K] (K-major, b_mn = 0, "x W^T") or row-major [K, N] (MN-major,
// b_mn = 1, "x W"); B2 has the same major-ness. With splits > 1 the K range is cut into slices
// whose partial products are written side by side (fixed-order reduction left to the caller).
// The optional (A2, B2) pair is a second contraction appended along K; the LoRA path uses it
// to fold s (x A^T) B^T into the same accumulator as the frozen base.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

struct GemmArgs {
  int M = 0, N = 0, K = 0;
  const __nv_bfloat16* A = nullptr;   // [M, K], row stride lda
  int64_t lda = 0;
  const __nv_bfloat16* B = nullptr;   // b_mn=0: [N, K]; b_mn=1: [K, N]; row stride ldb
  int64_t ldb = 0;
  int b_mn = 0;
  const __nv_bfloat16* A2 = nullptr;  // optional [M, K2]
  int64_t lda2 = 0;
  const __nv_bfloat16* B2 = nullptr;  // optional b_mn=0: [N, K2]; b_mn=1: [K2, N]
  int64_t ldb2 = 0;
  int K2 = 0;
  void* C = nullptr;                  // [M, N] row stride ldc; fp32 if c_f32 else bf16
  int64_t ldc = 0;
  int c_f32 = 0;
  float alpha = 1.0f;
  const float* bias = nullptr;        // [N] or null
  const float* R = nullptr;           // fp32 residual [M, N] row stride ldr, or null
  int64_t ldr = 0;
  int a_mn = 0;                       // 1: A is row-major [K, M] (MN-major); needs b_mn = 1
  int splits = 1;                     // split-K: partial results at C + z * split_stride
  int64_t split_stride = 0;
  // Rotary embedding fused into the epilogue (q and k of a fused q/k/v projection): output
  // columns [0, rope_end) form heads of rope_hd columns whose pairs (j, j + rope_hd/2) are rotated
  // by the angle of position (row mod rope_S), tables rope_cos / rope_sin [rope_S, rope_hd/2].
  const float* rope_cos = nullptr;
  const float* rope_sin = nullptr;
  int rope_end = 0, rope_hd = 0, rope_S = 0;
  // Store mode for the LoRA gradients (result [M, snseg * sr], fp32, scaled by alpha):
  //   1: column p*sr + j of row i -> sdst[p][j * M + i]                        (dA, [r, in])
  //   2: row o of segment p (sbounds), column p*sr + j -> sdst[p][(o - sbounds[p]) * sr + j] (dB)
  int epi_mode = 0;
  float* sdst[3] = {nullptr, nullptr, nullptr};
  int sr = 0, snseg = 0;
  int sbounds[4] = {0, 0, 0, 0};
  // Split-K with the reduction in the kernel: C receives the fp32 partials; the last CTA of each
  // output tile sums them in split order and writes bf16(kscale * sum) to kout [M, N] (row stride
  // ldk). sem: one int per output tile, zero before the call and left zero after it.
  __nv_bfloat16* kout = nullptr;
  int64_t ldk = 0;
  float kscale = 1.0f;
  int* sem = nullptr;
};

// Returns cudaSuccess or the launch / argument error. Deterministic: no split-K, no atomics.
cudaError_t gemm_bf16(const GemmArgs& a, cudaStream_t s);

}  // namespace lst
