// bf16 tensor-core GEMM for sm_100a (tcgen05 + TMEM + TMA), host interface.
//
//   C[m, n] = alpha * ( sum_k A[m, k] B(n, k)  +  sum_j A2[m, j] B2(n, j) ) + bias[n] + R[m, n]
//
// A, A2 are row-major [M, K] / [M, K2] (K-major), or A is row-major [K, M] (a_mn = 1, "X^T ...").
// B is either row-major [N, K] (K-major, b_mn = 0, "x W^T") or row-major [K, N] (MN-major,
// b_mn = 1, "x W"); B2 has the same major-ness. The optional (A2, B2) pair is a second
// contraction appended along K; the LoRA path uses it to fold s (x A^T) B^T into the same
// accumulator as the frozen base.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

// A bf16 weight matrix W [rows, cols] (row-major, cols a multiple of 64) held as up to three NF4
// tensors stacked along its rows (q/k/v or gate/up of a layer), each in the format of nf4.cu:
// tensor g covers rows [row_end[g-1], row_end[g]) (row_end[-1] = 0) and its element (r, c) is
// element (r - row_end[g-1]) * cols + c of the tensor, so that with cols % 64 == 0 every 64-wide
// column block of a row is exactly one NF4 block.
struct Nf4Mat {
  int nseg = 0;
  int cols = 0;
  int row_end[3] = {0, 0, 0};
  const uint8_t* packed[3] = {};
  const int8_t* qabs[3] = {};
  const float* gscale[3] = {};
  const float* mean[3] = {};
  float cb[16] = {};  // the codebook
};

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
  // Rotary embedding fused into the epilogue (q and k of a fused q/k/v projection): output
  // columns [0, rope_end) form heads of rope_hd columns whose pairs (j, j + rope_hd/2) are rotated
  // by the angle of position (row mod rope_S), tables rope_cos / rope_sin [rope_S, rope_hd/2].
  const float* rope_cos = nullptr;
  const float* rope_sin = nullptr;
  int rope_end = 0, rope_hd = 0, rope_S = 0;
  // Optional: B dequantised from NF4 inside the GEMM (B and ldb are then not used). b_mn = 0:
  // B(n, k) = W[n][k] (W [N, K], "x W^T"); b_mn = 1: B(k, n) = W[k][n] (W [K, N], "x W"). The
  // values equal those of nf4_dequant bit for bit, so the result equals the GEMM on the
  // dequantised matrix byte for byte. Needs a_mn = 0 and W's row length (K or N) % 64 == 0.
  const Nf4Mat* Bq = nullptr;
};

// Returns cudaSuccess or the launch / argument error. Deterministic: no split-K, no atomics.
cudaError_t gemm_bf16(const GemmArgs& a, cudaStream_t s);

// 2D bf16 TMA descriptor over a row-major [rows, cols] matrix with row stride ld (elements):
// box = [box_rows rows, 64 columns], 128-byte swizzle, zero fill out of bounds. False if the
// driver entry point is missing or the encoder rejects the arguments.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows);

}  // namespace lst
