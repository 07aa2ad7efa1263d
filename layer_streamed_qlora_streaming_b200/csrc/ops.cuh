// Memory-bound kernels of the decoder layer and the LoRA side path (host interface). See ops.cu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

using bf16 = __nv_bfloat16;

// y = bf16(x * rstd * g), rstd = 1/sqrt(mean(x^2) + eps) per row (x fp32: the residual stream);
// rstd saved [T].
cudaError_t rmsnorm_fwd(const float* x, const float* g, int64_t T, int d, float eps, bf16* y, float* rstd,
                        cudaStream_t s);
// dx = dres + rstd * (dy*g - xhat * mean(dy*g*xhat)); writes fp32 dx and (optional) bf16 copy.
cudaError_t rmsnorm_bwd(const float* dy, const float* x, const float* g, const float* rstd, const float* dres,
                        int64_t T, int d, float* dx, bf16* dx_bf16, cudaStream_t s);

// Rotate pairs (j, j + hd/2) of the first nh heads of each row of buf (row stride ld) by the
// angle of position (t mod S): cos/sin tables [S_max, hd/2]. inverse = 1 rotates backwards.
cudaError_t rope(bf16* buf, int64_t ld, int64_t T, int S, int col0, int nh, int hd, const float* cos_t,
                 const float* sin_t, int inverse, cudaStream_t s);
// cos/sin of pos * theta^(-2j/hd) computed in fp64, stored fp32 [S, hd/2].
cudaError_t rope_tables(int S, int hd, double theta, float* cos_t, float* sin_t, cudaStream_t s);

// m = bf16(silu(g) * u) where gu = [g | u] along columns ([T, 2F]).
cudaError_t swiglu_fwd(const bf16* gu, int64_t T, int F, bf16* m, cudaStream_t s);
// dgu = [dm * u * silu'(g) | dm * silu(g)] (bf16), dm fp32 [T, F].
cudaError_t swiglu_bwd(const float* dm, const bf16* gu, int64_t T, int F, bf16* dgu, cudaStream_t s);

// x[t] = E[tok[t]] as fp32 (the residual stream); out-of-range ids set the device error word.
cudaError_t embed(const int32_t* tok, const bf16* E, int64_t T, int d, int vocab, float* x, cudaStream_t s);

// Cross-entropy rows: loss_t = lse_t - logit[t, y_t]; dlogits = (softmax - onehot) * inv_T (bf16).
cudaError_t cross_entropy(const float* logits, int64_t T, int V, const int32_t* targets, float inv_T,
                          float* loss_rows, bf16* dlogits, cudaStream_t s);
// out = mean of v[0..n) with a fixed summation order.
cudaError_t mean_fixed(const float* v, int64_t n, float* out, cudaStream_t s);

// Preference (DPO) head pieces. Row statistics of fp32 logits [T, V]: lse[t] and
// logp[t] = logits[t][y_t] - lse[t].
cudaError_t ce_stats(const float* logits, int64_t T, int V, const int32_t* targets, float* lse, float* logp,
                     cudaStream_t s);
// out[q] = sum over the S rows of sequence q of mask * v (mask NULL = all ones), fixed order.
cudaError_t seq_sum(const float* v, const int32_t* mask, int nseq, int S, float* out, cudaStream_t s);
// DPO over P pairs (sequences [0, P) chosen, [P, 2P) rejected): loss = mean_p -log sigmoid(z_p),
// z_p = beta ((pi_p - ref_p) - (pi_{P+p} - ref_{P+p})); w[q] = -dloss/dpi_q.
cudaError_t dpo_loss(const float* pi, const float* ref, int P, float beta, float* loss, float* w, cudaStream_t s);
// dlogits of rows [row0, row0 + rows) (logits / dlog point at row row0):
// dlog = bf16(w[row / S] * mask[row] * (softmax(logits_row) - onehot(y_row))).
cudaError_t ce_grad(const float* logits, int64_t rows, int64_t row0, int V, const int32_t* targets, const float* lse,
                    const float* w, const int32_t* mask, int S, __nv_bfloat16* dlog, cudaStream_t s);
// out = sum_i a[i] * b[i] with a fixed order; partials: scratch of 1024 floats.
cudaError_t dot_fixed(const float* a, const bf16* b, int64_t n, float* partials, float* out, cudaStream_t s);

cudaError_t f32_to_bf16(const float* x, int64_t n, bf16* y, cudaStream_t s);
// bytes (a multiple of 16, both pointers 16-byte aligned) from src to dst on stream s
cudaError_t copy16(const void* src, void* dst, int64_t bytes, cudaStream_t s);
cudaError_t bf16_to_f32(const bf16* x, int64_t n, float* y, cudaStream_t s);

}  // namespace lst
