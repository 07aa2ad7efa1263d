// AdamW update of the resident LoRA adapters, fused with the refresh of their bf16 GEMM operands.
//
// The adapters are the only trained parameters and they stay on the GPU with their optimizer
// state ("Fine-tune Llama 3.1 8B on a 4GB GPU with Soup", first paragraph and "Step 5": LoRA
// r 16, alpha 32, lr 2e-4; "Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU", section
// "Why GPU Memory Has Always Been the Bottleneck": Adam keeps two extra tensors per parameter).
// The update is the decoupled-weight-decay Adam of Loshchilov & Hutter:
//   m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
//   p <- p (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// in fp32, element by element (deterministic). The same pass writes the split bf16 pair
// (bf16(p), bf16(p - bf16(p))) to the places the element occupies in the group operands
// (Acat [KP, in] or Bexp [out, KP]) the GEMMs read.
#include "common.cuh"
#include "pdl.cuh"
#include "optim.cuh"

namespace lst {
namespace {

__global__ void k_adamw(const AdamTensor* __restrict__ tab, float* __restrict__ p, const float* __restrict__ g,
                        float* __restrict__ m, float* __restrict__ v, const AdamHyper h) {
  pdl_wait();
  pdl_trigger();
  const AdamTensor t = tab[blockIdx.y];
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < t.n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = t.off + e;
    const float gi = g[i];
    const float mi = h.b1 * m[i] + (1.0f - h.b1) * gi;
    const float vi = h.b2 * v[i] + (1.0f - h.b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    const float denom = sqrtf(vi) / h.sqrt_bc2 + h.eps;
    const float pi = p[i] * (1.0f - h.lr * h.wd) - h.step_size * (mi / denom);
    p[i] = pi;
    const int row = (int)(e / t.cols), col = (int)(e % t.cols);
    __nv_bfloat16* e0 = t.dst + (int64_t)(t.dst_row0 + row) * t.dst_ld + t.dst_col0 + col;
    const __nv_bfloat16 hi = __float2bfloat16_rn(pi);
    e0[0] = hi;
    e0[t.sec] = hi;
    e0[2 * t.sec] = __float2bfloat16_rn(pi - __bfloat162float(hi));
  }
}

}  // namespace

cudaError_t adamw_update(const AdamTensor* tab_dev, int ntensors, int64_t max_numel, float* params,
                         const float* grads, float* m, float* v, const AdamHyper& h, cudaStream_t s) {
  if (ntensors <= 0 || max_numel <= 0) return cudaErrorInvalidValue;
  int64_t bx = (max_numel + 255) / 256;
  if (bx > 64) bx = 64;  // grid-stride inside each tensor
  dim3 grid((unsigned)bx, (unsigned)ntensors);
  const cudaError_t e = launch_k(k_adamw, grid, dim3(256), 0, s, 0, tab_dev, params, grads, m, v, h);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lst
