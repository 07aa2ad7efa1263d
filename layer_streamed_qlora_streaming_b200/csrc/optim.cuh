// AdamW update of the LoRA adapters (host interface). See optim.cu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

// One adapter tensor [rows, cols] at `off` in the parameter / gradient / moment buffers, and the
// split bf16 operand it is mirrored into: element (row, col) = p goes to
// e = dst + (dst_row0 + row) * dst_ld + dst_col0 + col as e[0] = e[sec] = bf16(p) and
// e[2 sec] = bf16(p - bf16(p)), sec being the section stride (elements) of the operand.
struct AdamTensor {
  int64_t off, n;
  int rows, cols;
  __nv_bfloat16* dst;
  int64_t dst_ld;
  int dst_row0, dst_col0;
  int64_t sec;
};

struct AdamHyper {
  float lr, b1, b2, eps, wd;
  float step_size;  // lr / (1 - b1^t)
  float sqrt_bc2;   // sqrt(1 - b2^t)
};

cudaError_t adamw_update(const AdamTensor* tab_dev, int ntensors, int64_t max_numel, float* params,
                         const float* grads, float* m, float* v, const AdamHyper& h, cudaStream_t s);

}  // namespace lst
