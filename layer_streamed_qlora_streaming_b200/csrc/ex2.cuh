// 2^x by the SFU's approximate base-2 exponential (PTX ex2.approx.ftz.f32: one instruction, about
// 2 ulp of relative error, results below 2^-126 flushed to zero, 2^-inf = 0). The softmax kernels
// take every exponential this way: their results are rounded to fp16 / bf16 or summed in fp32,
// where that error is far below the rounding.
#pragma once

namespace lst {
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
}  // namespace lst
