// Causal GQA attention (host interface). See attention.cu.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

struct AttnArgs {
  const __nv_bfloat16* q;  // [T, ldq], head h at column h*hd
  const __nv_bfloat16* k;  // [T, ldk], kv head j at column j*hd
  const __nv_bfloat16* v;  // [T, ldv]
  __nv_bfloat16* o;        // [T, ldo]
  float* lse;              // [T, hq] natural-log sum-exp of the scaled scores
  float* o32 = nullptr;    // optional [T, hq*hd] fp32 copy of o before rounding (for the backward)
  int64_t ldq, ldk, ldv, ldo;
  int64_t T;               // batch * S tokens
  int S, hq, hkv, hd;      // hd in {64, 128}
  float scale;             // 1/sqrt(hd)
};

struct AttnBwdArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;  // dL/do, [T, lddo]
  const float* lse;           // from the forward
  float* D;                   // scratch [T, hq]: rowsum(dout * o)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int64_t ldq, ldk, ldv, ldo, lddo, lddq, lddk, lddv;
  int64_t T;
  int S, hq, hkv, hd;
  float scale;
  const float* o32 = nullptr;  // optional fp32 forward output [T, hq*hd]; D uses it when given
  // optional: undo the rotary embedding on dq and dk before they are stored (tables [S, hd/2])
  const float* rope_cos = nullptr;
  const float* rope_sin = nullptr;
};

cudaError_t attention_fwd(const AttnArgs& a, cudaStream_t s);
cudaError_t attention_bwd(const AttnBwdArgs& a, cudaStream_t s);

}  // namespace lst
