// NF4 quantisation / dequantisation (host interface). See nf4.cu for the format.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lst {

struct Nf4Table {
  float cb[16];    // codebook, ascending, cb[7] == 0
  float mid[16];   // mid[j] = (cb[j] + cb[j+1]) / 2 for j < 15; mid[15] is a sentinel
};

// The 16 NF4 values: 8 positive and 7 negative standard-normal quantiles at levels
// delta - j (delta - 1/2) / 8 and / 7 with delta = ((1 - 1/30) + (1 - 1/32)) / 2, plus 0,
// sorted and divided by the quantile at delta; computed in fp64, rounded once to fp32.
void nf4_codebook(float out[16]);
Nf4Table nf4_table();

// Device pointers of one quantised tensor of n elements.
struct Nf4Out {
  uint8_t* packed;   // [n / 2]
  int8_t* qabs;      // [n / 64]
  float* gscale;     // [ceil(n / 64 / 256)]
  float* mean;       // [1]
};

// Quantise fp32 device tensor w (n a multiple of 64). Scratch: n/64 floats, ceil(n/64/256) doubles.
cudaError_t nf4_quantize(const float* w, int64_t n, const Nf4Out& o, float* scratch_absmax,
                         double* scratch_gsum, cudaStream_t s);

struct Nf4Seg {
  const uint8_t* packed;
  const int8_t* qabs;
  const float* gscale;
  const float* mean;
  int64_t n;           // elements (multiple of 64)
  int64_t out_offset;  // element offset of this tensor in the output (multiple of 8)
};
constexpr int kMaxNf4Segs = 8;

// Dequantise up to 8 tensors into one bf16 buffer (each at its out_offset).
cudaError_t nf4_dequant(const Nf4Seg* segs, int nseg, __nv_bfloat16* out, cudaStream_t s);

}  // namespace lst
