// NF4 4-bit quantisation with double-quantised absmax, and its bit-exact dequantisation.
//
// Format ("Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU", section "Quantization:
// Shrink the Weights": NF4 with nested quantisation of the constants; construction after QLoRA,
// Dettmers et al. 2023, section 3):
//   * blocks of 64 consecutive elements of the row-major flattened tensor, absmax per block;
//   * code = number of codebook midpoints strictly below w / absmax (fp32 division);
//   * two codes per byte, element 2i in the high nibble;
//   * absmax - mean(absmax) quantised symmetric int8 (x127, round half to even) in groups of 256
//     blocks, one fp32 scale per group; mean = fp64 sums (in each group in order, then over the
//     groups in order) / count, rounded to fp32;
//   * dequant: a^ = (q * s) / 127 + mean and w^ = bf16_rne(code_value * a^), every operation a
//     single fp32 rounding (explicit _rn intrinsics, so no multiply-add contraction).
#include "common.cuh"
#include "pdl.cuh"
#include "nf4.cuh"

#include <algorithm>
#include <cmath>

namespace lst {

// ---------------------------------------------------------------------------------- codebook
namespace {
double normal_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }
double normal_pdf(double z) { return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI); }
// Inverse normal CDF by Newton iteration on the CDF (converges to ~1 ulp for p in (0.5, 1)).
double normal_quantile(double p) {
  double z = 0.0;
  for (int i = 0; i < 100; ++i) {
    double step = (normal_cdf(z) - p) / normal_pdf(z);
    z -= step;
    if (std::fabs(step) < 1e-17 * std::max(1.0, std::fabs(z))) break;
  }
  return z;
}
}  // namespace

void nf4_codebook(float out[16]) {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double v[16];
  int n = 0;
  for (int j = 0; j < 8; ++j) v[n++] = normal_quantile(delta - j * (delta - 0.5) / 8.0);
  for (int j = 0; j < 7; ++j) v[n++] = -normal_quantile(delta - j * (delta - 0.5) / 7.0);
  v[n++] = 0.0;
  std::sort(v, v + 16);
  const double scale = normal_quantile(delta);
  for (int i = 0; i < 16; ++i) out[i] = (float)(v[i] / scale);
}

Nf4Table nf4_table() {
  Nf4Table t;
  nf4_codebook(t.cb);
  for (int j = 0; j < 15; ++j) t.mid[j] = (t.cb[j] + t.cb[j + 1]) * 0.5f;
  t.mid[15] = 2.0f;  // sentinel, never below x
  return t;
}

// ---------------------------------------------------------------------------------- quantise
namespace {

// One warp per 64-element block: lane i owns elements 2i, 2i+1 and writes byte i.
__global__ void k_q_codes(const float* __restrict__ w, int64_t nblocks, uint8_t* __restrict__ packed,
                          float* __restrict__ absmax, const Nf4Table tab) {
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= nblocks) return;
  const float2 v = reinterpret_cast<const float2*>(w + warp_global * 64)[lane];
  const float a = warp_max(fmaxf(fabsf(v.x), fabsf(v.y)));
  uint32_t c0 = 7, c1 = 7;
  if (a > 0.0f) {
    const float x0 = __fdiv_rn(v.x, a), x1 = __fdiv_rn(v.y, a);
    c0 = 0;
    c1 = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) {
      c0 += tab.mid[j] < x0;
      c1 += tab.mid[j] < x1;
    }
  }
  packed[warp_global * 32 + lane] = (uint8_t)((c0 << 4) | c1);
  if (lane == 0) absmax[warp_global] = a;
}

// One thread per group of 256 absmax values: fp64 sum in index order.
__global__ void k_q_group_sums(const float* __restrict__ absmax, int64_t nblocks, double* __restrict__ gsum) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t ng = (nblocks + 255) / 256;
  if (g >= ng) return;
  double s = 0.0;
  const int64_t end = min((g + 1) * 256, nblocks);
  for (int64_t b = g * 256; b < end; ++b) s += (double)absmax[b];
  gsum[g] = s;
}

// Single thread: group sums in index order, divided by the count, rounded to fp32.
__global__ void k_q_mean(const double* __restrict__ gsum, int64_t nblocks, float* __restrict__ mean) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int64_t ng = (nblocks + 255) / 256;
  double s = 0.0;
  for (int64_t g = 0; g < ng; ++g) s += gsum[g];
  *mean = (float)(s / (double)nblocks);
}

// One 256-thread block per group: c = a - mean, s = max|c|, q = rint(c / s * 127).
__global__ void k_q_double(const float* __restrict__ absmax, int64_t nblocks, const float* __restrict__ mean,
                           int8_t* __restrict__ qabs, float* __restrict__ gscale) {
  __shared__ float red[8];
  const int64_t g = blockIdx.x;
  const int64_t b = g * 256 + threadIdx.x;
  const float mu = *mean;
  const float c = b < nblocks ? __fsub_rn(absmax[b], mu) : 0.0f;
  float m = warp_max(fabsf(c));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float s = red[0];
  for (int i = 1; i < 8; ++i) s = fmaxf(s, red[i]);
  if (threadIdx.x == 0) gscale[g] = s;
  if (b < nblocks) {
    int q = 0;
    if (s > 0.0f) {
      const float u = __fmul_rn(__fdiv_rn(c, s), 127.0f);
      q = (int)rintf(u);
      q = max(-127, min(127, q));
    }
    qabs[b] = (int8_t)q;
  }
}

}  // namespace

cudaError_t nf4_quantize(const float* w, int64_t n, const Nf4Out& o, float* scratch_absmax,
                         double* scratch_gsum, cudaStream_t s) {
  if (n <= 0 || (n % 64) != 0) return cudaErrorInvalidValue;
  const int64_t nb = n / 64;
  const int64_t ng = (nb + 255) / 256;
  const Nf4Table tab = nf4_table();
  {
    const int64_t threads = nb * 32;
    k_q_codes<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(w, nb, o.packed, scratch_absmax, tab);
  }
  k_q_group_sums<<<(unsigned)((ng + 127) / 128), 128, 0, s>>>(scratch_absmax, nb, scratch_gsum);
  k_q_mean<<<1, 32, 0, s>>>(scratch_gsum, nb, o.mean);
  k_q_double<<<(unsigned)ng, 256, 0, s>>>(scratch_absmax, nb, o.mean, o.qabs, o.gscale);
  note_launch(4);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------- dequantise
namespace {

struct DequantJob {
  Nf4Seg seg[kMaxNf4Segs];
  int nseg;
  Nf4Table tab;
};

// Each thread expands 16 codes (8 packed bytes) into 16 bf16 values (two 16-byte stores).
__global__ void __launch_bounds__(256) k_dequant(const DequantJob job, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = job.tab.cb[threadIdx.x];
  __syncthreads();
  const int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 16-element chunk index
  int64_t e0 = chunk * 16;
  int si = 0;
  int64_t base = 0;
  for (; si < job.nseg; ++si) {
    if (e0 < base + job.seg[si].n) break;
    base += job.seg[si].n;
  }
  if (si >= job.nseg) return;
  const Nf4Seg& sg = job.seg[si];
  const int64_t le = e0 - base;               // element index inside the tensor
  const int64_t blk = le >> 6;
  const float qs = __fmul_rn((float)sg.qabs[blk], sg.gscale[blk >> 8]);
  const float ahat = __fadd_rn(__fdiv_rn(qs, 127.0f), *sg.mean);
  const uint2 pk = *reinterpret_cast<const uint2*>(sg.packed + (le >> 1));
  const uint8_t* bytes = reinterpret_cast<const uint8_t*>(&pk);
  uint4 o[2];
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(o);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float hi = __fmul_rn(cb[bytes[i] >> 4], ahat);
    const float lo = __fmul_rn(cb[bytes[i] & 15], ahat);
    h[i] = __halves2bfloat162(__float2bfloat16_rn(hi), __float2bfloat16_rn(lo));
  }
  uint4* dst = reinterpret_cast<uint4*>(out + sg.out_offset + le);
  dst[0] = o[0];
  dst[1] = o[1];
}

}  // namespace

cudaError_t nf4_dequant(const Nf4Seg* segs, int nseg, __nv_bfloat16* out, cudaStream_t s) {
  if (nseg <= 0 || nseg > kMaxNf4Segs) return cudaErrorInvalidValue;
  DequantJob job;
  int64_t total = 0;
  for (int i = 0; i < nseg; ++i) {
    job.seg[i] = segs[i];
    if (segs[i].n % 64) return cudaErrorInvalidValue;
    total += segs[i].n;
  }
  job.nseg = nseg;
  job.tab = nf4_table();
  const int64_t chunks = total / 16;
  const cudaError_t e = launch_k(k_dequant, dim3((unsigned)((chunks + 255) / 256)), dim3(256), 0, s, 0, job, out);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lst
