// Memory-bound kernels of the decoder layer (RMSNorm, RoPE, SwiGLU, embedding, cross-entropy) and
// the LoRA side path (x A^T projections, fixed-order dA / dB reductions, operand preparation).
//
// Every reduction has a fixed order (per-thread sequential sums, xor-butterfly inside a warp, warp
// partials summed in index order), so results do not depend on scheduling: the streamed and the
// resident schedule run the same launches and give the same bytes.
#include "common.cuh"
#include "pdl.cuh"
#include "ex2.cuh"
#include "ops.cuh"

namespace lst {
namespace {

constexpr int kThreads = 256;

// Block-wide sum with a fixed order; every thread returns the same value.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float s = -INFINITY;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) s = fmaxf(s, red[i]);
  return s;
}

// ------------------------------------------------------------------------------- RMSNorm
// Forward: one CTA per row, the row held in registers: thread t owns the float4 columns t,
// t + blockDim, ..., t + (kRnV - 1) blockDim (coalesced), so the row crosses HBM once and the
// normalisation reads it from registers after the block reduction; blockDim = rn_threads(d).
// Backward: one CTA of 256 threads per row, two passes over dy and x (the second from cache).
constexpr int kRnV = 8;  // float4 per thread: rows of up to 32 * blockDim elements
__host__ __device__ inline int rn_threads(int d) {
  const int n = (d / 4 + kRnV - 1) / kRnV;
  return n <= 32 ? 32 : ((n + 31) / 32) * 32;
}

__global__ void k_rmsnorm_fwd(const float* __restrict__ x, const float* __restrict__ g, int d, float eps,
                              bf16* __restrict__ y, float* __restrict__ rstd) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int n4 = d / 4;
  const float4* xr = reinterpret_cast<const float4*>(x + row * d);
  float4 v[kRnV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kRnV; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    v[i] = c < n4 ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[i].x * v[i].x;
    ss += v[i].y * v[i].y;
    ss += v[i].z * v[i].z;
    ss += v[i].w * v[i].w;
  }
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  if (threadIdx.x == 0) rstd[row] = r;
  const float4* g4 = reinterpret_cast<const float4*>(g);
#pragma unroll
  for (int i = 0; i < kRnV; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c >= n4) break;
    const float4 gg = g4[c];
    __nv_bfloat162 o[2];
    o[0] = __floats2bfloat162_rn(v[i].x * r * gg.x, v[i].y * r * gg.y);
    o[1] = __floats2bfloat162_rn(v[i].z * r * gg.z, v[i].w * r * gg.w);
    *reinterpret_cast<uint2*>(y + row * d + 4 * c) = *reinterpret_cast<const uint2*>(o);
  }
}

__global__ void k_rmsnorm_bwd(const float* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ g,
                              const float* __restrict__ rstd, const float* __restrict__ dres, int d,
                              float* __restrict__ dx, bf16* __restrict__ dxb) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const float r = rstd[row];
  const float* dyr = dy + row * d;
  const float* xr = x + row * d;
  float dot = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 a = *reinterpret_cast<const float4*>(dyr + c);
    const float4 b = *reinterpret_cast<const float4*>(xr + c);
    dot += a.x * g[c] * (b.x * r);
    dot += a.y * g[c + 1] * (b.y * r);
    dot += a.z * g[c + 2] * (b.z * r);
    dot += a.w * g[c + 3] * (b.w * r);
  }
  dot = block_sum(dot, red) / (float)d;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 a = *reinterpret_cast<const float4*>(dyr + c);
    const float4 b = *reinterpret_cast<const float4*>(xr + c);
    float v[4] = {r * (a.x * g[c] - b.x * r * dot), r * (a.y * g[c + 1] - b.y * r * dot),
                  r * (a.z * g[c + 2] - b.z * r * dot), r * (a.w * g[c + 3] - b.w * r * dot)};
    if (dres) {
      const float4 q = *reinterpret_cast<const float4*>(dres + row * d + c);
      v[0] += q.x;
      v[1] += q.y;
      v[2] += q.z;
      v[3] += q.w;
    }
    *reinterpret_cast<float4*>(dx + row * d + c) = make_float4(v[0], v[1], v[2], v[3]);
    if (dxb) {
      __nv_bfloat162 h[2] = {__floats2bfloat162_rn(v[0], v[1]), __floats2bfloat162_rn(v[2], v[3])};
      *reinterpret_cast<uint2*>(dxb + row * d + c) = *reinterpret_cast<const uint2*>(h);
    }
  }
}

// ------------------------------------------------------------------------------- RoPE
__global__ void k_rope(bf16* __restrict__ buf, int64_t ld, int64_t T, int S, int col0, int nh, int hd,
                       const float* __restrict__ ct, const float* __restrict__ st, int inverse) {
  const int half = hd / 2;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * nh * half) return;
  const int j = (int)(i % half);
  const int h = (int)((i / half) % nh);
  const int64_t t = i / ((int64_t)half * nh);
  const int pos = (int)(t % S);
  bf16* p = buf + t * ld + col0 + (int64_t)h * hd;
  const float x1 = __bfloat162float(p[j]), x2 = __bfloat162float(p[j + half]);
  const float c = ct[pos * half + j], sn = st[pos * half + j];
  float y1, y2;
  if (!inverse) {
    y1 = x1 * c - x2 * sn;
    y2 = x2 * c + x1 * sn;
  } else {
    y1 = x1 * c + x2 * sn;
    y2 = x2 * c - x1 * sn;
  }
  p[j] = __float2bfloat16_rn(y1);
  p[j + half] = __float2bfloat16_rn(y2);
}

__global__ void k_rope_tables(int S, int hd, double theta, float* ct, float* st) {
  const int half = hd / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= S * half) return;
  const int pos = i / half, j = i % half;
  const double ang = (double)pos * pow(theta, -2.0 * (double)j / (double)hd);
  ct[i] = (float)cos(ang);
  st[i] = (float)sin(ang);
}

// ------------------------------------------------------------------------------- SwiGLU
// 8 consecutive elements per thread (16-byte loads and stores); F is a multiple of 8.
// sigmoid(g) = 1 / (1 + 2^(-g log2 e)) with the SFU's approximate exp2 (about 2 ulp) and a correctly
// rounded reciprocal; the results are rounded to bf16.
constexpr float kLog2e = 1.4426950408889634f;
__device__ __forceinline__ float sigmoid_fast(float g) { return __frcp_rn(1.0f + ex2_approx(-g * kLog2e)); }
__global__ void k_swiglu_fwd(const bf16* __restrict__ gu, int64_t T, int F, bf16* __restrict__ m) {
  pdl_wait();
  pdl_trigger();
  const int f8 = F / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * f8) return;
  const int64_t t = i / f8;
  const int j = (int)(i % f8) * 8;
  const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + j);
  const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + j);
  const bf16* g8 = reinterpret_cast<const bf16*>(&gv);
  const bf16* u8 = reinterpret_cast<const bf16*>(&uv);
  uint4 o;
  __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float r[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float g = __bfloat162float(g8[2 * e + k]), u = __bfloat162float(u8[2 * e + k]);
      const float sg = sigmoid_fast(g);
      r[k] = g * sg * u;
    }
    o2[e] = __floats2bfloat162_rn(r[0], r[1]);
  }
  *reinterpret_cast<uint4*>(m + t * F + j) = o;
}

__global__ void k_swiglu_bwd(const float* __restrict__ dm, const bf16* __restrict__ gu, int64_t T, int F,
                             bf16* __restrict__ dgu) {
  pdl_wait();
  pdl_trigger();
  const int f8 = F / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * f8) return;
  const int64_t t = i / f8;
  const int j = (int)(i % f8) * 8;
  const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + j);
  const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + j);
  const float4 d0 = *reinterpret_cast<const float4*>(dm + t * F + j);
  const float4 d1 = *reinterpret_cast<const float4*>(dm + t * F + j + 4);
  const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
  const bf16* g8 = reinterpret_cast<const bf16*>(&gv);
  const bf16* u8 = reinterpret_cast<const bf16*>(&uv);
  uint4 og, ou;
  __nv_bfloat162* og2 = reinterpret_cast<__nv_bfloat162*>(&og);
  __nv_bfloat162* ou2 = reinterpret_cast<__nv_bfloat162*>(&ou);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float rg[2], ru[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float g = __bfloat162float(g8[2 * e + k]), u = __bfloat162float(u8[2 * e + k]);
      const float sg = sigmoid_fast(g);
      const float d = dd[2 * e + k];
      rg[k] = d * u * sg * (1.0f + g * (1.0f - sg));
      ru[k] = d * g * sg;
    }
    og2[e] = __floats2bfloat162_rn(rg[0], rg[1]);
    ou2[e] = __floats2bfloat162_rn(ru[0], ru[1]);
  }
  *reinterpret_cast<uint4*>(dgu + t * 2 * F + j) = og;
  *reinterpret_cast<uint4*>(dgu + t * 2 * F + F + j) = ou;
}

// ------------------------------------------------------------------------------- embedding
__global__ void k_embed(const int32_t* __restrict__ tok, const bf16* __restrict__ E, int64_t T, int d, int V,
                        float* __restrict__ x) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8-element vector index
  const int nv = d / 8;
  if (i >= T * nv) return;
  const int64_t t = i / nv;
  const int c = (int)(i % nv) * 8;
  const int id = tok[t];
  uint4 v = make_uint4(0, 0, 0, 0);
  if (id >= 0 && id < V) v = *reinterpret_cast<const uint4*>(E + (int64_t)id * d + c);
  else if (c == 0) dev_fail(DEV_ERR_BAD_INDEX);
  const bf16* h = reinterpret_cast<const bf16*>(&v);
  float4* o = reinterpret_cast<float4*>(x + t * d + c);
  o[0] = make_float4(__bfloat162float(h[0]), __bfloat162float(h[1]), __bfloat162float(h[2]), __bfloat162float(h[3]));
  o[1] = make_float4(__bfloat162float(h[4]), __bfloat162float(h[5]), __bfloat162float(h[6]), __bfloat162float(h[7]));
}

// ------------------------------------------------------------------------------- cross-entropy
// One CTA per row. Pass 1 reads the row once and keeps a running (max, sum of exp) pair per thread,
// rescaling the sum when the max grows (the online normaliser of Milakov & Gimelshein, "Online
// normalizer calculation for softmax", 2018); the pairs are merged in a fixed tree. Pass 2 reads
// the row again, usually from L2 (one 1024-thread CTA per SM keeps ~148 rows in flight), and writes
// dlogits. Deterministic: the thread-to-element map and the merge order depend only on V.
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;  // both empty
  s = s * expf(m - M) + s2 * expf(m2 - M);
  m = M;
}
__device__ __forceinline__ void ms_add4(float& m, float& s, float4 v) {
  const float M = fmaxf(fmaxf(m, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
  s = s * expf(m - M) + (expf(v.x - M) + expf(v.y - M)) + (expf(v.z - M) + expf(v.w - M));
  m = M;
}

__global__ void __launch_bounds__(1024, 1)
k_ce(const float* __restrict__ logits, int V, const int32_t* __restrict__ y, float inv_T,
     float* __restrict__ loss_rows, bf16* __restrict__ dlog) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sm[32], ss[32];
  const int64_t row = blockIdx.x;
  const float* lr = logits + row * V;
  bf16* dr = dlog + row * V;
  const bool vec = (V % 4) == 0;  // rows then start 16-byte aligned
  float m = -INFINITY, s = 0.f;
  if (vec) {
    const float4* l4 = reinterpret_cast<const float4*>(lr);
    for (int c = threadIdx.x; c < V / 4; c += blockDim.x) ms_add4(m, s, __ldg(l4 + c));
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) ms_add4(m, s, make_float4(lr[c], -INFINITY, -INFINITY, -INFINITY));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_merge(m, s, m2, s2);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sm[w] = m;
    ss[w] = s;
  }
  __syncthreads();
  m = sm[0];
  s = ss[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) ms_merge(m, s, sm[i], ss[i]);
  const float lse = m + logf(s);
  int tgt = y[row];
  if (tgt < 0 || tgt >= V) {
    if (threadIdx.x == 0) dev_fail(DEV_ERR_BAD_INDEX);
    tgt = 0;
  }
  if (threadIdx.x == 0) loss_rows[row] = lse - lr[tgt];
  if (vec) {
    const float4* l4 = reinterpret_cast<const float4*>(lr);
    for (int c = threadIdx.x; c < V / 4; c += blockDim.x) {
      const float4 v = __ldg(l4 + c);
      float p[4] = {expf(v.x - lse), expf(v.y - lse), expf(v.z - lse), expf(v.w - lse)};
      const int d = tgt - 4 * c;
      if (d >= 0 && d < 4) p[d] -= 1.0f;
      const __nv_bfloat162 h[2] = {__floats2bfloat162_rn(p[0] * inv_T, p[1] * inv_T),
                                   __floats2bfloat162_rn(p[2] * inv_T, p[3] * inv_T)};
      *reinterpret_cast<uint2*>(dr + 4 * c) = *reinterpret_cast<const uint2*>(h);
    }
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) {
      float p = expf(lr[c] - lse);
      if (c == tgt) p -= 1.0f;
      dr[c] = __float2bfloat16_rn(p * inv_T);
    }
  }
}

// Cross-entropy rows that read each logit once: a thread-block cluster of cs CTAs holds one row
// in shared memory, CTA z the slice [z * slice, (z + 1) * slice), brought in by kCeChunks bulk
// asynchronous copies issued at once (the copy engine keeps the whole slice in flight, and the
// first pass starts on a chunk as soon as it has landed). On the slice in shared memory: its max,
// then its sum of exp(x - max) in a fixed order; the cs (max, sum) pairs are merged in rank order
// through distributed shared memory (every CTA gets the same lse); then each CTA writes dlogits of
// its slice, and the CTA holding the target writes the row's loss. exp(t) is taken as 2^(t log2 e)
// (the SFU's approximate exp2 on the product, formed with one fma). Needs V % 4 == 0 (16-byte
// aligned slices).
constexpr int kCeThreads = 256, kCeChunks = 4;
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// block-wide max / sum of one value per thread (kCeThreads), fixed tree; every thread gets it
__device__ __forceinline__ float ce_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int i = 1; i < kCeThreads / 32; ++i) v = fmaxf(v, red[i]);
  return v;
}
__device__ __forceinline__ float ce_block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int i = 1; i < kCeThreads / 32; ++i) v += red[i];
  return v;
}

__global__ void __launch_bounds__(kCeThreads)
k_ce_cluster(const float* __restrict__ logits, int V, int slice, const int32_t* __restrict__ y, float inv_T,
             float* __restrict__ loss_rows, bf16* __restrict__ dlog) {
  // [slice] floats, the CTA's (max, sum) pair, kCeChunks mbarriers
  extern __shared__ __align__(128) float row_s[];
  __shared__ float red_m[kCeThreads / 32], red_s[kCeThreads / 32];
  const int cs = (int)cluster_size_x();
  const int z = (int)cluster_rank();
  const int64_t row = blockIdx.x / cs;
  const int c0 = z * slice, n = max(0, min(V - c0, slice));
  const int n4 = n / 4, q4 = (n4 + kCeChunks - 1) / kCeChunks;  // float4s in the slice, in a chunk
  float* pair = row_s + slice;
  uint64_t* bar = reinterpret_cast<uint64_t*>(pair + 2);
  if (threadIdx.x == 0) {
    for (int k = 0; k < kCeChunks; ++k) mbar_init(bar + k, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // the logits of the previous kernel are complete from here on
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int k = 0; k < kCeChunks; ++k) {
      const int a = min(n4, k * q4), b = min(n4, a + q4);
      mbar_arrive_expect_tx(bar + k, (uint32_t)(b - a) * 16);
      if (b > a) bulk_load(row_s + 4 * a, logits + row * V + c0 + 4 * a, (uint32_t)(b - a) * 16, bar + k);
    }
  }
  int tgt = y[row];
  const float4* r4 = reinterpret_cast<const float4*>(row_s);
  float m = -INFINITY;
  for (int k = 0; k < kCeChunks; ++k) {
    const int a = min(n4, k * q4), b = min(n4, a + q4);
    mbar_wait(bar + k, 0);
    for (int c = a + threadIdx.x; c < b; c += kCeThreads) {
      const float4 v = r4[c];
      m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
  }
  m = ce_block_max(m, red_m);
  float sum = 0.f;
  if (m != -INFINITY) {
    const float ml = m * kLog2e;
    for (int c = threadIdx.x; c < n4; c += kCeThreads) {
      const float4 v = r4[c];
      sum += (ex2_approx(fmaf(v.x, kLog2e, -ml)) + ex2_approx(fmaf(v.y, kLog2e, -ml))) +
             (ex2_approx(fmaf(v.z, kLog2e, -ml)) + ex2_approx(fmaf(v.w, kLog2e, -ml)));
    }
  }
  sum = ce_block_sum(sum, red_s);
  if (threadIdx.x == 0) {
    pair[0] = m;
    pair[1] = sum;
  }
  cluster_sync_all();  // every CTA's pair is in place
  const uint32_t pa = smem_u32(pair);
  float M = -INFINITY;
  for (int q = 0; q < cs; ++q) M = fmaxf(M, ld_cluster_f2(cluster_map(pa, (uint32_t)q)).x);
  float S = 0.f;
  for (int q = 0; q < cs; ++q) {
    const float2 v = ld_cluster_f2(cluster_map(pa, (uint32_t)q));
    if (v.x != -INFINITY) S += v.y * ex2_approx((v.x - M) * kLog2e);
  }
  cluster_sync_all();  // no CTA leaves while another still reads its pair
  const float lse = M + logf(S);
  if (tgt < 0 || tgt >= V) {
    if (threadIdx.x == 0 && z == 0) dev_fail(DEV_ERR_BAD_INDEX);
    tgt = 0;
  }
  if (threadIdx.x == 0 && tgt >= c0 && tgt < c0 + n) loss_rows[row] = lse - row_s[tgt - c0];
  bf16* dr = dlog + row * V + c0;
  const float ll = lse * kLog2e;
  for (int c = threadIdx.x; c < n4; c += kCeThreads) {
    const float4 v = r4[c];
    float p[4] = {ex2_approx(fmaf(v.x, kLog2e, -ll)), ex2_approx(fmaf(v.y, kLog2e, -ll)),
                  ex2_approx(fmaf(v.z, kLog2e, -ll)), ex2_approx(fmaf(v.w, kLog2e, -ll))};
    const int d = tgt - c0 - 4 * c;
    if (d >= 0 && d < 4) p[d] -= 1.0f;
    const __nv_bfloat162 h[2] = {__floats2bfloat162_rn(p[0] * inv_T, p[1] * inv_T),
                                 __floats2bfloat162_rn(p[2] * inv_T, p[3] * inv_T)};
    *reinterpret_cast<uint2*>(dr + 4 * c) = *reinterpret_cast<const uint2*>(h);
  }
}

// Row (max, sum of exp) of a logits row by the online rule of k_ce, merged in a fixed tree.
__device__ __forceinline__ float row_lse(const float* __restrict__ lr, int V, float* sm, float* ss) {
  float m = -INFINITY, s = 0.f;
  if ((V % 4) == 0) {
    const float4* l4 = reinterpret_cast<const float4*>(lr);
    for (int c = threadIdx.x; c < V / 4; c += blockDim.x) ms_add4(m, s, __ldg(l4 + c));
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) ms_add4(m, s, make_float4(lr[c], -INFINITY, -INFINITY, -INFINITY));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_merge(m, s, m2, s2);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sm[w] = m;
    ss[w] = s;
  }
  __syncthreads();
  m = sm[0];
  s = ss[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) ms_merge(m, s, sm[i], ss[i]);
  return m + logf(s);
}

__global__ void __launch_bounds__(1024, 1)
k_ce_stats(const float* __restrict__ logits, int V, const int32_t* __restrict__ y, float* __restrict__ lse_out,
           float* __restrict__ logp_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sm[32], ss[32];
  const int64_t row = blockIdx.x;
  const float* lr = logits + row * V;
  const float lse = row_lse(lr, V, sm, ss);
  if (threadIdx.x == 0) {
    int tgt = y[row];
    if (tgt < 0 || tgt >= V) {
      dev_fail(DEV_ERR_BAD_INDEX);
      tgt = 0;
    }
    lse_out[row] = lse;
    logp_out[row] = lr[tgt] - lse;
  }
}

// One block per sequence; the block_sum tree fixes the order.
__global__ void k_seq_sum(const float* __restrict__ v, const int32_t* __restrict__ mask, int S, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int64_t base = (int64_t)blockIdx.x * S;
  float acc = 0.f;
  for (int t = threadIdx.x; t < S; t += blockDim.x) acc += mask ? (float)mask[base + t] * v[base + t] : v[base + t];
  acc = block_sum(acc, red);
  if (threadIdx.x == 0) out[blockIdx.x] = acc;
}

__global__ void k_dpo(const float* __restrict__ pi, const float* __restrict__ ref, int P, float beta,
                      float* __restrict__ loss, float* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  float part = 0.f;
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const float z = beta * ((pi[p] - ref[p]) - (pi[P + p] - ref[P + p]));
    part += fmaxf(-z, 0.f) + log1pf(expf(-fabsf(z)));  // -log sigmoid(z), overflow-free
    const float g = (1.0f / (1.0f + expf(-z)) - 1.0f) * beta / (float)P;  // dloss/dpi of the chosen one
    w[p] = -g;
    w[P + p] = g;
  }
  part = block_sum(part, red);
  if (threadIdx.x == 0) *loss = part / (float)P;
}

__global__ void __launch_bounds__(1024, 1)
k_ce_grad(const float* __restrict__ logits, int64_t row0, int V, const int32_t* __restrict__ y,
          const float* __restrict__ lse_rows, const float* __restrict__ wseq, const int32_t* __restrict__ mask, int S,
          bf16* __restrict__ dlog) {
  pdl_wait();
  pdl_trigger();
  const int64_t lrow = blockIdx.x, row = row0 + lrow;
  const float* lr = logits + lrow * V;
  bf16* dr = dlog + lrow * V;
  const float lse = lse_rows[row];
  const float w = wseq[row / S] * (mask ? (float)mask[row] : 1.0f);
  int tgt = y[row];
  if (tgt < 0 || tgt >= V) tgt = 0;  // reported by k_ce_stats
  if ((V % 4) == 0) {
    const float4* l4 = reinterpret_cast<const float4*>(lr);
    for (int c = threadIdx.x; c < V / 4; c += blockDim.x) {
      const float4 v = __ldg(l4 + c);
      float p[4] = {expf(v.x - lse), expf(v.y - lse), expf(v.z - lse), expf(v.w - lse)};
      const int d = tgt - 4 * c;
      if (d >= 0 && d < 4) p[d] -= 1.0f;
      const __nv_bfloat162 h[2] = {__floats2bfloat162_rn(p[0] * w, p[1] * w), __floats2bfloat162_rn(p[2] * w, p[3] * w)};
      *reinterpret_cast<uint2*>(dr + 4 * c) = *reinterpret_cast<const uint2*>(h);
    }
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) {
      float p = expf(lr[c] - lse);
      if (c == tgt) p -= 1.0f;
      dr[c] = __float2bfloat16_rn(p * w);
    }
  }
}

__global__ void k_mean(const float* __restrict__ v, int64_t n, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += v[i];
  s = block_sum(s, red);
  if (threadIdx.x == 0) *out = s / (float)n;
}

__global__ void k_dot_partial(const float* __restrict__ a, const bf16* __restrict__ b, int64_t n,
                              float* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int64_t per = (n + gridDim.x - 1) / gridDim.x;
  const int64_t lo = blockIdx.x * per, hi = min(n, lo + per);
  float s = 0.f;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) s += a[i] * __bfloat162float(b[i]);
  s = block_sum(s, red);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}
__global__ void k_sum_in_order(const float* __restrict__ part, int n, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < n; ++i) s += part[i];
    *out = s;
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ x, int64_t n, bf16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __float2bfloat16_rn(x[i]);
}
// 16-byte words src -> dst (n words), grid-stride
__global__ void k_copy16(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

__global__ void k_bf16_to_f32(const bf16* __restrict__ x, int64_t n, float* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __bfloat162float(x[i]);
}

inline unsigned nblk(int64_t n, int t = kThreads) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t rmsnorm_fwd(const float* x, const float* g, int64_t T, int d, float eps, bf16* y, float* rstd,
                        cudaStream_t s) {
  if (d % 8 || rn_threads(d) > 1024) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_rmsnorm_fwd, dim3((unsigned)T), dim3(rn_threads(d)), 0, s, 0, x, g, d, eps, y, rstd);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t rmsnorm_bwd(const float* dy, const float* x, const float* g, const float* rstd, const float* dres,
                        int64_t T, int d, float* dx, bf16* dxb, cudaStream_t s) {
  if (d % 8) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_rmsnorm_bwd, dim3((unsigned)T), dim3(256), 0, s, 0, dy, x, g, rstd, dres, d, dx, dxb);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t rope(bf16* buf, int64_t ld, int64_t T, int S, int col0, int nh, int hd, const float* ct,
                 const float* st, int inverse, cudaStream_t s) {
  k_rope<<<nblk(T * nh * (hd / 2)), kThreads, 0, s>>>(buf, ld, T, S, col0, nh, hd, ct, st, inverse);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t rope_tables(int S, int hd, double theta, float* ct, float* st, cudaStream_t s) {
  k_rope_tables<<<nblk((int64_t)S * (hd / 2)), kThreads, 0, s>>>(S, hd, theta, ct, st);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t swiglu_fwd(const bf16* gu, int64_t T, int F, bf16* m, cudaStream_t s) {
  if (F % 8) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_swiglu_fwd, dim3(nblk(T * (F / 8))), dim3(kThreads), 0, s, 0, gu, T, F, m);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t swiglu_bwd(const float* dm, const bf16* gu, int64_t T, int F, bf16* dgu, cudaStream_t s) {
  if (F % 8) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_swiglu_bwd, dim3(nblk(T * (F / 8))), dim3(kThreads), 0, s, 0, dm, gu, T, F, dgu);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t embed(const int32_t* tok, const bf16* E, int64_t T, int d, int V, float* x, cudaStream_t s) {
  if (d % 8) return cudaErrorInvalidValue;
  const cudaError_t e = launch_k(k_embed, dim3(nblk(T * (d / 8))), dim3(kThreads), 0, s, 0, tok, E, T, d, V, x);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t cross_entropy(const float* logits, int64_t T, int V, const int32_t* y, float inv_T, float* loss_rows,
                          bf16* dlog, cudaStream_t s) {
  // cluster of 1-8 CTAs with slices of about 64 KB (two or three CTAs an SM); 16-byte slices need
  // V % 4 == 0, and a slice must fit one CTA's shared memory
  constexpr int64_t kTargetBytes = 64 * 1024, kMaxSliceBytes = 200 * 1024;
  int cs = 1;
  while (cs < 8 && (((int64_t)V + cs - 1) / cs) * 4 > kTargetBytes) cs *= 2;
  const int slice = (int)((((int64_t)V + cs - 1) / cs + 3) / 4 * 4);
  if ((V % 4) || (int64_t)slice * 4 > kMaxSliceBytes || T * cs > INT32_MAX) {
    const cudaError_t e = launch_k(k_ce, dim3((unsigned)T), dim3(1024), 0, s, 0, logits, V, y, inv_T, loss_rows,
                                   dlog);  // the two-pass form
    note_launch(1);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const int smem = slice * 4 + 8 + 8 * kCeChunks;  // the slice, the (max, sum) pair and the mbarriers
  static std::atomic<unsigned long long> attr_done{0};
  if (!done_on_device(attr_done)) {
    const cudaError_t e = cudaFuncSetAttribute(k_ce_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)(kMaxSliceBytes + 8 + 8 * kCeChunks));
    if (e != cudaSuccess) return e;
    mark_done_on_device(attr_done);
  }
  const cudaError_t e = launch_k(k_ce_cluster, dim3((unsigned)(T * cs)), dim3(kCeThreads), (size_t)smem, s,
                                 (unsigned)cs, logits, V, slice, y, inv_T, loss_rows, dlog);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t ce_stats(const float* logits, int64_t T, int V, const int32_t* y, float* lse, float* logp, cudaStream_t s) {
  const cudaError_t e = launch_k(k_ce_stats, dim3((unsigned)T), dim3(1024), 0, s, 0, logits, V, y, lse, logp);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t seq_sum(const float* v, const int32_t* mask, int nseq, int S, float* out, cudaStream_t s) {
  const cudaError_t e = launch_k(k_seq_sum, dim3(nseq), dim3(256), 0, s, 0, v, mask, S, out);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t dpo_loss(const float* pi, const float* ref, int P, float beta, float* loss, float* w, cudaStream_t s) {
  const cudaError_t e = launch_k(k_dpo, dim3(1), dim3(256), 0, s, 0, pi, ref, P, beta, loss, w);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t ce_grad(const float* logits, int64_t rows, int64_t row0, int V, const int32_t* y, const float* lse,
                    const float* w, const int32_t* mask, int S, bf16* dlog, cudaStream_t s) {
  const cudaError_t e = launch_k(k_ce_grad, dim3((unsigned)rows), dim3(1024), 0, s, 0, logits, row0, V, y, lse, w, mask, S, dlog);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t mean_fixed(const float* v, int64_t n, float* out, cudaStream_t s) {
  const cudaError_t e = launch_k(k_mean, dim3(1), dim3(1024), 0, s, 0, v, n, out);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t dot_fixed(const float* a, const bf16* b, int64_t n, float* part, float* out, cudaStream_t s) {
  cudaError_t e = launch_k(k_dot_partial, dim3(1024), dim3(256), 0, s, 0, a, b, n, part);
  if (e == cudaSuccess) e = launch_k(k_sum_in_order, dim3(1), dim3(32), 0, s, 0, part, 1024, out);
  note_launch(2);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t f32_to_bf16(const float* x, int64_t n, bf16* y, cudaStream_t s) {
  const cudaError_t e = launch_k(k_f32_to_bf16, dim3(nblk(n)), dim3(kThreads), 0, s, 0, x, n, y);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t bf16_to_f32(const bf16* x, int64_t n, float* y, cudaStream_t s) {
  const cudaError_t e = launch_k(k_bf16_to_f32, dim3(nblk(n)), dim3(kThreads), 0, s, 0, x, n, y);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}
cudaError_t copy16(const void* src, void* dst, int64_t bytes, cudaStream_t s) {
  if (bytes <= 0) return cudaSuccess;
  if (bytes % 16 || (reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
    return cudaErrorInvalidValue;
  const int64_t n = bytes / 16;
  const cudaError_t e = launch_k(k_copy16, dim3((unsigned)std::min<int64_t>((n + kThreads - 1) / kThreads, 1024)),
                                 dim3(kThreads), 0, s, 0, reinterpret_cast<const uint4*>(src),
                                 reinterpret_cast<uint4*>(dst), n);
  note_launch(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lst
