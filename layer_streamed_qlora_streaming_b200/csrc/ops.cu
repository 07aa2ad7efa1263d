// Memory-bound kernels of the decoder layer (RMSNorm, RoPE, SwiGLU, embedding, cross-entropy) and
// the LoRA side path (x A^T projections, fixed-order dA / dB reductions, operand preparation).
//
// Every reduction has a fixed order (per-thread sequential sums, xor-butterfly inside a warp, warp
// partials summed in index order), so results do not depend on scheduling: the streamed and the
// resident schedule run the same launches and give the same bytes.
#include "common.cuh"
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
__global__ void k_rmsnorm_fwd(const float* __restrict__ x, const float* __restrict__ g, int d, float eps,
                              bf16* __restrict__ y, float* __restrict__ rstd) {
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const float* xr = x + row * d;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 u = *reinterpret_cast<const float4*>(xr + c);
    ss += u.x * u.x;
    ss += u.y * u.y;
    ss += u.z * u.z;
    ss += u.w * u.w;
  }
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  if (threadIdx.x == 0) rstd[row] = r;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 u = *reinterpret_cast<const float4*>(xr + c);
    __nv_bfloat162 o[2];
    o[0] = __floats2bfloat162_rn(u.x * r * g[c], u.y * r * g[c + 1]);
    o[1] = __floats2bfloat162_rn(u.z * r * g[c + 2], u.w * r * g[c + 3]);
    *reinterpret_cast<uint2*>(y + row * d + c) = *reinterpret_cast<const uint2*>(o);
  }
}

__global__ void k_rmsnorm_bwd(const float* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ g,
                              const float* __restrict__ rstd, const float* __restrict__ dres, int d,
                              float* __restrict__ dx, bf16* __restrict__ dxb) {
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const float r = rstd[row];
  const float* dyr = dy + row * d;
  const float* xr = x + row * d;
  float dot = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) dot += dyr[c] * g[c] * (xr[c] * r);
  dot = block_sum(dot, red) / (float)d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float xh = xr[c] * r;
    float v = r * (dyr[c] * g[c] - xh * dot);
    if (dres) v += dres[row * d + c];
    dx[row * d + c] = v;
    if (dxb) dxb[row * d + c] = __float2bfloat16_rn(v);
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
__global__ void k_swiglu_fwd(const bf16* __restrict__ gu, int64_t T, int F, bf16* __restrict__ m) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * F) return;
  const int64_t t = i / F;
  const int j = (int)(i % F);
  const float g = __bfloat162float(gu[t * 2 * F + j]);
  const float u = __bfloat162float(gu[t * 2 * F + F + j]);
  const float sg = 1.0f / (1.0f + expf(-g));
  m[i] = __float2bfloat16_rn(g * sg * u);
}

__global__ void k_swiglu_bwd(const float* __restrict__ dm, const bf16* __restrict__ gu, int64_t T, int F,
                             bf16* __restrict__ dgu) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * F) return;
  const int64_t t = i / F;
  const int j = (int)(i % F);
  const float g = __bfloat162float(gu[t * 2 * F + j]);
  const float u = __bfloat162float(gu[t * 2 * F + F + j]);
  const float sg = 1.0f / (1.0f + expf(-g));
  const float d = dm[i];
  dgu[t * 2 * F + j] = __float2bfloat16_rn(d * u * sg * (1.0f + g * (1.0f - sg)));
  dgu[t * 2 * F + F + j] = __float2bfloat16_rn(d * g * sg);
}

// ------------------------------------------------------------------------------- embedding
__global__ void k_embed(const int32_t* __restrict__ tok, const bf16* __restrict__ E, int64_t T, int d, int V,
                        float* __restrict__ x) {
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
__global__ void k_ce(const float* __restrict__ logits, int V, const int32_t* __restrict__ y, float inv_T,
                     float* __restrict__ loss_rows, bf16* __restrict__ dlog) {
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const float* lr = logits + row * V;
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < V; c += blockDim.x) mx = fmaxf(mx, lr[c]);
  mx = block_max(mx, red);
  float se = 0.f;
  for (int c = threadIdx.x; c < V; c += blockDim.x) se += expf(lr[c] - mx);
  se = block_sum(se, red);
  const float lse = mx + logf(se);
  int tgt = y[row];
  if (tgt < 0 || tgt >= V) {
    if (threadIdx.x == 0) dev_fail(DEV_ERR_BAD_INDEX);
    tgt = 0;
  }
  if (threadIdx.x == 0) loss_rows[row] = lse - lr[tgt];
  bf16* dr = dlog + row * V;
  for (int c = threadIdx.x; c < V; c += blockDim.x) {
    float p = expf(lr[c] - lse);
    if (c == tgt) p -= 1.0f;
    dr[c] = __float2bfloat16_rn(p * inv_T);
  }
}

__global__ void k_mean(const float* __restrict__ v, int64_t n, float* __restrict__ out) {
  __shared__ float red[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += v[i];
  s = block_sum(s, red);
  if (threadIdx.x == 0) *out = s / (float)n;
}

__global__ void k_dot_partial(const float* __restrict__ a, const bf16* __restrict__ b, int64_t n,
                              float* __restrict__ part) {
  __shared__ float red[32];
  const int64_t per = (n + gridDim.x - 1) / gridDim.x;
  const int64_t lo = blockIdx.x * per, hi = min(n, lo + per);
  float s = 0.f;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) s += a[i] * __bfloat162float(b[i]);
  s = block_sum(s, red);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}
__global__ void k_sum_in_order(const float* __restrict__ part, int n, float* __restrict__ out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < n; ++i) s += part[i];
    *out = s;
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ x, int64_t n, bf16* __restrict__ y) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __float2bfloat16_rn(x[i]);
}
__global__ void k_bf16_to_f32(const bf16* __restrict__ x, int64_t n, float* __restrict__ y) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __bfloat162float(x[i]);
}

// ------------------------------------------------------------------------------- LoRA
// One warp per token row; the A columns are staged 128 at a time in shared memory.
template <int RP>
__global__ void __launch_bounds__(256) k_lora_project(const bf16* __restrict__ X, int64_t ldx, int64_t T, int in,
                                                      const float* __restrict__ A, int64_t lda, int R, float s,
                                                      float* __restrict__ U, bf16* __restrict__ Us, int64_t ldus) {
  __shared__ __align__(16) float As[RP][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  float acc[RP];
#pragma unroll
  for (int j = 0; j < RP; ++j) acc[j] = 0.f;
  for (int c0 = 0; c0 < in; c0 += 128) {
    __syncthreads();
    for (int i = threadIdx.x; i < RP * 128; i += 256) {
      const int j = i >> 7, c = i & 127;
      As[j][c] = (j < R && c0 + c < in) ? A[(int64_t)j * lda + c0 + c] : 0.f;
    }
    __syncthreads();
    if (t < T) {
      const int c = c0 + lane * 4;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      const bf16* xr = X + t * ldx;
      if (c + 3 < in) {
        const uint2 u = *reinterpret_cast<const uint2*>(xr + c);
        const bf16* h = reinterpret_cast<const bf16*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __bfloat162float(h[e]);
      } else {
        for (int e = 0; e < 4; ++e)
          if (c + e < in) x[e] = __bfloat162float(xr[c + e]);
      }
#pragma unroll
      for (int j = 0; j < RP; ++j) {
        const float4 a = *reinterpret_cast<const float4*>(&As[j][lane * 4]);
        float v = acc[j];
        v = fmaf(x[0], a.x, v);
        v = fmaf(x[1], a.y, v);
        v = fmaf(x[2], a.z, v);
        v = fmaf(x[3], a.w, v);
        acc[j] = v;
      }
    }
  }
  if (t >= T) return;
#pragma unroll
  for (int j = 0; j < RP; ++j) {
    const float v = warp_sum(acc[j]);
    if (lane == 0 && j < R) {
      U[t * R + j] = v;
      Us[t * ldus + j] = __float2bfloat16_rn(s * v);
    }
  }
}

// Partial sums over a chunk of 128 tokens: thread = column.
template <int JR>
__global__ void __launch_bounds__(128) k_lora_grad_partial(const LoraGradArgs a) {
  __shared__ float Ps[128][64];
  const int c = blockIdx.x * 128 + threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.y * 128;
  const int nt = (int)min((int64_t)128, a.T - t0);
  for (int i = threadIdx.x; i < nt * a.R; i += 128) Ps[i / a.R][i % a.R] = a.P[(t0 + i / a.R) * a.R + i % a.R];
  __syncthreads();
  if (c >= a.C) return;
  int jb = 0;
  if (a.seg_r) {
    int p = 0;
    while (p + 1 < a.nseg && c >= a.bounds[p + 1]) ++p;
    jb = p * a.seg_r;
  }
  float acc[JR];
#pragma unroll
  for (int j = 0; j < JR; ++j) acc[j] = 0.f;
  const bf16* q = a.Q + t0 * a.ldq + c;
  for (int tt = 0; tt < nt; ++tt) {
    const float qv = __bfloat162float(q[(int64_t)tt * a.ldq]);
#pragma unroll
    for (int j = 0; j < JR; ++j) acc[j] = fmaf(Ps[tt][jb + j], qv, acc[j]);
  }
  float* out = a.partial + (int64_t)blockIdx.y * JR * a.C;
#pragma unroll
  for (int j = 0; j < JR; ++j) out[(int64_t)j * a.C + c] = acc[j];
}

__global__ void k_lora_grad_reduce(const LoraGradArgs a, int JR, int nchunks) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)JR * a.C) return;
  const int j = (int)(i / a.C), c = (int)(i % a.C);
  float s = 0.f;
  for (int k = 0; k < nchunks; ++k) s += a.partial[((int64_t)k * JR + j) * a.C + c];
  s *= a.s;
  if (a.seg_r) {
    int p = 0;
    while (p + 1 < a.nseg && c >= a.bounds[p + 1]) ++p;
    a.dst[p][(int64_t)(c - a.bounds[p]) * a.seg_r + j] = s;
  } else {
    a.dst[j / a.rows_per_dst][(int64_t)(j % a.rows_per_dst) * a.C + c] = s;
  }
}

__global__ void k_lora_prep(const LoraPrepArgs a) {
  const int R = a.nseg * a.r;
  const int out = a.bounds[a.nseg];
  const int64_t n1 = (int64_t)a.KP * a.in;      // Acat16 (covers Acat32 rows < R)
  const int64_t n2 = (int64_t)out * a.KP;       // Bexp16 (covers BexpT32 entries j < R)
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n1; i += stride) {
    const int j = (int)(i / a.in), c = (int)(i % a.in);
    float v = 0.f;
    if (j < R) {
      v = a.A[j / a.r][(int64_t)(j % a.r) * a.in + c];
      a.Acat32[i] = v;
    }
    a.Acat16[i] = __float2bfloat16_rn(v);
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += stride) {
    const int o = (int)(i / a.KP), j = (int)(i % a.KP);
    int p = 0;
    while (p + 1 < a.nseg && o >= a.bounds[p + 1]) ++p;
    float v = 0.f;
    if (j < R && j / a.r == p) v = a.B[p][(int64_t)(o - a.bounds[p]) * a.r + (j % a.r)];
    a.Bexp16[i] = __float2bfloat16_rn(v);
    if (j < R) a.BexpT32[(int64_t)j * out + o] = v;
  }
}

inline unsigned nblk(int64_t n, int t = kThreads) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t rmsnorm_fwd(const float* x, const float* g, int64_t T, int d, float eps, bf16* y, float* rstd,
                        cudaStream_t s) {
  if (d % 8) return cudaErrorInvalidValue;
  k_rmsnorm_fwd<<<(unsigned)T, d >= 2048 ? 256 : 128, 0, s>>>(x, g, d, eps, y, rstd);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t rmsnorm_bwd(const float* dy, const float* x, const float* g, const float* rstd, const float* dres,
                        int64_t T, int d, float* dx, bf16* dxb, cudaStream_t s) {
  k_rmsnorm_bwd<<<(unsigned)T, 256, 0, s>>>(dy, x, g, rstd, dres, d, dx, dxb);
  note_launch(1);
  return cudaGetLastError();
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
  k_swiglu_fwd<<<nblk(T * F), kThreads, 0, s>>>(gu, T, F, m);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t swiglu_bwd(const float* dm, const bf16* gu, int64_t T, int F, bf16* dgu, cudaStream_t s) {
  k_swiglu_bwd<<<nblk(T * F), kThreads, 0, s>>>(dm, gu, T, F, dgu);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t embed(const int32_t* tok, const bf16* E, int64_t T, int d, int V, float* x, cudaStream_t s) {
  if (d % 8) return cudaErrorInvalidValue;
  k_embed<<<nblk(T * (d / 8)), kThreads, 0, s>>>(tok, E, T, d, V, x);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t cross_entropy(const float* logits, int64_t T, int V, const int32_t* y, float inv_T, float* loss_rows,
                          bf16* dlog, cudaStream_t s) {
  k_ce<<<(unsigned)T, 512, 0, s>>>(logits, V, y, inv_T, loss_rows, dlog);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t mean_fixed(const float* v, int64_t n, float* out, cudaStream_t s) {
  k_mean<<<1, 1024, 0, s>>>(v, n, out);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t dot_fixed(const float* a, const bf16* b, int64_t n, float* part, float* out, cudaStream_t s) {
  k_dot_partial<<<1024, 256, 0, s>>>(a, b, n, part);
  k_sum_in_order<<<1, 32, 0, s>>>(part, 1024, out);
  note_launch(2);
  return cudaGetLastError();
}
cudaError_t f32_to_bf16(const float* x, int64_t n, bf16* y, cudaStream_t s) {
  k_f32_to_bf16<<<nblk(n), kThreads, 0, s>>>(x, n, y);
  note_launch(1);
  return cudaGetLastError();
}
cudaError_t bf16_to_f32(const bf16* x, int64_t n, float* y, cudaStream_t s) {
  k_bf16_to_f32<<<nblk(n), kThreads, 0, s>>>(x, n, y);
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t lora_project(const bf16* X, int64_t ldx, int64_t T, int in, const float* A, int64_t lda, int R,
                         float s, float* U, bf16* Us, int64_t ldus, cudaStream_t st) {
  if (R <= 0 || R > 64 || (ldx % 4)) return cudaErrorInvalidValue;
  const unsigned g = (unsigned)((T + 7) / 8);
  if (R <= 16) k_lora_project<16><<<g, 256, 0, st>>>(X, ldx, T, in, A, lda, R, s, U, Us, ldus);
  else if (R <= 32) k_lora_project<32><<<g, 256, 0, st>>>(X, ldx, T, in, A, lda, R, s, U, Us, ldus);
  else if (R <= 48) k_lora_project<48><<<g, 256, 0, st>>>(X, ldx, T, in, A, lda, R, s, U, Us, ldus);
  else k_lora_project<64><<<g, 256, 0, st>>>(X, ldx, T, in, A, lda, R, s, U, Us, ldus);
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t lora_grad(const LoraGradArgs& a, cudaStream_t st) {
  const int JR = a.seg_r ? a.seg_r : a.R;
  if (a.R <= 0 || a.R > 64 || a.C <= 0 || a.T <= 0) return cudaErrorInvalidValue;
  const int nchunks = (int)((a.T + 127) / 128);
  dim3 grid((a.C + 127) / 128, nchunks);
  switch (JR) {
    case 8: k_lora_grad_partial<8><<<grid, 128, 0, st>>>(a); break;
    case 16: k_lora_grad_partial<16><<<grid, 128, 0, st>>>(a); break;
    case 24: k_lora_grad_partial<24><<<grid, 128, 0, st>>>(a); break;
    case 32: k_lora_grad_partial<32><<<grid, 128, 0, st>>>(a); break;
    case 48: k_lora_grad_partial<48><<<grid, 128, 0, st>>>(a); break;
    case 64: k_lora_grad_partial<64><<<grid, 128, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  k_lora_grad_reduce<<<nblk((int64_t)JR * a.C), kThreads, 0, st>>>(a, JR, nchunks);
  note_launch(2);
  return cudaGetLastError();
}

cudaError_t lora_prep(const LoraPrepArgs& a, cudaStream_t st) {
  if (a.nseg < 1 || a.nseg > 3 || a.nseg * a.r > a.KP) return cudaErrorInvalidValue;
  k_lora_prep<<<1024, kThreads, 0, st>>>(a);
  note_launch(1);
  return cudaGetLastError();
}

}  // namespace lst
