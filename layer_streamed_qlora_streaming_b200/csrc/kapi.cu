// C ABI of the individual kernels (include/lst_kernels.h): argument checks and marshalling only.
#include "../../include/lst_kernels.h"
#include "attention.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "lora.cuh"
#include "nf4.cuh"
#include "ops.cuh"

#include <atomic>

namespace lst {
extern std::atomic<long long> g_launch_count;
}

using namespace lst;

namespace {
inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }
inline const bf16* B16(const uint16_t* p) { return reinterpret_cast<const bf16*>(p); }
inline bf16* B16(uint16_t* p) { return reinterpret_cast<bf16*>(p); }
inline lst_status st(cudaError_t e) {
  if (e == cudaSuccess) return LST_OK;
  cudaGetLastError();
  return e == cudaErrorInvalidValue ? LST_ERR_ARG : LST_ERR_CUDA;
}
}  // namespace

extern "C" {

lst_status lst_k_nf4_quantize(const float* w, int64_t n, uint8_t* packed, int8_t* qabs, float* gscale, float* mean,
                              void* stream) {
  if (!w || !packed || !qabs || !gscale || !mean || n <= 0 || n % 64) return LST_ERR_ARG;
  const int64_t nb = n / 64, ng = (nb + 255) / 256;
  float* absmax = nullptr;
  double* gsum = nullptr;
  if (cudaMalloc(&absmax, nb * 4) != cudaSuccess) return LST_ERR_OOM;
  if (cudaMalloc(&gsum, ng * 8) != cudaSuccess) {
    cudaFree(absmax);
    return LST_ERR_OOM;
  }
  Nf4Out o{packed, qabs, gscale, mean};
  cudaError_t e = nf4_quantize(w, n, o, absmax, gsum, S(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
  cudaFree(absmax);
  cudaFree(gsum);
  return st(e);
}

lst_status lst_k_nf4_dequant(const uint8_t* packed, const int8_t* qabs, const float* gscale, const float* mean,
                             int64_t n, uint16_t* out, void* stream) {
  if (!packed || !qabs || !gscale || !mean || !out || n <= 0 || n % 64) return LST_ERR_ARG;
  Nf4Seg s{packed, qabs, gscale, mean, n, 0};
  return st(nf4_dequant(&s, 1, B16(out), S(stream)));
}

lst_status lst_k_gemm(int32_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda, int32_t a_mn, const uint16_t* B,
                      int64_t ldb,
                      int32_t b_mn, const uint16_t* A2, int64_t lda2, const uint16_t* B2, int64_t ldb2, int32_t K2,
                      void* C, int64_t ldc, int32_t c_f32, float alpha, const float* bias, const float* R,
                      int64_t ldr, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || !A || !B || !C) return LST_ERR_ARG;
  if ((A2 == nullptr) != (B2 == nullptr)) return LST_ERR_ARG;
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.A = B16(A);
  a.lda = lda;
  a.B = B16(B);
  a.ldb = ldb;
  a.b_mn = b_mn ? 1 : 0;
  a.a_mn = a_mn ? 1 : 0;
  a.A2 = B16(A2);
  a.lda2 = lda2;
  a.B2 = B16(B2);
  a.ldb2 = ldb2;
  a.K2 = A2 ? K2 : 0;
  a.C = C;
  a.ldc = ldc;
  a.c_f32 = c_f32 ? 1 : 0;
  a.alpha = alpha;
  a.bias = bias;
  a.R = R;
  a.ldr = ldr;
  return st(gemm_bf16(a, S(stream)));
}

lst_status lst_k_gemm_nf4(int32_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda, const lst_nf4_part* parts,
                          int32_t nparts, int32_t b_mn, const uint16_t* A2, int64_t lda2, const uint16_t* B2,
                          int64_t ldb2, int32_t K2, void* C, int64_t ldc, int32_t c_f32, float alpha, const float* bias,
                          const float* R, int64_t ldr, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || !A || !C || !parts || nparts < 1 || nparts > 3) return LST_ERR_ARG;
  if ((A2 == nullptr) != (B2 == nullptr)) return LST_ERR_ARG;
  Nf4Mat q;
  q.nseg = nparts;
  q.cols = b_mn ? N : K;
  int rows = 0;
  for (int g = 0; g < nparts; ++g) {
    if (parts[g].rows <= 0 || ((int64_t)parts[g].rows * q.cols) % 64) return LST_ERR_ARG;
    rows += parts[g].rows;
    q.row_end[g] = rows;
    q.packed[g] = parts[g].packed;
    q.qabs[g] = parts[g].qabs;
    q.gscale[g] = parts[g].gscale;
    q.mean[g] = parts[g].mean;
  }
  if (rows != (b_mn ? K : N)) return LST_ERR_ARG;
  nf4_codebook(q.cb);
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.A = B16(A);
  a.lda = lda;
  a.b_mn = b_mn ? 1 : 0;
  a.Bq = &q;
  a.A2 = B16(A2);
  a.lda2 = lda2;
  a.B2 = B16(B2);
  a.ldb2 = ldb2;
  a.K2 = A2 ? K2 : 0;
  a.C = C;
  a.ldc = ldc;
  a.c_f32 = c_f32 ? 1 : 0;
  a.alpha = alpha;
  a.bias = bias;
  a.R = R;
  a.ldr = ldr;
  return st(gemm_bf16(a, S(stream)));
}

lst_status lst_k_attention_fwd(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk, const uint16_t* v,
                               int64_t ldv, uint16_t* o, int64_t ldo, float* lse, int64_t T, int32_t Sq, int32_t hq,
                               int32_t hkv, int32_t hd, void* stream) {
  if (!q || !k || !v || !o || !lse) return LST_ERR_ARG;
  AttnArgs a{B16(q), B16(k), B16(v), B16(o), lse, nullptr, ldq, ldk, ldv, ldo, T, Sq, hq, hkv, hd, 0.f};
  a.scale = 1.0f / sqrtf((float)hd);
  return st(attention_fwd(a, S(stream)));
}

lst_status lst_k_attention_bwd(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk, const uint16_t* v,
                               int64_t ldv, const uint16_t* o, int64_t ldo, const uint16_t* dout, int64_t lddo,
                               const float* lse, float* D, uint16_t* dq, int64_t lddq, uint16_t* dk, int64_t lddk,
                               uint16_t* dv, int64_t lddv, int64_t T, int32_t Sq, int32_t hq, int32_t hkv, int32_t hd,
                               void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !D || !dq || !dk || !dv) return LST_ERR_ARG;
  AttnBwdArgs a;
  a.q = B16(q);
  a.k = B16(k);
  a.v = B16(v);
  a.o = B16(o);
  a.dout = B16(dout);
  a.lse = lse;
  a.D = D;
  a.dq = B16(dq);
  a.dk = B16(dk);
  a.dv = B16(dv);
  a.ldq = ldq;
  a.ldk = ldk;
  a.ldv = ldv;
  a.ldo = ldo;
  a.lddo = lddo;
  a.lddq = lddq;
  a.lddk = lddk;
  a.lddv = lddv;
  a.T = T;
  a.S = Sq;
  a.hq = hq;
  a.hkv = hkv;
  a.hd = hd;
  a.scale = 1.0f / sqrtf((float)hd);
  return st(attention_bwd(a, S(stream)));
}

lst_status lst_k_rmsnorm_fwd(const float* x, const float* g, int64_t T, int32_t d, float eps, uint16_t* y,
                             float* rstd, void* stream) {
  if (!x || !g || !y || !rstd || T <= 0 || d <= 0) return LST_ERR_ARG;
  return st(rmsnorm_fwd(x, g, T, d, eps, B16(y), rstd, S(stream)));
}

lst_status lst_k_rmsnorm_bwd(const float* dy, const float* x, const float* g, const float* rstd, const float* dres,
                             int64_t T, int32_t d, float* dx, uint16_t* dxb, void* stream) {
  if (!dy || !x || !g || !rstd || !dx || T <= 0 || d <= 0) return LST_ERR_ARG;
  return st(rmsnorm_bwd(dy, x, g, rstd, dres, T, d, dx, B16(dxb), S(stream)));
}

lst_status lst_k_rope_tables(int32_t Sq, int32_t hd, double theta, float* ct, float* sn, void* stream) {
  if (!ct || !sn || Sq <= 0 || hd <= 0 || hd % 2) return LST_ERR_ARG;
  return st(rope_tables(Sq, hd, theta, ct, sn, S(stream)));
}

lst_status lst_k_rope(uint16_t* buf, int64_t ld, int64_t T, int32_t Sq, int32_t col0, int32_t nh, int32_t hd,
                      const float* ct, const float* sn, int32_t inverse, void* stream) {
  if (!buf || !ct || !sn || T <= 0 || Sq <= 0) return LST_ERR_ARG;
  return st(rope(B16(buf), ld, T, Sq, col0, nh, hd, ct, sn, inverse, S(stream)));
}

lst_status lst_k_swiglu_fwd(const uint16_t* gu, int64_t T, int32_t F, uint16_t* m, void* stream) {
  if (!gu || !m || T <= 0 || F <= 0) return LST_ERR_ARG;
  return st(swiglu_fwd(B16(gu), T, F, B16(m), S(stream)));
}

lst_status lst_k_swiglu_bwd(const float* dm, const uint16_t* gu, int64_t T, int32_t F, uint16_t* dgu, void* stream) {
  if (!dm || !gu || !dgu || T <= 0 || F <= 0) return LST_ERR_ARG;
  return st(swiglu_bwd(dm, B16(gu), T, F, B16(dgu), S(stream)));
}

lst_status lst_k_cross_entropy(const float* logits, int64_t T, int32_t V, const int32_t* targets, float inv_T,
                               float* loss_rows, uint16_t* dlogits, void* stream) {
  if (!logits || !targets || !loss_rows || !dlogits || T <= 0 || V <= 0) return LST_ERR_ARG;
  return st(cross_entropy(logits, T, V, targets, inv_T, loss_rows, B16(dlogits), S(stream)));
}

lst_status lst_k_lora_skinny(const uint16_t* X, int64_t ldx, int64_t T, int32_t K, const uint16_t* Bop, int64_t ldb,
                             int32_t b_mn, int32_t KP, float s, uint16_t* Us, void* stream) {
  if (!X || !Bop || !Us || T <= 0 || K <= 0 || KP <= 0 || (KP % 8)) return LST_ERR_ARG;
  return st(lora_skinny(B16(X), ldx, T, K, B16(Bop), ldb, b_mn ? 1 : 0, KP, s, B16(Us), S(stream)));
}

lst_status lst_k_lora_skinny_split(const uint16_t* X, int64_t ldx, int64_t T, int32_t K, const uint16_t* Bop,
                                   int64_t ldb, int32_t b_mn, int32_t R, int32_t RS, int32_t KP, float s, uint16_t* Us,
                                   void* stream) {
  if (!X || !Bop || !Us || T <= 0 || K <= 0 || R <= 0 || R > RS || RS > 64 || (RS % 8) || 3 * RS > KP || (KP % 8))
    return LST_ERR_ARG;
  return st(lora_skinny_split(B16(X), ldx, T, K, B16(Bop), ldb, b_mn ? 1 : 0, R, RS, KP, s, B16(Us), S(stream)));
}

lst_status lst_k_lora_grads(const uint16_t* X, int64_t ldx, int32_t in, const uint16_t* dY, int64_t ldy,
                            int32_t out, int64_t T, const uint16_t* Us, const uint16_t* Vs, int32_t KP, int32_t nseg,
                            int32_t r, const int32_t* bounds, float* const* dA, float* const* dB, void* stream) {
  if (!X || !dY || !Us || !Vs || !bounds || !dA || !dB || T <= 0 || in <= 0 || out <= 0) return LST_ERR_ARG;
  if (nseg < 1 || nseg > 3 || r <= 0 || nseg * r > KP || (KP % 8)) return LST_ERR_ARG;
  int b[4] = {0, 0, 0, 0};
  for (int p = 0; p <= nseg; ++p) b[p] = bounds[p];
  for (int p = 0; p < nseg; ++p)
    if (!dA[p] || !dB[p] || b[p + 1] <= b[p]) return LST_ERR_ARG;
  if (b[0] != 0 || b[nseg] != out) return LST_ERR_ARG;
  return st(lora_grads(B16(X), ldx, in, B16(dY), ldy, out, T, B16(Us), B16(Vs), KP, nseg, r, b, dA, dB, S(stream)));
}

lst_status lst_k_lora_grads_multi(const lst_lora_grad_group* groups, int32_t n, int64_t T, void* stream) {
  if (!groups || n < 1 || n > 4 || T <= 0) return LST_ERR_ARG;
  LoraGradProb q[4];
  for (int i = 0; i < n; ++i) {
    const lst_lora_grad_group& g = groups[i];
    if (!g.X || !g.dY || !g.Us || !g.Vs || g.in <= 0 || g.out <= 0) return LST_ERR_ARG;
    if (g.nseg < 1 || g.nseg > 3 || g.r <= 0 || g.nseg * g.r > g.KP || (g.KP % 8)) return LST_ERR_ARG;
    if (g.bounds[0] != 0 || g.bounds[g.nseg] != g.out) return LST_ERR_ARG;
    q[i] = LoraGradProb{};
    q[i].X = B16(g.X);
    q[i].ldx = g.ldx;
    q[i].in = g.in;
    q[i].dY = B16(g.dY);
    q[i].ldy = g.ldy;
    q[i].out = g.out;
    q[i].Us = B16(g.Us);
    q[i].Vs = B16(g.Vs);
    q[i].KP = g.KP;
    q[i].nseg = g.nseg;
    q[i].r = g.r;
    for (int p = 0; p <= g.nseg; ++p) q[i].bounds[p] = g.bounds[p];
    for (int p = 0; p < g.nseg; ++p) {
      if (!g.dA[p] || !g.dB[p] || g.bounds[p + 1] <= g.bounds[p]) return LST_ERR_ARG;
      q[i].dA[p] = g.dA[p];
      q[i].dB[p] = g.dB[p];
    }
  }
  return st(lora_grads_multi(q, n, T, S(stream)));
}

int64_t lst_k_launch_count(void) { return g_launch_count.load(); }

}  // extern "C"
