/*
 * lst_kernels.h -- the individual device kernels of liblst.so behind a C ABI, so each can be
 * checked on its own against the CPU oracle. All pointers are DEVICE pointers unless stated;
 * `stream` is a cudaStream_t (NULL = legacy default stream). Calls enqueue work and return
 * without synchronising; errors in the arguments return LST_ERR_ARG before anything is
 * launched, a failed launch returns LST_ERR_CUDA. bf16 buffers are passed as uint16_t bits.
 */
#ifndef LST_KERNELS_H_
#define LST_KERNELS_H_

#include <stdint.h>

#include "lst.h"

#ifdef __cplusplus
extern "C" {
#endif

/* NF4 quantisation of w [n] fp32 (n a multiple of 64), as defined in "Fine-Tuning an 8B Parameter
 * Model on a 4 GB Laptop GPU", section "Quantization" (NF4 + nested quantisation; construction
 * after QLoRA): packed [n/2] (element 2i in the high nibble), qabs [n/64] int8,
 * gscale [ceil(n/64/256)] fp32, mean [1] fp32. Allocates and frees its own scratch. */
lst_status lst_k_nf4_quantize(const float* w, int64_t n, uint8_t* packed, int8_t* qabs,
                              float* gscale, float* mean, void* stream);

/* Same result as lst_k_nf4_quantize, for callers that cannot allocate device memory: code whose
 * GPU memory is all reserved by its own caching allocator, or code that must not trigger the
 * device-wide synchronisation of cudaMalloc / cudaFree while other streams run. The pages have no
 * counterpart of this entry point; it is an interface variant of this library.
 *  - Scratch comes from one fixed device array inside the library (4 MiB + 32 KiB), present on
 *    every GPU that loads the library until the process exits. It allocates nothing and calls no
 *    allocating routine.
 *  - n is limited to 67,108,864 elements (1 << 26); larger n returns LST_ERR_ARG and launches
 *    nothing, as does n not a multiple of 64 or a null pointer.
 *  - Every call looks up the array's address on the current device (cudaGetSymbolAddress, which
 *    allocates nothing), so the entry point stays valid across a device reset. The first call on
 *    a device may load the library's device code there; make it before any stream capture.
 *  - Asynchronous on `stream`. All calls share the one array, which keeps the last call's
 *    contents (nothing in it needs clearing: it is fully rewritten before being read), so calls
 *    whose work overlaps on the GPU (other streams, other threads) race on it: order them. */
lst_status lst_k_nf4_quantize_noalloc(const float* w, int64_t n, uint8_t* packed, int8_t* qabs,
                                      float* gscale, float* mean, void* stream);

/* Dequantise one NF4 tensor into bf16 [n]: a^ = (q * s) / 127 + mean, w^ = bf16(code * a^),
 * each operation one fp32 rounding; bit-exact by construction. */
lst_status lst_k_nf4_dequant(const uint8_t* packed, const int8_t* qabs, const float* gscale,
                             const float* mean, int64_t n, uint16_t* out, void* stream);

/* C = alpha * (A' B' + A2 B2') + bias + R on the tcgen05 tensor cores (fp32 accumulate).
 * A' = A with A [M, K] (a_mn = 0) or A' = A^T with A [K, M] (a_mn = 1, needs b_mn = 1), row
 * stride lda; B' = B^T with B [N, K] (b_mn = 0) or B' = B with B [K, N] (b_mn = 1),
 * row stride ldb; (A2 [M, K2], B2) optional second pair of the same major-ness (NULL to skip);
 * C [M, N] fp32 (c_f32 = 1) or bf16; bias [N] fp32 or NULL; R [M, N] fp32 (residual) or NULL.
 * Leading dimensions must be multiples of 8 and A/B/A2/B2 16-byte aligned. */
lst_status lst_k_gemm(int32_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda,
                      int32_t a_mn, const uint16_t* B, int64_t ldb, int32_t b_mn, const uint16_t* A2,
                      int64_t lda2, const uint16_t* B2, int64_t ldb2, int32_t K2, void* C,
                      int64_t ldc, int32_t c_f32, float alpha, const float* bias,
                      const float* R, int64_t ldr, void* stream);

/* One NF4 tensor (format of lst_k_nf4_quantize) of a weight matrix stacked from up to three
 * such tensors along its rows (q/k/v, gate/up), covering `rows` consecutive rows. */
typedef struct {
  const uint8_t* packed;  /* [rows * cols / 2], 16-byte aligned */
  const int8_t* qabs;     /* [rows * cols / 64] */
  const float* gscale;    /* [ceil(rows * cols / 64 / 256)] */
  const float* mean;      /* [1] */
  int32_t rows;
} lst_nf4_part;

/* lst_k_gemm with the frozen base B dequantised from NF4 inside the GEMM ("Fine-Tuning an 8B
 * Parameter Model on a 4 GB Laptop GPU", section "Quantization: Shrink the Weights": the 4-bit
 * base is expanded to 16 bits for the matrix product): W = the nparts (1..3) tensors stacked
 * along rows; b_mn = 0: C = A W^T with W [N, K]; b_mn = 1: C = A W with W [K, N]. W's row length
 * (K or N) must be a multiple of 64, a_mn is 0, the parts must cover W's rows. The operand equals
 * lst_k_nf4_dequant of the parts bit for bit, so C equals lst_k_gemm on the dequantised matrix
 * byte for byte. parts is a HOST array. Other arguments as lst_k_gemm. */
lst_status lst_k_gemm_nf4(int32_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda,
                          const lst_nf4_part* parts, int32_t nparts, int32_t b_mn,
                          const uint16_t* A2, int64_t lda2, const uint16_t* B2, int64_t ldb2,
                          int32_t K2, void* C, int64_t ldc, int32_t c_f32, float alpha,
                          const float* bias, const float* R, int64_t ldr, void* stream);

/* Causal GQA attention forward over T = batch*S tokens: q [T, ldq], k [T, ldk], v [T, ldv]
 * (head h at column h*hd), o [T, ldo] bf16, lse [T, hq] fp32. hd in {64, 128}; row strides
 * multiples of 8 and bases 16-byte aligned (the tiles are loaded by TMA). The probabilities enter
 * the P V product as fp16 with V converted to fp16, exact for |v| in [2^-14, 65504]: entries of v
 * must stay below 65504 in magnitude (larger ones would overflow to infinity). */
lst_status lst_k_attention_fwd(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk,
                               const uint16_t* v, int64_t ldv, uint16_t* o, int64_t ldo,
                               float* lse, int64_t T, int32_t S, int32_t hq, int32_t hkv,
                               int32_t hd, void* stream);

/* Attention backward: dq [T, lddq], dk [T, lddk], dv [T, lddv] bf16 from dout [T, lddo] and the
 * forward's o and lse; D is scratch [T, hq] fp32. Deterministic (no atomics). */
lst_status lst_k_attention_bwd(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk,
                               const uint16_t* v, int64_t ldv, const uint16_t* o, int64_t ldo,
                               const uint16_t* dout, int64_t lddo, const float* lse, float* D,
                               uint16_t* dq, int64_t lddq, uint16_t* dk, int64_t lddk,
                               uint16_t* dv, int64_t lddv, int64_t T, int32_t S, int32_t hq,
                               int32_t hkv, int32_t hd, void* stream);

/* RMSNorm forward of the fp32 residual stream x [T, d]: y = bf16(x * rstd * g), rstd [T]. */
lst_status lst_k_rmsnorm_fwd(const float* x, const float* g, int64_t T, int32_t d, float eps,
                             uint16_t* y, float* rstd, void* stream);
/* RMSNorm backward: dx = dres + rstd (dy g - xhat mean(dy g xhat)); dres and dx_bf16 may be NULL. */
lst_status lst_k_rmsnorm_bwd(const float* dy, const float* x, const float* g,
                             const float* rstd, const float* dres, int64_t T, int32_t d,
                             float* dx, uint16_t* dx_bf16, void* stream);

/* RoPE in place on nh heads starting at column col0 of buf [T, ld]; cos/sin tables [S, hd/2]
 * from lst_k_rope_tables; inverse != 0 applies the transpose (backward). */
lst_status lst_k_rope_tables(int32_t S, int32_t hd, double theta, float* cos_t, float* sin_t,
                             void* stream);
lst_status lst_k_rope(uint16_t* buf, int64_t ld, int64_t T, int32_t S, int32_t col0, int32_t nh,
                      int32_t hd, const float* cos_t, const float* sin_t, int32_t inverse,
                      void* stream);

/* SwiGLU: m = silu(g) * u with gu = [g | u] [T, 2F]; backward gives dgu [T, 2F] from dm fp32. */
lst_status lst_k_swiglu_fwd(const uint16_t* gu, int64_t T, int32_t F, uint16_t* m, void* stream);
lst_status lst_k_swiglu_bwd(const float* dm, const uint16_t* gu, int64_t T, int32_t F,
                            uint16_t* dgu, void* stream);

/* Cross-entropy rows over fp32 logits [T, V]: loss_rows [T], dlogits bf16 [T, V] scaled by inv_T. */
lst_status lst_k_cross_entropy(const float* logits, int64_t T, int32_t V, const int32_t* targets,
                               float inv_T, float* loss_rows, uint16_t* dlogits, void* stream);

/* LoRA skinny projection Us = bf16(s * X Bop) of the side path ("Fine-Tuning an 8B Parameter
 * Model on a 4 GB Laptop GPU", section "LoRA and QLoRA"): X bf16 [T, K] (row stride ldx); Bop bf16
 * K-major [KP, K] (b_mn = 0: Us = s X Bop^T) or MN-major [K, KP] (b_mn = 1: Us = s X Bop);
 * Us [T, KP] contiguous, KP a multiple of 8; ldx, ldb multiples of 8 and X, Bop 16-byte aligned.
 * The K range is split over a thread-block cluster whose partial tiles are summed in slice order
 * through distributed shared memory: deterministic, no scratch. */
lst_status lst_k_lora_skinny(const uint16_t* X, int64_t ldx, int64_t T, int32_t K,
                             const uint16_t* Bop, int64_t ldb, int32_t b_mn, int32_t KP, float s,
                             uint16_t* Us, void* stream);

/* The same projection at fp32-level precision for adapters kept in full precision (same section):
 * each adapter value is stored as the bf16 pair hi = bf16(a), lo = bf16(a - hi), hi in sections
 * [0, RS) and [RS, 2 RS) and lo in [2 RS, 3 RS) of the KP-wide dimension of Bop (rows when
 * b_mn = 0, columns when b_mn = 1). U = s X (hi + lo) is accumulated in fp32 and its columns
 * j < R are stored as bf16 pairs too: Us[t][j] = Us[t][2 RS + j] = bf16(U), Us[t][RS + j] =
 * bf16(U - bf16(U)); the other columns of Us [T, KP] are not written. Sections [hi | lo | hi] of
 * Us against [hi | hi | lo] of the operand form, in one extra K block of the base GEMM, the
 * product of U and the adapter up to the lo x lo term. R <= RS <= 64, RS a multiple of 8,
 * 3 RS <= KP, KP a multiple of 8. Deterministic, no scratch. */
lst_status lst_k_lora_skinny_split(const uint16_t* X, int64_t ldx, int64_t T, int32_t K,
                                   const uint16_t* Bop, int64_t ldb, int32_t b_mn, int32_t R,
                                   int32_t RS, int32_t KP, float s, uint16_t* Us, void* stream);

/* LoRA adapter gradients of one fused projection group (same section): nseg (1..3) segments of rank
 * r sharing the input X bf16 [T, in] (row stride ldx), with output-gradient dY bf16 [T, out] (row
 * stride ldy) whose columns [bounds[p], bounds[p+1]) belong to segment p (bounds: HOST array of
 * nseg + 1 ints, bounds[0] = 0, bounds[nseg] = out). Us = bf16(s X A_cat^T), Vs = bf16(s dY B_exp)
 * [T, KP] (column p*r + j = rank j of segment p; only columns < nseg*r are read, so the hi section
 * of a split Us / Vs serves as well). Writes, fp32:
 *   dA[p] [r, in]:        dA_p[j][i] = sum_t Vs[t][p*r + j] X[t][i]
 *   dB[p] [out_p, r]:     dB_p[o][j] = sum_t dY[t][bounds[p] + o] Us[t][p*r + j]
 * dA, dB: HOST arrays of nseg device pointers. Sums over t in a fixed order (deterministic). */
lst_status lst_k_lora_grads(const uint16_t* X, int64_t ldx, int32_t in, const uint16_t* dY,
                            int64_t ldy, int32_t out, int64_t T, const uint16_t* Us,
                            const uint16_t* Vs, int32_t KP, int32_t nseg, int32_t r,
                            const int32_t* bounds, float* const* dA, float* const* dB,
                            void* stream);

/* One fused group of lst_k_lora_grads_multi: the arguments of lst_k_lora_grads, with bounds, dA and
 * dB held in the struct (dA / dB: nseg device pointers; unused entries ignored). */
typedef struct {
  const uint16_t* X;
  int64_t ldx;
  int32_t in;
  const uint16_t* dY;
  int64_t ldy;
  int32_t out;
  const uint16_t* Us;
  const uint16_t* Vs;
  int32_t KP, nseg, r;
  int32_t bounds[4];
  float* dA[3];
  float* dB[3];
} lst_lora_grad_group;

/* The adapter gradients of n (1..4) fused groups of the same T in one launch -- what a layer's
 * backward issues for its four groups -- each group's results as lst_k_lora_grads defines them.
 * How far the T sums are split over a thread-block cluster follows the launch's total number of
 * output tiles, so a group's fp32 sums may round differently alone and in company (the bytes are
 * fixed for a given set of groups). groups: HOST array of n structs. */
lst_status lst_k_lora_grads_multi(const lst_lora_grad_group* groups, int32_t n, int64_t T, void* stream);

/* Read and clear the device error word of the current device: 0 when no kernel reported a
 * problem, else the code of the first report (1: a bounded wait gave up, 2: an index was out of
 * range). Synchronises the device. Returns -1 if the word cannot be read. */
int32_t lst_k_device_error(void);

/* Kernel launches made by this library so far in this process (all contexts). Needs no GPU. */
int64_t lst_k_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LST_KERNELS_H_ */
