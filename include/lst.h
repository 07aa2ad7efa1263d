/*
 * lst.h -- layer-streamed LoRA fine-tuning on one GPU: the C ABI of liblst.so.
 *
 * What it computes (sources by page title and section):
 *  - "Soup: Fine-Tuning an 8B Model on a 4 GB Laptop GPU, One Layer at a Time" (toknow.ai),
 *    first paragraph: the frozen base stays in CPU RAM and is copied to the GPU one layer at a
 *    time, double-buffered so the next layer loads while the current one computes; the base can
 *    be 4-bit (NF4) or unquantised 16-bit; second paragraph: the forward pass is bit-exact
 *    against a resident run.
 *  - Tutorial "Fine-tune Llama 3.1 8B on a 4GB GPU with Soup" (lachieslifestyle.com), section
 *    "What Soup layer streaming changes": a two-buffer VRAM pool; each decoder layer is read in
 *    the forward pass and read again for backward recomputation; LoRA adapters stay on the GPU.
 *  - "Soup CLI fine-tunes Llama-3.1-8B on a 4 GB laptop GPU, ..." (thetesserapress.com),
 *    second paragraph: copies run on a dedicated CUDA stream; logits stay resident.
 *  - "Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU" (codeinktechnologies.com),
 *    sections "Quantization" (NF4 with nested quantisation of the constants) and "LoRA and
 *    QLoRA" (frozen quantised base, full-precision adapters).
 *
 * One step = embedding -> L pre-norm decoder layers (RMSNorm, q/k/v with RoPE, causal GQA
 * attention, o, RMSNorm, SwiGLU MLP; every projection y = x W^T + (alpha/r) (x A^T) B^T) ->
 * final RMSNorm -> LM head -> mean cross-entropy, then the analytic backward with each layer
 * recomputed from its saved input. Outputs: the loss and dL/dA, dL/dB of every adapter.
 *
 * Conventions
 *  - Every call returns an lst_status; no exception or abort crosses the ABI. After a non-OK
 *    status, lst_last_error(ctx) describes it (valid until the next call on ctx).
 *  - Matrices are row-major; a projection's W is [out, in], its A is [r, in], its B is [out, r].
 *  - Projection order everywhere: q, k, v, o, gate, up, down (LST_PROJ_*).
 *  - Pointer arguments may be host or device memory unless stated; the library detects which.
 *    The library copies what it needs before returning; the caller keeps ownership.
 *  - A context is bound to the device current at lst_create and is not thread-safe.
 *  - Device faults are never used for error reporting: device code records an error word that
 *    the host turns into LST_ERR_DEVICE, and waits are bounded (LST_ERR_TIMEOUT).
 */
#ifndef LST_H_
#define LST_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lst_ctx lst_ctx;

typedef enum {
  LST_OK = 0,
  LST_ERR_ARG = 1,      /* bad argument: null pointer, shape beyond the config, bad index */
  LST_ERR_STATE = 2,    /* call out of order: e.g. a step before every layer is registered */
  LST_ERR_OOM = 3,      /* device or pinned host allocation failed */
  LST_ERR_CUDA = 4,     /* a CUDA runtime call failed */
  LST_ERR_TIMEOUT = 5,  /* the step did not complete within timeout_ms */
  LST_ERR_DEVICE = 6    /* device code reported an error (bad token id, a bounded wait ran out) */
} lst_status;

enum { LST_BASE_NF4 = 0, LST_BASE_BF16 = 1 };
enum {
  LST_PROJ_Q = 0, LST_PROJ_K = 1, LST_PROJ_V = 2, LST_PROJ_O = 3,
  LST_PROJ_GATE = 4, LST_PROJ_UP = 5, LST_PROJ_DOWN = 6, LST_NUM_PROJ = 7
};

typedef struct {
  int32_t n_layers;     /* L >= 1 */
  int32_t d_model;      /* d, multiple of 8 */
  int32_t n_heads;      /* hq */
  int32_t n_kv_heads;   /* hkv, divides hq */
  int32_t head_dim;     /* 64 or 128 */
  int32_t ffn;          /* F, multiple of 8 */
  int32_t vocab;        /* V; 0 = headless stack (use lst_step_hidden) */
  float rms_eps;
  float rope_theta;     /* rotate-half RoPE, angle pos * theta^(-2j/hd) */
  int32_t qkv_bias;     /* 1: q, k, v projections carry a frozen bias */
  int32_t lora_rank;    /* r; 3*r <= 64 */
  float lora_alpha;     /* LoRA scale s = alpha / r */
  int32_t base_format;  /* LST_BASE_NF4: 4-bit NF4, blocks of 64, absmax double-quantised to
                           int8 in groups of 256; LST_BASE_BF16: unquantised bf16 */
  int32_t max_batch;
  int32_t max_seq;
  int32_t streamed;     /* 1: base in pinned host RAM, copied per layer read into a two-buffer
                           device pool on a dedicated copy stream; 0: all layers resident on the
                           device (same kernels, same results) */
  int32_t timeout_ms;   /* host-side wait limit of one step; <= 0 means 600000 */
  int32_t head_chunk;   /* LM head + cross-entropy in passes of this many token rows, so logits
                           [rows, V] are never resident for the whole batch; <= 0: one pass.
                           The result does not depend on it. */
  int32_t reuse;        /* 1: a layer still in the pool is not copied again (the two layers at the
                           forward/backward turn, and layers 0, 1 from the end of the previous
                           step); 0: every read copies (2L reads per step). Same results. */
} lst_config;

typedef struct {
  const float* w[LST_NUM_PROJ];       /* frozen base W [out, in] fp32 */
  const float* bias[3];               /* q, k, v bias [out] fp32; required iff qkv_bias */
  const float* attn_norm;             /* RMSNorm gains before attention [d] fp32 */
  const float* mlp_norm;              /* RMSNorm gains before the MLP [d] fp32 */
  const float* lora_a[LST_NUM_PROJ];  /* A [r, in] fp32 */
  const float* lora_b[LST_NUM_PROJ];  /* B [out, r] fp32 */
} lst_layer_weights;

typedef struct {
  int64_t steps;               /* completed steps */
  int64_t launches_last_step;  /* kernels launched by the last step */
  int64_t layer_reads_last_step; /* layer blobs copied host -> device by the last step (2L) */
  int64_t h2d_bytes_last_step; /* bytes of layer copies of the last step */
  int64_t blob_bytes;          /* bytes of one layer's frozen base as stored */
  int64_t arena_bytes;         /* pinned host bytes (streamed) or device bytes (resident) of the base */
  int64_t device_bytes;        /* device bytes allocated by the context */
  /* filled when profiling is on (lst_set_profiling): device time of the last step by class */
  double gemm_ms, attention_ms, dequant_ms, other_ms, copy_ms, step_ms;
  int64_t gemm_launches, attention_launches, dequant_launches, copy_count;
  double gemm_flops;           /* algorithmic FLOPs of the GEMM launches of the last step */
  double lora_ms;              /* LoRA side path (skinny projections, dA / dB) */
  int64_t lora_launches;
} lst_stats;

/* Create a context. embed [V, d], final_norm [d], lm_head [V, d] are fp32 (host or device; the
 * library rounds E and H to bf16 and keeps them resident); all three must be NULL iff vocab == 0.
 * cuda_stream: cudaStream_t the steps run on, or NULL for a stream owned by the context (created
 * at the highest priority). The context adds a copy stream, a device-to-host stream and a prep
 * stream at the lowest priority for the dequant of the next layer read, which then only takes SM
 * slots the step stream leaves free: give a caller stream a priority above the lowest.
 * The context belongs to the device current at this call; every later call on it runs there and
 * restores the caller's current device (one thread may drive contexts on several GPUs).
 * Environment: LST_CANARY=1 checks guard bytes after the pool and scratch buffers after each step;
 * LST_FAULT injects host-side failures (pinned_alloc:N, device_alloc:N, memcpy:N, timeout).
 * Errors: LST_ERR_ARG (bad config), LST_ERR_OOM, LST_ERR_CUDA. On error *out is NULL. */
lst_status lst_create(const lst_config* cfg, const float* embed, const float* final_norm,
                      const float* lm_head, void* cuda_stream, lst_ctx** out);

/* Register layer `layer` (0 <= layer < L): quantise (NF4) or round (bf16) the base on the device,
 * lay it out as one contiguous blob, store it in the pinned arena (streamed) or on the device
 * (resident), and copy the LoRA A, B into resident device memory. May be called again to replace
 * a layer. Synchronous. Errors: LST_ERR_ARG, LST_ERR_OOM, LST_ERR_CUDA. */
lst_status lst_register_layer(lst_ctx* ctx, int32_t layer, const lst_layer_weights* w);

/* Replace the adapters of one projection (A [r, in], B [out, r] fp32). */
lst_status lst_set_lora(lst_ctx* ctx, int32_t layer, int32_t proj, const float* a, const float* b);

/* Number of fp32 values in the gradient (and parameter) layout: for each layer, for each
 * projection in LST_PROJ order, dA [r, in] then dB [out, r]. */
int64_t lst_lora_numel(const lst_ctx* ctx);

/* AdamW on the adapters ("Fine-tune Llama 3.1 8B on a 4GB GPU with Soup", "Step 5": lr 2e-4;
 * "Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU": Adam keeps two extra tensors per
 * parameter). With an optimizer set, every step ends with
 *   m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;
 *   p <- p (1 - lr wd) - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * on every adapter element (fp32, t = 1, 2, ... counted from lst_set_optimizer), after the step's
 * gradients are complete; the next step computes with the updated adapters. */
typedef struct {
  float lr;            /* learning rate */
  float beta1, beta2;  /* moment decay rates, in [0, 1) */
  float eps;           /* > 0 */
  float weight_decay;  /* decoupled weight decay, >= 0 */
  int32_t deferred;    /* 0: applied by every step with its own gradients; 1: applied only by
                          lst_apply_optimizer, with the caller's gradients */
} lst_adamw;

/* Enable (cfg non-NULL: moments reset to zero, t reset) or disable (NULL) the update. */
lst_status lst_set_optimizer(lst_ctx* ctx, const lst_adamw* cfg);

/* One AdamW update of the adapters with the gradient g (lst_lora_numel fp32 values in the gradient
 * layout, host or device), using the moments and step count of lst_set_optimizer. For data-parallel
 * training: each replica's step leaves its gradients, the caller averages them over the replicas
 * (e.g. an NCCL all-reduce on the context's stream) and applies the average here, so every replica
 * takes the same update. Needs the optimizer set with deferred = 1 (else LST_ERR_STATE).
 * Enqueued on the context's stream; returns when the update is done. */
lst_status lst_apply_optimizer(lst_ctx* ctx, const float* g);

/* Copy the current adapters (lst_lora_numel fp32 values, gradient layout) to dst (host or device). */
lst_status lst_get_lora(lst_ctx* ctx, float* dst);

/* One forward + backward step of the model with a head: tokens and targets are int32
 * [batch * seq] (host or device), the loss is the mean cross-entropy over all tokens (written to
 * *loss, host memory). grads (host or device, may be NULL) receives lst_lora_numel() fp32 values.
 * Requires vocab > 0, every layer registered (else LST_ERR_STATE), batch <= max_batch,
 * seq <= max_seq. Blocks until the step is done or timeout_ms passed (LST_ERR_TIMEOUT). */
lst_status lst_step(lst_ctx* ctx, const int32_t* tokens, const int32_t* targets, int32_t batch,
                    int32_t seq, float* loss, float* grads);

/* Headless step of the decoder stack: x and g are bf16 bit patterns [batch * seq, d] (host or
 * device); the loss is sum(x_L * g) over all elements, so dL/dx_L = g. Same outputs and rules as
 * lst_step; requires vocab == 0. */
lst_status lst_step_hidden(lst_ctx* ctx, const uint16_t* x, const uint16_t* g, int32_t batch,
                           int32_t seq, float* loss, float* grads);

/* One DPO training step over the streamed base ("Soup CLI fine-tunes Llama-3.1-8B on a 4 GB laptop
 * GPU, and that changes who owns AI", paragraph on the economics: preference training with the
 * reference model being the same streamed base with its adapters switched off; loss of Rafailov et
 * al., "Direct Preference Optimization", 2023). The batch is 2 * n_pairs sequences of `seq` tokens:
 * the n_pairs chosen sequences, then the n_pairs rejected ones in the same pair order. tokens,
 * targets and mask are int32 [2 * n_pairs * seq] (host or device); mask (NULL = all ones) marks the
 * positions whose target log-likelihood counts towards a sequence's log-likelihood pi.
 * The step runs the reference forward with the adapters off (L layer reads), then the policy
 * forward, head and backward (2L reads): 3L reads, or fewer with reuse. *loss (host) = mean over
 * the pairs of -log sigmoid(beta * ((pi_w - ref_w) - (pi_l - ref_l))); grads as in lst_step.
 * Needs vocab > 0, 2 * n_pairs <= max_batch, beta > 0. */
lst_status lst_step_dpo(lst_ctx* ctx, const int32_t* tokens, const int32_t* targets,
                        const int32_t* mask, int32_t n_pairs, int32_t seq, float beta, float* loss,
                        float* grads);

/* Copy the last step's logits [batch * seq, V] fp32 to dst (host or device). */
lst_status lst_get_logits(lst_ctx* ctx, float* dst);

/* Inspect activations of the last step (for checking a step stage by stage). `which`:
 *  LST_ACT_X  : the fp32 residual-stream input of decoder layer `layer` [T, d] (layer == L gives
 *               the output of the last layer);
 *  LST_ACT_N1, _QKV, _O, _N2, _GU, _M : bf16 intermediates [T, d], [T, dq+2dkv] (q and k after
 *               RoPE), [T, dq], [T, d], [T, 2F], [T, F]; LST_ACT_H : fp32 [T, d];
 *               these hold the most recently computed layer, which after a step is layer 0
 *               (`layer` must be 0).
 * dst: host or device memory of the stated size. */
enum { LST_ACT_X = 0, LST_ACT_N1 = 1, LST_ACT_QKV = 2, LST_ACT_O = 3, LST_ACT_H = 4, LST_ACT_N2 = 5,
       LST_ACT_GU = 6, LST_ACT_M = 7 };
lst_status lst_get_activation(lst_ctx* ctx, int32_t which, int32_t layer, void* dst);

/* Record per-class device times of every step (CUDA events around each launch) when on != 0. */
lst_status lst_set_profiling(lst_ctx* ctx, int32_t on);

/* Per-read timeline of the last step run with profiling on (the library's own CUDA events; stands
 * in for a trace). One row of 8 floats per layer read, in read order: layer, kind (0 reference
 * forward, 1 forward, 2 backward with recompute), then milliseconds from the start of the step:
 * copy start, copy end (copy stream), dequant start, dequant end (prep stream, NF4 base), compute
 * start (compute stream, once the read's first weight group is in place), compute end. A time is
 * -1 where the read had no copy or dequant of its own (reuse, bf16 base). *n_reads receives the
 * number of reads; out must hold max_reads >= that many rows (else LST_ERR_ARG). LST_ERR_STATE if
 * no profiled step has run. Host only; no synchronisation (the step has completed). */
lst_status lst_get_read_timeline(const lst_ctx* ctx, float* out, int32_t max_reads, int32_t* n_reads);

/* Split copies over several GPUs (one process per GPU, each with its own context holding the same
 * base): each layer read copies only this rank's slice of the blob over its own host link, and an
 * in-place NCCL all-gather on the copy stream assembles the whole blob in every rank's pool slot
 * over NVLink / NVSwitch, so N GPUs divide the host-link bytes of every read by N. All ranks must
 * run the same steps in the same order (the reads are collective). The library loads
 * libnccl.so.2 on first use (LST_ERR_STATE if it cannot); the communicator is created here
 * (ncclCommInitRank, collective over the ranks) and destroyed with the context. unique_id: the 128
 * bytes of lst_nccl_unique_id from one rank, passed to every rank. world == 1 runs the same path
 * on one GPU (the whole blob is this rank's slice; the all-gather is a one-rank collective). Needs
 * a streamed context; call once, before the first step. The results are the same bytes as
 * without it (the assembled blob is the same). */
lst_status lst_set_split_copy(lst_ctx* ctx, int32_t rank, int32_t world, const void* unique_id);

/* A fresh NCCL unique id (128 bytes into out) for lst_set_split_copy. LST_ERR_STATE without NCCL. */
lst_status lst_nccl_unique_id(void* out);

/* The split-copy plan of a blob of blob_bytes (host only, no GPU): rank `rank` of `world` copies
 * bytes [*offset, *offset + *bytes) of the blob (*bytes may be 0) and contributes *count bytes
 * (a multiple of 256) from offset *offset of its pool slot to the all-gather of world * *count
 * bytes, whose first blob_bytes are the blob. */
lst_status lst_split_plan(int64_t blob_bytes, int32_t world, int32_t rank, int64_t* offset, int64_t* bytes,
                          int64_t* count);

/* The copy / dequant plan of one step, host only (no context, no GPU), for inspection and tests.
 * reads: the layer of each read in order (an SFT step reads 0..L-1 then L-1..0; a DPO step reads
 * 0..L-1 once more first); reuse / nf4: the config's reuse and base_format == LST_BASE_NF4;
 * held[2] / wheld[2]: the layers the two pool slots / two bf16 weight scratches hold before the step
 * (-1 = nothing), overwritten with what they hold after it. out: n_reads rows of 8 int32:
 * slot, copy (0/1), wait_free (the read the copy waits for, -1 none: until its compute has finished,
 * or, in a step whose NF4 base is dequantised in a separate pass with reuse off, until its dequant
 * has -- the compute then reads only the bf16 scratch and a copy of the blob's header), loaded_by
 * (the read whose copy filled the slot, -1 an earlier step), wslot, dequant (0/1), wwait,
 * wfilled_by (the same for the weight scratch; -1 / 0 for a bf16 base).
 * prefetch (may be NULL: no prefetch, as with lst_set_prefetch(ctx, 0)): in, prefetch[0] = the slot
 * a previous step already copied this step's first read into (-1 none; used with reuse off only);
 * out, prefetch[0] / prefetch[1] = the slot this step copies the next step's first read into and the
 * read that copy waits for, as wait_free (-1 / -1 with reuse on). A prefetched first read has
 * copy 0 and loaded_by -1. LST_ERR_ARG on a null pointer (other than prefetch), n_reads <= 0, a
 * negative layer or prefetch[0] outside -1..1. */
lst_status lst_plan_reads(const int32_t* reads, int32_t n_reads, int32_t reuse, int32_t nf4,
                          int32_t* held, int32_t* wheld, int32_t* prefetch, int32_t* out);

/* Where an NF4 base is dequantised in the next steps: 0 (default) in a separate pass that writes
 * each layer read's bf16 weights to a device scratch, one read ahead on a low-priority stream;
 * 1 inside the GEMMs, which build the bf16 operand tile by tile in shared memory from the NF4 blob
 * (groups whose rows are not whole 64-element blocks keep the separate pass). The results are the
 * same bytes. LST_ERR_ARG for other values. */
lst_status lst_set_dequant_mode(lst_ctx* ctx, int32_t mode);

/* Switch the copy schedule of the next steps (the config's `reuse`): 1 keeps layers that are still
 * in the pool instead of copying them again, 0 copies every read. Results are the same bytes. */
lst_status lst_set_reuse(lst_ctx* ctx, int32_t reuse);

/* Copy ahead, at the end of each step with reuse off, the next step's first read (layer 0) into the
 * pool slot that the step's last read does not use, as soon as the read before it has finished: that
 * copy overlaps the step's last layer and the optimizer instead of starting the next step. Every step
 * still copies 2L (3L for DPO) layer blobs -- one of them issued by the step before -- and returns
 * only once that copy has landed. On (1) by default; 0 switches it off. Results are the same bytes. */
lst_status lst_set_prefetch(lst_ctx* ctx, int32_t on);
lst_status lst_get_stats(const lst_ctx* ctx, lst_stats* out);

const char* lst_last_error(const lst_ctx* ctx);

/* Free everything the context owns. NULL-safe. */
void lst_destroy(lst_ctx* ctx);

/* The 16 NF4 values (fp32, ascending) the library quantises with: 8 positive and 7 negative
 * standard-normal quantiles and an exact 0, scaled to [-1, 1]. Needs no GPU. */
lst_status lst_nf4_codebook(float out[16]);

/* Bytes of one layer blob for a config (needs no GPU). */
int64_t lst_blob_bytes(const lst_config* cfg);

#ifdef __cplusplus
}
#endif

#endif /* LST_H_ */
