// Streaming engine and the C ABI of include/lst.h.
//
// The frozen base of every decoder layer is one contiguous, group-major blob. In streamed mode the
// blobs live in one pinned host arena; an SFT step makes 2L layer reads (layers 0..L-1 forward,
// then L-1..0 backward with recompute), a DPO step 3L (a reference forward with the adapters off
// first). Each read computes from one of two device pool slots, filled with cudaMemcpyAsync on a
// dedicated copy stream in four chunks (q/k/v with the small tensors, o, gate/up, down), and for
// an NF4 base from one of two bf16 weight scratches, filled chunk by chunk on a low-priority prep
// stream one read ahead. Events fence the streams: the compute of a weight group waits for its
// chunk's copy and dequant; a copy into a slot waits for "free" of the last read that computed from
// it. So the next layer streams in while the current one computes ("Soup: Fine-Tuning an 8B Model
// on a 4 GB Laptop GPU, One Layer at a Time", first paragraph: double buffering; tutorial
// "Fine-tune Llama 3.1 8B on a 4GB GPU with Soup", section "What Soup layer streaming changes":
// two-buffer pool, forward read plus backward-recomputation read; "Soup CLI fine-tunes
// Llama-3.1-8B on a 4 GB laptop GPU", second paragraph: a dedicated CUDA stream for the copies).
// plan_reads fixes, before a step, every read's slot and scratch and which copies and dequants run
// (with `reuse`, a layer still held by a slot or scratch is not fetched again).
//
// The forward keeps only each layer's input; the backward reads the layer again, recomputes its
// forward (keeping the intermediates) and runs its backward. A pinned host gradient buffer is
// filled layer by layer on a device-to-host stream during the backward. Resident mode runs the same
// launches on blobs that stay on the device, so every mode and schedule gives the same bytes.
#include "../../include/lst.h"
#include "../../include/lst_kernels.h"
#include "attention.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "lora.cuh"
#include "nf4.cuh"
#include "ops.cuh"
#include "optim.cuh"

#include <atomic>
#include <cstdio>
#include <dlfcn.h>
#include <nvtx3/nvToolsExt.h>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

namespace lst {
__device__ int g_lst_dev_error = 0;
std::atomic<long long> g_launch_count{0};
}  // namespace lst

using namespace lst;

namespace {

constexpr int NPROJ = 7;
enum { G_QKV = 0, G_O = 1, G_GU = 2, G_DOWN = 3, NGROUP = 4 };

inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// ------------------------------------------------------------------------- host fault injection
// LST_FAULT=pinned_alloc:N | device_alloc:N | memcpy:N | timeout  -- fail the N-th (1-based)
// pinned allocation / device allocation / layer-copy enqueue, or report a step timeout.
struct Faults {
  long pinned_at = 0, device_at = 0, memcpy_at = 0;
  bool timeout = false;
  long pinned_n = 0, device_n = 0, memcpy_n = 0;
  Faults() {
    const char* e = std::getenv("LST_FAULT");
    if (!e) return;
    std::string s(e);
    auto num = [&](const char* key) -> long {
      auto p = s.find(key);
      if (p == std::string::npos) return 0;
      return std::atol(s.c_str() + p + std::strlen(key));
    };
    pinned_at = num("pinned_alloc:");
    device_at = num("device_alloc:");
    memcpy_at = num("memcpy:");
    timeout = s.find("timeout") != std::string::npos;
  }
  bool fail_pinned() { return pinned_at && ++pinned_n == pinned_at; }
  bool fail_device() { return device_at && ++device_n == device_at; }
  bool fail_memcpy() { return memcpy_at && ++memcpy_n == memcpy_at; }
};

struct Group {
  int nseg = 0;
  int proj[3] = {0, 0, 0};
  int in = 0, out = 0;
  int bounds[4] = {0, 0, 0, 0};
  // LoRA side path: R = nseg * r adapter ranks; the split operands hold sections [hi | hi | lo] of
  // RS = round_up(R, 8) each, padded to KP = round_up(3 RS, 64) (the GEMMs' extra K block)
  int R = 0, RS = 0, KP = 0;
  int64_t woff = 0;  // element offset of the group's W in the concatenated bf16 weights
};

// A layer blob is group-major: the small fp32 tensors first (NF4 means, norm gains, q/k/v bias),
// then the projection groups in compute order (q/k/v, o, gate/up, down), each group holding its
// packed codes, absmax codes and group scales (NF4) or its bf16 matrices. Chunk g spans
// [chunk[g], chunk[g + 1]): chunk 0 = the small tensors + q/k/v, then o, gate/up, down, so a layer
// can be copied (and dequantised) group by group and its compute start on the first group.
constexpr int NCHUNK = 4;
struct Layout {
  int64_t n[NPROJ], outd[NPROJ], ind[NPROJ], woff[NPROJ];
  int64_t P = 0;
  int64_t packed[NPROJ], qabs[NPROJ], gscale[NPROJ], means = 0, w16 = 0, norms = 0, bias = 0, total = 0;
  int64_t chunk[NCHUNK + 1];
};

bool valid_config(const lst_config* c, std::string* why) {
  auto bad = [&](const char* m) {
    if (why) *why = m;
    return false;
  };
  if (!c) return bad("null config");
  if (c->n_layers < 1) return bad("n_layers must be >= 1");
  if (c->d_model <= 0 || c->d_model % 8) return bad("d_model must be a positive multiple of 8");
  if (c->n_heads <= 0 || c->n_kv_heads <= 0 || c->n_heads % c->n_kv_heads) return bad("bad head counts");
  if (c->head_dim != 64 && c->head_dim != 128) return bad("head_dim must be 64 or 128");
  if (c->ffn <= 0 || c->ffn % 8) return bad("ffn must be a positive multiple of 8");
  if (c->vocab < 0) return bad("vocab must be >= 0");
  if (c->lora_rank <= 0 || 3 * c->lora_rank > 64) return bad("lora_rank must be in [1, 21]");
  if (!(c->lora_alpha == c->lora_alpha)) return bad("lora_alpha is NaN");
  if (c->base_format != LST_BASE_NF4 && c->base_format != LST_BASE_BF16) return bad("bad base_format");
  if (c->max_batch <= 0 || c->max_seq <= 0) return bad("max_batch and max_seq must be positive");
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 0.f)) return bad("rms_eps and rope_theta must be positive");
  const int64_t dq = (int64_t)c->n_heads * c->head_dim, dkv = (int64_t)c->n_kv_heads * c->head_dim;
  if ((dq * c->d_model) % 64 || (dkv * c->d_model) % 64 || ((int64_t)c->ffn * c->d_model) % 64)
    return bad("every projection must have a multiple of 64 elements");
  return true;
}

Layout make_layout(const lst_config& c) {
  Layout L{};
  const int64_t d = c.d_model, dq = (int64_t)c.n_heads * c.head_dim, dkv = (int64_t)c.n_kv_heads * c.head_dim,
                F = c.ffn;
  const int64_t outs[NPROJ] = {dq, dkv, dkv, d, F, F, d};
  const int64_t ins[NPROJ] = {d, d, d, dq, d, d, F};
  int64_t acc = 0;
  for (int p = 0; p < NPROJ; ++p) {
    L.outd[p] = outs[p];
    L.ind[p] = ins[p];
    L.n[p] = outs[p] * ins[p];
    L.woff[p] = acc;
    acc += L.n[p];
  }
  L.P = acc;
  static const int kGroupProj[NCHUNK + 1] = {0, 3, 4, 6, 7};  // projections of each chunk
  int64_t off = 0;
  if (c.base_format == LST_BASE_NF4) {
    L.means = off;
    off = align256(off + NPROJ * 4);
  }
  L.norms = off;
  off = align256(off + 2 * d * 4);
  L.bias = off;
  if (c.qkv_bias) off = align256(off + (dq + 2 * dkv) * 4);
  L.chunk[0] = 0;
  if (c.base_format == LST_BASE_NF4) {
    for (int g = 0; g < NCHUNK; ++g) {
      for (int p = kGroupProj[g]; p < kGroupProj[g + 1]; ++p) { L.packed[p] = off; off = align256(off + L.n[p] / 2); }
      for (int p = kGroupProj[g]; p < kGroupProj[g + 1]; ++p) { L.qabs[p] = off; off = align256(off + L.n[p] / 64); }
      for (int p = kGroupProj[g]; p < kGroupProj[g + 1]; ++p) {
        L.gscale[p] = off;
        off = align256(off + ((L.n[p] / 64 + 255) / 256) * 4);
      }
      L.chunk[g + 1] = off;
    }
  } else {
    L.w16 = off;  // the 7 matrices back to back, so q/k/v and gate/up are single matrices
    for (int g = 0; g < NCHUNK; ++g) L.chunk[g + 1] = L.w16 + L.woff[kGroupProj[g + 1] - 1] * 2 + L.n[kGroupProj[g + 1] - 1] * 2;
    off = align256(off + L.P * 2);
    L.chunk[NCHUNK] = off;
  }
  L.total = off;
  return L;
}

constexpr int64_t kGuardBytes = 4096;
constexpr uint8_t kGuardByte = 0xA5;

bool is_pinned_host_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// ------------------------------------------------------------------------- NCCL, loaded on demand
// The split-copy mode (lst_set_split_copy) all-gathers each layer blob over NVLink with NCCL. The
// library does not link NCCL: the few entry points it uses are looked up in libnccl.so.2 the first
// time the mode is switched on (the copy a process already loaded, e.g. torch's, is found first).
// Declarations follow NCCL's public API (nccl.h); ncclUniqueId is 128 opaque bytes.
struct NcclUid {
  char internal[128];
};
typedef struct NcclComm* NcclCommT;
enum { kNcclUint8 = 1 };  // ncclUint8 in nccl.h's ncclDataType_t
struct NcclApi {
  bool ok = false;
  int (*get_unique_id)(NcclUid*) = nullptr;
  int (*comm_init_rank)(NcclCommT*, int, NcclUid, int) = nullptr;
  int (*all_gather)(const void*, void*, size_t, int, NcclCommT, cudaStream_t) = nullptr;
  int (*comm_destroy)(NcclCommT) = nullptr;
  const char* (*error_string)(int) = nullptr;
};
const NcclApi& nccl() {
  static NcclApi api = [] {
    NcclApi a;
    void* h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("libnccl.so", RTLD_NOW | RTLD_GLOBAL);
    if (!h) return a;
    a.get_unique_id = reinterpret_cast<int (*)(NcclUid*)>(dlsym(h, "ncclGetUniqueId"));
    a.comm_init_rank = reinterpret_cast<int (*)(NcclCommT*, int, NcclUid, int)>(dlsym(h, "ncclCommInitRank"));
    a.all_gather = reinterpret_cast<int (*)(const void*, void*, size_t, int, NcclCommT, cudaStream_t)>(
        dlsym(h, "ncclAllGather"));
    a.comm_destroy = reinterpret_cast<int (*)(NcclCommT)>(dlsym(h, "ncclCommDestroy"));
    a.error_string = reinterpret_cast<const char* (*)(int)>(dlsym(h, "ncclGetErrorString"));
    a.ok = a.get_unique_id && a.comm_init_rank && a.all_gather && a.comm_destroy && a.error_string;
    return a;
  }();
  return api;
}

// The slice of a blob of `blob` bytes that rank `rank` of `world` copies in split-copy mode: every
// rank contributes `count` bytes (a multiple of 256) to an all-gather of world * count bytes;
// rank r's part is [r * count, r * count + count) clipped to the blob (possibly empty).
void split_plan(int64_t blob, int world, int rank, int64_t* off, int64_t* bytes, int64_t* count) {
  const int64_t c = ((blob + (int64_t)world * 256 - 1) / ((int64_t)world * 256)) * 256;
  const int64_t o = (int64_t)rank * c;
  *count = c;
  *off = o;
  *bytes = o >= blob ? 0 : std::min(c, blob - o);
}

// Profiling classes
enum { PC_GEMM = 0, PC_ATTN = 1, PC_DEQ = 2, PC_OTHER = 3, PC_COPY = 4, PC_LORA = 5, PC_N = 6 };

}  // namespace

enum ReadKind { RD_REF = 0, RD_FWD = 1, RD_BWD = 2 };

// NVTX range on the host thread for the scope (shows the enqueue of each read and copy in a
// timeline tool; costs nothing when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* fmt, int a, int b) {
    char name[64];
    std::snprintf(name, sizeof(name), fmt, a, b);
    nvtxRangePushA(name);
  }
  ~NvtxRange() { nvtxRangePop(); }
};
enum HeadMode { HEAD_SFT = 0, HEAD_HIDDEN = 1, HEAD_DPO = 2 };

struct ReadPlan {
  int slot = 0;         // pool slot the read computes from
  bool copy = true;     // the layer is copied into the slot for this read
  int wait_free = -1;   // the copy waits for this read's compute to finish (-1: nothing to wait for)
  int loaded_by = -1;   // read whose copy filled the slot (-1: filled by an earlier step)
  // NF4 base: bf16 weight scratch the read computes from
  int wslot = 0;
  bool deq = true;      // the layer is dequantised into the scratch for this read
  int wwait = -1;       // the dequant waits for this read's compute to finish
  int wfilled_by = -1;  // read whose dequant filled the scratch (-1: an earlier step)
};

struct lst_ctx {
  lst_config cfg{};
  int dev = 0;
  cudaStream_t stream = nullptr, copy_stream = nullptr;
  cudaStream_t prep_stream = nullptr;  // dequant of the next read, below the compute stream's priority
  cudaStream_t d2h_stream = nullptr;   // gradients to pinned host memory, layer by layer
  // guard bytes after the pool slots and weight scratches, checked after each step when the
  // environment sets LST_CANARY=1 (a kernel or copy writing past one of them is reported)
  std::vector<uint8_t*> guards;
  bool check_guards = [] {
    const char* e = std::getenv("LST_CANARY");
    return e && e[0] && std::strcmp(e, "0") != 0;
  }();
  float* grads_host = nullptr;         // pinned host destination of this step's gradients (or null)
  // split-copy mode: this rank copies its slice of each blob, NCCL all-gathers the rest (world > 1)
  int split_world = 1, split_rank = 0;
  NcclCommT nccl_comm = nullptr;
  int64_t pool_bytes = 0;               // bytes of each pool slot before its guard
  // NF4 base: where the weights are dequantised -- 0: a separate pass into a bf16 scratch, one read
  // ahead on the prep stream; 1: inside the GEMMs, for every group whose rows are whole NF4 blocks
  int deq_mode = 0;
  bool fuse_ok[NGROUP] = {false, false, false, false};
  cudaEvent_t ev_d2h = nullptr;
  bool own_stream = false;
  std::string err;
  Faults faults;

  int d = 0, hq = 0, hkv = 0, hd = 0, F = 0, V = 0, L = 0, r = 0;
  int64_t dq = 0, dkv = 0, dqkv = 0, Tmax = 0;
  float s = 1.f;
  Layout lay{};
  Group grp[NGROUP];

  uint8_t* arena = nullptr;     // pinned host, L blobs (streamed)
  uint8_t* resident = nullptr;  // device, L blobs (resident)
  uint8_t* pool[2] = {nullptr, nullptr};
  std::vector<char> registered;

  __nv_bfloat16 *E = nullptr, *H = nullptr;
  float* gf = nullptr;

  float* lora = nullptr;
  int64_t lora_numel = 0;
  std::vector<int64_t> offA, offB;
  struct Derived {                 // bf16 operands of the LoRA side path, per fused group
    __nv_bfloat16* Acat16 = nullptr;  // [KP, in], split rows (hi, hi, lo)
    __nv_bfloat16* Bexp16 = nullptr;  // [out, KP], split columns (hi, hi, lo)
  };
  std::vector<Derived> der;  // L * NGROUP
  float* grads = nullptr;

  float* xs = nullptr;  // residual stream: the input of every layer and the final output, fp32
  float* h = nullptr;   // residual after attention, fp32
  __nv_bfloat16 *n1 = nullptr, *qkv = nullptr, *o = nullptr, *n2 = nullptr, *gu = nullptr, *m = nullptr,
                *wscr[2] = {nullptr, nullptr};
  // NF4 base: the blob's header (means, norm gains, bias) of the layer each weight scratch holds,
  // copied by the dequant pass, so that a read's compute needs nothing from its pool slot
  uint8_t* whdr[2] = {nullptr, nullptr};
  int64_t hdr_bytes = 0;
  // this step's pool slots are released by the dequant that read them, not by the compute (NF4
  // base dequantised in a separate pass, reuse off): a copy waits for that dequant only
  bool release_at_deq = false;
  float *rstd1 = nullptr, *rstd2 = nullptr, *lse = nullptr, *Dbuf = nullptr;
  float* o32 = nullptr;  // attention output before rounding (recompute pass), for the backward's D
  LoraGradProb gq[NGROUP];  // adapter-gradient reductions queued by the layer's group backwards
  int n_gq = 0;
  __nv_bfloat16* Us[NGROUP] = {};  // split bf16 s * x A^T per group [T, KP] (sections hi, lo, hi)
  __nv_bfloat16* Vs[NGROUP] = {};  // split bf16 s * dy B per group [T, KP]
  float *ga = nullptr, *gb = nullptr, *dn = nullptr, *dm = nullptr;
  __nv_bfloat16 *dout_b = nullptr, *dh_b = nullptr, *do_b = nullptr, *dqkvb = nullptr, *dgu = nullptr;
  __nv_bfloat16* nf = nullptr;
  float *rstdf = nullptr, *logits = nullptr, *loss_rows = nullptr, *loss_dev = nullptr, *dot_part = nullptr;
  __nv_bfloat16* dlog = nullptr;
  int64_t head_rows = 0;      // token rows per head pass (logits / dlogits buffers hold this many)
  // preference (DPO) step
  bool adapters_off = false;  // the layer GEMMs skip the LoRA term (reference pass)
  float* lse_rows = nullptr;  // [T] row logsumexp of the logits
  float *seq_pi = nullptr, *seq_ref = nullptr, *w_seq = nullptr;  // [max_batch] per sequence
  int32_t* mask_dev = nullptr;  // [T] positions that count (DPO)
  bool have_mask = false;
  float dpo_beta = 0.f;
  bool logits_whole = false;  // the last step's logits are all in `logits`
  __nv_bfloat16* gbuf = nullptr;
  int32_t *tok = nullptr, *tgt = nullptr;
  float *cos_t = nullptr, *sin_t = nullptr;
  float* host_loss = nullptr;

  std::vector<cudaEvent_t> ev_chunk, ev_free;  // ev_chunk[n * NCHUNK + g]: chunk g of read n copied
  // the step's layer reads in order: layer index and kind (reference forward, forward, backward)
  std::vector<int> rd_layer, rd_kind;
  // pool slot use per read (see plan_reads)
  std::vector<ReadPlan> plan;
  int plan_held[2] = {-1, -1};   // layers the slots hold once the planned step has run
  int slot_layer[2] = {-1, -1};  // layers the slots hold after the last completed step (-1: unknown)
  int plan_wheld[2] = {-1, -1};  // layers the weight scratches hold once the planned step has run
  int w_layer[2] = {-1, -1};     // layers the weight scratches hold after the last completed step
  // prefetch of the next step's first read (reuse off): on between steps unless switched off
  bool prefetch_on = true;
  int pre_slot = -1, pre_layer = -1;  // slot holding the next step's first read, copied by the last step
  int64_t pre_bytes = 0;              // bytes that copy moved over this rank's link
  int plan_pre[2] = {-1, -1};         // this step's prefetch: slot, read whose compute it waits for
  bool pre_issued = false;            // the prefetch is enqueued; the step ends when ev_pre has fired
  cudaEvent_t ev_pre = nullptr;
  std::vector<cudaEvent_t> ev_deqg;  // [n * NCHUNK + g]: chunk g of read n dequantised
  // what the compute stream still waits on for the current read, per chunk: its copy, its dequant
  cudaEvent_t cur_wait[NCHUNK][2] = {};
  cudaEvent_t ev_done = nullptr, ev_start = nullptr;

  float* stage_w = nullptr;
  uint8_t* stage_blob = nullptr;
  float* stage_absmax = nullptr;
  double* stage_gsum = nullptr;

  std::vector<void*> dev_allocs;
  int64_t dev_bytes = 0;
  int64_t curT = 0, curB = 0, curS = 0;
  bool have_logits = false;

  lst_stats st{};
  // AdamW on the adapters (off until lst_set_optimizer)
  bool opt_on = false;
  lst_adamw opt{};
  int64_t opt_t = 0;
  float *opt_m = nullptr, *opt_v = nullptr;
  AdamTensor* opt_tab = nullptr;  // device table of every adapter tensor and its bf16 mirror
  int opt_ntab = 0;
  int64_t opt_maxn = 0;
  // profiling
  bool profiling = false;
  struct ProfRec {
    cudaEvent_t a, b;
    int cls;
    double flops;
  };
  std::vector<cudaEvent_t> prof_pool;
  size_t prof_used = 0;
  std::vector<ProfRec> prof_recs;
  cudaEvent_t prof_step0 = nullptr, prof_step1 = nullptr;
  int64_t launches_at_step_start = 0;
  // per-read timeline of the last profiled step: events [read][TL_N] and the times they gave (ms
  // from the step's start; -1: the read had no copy / dequant of its own)
  enum { TL_COPY0 = 0, TL_COPY1, TL_DEQ0, TL_DEQ1, TL_COMP0, TL_COMP1, TL_N };
  std::vector<cudaEvent_t> tl_ev;
  std::vector<char> tl_set;
  std::vector<float> tl_ms;
  int tl_reads = 0;
};

namespace {

lst_status fail(lst_ctx* c, lst_status s, const std::string& m) {
  if (c) c->err = m;
  return s;
}
lst_status cuda_fail(lst_ctx* c, cudaError_t e, const char* where) {
  cudaGetLastError();
  return fail(c, e == cudaErrorMemoryAllocation ? LST_ERR_OOM : LST_ERR_CUDA,
              std::string(where) + ": " + cudaGetErrorString(e));
}

#define CK(call)                                           \
  do {                                                     \
    cudaError_t e__ = (call);                              \
    if (e__ != cudaSuccess) return cuda_fail(c, e__, #call); \
  } while (0)

template <class T>
lst_status dalloc(lst_ctx* c, T** p, int64_t n, bool zero = false) {
  *p = nullptr;
  if (n <= 0) n = 1;
  if (c->faults.fail_device()) return fail(c, LST_ERR_OOM, "device allocation failed (injected)");
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, (size_t)n * sizeof(T));
  if (e != cudaSuccess) return cuda_fail(c, e, "cudaMalloc");
  c->dev_allocs.push_back(q);
  c->dev_bytes += n * (int64_t)sizeof(T);
  if (zero) {
    e = cudaMemset(q, 0, (size_t)n * sizeof(T));
    if (e != cudaSuccess) return cuda_fail(c, e, "cudaMemset");
  }
  *p = static_cast<T*>(q);
  return LST_OK;
}

lst_status add_guard(lst_ctx* c, uint8_t* p) {
  CK(cudaMemset(p, kGuardByte, kGuardBytes));
  c->guards.push_back(p);
  return LST_OK;
}

lst_status check_guards(lst_ctx* c) {
  std::vector<uint8_t> h(kGuardBytes);
  for (size_t i = 0; i < c->guards.size(); ++i) {
    CK(cudaMemcpy(h.data(), c->guards[i], kGuardBytes, cudaMemcpyDeviceToHost));
    for (int64_t k = 0; k < kGuardBytes; ++k)
      if (h[k] != kGuardByte)
        return fail(c, LST_ERR_DEVICE, "guard bytes after device buffer " + std::to_string(i) + " were overwritten");
  }
  return LST_OK;
}


#define TRY(x)                        \
  do {                                \
    lst_status s__ = (x);             \
    if (s__ != LST_OK) return s__;    \
  } while (0)

// ------------------------------------------------------------------------- profiling helpers
cudaEvent_t prof_event(lst_ctx* c) {
  if (c->prof_used == c->prof_pool.size()) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    c->prof_pool.push_back(e);
  }
  return c->prof_pool[c->prof_used++];
}
struct ProfScope {
  lst_ctx* c;
  cudaStream_t s;
  int cls;
  double flops;
  cudaEvent_t a = nullptr;
  // the many small kernels of class "other" are not bracketed, to keep the event count low
  ProfScope(lst_ctx* c_, cudaStream_t s_, int cls_, double flops_ = 0) : c(c_), s(s_), cls(cls_), flops(flops_) {
    if (c->profiling && cls != PC_OTHER) {
      a = prof_event(c);
      cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    if (c->profiling && cls != PC_OTHER) {
      cudaEvent_t b = prof_event(c);
      cudaEventRecord(b, s);
      c->prof_recs.push_back({a, b, cls, flops});
    }
  }
};

// Timeline event `which` of read n on stream st (profiling only).
lst_status tl_record(lst_ctx* c, int n, int which, cudaStream_t st) {
  if (!c->profiling) return LST_OK;
  const size_t i = (size_t)n * lst_ctx::TL_N + which;
  if (i >= c->tl_ev.size()) return LST_OK;
  CK(cudaEventRecord(c->tl_ev[i], st));
  c->tl_set[i] = 1;
  return LST_OK;
}

// ------------------------------------------------------------------------- LoRA operands
lst_status prep_lora(lst_ctx* c, int layer) {
  for (int g = 0; g < NGROUP; ++g) {
    const Group& G = c->grp[g];
    const auto& D = c->der[layer * NGROUP + g];
    LoraPrepArgs a{};
    for (int k = 0; k < G.nseg; ++k) {
      a.A[k] = c->lora + c->offA[layer * NPROJ + G.proj[k]];
      a.B[k] = c->lora + c->offB[layer * NPROJ + G.proj[k]];
    }
    a.nseg = G.nseg;
    a.r = c->r;
    a.in = G.in;
    for (int k = 0; k <= G.nseg; ++k) a.bounds[k] = G.bounds[k];
    a.RS = G.RS;
    a.KP = G.KP;
    a.Acat16 = D.Acat16;
    a.Bexp16 = D.Bexp16;
    CK(lora_prep(a, c->stream));
  }
  return LST_OK;
}

// True when group g's GEMMs dequantise the NF4 blob themselves in the current mode.
bool fused_group(const lst_ctx* c, int g) { return c->deq_mode == 1 && c->fuse_ok[g]; }

// The NF4 tensors of group g in a blob, stacked along the output rows as the GEMMs see them.
Nf4Mat group_nf4(const lst_ctx* c, const uint8_t* blob, int g) {
  static const int first[NCHUNK + 1] = {0, 3, 4, 6, 7};
  Nf4Mat q;
  q.nseg = first[g + 1] - first[g];
  q.cols = c->grp[g].in;
  int rows = 0;
  for (int k = 0; k < q.nseg; ++k) {
    const int p = first[g] + k;
    rows += (int)c->lay.outd[p];
    q.row_end[k] = rows;
    q.packed[k] = blob + c->lay.packed[p];
    q.qabs[k] = reinterpret_cast<const int8_t*>(blob + c->lay.qabs[p]);
    q.gscale[k] = reinterpret_cast<const float*>(blob + c->lay.gscale[p]);
    q.mean[k] = reinterpret_cast<const float*>(blob + c->lay.means) + p;
  }
  nf4_codebook(q.cb);
  return q;
}

// ------------------------------------------------------------------------- layer compute
const __nv_bfloat16* group_w(lst_ctx* c, const __nv_bfloat16* W, int g) { return W + c->grp[g].woff; }

lst_status group_fwd(lst_ctx* c, int layer, int g, const uint8_t* blob, const __nv_bfloat16* W, const __nv_bfloat16* X,
                     int64_t ldx, void* Y, int64_t ldy, int y_f32, const float* bias, const float* resid, bool gemm) {
  const Group& G = c->grp[g];
  const auto& D = c->der[layer * NGROUP + g];
  const int64_t T = c->curT;
  const bool lora = !c->adapters_off;
  if (lora) {
    ProfScope ps(c, c->stream, PC_LORA);  // Us = split(s * X Acat^T)
    CK(lora_skinny_split(X, ldx, T, G.in, D.Acat16, G.in, 0, G.R, G.RS, G.KP, c->s, c->Us[g], c->stream));
  }
  if (!gemm) return LST_OK;
  GemmArgs a;
  a.M = (int)T;
  a.N = G.out;
  a.K = G.in;
  a.A = X;
  a.lda = ldx;
  a.B = group_w(c, W, g);
  a.ldb = G.in;
  a.b_mn = 0;
  Nf4Mat q;
  if (fused_group(c, g)) {
    q = group_nf4(c, blob, g);
    a.Bq = &q;
  }
  if (lora) {
    a.A2 = c->Us[g];
    a.lda2 = G.KP;
    a.B2 = D.Bexp16;
    a.ldb2 = G.KP;
    a.K2 = G.KP;
  }
  a.C = Y;
  a.ldc = ldy;
  a.c_f32 = y_f32;
  a.bias = bias;
  a.R = resid;
  a.ldr = c->d;
  if (g == G_QKV) {  // rotary embedding of q and k applied in the epilogue (one bf16 rounding)
    a.rope_cos = c->cos_t;
    a.rope_sin = c->sin_t;
    a.rope_end = (int)(c->dq + c->dkv);
    a.rope_hd = c->hd;
    a.rope_S = (int)c->curS;
  }
  ProfScope ps(c, c->stream, PC_GEMM, 2.0 * T * G.out * (double)(G.in + (lora ? G.KP : 0)));
  CK(gemm_bf16(a, c->stream));
  return LST_OK;
}

lst_status group_bwd(lst_ctx* c, int layer, int g, const uint8_t* blob, const __nv_bfloat16* W, const __nv_bfloat16* dY,
                     int64_t ldy, const __nv_bfloat16* X, int64_t ldx, void* dX, int dx_f32) {
  const Group& G = c->grp[g];
  const auto& D = c->der[layer * NGROUP + g];
  const int64_t T = c->curT;
  {
    ProfScope ps(c, c->stream, PC_LORA);  // Vs = split(s * dY Bexp)
    CK(lora_skinny_split(dY, ldy, T, G.out, D.Bexp16, G.KP, 1, G.R, G.RS, G.KP, c->s, c->Vs[g], c->stream));
  }
  {
    GemmArgs a;
    a.M = (int)T;
    a.N = G.in;
    a.K = G.out;
    a.A = dY;
    a.lda = ldy;
    a.B = group_w(c, W, g);
    a.ldb = G.in;
    a.b_mn = 1;
    Nf4Mat q;
    if (fused_group(c, g)) {
      q = group_nf4(c, blob, g);
      a.Bq = &q;
    }
    a.A2 = c->Vs[g];
    a.lda2 = G.KP;
    a.B2 = D.Acat16;
    a.ldb2 = G.in;
    a.K2 = G.KP;
    a.C = dX;
    a.ldc = G.in;
    a.c_f32 = dx_f32;
    ProfScope ps(c, c->stream, PC_GEMM, 2.0 * T * G.in * (double)(G.out + G.KP));
    CK(gemm_bf16(a, c->stream));
  }
  // dA = s V^T X and dB = s dY^T U, with s folded into Vs and Us (their hi sections: the gradients are
  // fp32 reductions of bf16 products, so the lo parts would only refine the last bits of V and U);
  // queued here, launched for all four groups of the layer at once (flush_grads)
  if (c->n_gq >= NGROUP) return fail(c, LST_ERR_STATE, "adapter-gradient queue full");
  LoraGradProb& q = c->gq[c->n_gq++];
  q = LoraGradProb{};
  q.X = X;
  q.ldx = ldx;
  q.in = G.in;
  q.dY = dY;
  q.ldy = ldy;
  q.out = G.out;
  q.Us = c->Us[g];
  q.Vs = c->Vs[g];
  q.KP = G.KP;
  q.nseg = G.nseg;
  q.r = c->r;
  for (int k = 0; k <= G.nseg; ++k) q.bounds[k] = G.bounds[k];
  for (int k = 0; k < G.nseg; ++k) {
    q.dA[k] = c->grads + c->offA[layer * NPROJ + G.proj[k]];
    q.dB[k] = c->grads + c->offB[layer * NPROJ + G.proj[k]];
  }
  return LST_OK;
}

// The queued adapter-gradient reductions of the layer's groups in one launch. Their inputs (each
// group's X, dY, Us and Vs) are all still in place: the layer's backward writes none of them after
// they are made, and the launch comes before the last RMSNorm backward overwrites dL/dx_{i+1}.
lst_status flush_grads(lst_ctx* c) {
  if (c->n_gq == 0) return LST_OK;
  ProfScope ps(c, c->stream, PC_LORA);
  const int n = c->n_gq;
  c->n_gq = 0;
  CK(lora_grads_multi(c->gq, n, c->curT, c->stream));
  return LST_OK;
}

// Weights of a layer read: the bf16 [P] matrix the GEMMs consume.
// NF4 blob -> bf16 weights of the projections of chunk g (q/k/v, o, gate/up or down), written to
// dst in the concatenated [q;k;v], o, [gate;up], down order, on stream st.
lst_status dequant_chunk(lst_ctx* c, const uint8_t* blob, __nv_bfloat16* dst, int g, cudaStream_t st) {
  static const int first[NCHUNK + 1] = {0, 3, 4, 6, 7};
  Nf4Seg segs[NPROJ];
  int k = 0;
  for (int p = first[g]; p < first[g + 1]; ++p, ++k) {
    segs[k].packed = blob + c->lay.packed[p];
    segs[k].qabs = reinterpret_cast<const int8_t*>(blob + c->lay.qabs[p]);
    segs[k].gscale = reinterpret_cast<const float*>(blob + c->lay.gscale[p]);
    segs[k].mean = reinterpret_cast<const float*>(blob + c->lay.means) + p;
    segs[k].n = c->lay.n[p];
    segs[k].out_offset = c->lay.woff[p];
  }
  ProfScope ps(c, st, PC_DEQ);
  CK(nf4_dequant(segs, k, dst, st));
  return LST_OK;
}

// Make the compute stream wait until chunk g of the current read (its bytes and, for an NF4 base,
// its dequantised weights) is in place; a no-op once waited or when nothing is pending.
lst_status wait_chunk(lst_ctx* c, int g) {
  for (int k = 0; k < 2; ++k) {
    if (c->cur_wait[g][k]) {
      CK(cudaStreamWaitEvent(c->stream, c->cur_wait[g][k], 0));
      c->cur_wait[g][k] = nullptr;
    }
  }
  return LST_OK;
}

// blob: the layer's pool slot (or resident copy); hdr: where its header (norm gains, bias) is read
// from -- the blob itself, or the copy the dequant pass made next to the weight scratch.
lst_status layer_fwd(lst_ctx* c, int i, const uint8_t* blob, const uint8_t* hdr, const __nv_bfloat16* W,
                     bool recompute) {
  const int64_t T = c->curT;
  const int S = (int)c->curS;
  const float* g1 = reinterpret_cast<const float*>(hdr + c->lay.norms);
  const float* g2 = g1 + c->d;
  const float* bias = c->cfg.qkv_bias ? reinterpret_cast<const float*>(hdr + c->lay.bias) : nullptr;
  const float* x = c->xs + (int64_t)i * c->Tmax * c->d;
  TRY(wait_chunk(c, 0));  // norm gains, bias and the q/k/v weights
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_fwd(x, g1, T, c->d, c->cfg.rms_eps, c->n1, c->rstd1, c->stream));
  }
  TRY(group_fwd(c, i, G_QKV, blob, W, c->n1, c->d, c->qkv, c->dqkv, 0, bias, nullptr, true));
  {
    AttnArgs a;
    a.q = c->qkv;
    a.k = c->qkv + c->dq;
    a.v = c->qkv + c->dq + c->dkv;
    a.o = c->o;
    a.lse = c->lse;
    a.o32 = recompute ? c->o32 : nullptr;  // only the backward of a recomputed layer reads it
    a.ldq = a.ldk = a.ldv = c->dqkv;
    a.ldo = c->dq;
    a.T = T;
    a.S = S;
    a.hq = c->hq;
    a.hkv = c->hkv;
    a.hd = c->hd;
    a.scale = 1.0f / std::sqrt((float)c->hd);
    ProfScope ps(c, c->stream, PC_ATTN);
    CK(attention_fwd(a, c->stream));
  }
  TRY(wait_chunk(c, 1));
  TRY(group_fwd(c, i, G_O, blob, W, c->o, c->dq, c->h, c->d, 1, nullptr, x, true));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_fwd(c->h, g2, T, c->d, c->cfg.rms_eps, c->n2, c->rstd2, c->stream));
  }
  TRY(wait_chunk(c, 2));
  TRY(group_fwd(c, i, G_GU, blob, W, c->n2, c->d, c->gu, 2 * c->F, 0, nullptr, nullptr, true));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(swiglu_fwd(c->gu, T, c->F, c->m, c->stream));
  }
  TRY(wait_chunk(c, 3));  // also before a recompute: the backward that follows needs W_down
  // the recompute pass needs only the LoRA projection of m (for dB of down), not the output
  TRY(group_fwd(c, i, G_DOWN, blob, W, c->m, c->F, c->xs + (int64_t)(i + 1) * c->Tmax * c->d, c->d, 1, nullptr,
                c->h, !recompute));
  return LST_OK;
}

// dL/dx_{i+1} is in c->ga (fp32) and c->dout_b (bf16); leaves dL/dx_i there.
lst_status layer_bwd(lst_ctx* c, int i, const uint8_t* blob, const uint8_t* hdr, const __nv_bfloat16* W) {
  const int64_t T = c->curT;
  const int S = (int)c->curS;
  const float* g1 = reinterpret_cast<const float*>(hdr + c->lay.norms);
  const float* g2 = g1 + c->d;
  const float* x = c->xs + (int64_t)i * c->Tmax * c->d;
  c->n_gq = 0;
  TRY(group_bwd(c, i, G_DOWN, blob, W, c->dout_b, c->d, c->m, c->F, c->dm, 1));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(swiglu_bwd(c->dm, c->gu, T, c->F, c->dgu, c->stream));
  }
  TRY(group_bwd(c, i, G_GU, blob, W, c->dgu, 2 * c->F, c->n2, c->d, c->dn, 1));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_bwd(c->dn, c->h, g2, c->rstd2, c->ga, T, c->d, c->gb, c->dh_b, c->stream));
  }
  TRY(group_bwd(c, i, G_O, blob, W, c->dh_b, c->d, c->o, c->dq, c->do_b, 0));
  {
    AttnBwdArgs a;
    a.q = c->qkv;
    a.k = c->qkv + c->dq;
    a.v = c->qkv + c->dq + c->dkv;
    a.o = c->o;
    a.dout = c->do_b;
    a.lse = c->lse;
    a.o32 = c->o32;
    a.D = c->Dbuf;
    a.dq = c->dqkvb;
    a.dk = c->dqkvb + c->dq;
    a.dv = c->dqkvb + c->dq + c->dkv;
    a.ldq = a.ldk = a.ldv = c->dqkv;
    a.ldo = c->dq;
    a.lddo = c->dq;
    a.lddq = a.lddk = a.lddv = c->dqkv;
    a.T = T;
    a.S = S;
    a.hq = c->hq;
    a.hkv = c->hkv;
    a.hd = c->hd;
    a.scale = 1.0f / std::sqrt((float)c->hd);
    a.rope_cos = c->cos_t;  // dq and dk leave the kernel with the rotary embedding undone
    a.rope_sin = c->sin_t;
    ProfScope ps(c, c->stream, PC_ATTN);
    CK(attention_bwd(a, c->stream));
  }
  TRY(group_bwd(c, i, G_QKV, blob, W, c->dqkvb, c->dqkv, c->n1, c->d, c->dn, 1));
  TRY(flush_grads(c));  // before dout_b (the down group's dY) is overwritten below
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_bwd(c->dn, x, g1, c->rstd1, c->gb, T, c->d, c->ga, c->dout_b, c->stream));
  }
  return LST_OK;
}

// Final RMSNorm, LM head, cross-entropy and the head's backward, in passes of at most head_rows
// token rows: logits [rows, V] fp32 and dlogits [rows, V] bf16 exist for one pass at a time. Every
// row is independent, so the result does not depend on the pass size.
lst_status head_fwd_bwd(lst_ctx* c) {
  const int64_t T = c->curT;
  const float* xL = c->xs + (int64_t)c->L * c->Tmax * c->d;
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_fwd(xL, c->gf, T, c->d, c->cfg.rms_eps, c->nf, c->rstdf, c->stream));
  }
  for (int64_t r0 = 0; r0 < T; r0 += c->head_rows) {
    const int64_t rows = std::min<int64_t>(c->head_rows, T - r0);
    {
      GemmArgs a;
      a.M = (int)rows;
      a.N = c->V;
      a.K = c->d;
      a.A = c->nf + r0 * c->d;
      a.lda = c->d;
      a.B = c->H;
      a.ldb = c->d;
      a.b_mn = 0;
      a.C = c->logits;
      a.ldc = c->V;
      a.c_f32 = 1;
      ProfScope ps(c, c->stream, PC_GEMM, 2.0 * rows * c->V * (double)c->d);
      CK(gemm_bf16(a, c->stream));
    }
    {
      ProfScope ps(c, c->stream, PC_OTHER);
      CK(cross_entropy(c->logits, rows, c->V, c->tgt + r0, 1.0f / (float)T, c->loss_rows + r0, c->dlog, c->stream));
    }
    {
      GemmArgs a;
      a.M = (int)rows;
      a.N = c->d;
      a.K = c->V;
      a.A = c->dlog;
      a.lda = c->V;
      a.B = c->H;
      a.ldb = c->d;
      a.b_mn = 1;
      a.C = c->dn + r0 * c->d;
      a.ldc = c->d;
      a.c_f32 = 1;
      ProfScope ps(c, c->stream, PC_GEMM, 2.0 * rows * c->V * (double)c->d);
      CK(gemm_bf16(a, c->stream));
    }
  }
  ProfScope ps(c, c->stream, PC_OTHER);
  CK(mean_fixed(c->loss_rows, T, c->loss_dev, c->stream));
  CK(rmsnorm_bwd(c->dn, xL, c->gf, c->rstdf, nullptr, T, c->d, c->ga, c->dout_b, c->stream));
  c->logits_whole = T <= c->head_rows;
  return LST_OK;
}

// logits of token rows [r0, r0 + rows) into c->logits
lst_status head_logits(lst_ctx* c, int64_t r0, int64_t rows) {
  GemmArgs a;
  a.M = (int)rows;
  a.N = c->V;
  a.K = c->d;
  a.A = c->nf + r0 * c->d;
  a.lda = c->d;
  a.B = c->H;
  a.ldb = c->d;
  a.b_mn = 0;
  a.C = c->logits;
  a.ldc = c->V;
  a.c_f32 = 1;
  ProfScope ps(c, c->stream, PC_GEMM, 2.0 * rows * c->V * (double)c->d);
  CK(gemm_bf16(a, c->stream));
  return LST_OK;
}

// Final norm, logits and per-sequence log-likelihood of the targets (masked positions) into out;
// leaves lse_rows and, when one pass covers every row, the logits.
lst_status head_seq_logp(lst_ctx* c, float* out) {
  const int64_t T = c->curT;
  const float* xL = c->xs + (int64_t)c->L * c->Tmax * c->d;
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(rmsnorm_fwd(xL, c->gf, T, c->d, c->cfg.rms_eps, c->nf, c->rstdf, c->stream));
  }
  for (int64_t r0 = 0; r0 < T; r0 += c->head_rows) {
    const int64_t rows = std::min<int64_t>(c->head_rows, T - r0);
    TRY(head_logits(c, r0, rows));
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(ce_stats(c->logits, rows, c->V, c->tgt + r0, c->lse_rows + r0, c->loss_rows + r0, c->stream));
  }
  ProfScope ps(c, c->stream, PC_OTHER);
  CK(seq_sum(c->loss_rows, c->have_mask ? c->mask_dev : nullptr, (int)c->curB, (int)c->curS, out, c->stream));
  return LST_OK;
}

// Reference model of the DPO step: the adapters-off pass just ran; keep its sequence log-likelihoods.
lst_status head_ref(lst_ctx* c) { return head_seq_logp(c, c->seq_ref); }

// Policy head of the DPO step: sequence log-likelihoods, the DPO loss and per-sequence weights,
// then dlogits = w (softmax - onehot) on masked rows and the head's backward (logits recomputed
// per pass when the head runs in more than one pass).
lst_status head_dpo(lst_ctx* c) {
  const int64_t T = c->curT;
  const float* xL = c->xs + (int64_t)c->L * c->Tmax * c->d;
  TRY(head_seq_logp(c, c->seq_pi));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(dpo_loss(c->seq_pi, c->seq_ref, (int)(c->curB / 2), c->dpo_beta, c->loss_dev, c->w_seq, c->stream));
  }
  const bool one_pass = T <= c->head_rows;
  for (int64_t r0 = 0; r0 < T; r0 += c->head_rows) {
    const int64_t rows = std::min<int64_t>(c->head_rows, T - r0);
    if (!one_pass) TRY(head_logits(c, r0, rows));
    {
      ProfScope ps(c, c->stream, PC_OTHER);
      CK(ce_grad(c->logits, rows, r0, c->V, c->tgt, c->lse_rows, c->w_seq, c->have_mask ? c->mask_dev : nullptr,
                 (int)c->curS, c->dlog, c->stream));
    }
    GemmArgs a;
    a.M = (int)rows;
    a.N = c->d;
    a.K = c->V;
    a.A = c->dlog;
    a.lda = c->V;
    a.B = c->H;
    a.ldb = c->d;
    a.b_mn = 1;
    a.C = c->dn + r0 * c->d;
    a.ldc = c->d;
    a.c_f32 = 1;
    ProfScope ps(c, c->stream, PC_GEMM, 2.0 * rows * c->V * (double)c->d);
    CK(gemm_bf16(a, c->stream));
  }
  ProfScope ps(c, c->stream, PC_OTHER);
  CK(rmsnorm_bwd(c->dn, xL, c->gf, c->rstdf, nullptr, T, c->d, c->ga, c->dout_b, c->stream));
  return LST_OK;
}

// An SFT step reads layers 0 .. L-1 (forward), then L-1 .. 0 (backward with recompute); a DPO step
// first reads 0 .. L-1 once more for the reference forward (adapters off): 2L or 3L reads.
// plan_reads decides, for each read, the pool slot it computes from and whether the layer is
// copied into that slot first:
//  - reuse off: every read copies, into slot n % 2 (2L copies per step);
//  - reuse on: a read whose layer is still held by a slot (the two layers at the forward/backward
//    turn; layers 0 and 1 left by the previous step's backward) uses it as it is; otherwise it copies
//    into the slot the previous read does not use (for read 0, the slot whose layer is needed last).
// A copy into a slot waits until the last read that used that slot no longer needs it: until its
// compute has finished, or -- in a step whose NF4 base is dequantised in a separate pass, with reuse
// off -- until its dequant has (that pass also copies the blob's header, the norm gains and bias,
// next to the bf16 scratch, so the compute reads nothing from the slot). The copies can then run
// up to four reads ahead of the compute: two in the slots, two in the scratches.
// An NF4 base is dequantised into one of two bf16 weight scratches by the same rule (a read reuses
// a scratch that still holds its layer only with reuse on), on the prep stream, one read ahead: the
// dequant of read n+1 overlaps the compute of read n.
// With reuse off a step can also copy the next step's first read ahead (pre != null): into the slot
// the step's last read does not use, once the last read that computed from that slot has finished,
// so the copy overlaps the step's last read and the optimizer; the step ends when it has landed.
// The next step then computes its first read from that slot without copying it (its copy was that
// prefetch): 2L copies per step all the same, one of them issued by the step before.
// The planning itself, on host data only: layers[n] is the layer of read n; held / wheld are the
// layers the two slots / weight scratches hold before the step (-1: nothing known) and are updated
// to what they hold after it. pre[0] is the slot a previous step prefetched this step's first read
// into (-1: none); on return pre[0] / pre[1] are the slot this step prefetches the next step's first
// read into and the read whose compute that copy waits for (-1 / -1 with reuse on).
void plan_schedule(const std::vector<int>& layers, bool reuse, bool nf4, int held[2], int wheld[2],
                   std::vector<ReadPlan>& plan, int* pre = nullptr) {
  const int R = (int)layers.size();
  const int pre_in = pre && !reuse && pre[0] >= 0 && pre[0] < 2 ? pre[0] : -1;
  if (!reuse) {
    held[0] = held[1] = wheld[0] = wheld[1] = -1;
    if (pre_in >= 0) held[pre_in] = layers[0];
  }
  int last_use[2] = {-1, -1}, loaded_by[2] = {-1, -1};
  int wlast[2] = {-1, -1}, wfill[2] = {-1, -1};
  auto first_need = [&](int layer) {
    for (int m = 0; m < R; ++m)
      if (layers[m] == layer) return m;
    return R;
  };
  plan.assign(R, ReadPlan{});
  for (int n = 0; n < R; ++n) {
    const int j = layers[n];
    ReadPlan& p = plan[n];
    p.slot = -1;
    if (reuse) {
      if (held[0] == j) p.slot = 0;
      else if (held[1] == j) p.slot = 1;
    } else if (n == 0 && pre_in >= 0) {
      p.slot = pre_in;  // copied by the previous step's prefetch
    }
    p.copy = p.slot < 0;
    if (p.copy) {
      if (n > 0) {
        p.slot = 1 - plan[n - 1].slot;
      } else {
        p.slot = first_need(held[1]) > first_need(held[0]) ? 1 : 0;
      }
      p.wait_free = last_use[p.slot];
      held[p.slot] = j;
      loaded_by[p.slot] = n;
    }
    p.loaded_by = loaded_by[p.slot];
    last_use[p.slot] = n;

    p.deq = false;
    if (!nf4) continue;
    p.wslot = -1;
    if (reuse) {
      if (wheld[0] == j) p.wslot = 0;
      else if (wheld[1] == j) p.wslot = 1;
    }
    if (p.wslot < 0) {
      p.deq = true;
      p.wslot = n > 0 ? 1 - plan[n - 1].wslot : (first_need(wheld[1]) > first_need(wheld[0]) ? 1 : 0);
      p.wwait = wlast[p.wslot];
      wheld[p.wslot] = j;
      wfill[p.wslot] = n;
    }
    p.wfilled_by = wfill[p.wslot];
    wlast[p.wslot] = n;
  }
  if (pre) {
    pre[0] = pre[1] = -1;
    if (!reuse) {
      const int s = 1 - plan[R - 1].slot;
      pre[0] = s;
      pre[1] = last_use[s];
      held[s] = layers[0];
    }
  }
}

void plan_reads(lst_ctx* c) {
  const bool reuse = c->cfg.reuse != 0;
  int held[2] = {c->slot_layer[0], c->slot_layer[1]};
  int wheld[2] = {c->w_layer[0], c->w_layer[1]};
  const bool pre = c->cfg.streamed && c->prefetch_on;
  c->plan_pre[0] = pre && c->pre_layer == c->rd_layer[0] ? c->pre_slot : -1;
  c->plan_pre[1] = -1;
  plan_schedule(c->rd_layer, reuse, c->cfg.base_format != LST_BASE_BF16, held, wheld, c->plan,
                pre ? c->plan_pre : nullptr);
  c->plan_held[0] = held[0];
  c->plan_held[1] = held[1];
  c->plan_wheld[0] = wheld[0];
  c->plan_wheld[1] = wheld[1];
}

// LST_COPY_WHOLE=1 copies each blob with one cudaMemcpyAsync instead of one per weight group (for
// measuring what the group copies cost; the compute of a read then starts only once all of it landed).
bool whole_blob_copies() {
  static const bool v = [] {
    const char* e = std::getenv("LST_COPY_WHOLE");
    return e && std::strcmp(e, "1") == 0;
  }();
  return v;
}

// Copy layer j's blob from the pinned arena into pool slot `slot` on the copy stream. chunk_ev
// (NCHUNK events, or null) is recorded after each weight group has landed; *bytes is what crossed
// this rank's link.
lst_status copy_layer(lst_ctx* c, int slot, int j, cudaEvent_t* chunk_ev, int64_t* bytes_out) {
  if (c->faults.fail_memcpy()) return fail(c, LST_ERR_CUDA, "layer copy enqueue failed (injected)");
  const uint8_t* src = c->arena + (int64_t)j * c->lay.total;
  if (c->nccl_comm) {
    // this rank's slice over its own link, then the whole blob from every rank's slice over
    // NVLink (in-place all-gather into the pool slot); the blob is complete for every chunk at once
    int64_t off = 0, bytes = 0, count = 0;
    split_plan(c->lay.total, c->split_world, c->split_rank, &off, &bytes, &count);
    if (bytes > 0)
      CK(cudaMemcpyAsync(c->pool[slot] + off, src + off, bytes, cudaMemcpyHostToDevice, c->copy_stream));
    const int r = nccl().all_gather(c->pool[slot] + off, c->pool[slot], (size_t)count, kNcclUint8, c->nccl_comm,
                                    c->copy_stream);
    if (r != 0) return fail(c, LST_ERR_CUDA, std::string("ncclAllGather: ") + nccl().error_string(r));
    if (chunk_ev)
      for (int g = 0; g < NCHUNK; ++g) CK(cudaEventRecord(chunk_ev[g], c->copy_stream));
    *bytes_out = bytes;
    return LST_OK;
  }
  if (whole_blob_copies()) {  // one copy per read; every group's event after it
    CK(cudaMemcpyAsync(c->pool[slot], src, c->lay.total, cudaMemcpyHostToDevice, c->copy_stream));
    if (chunk_ev)
      for (int g = 0; g < NCHUNK; ++g) CK(cudaEventRecord(chunk_ev[g], c->copy_stream));
    *bytes_out = c->lay.total;
    return LST_OK;
  }
  for (int g = 0; g < NCHUNK; ++g) {  // group by group, so compute can start on the first group
    CK(cudaMemcpyAsync(c->pool[slot] + c->lay.chunk[g], src + c->lay.chunk[g], c->lay.chunk[g + 1] - c->lay.chunk[g],
                       cudaMemcpyHostToDevice, c->copy_stream));
    if (chunk_ev) CK(cudaEventRecord(chunk_ev[g], c->copy_stream));
  }
  *bytes_out = c->lay.total;
  return LST_OK;
}

// The event after which read n no longer needs its pool slot: its dequant when the slots are
// released there, else the end of its compute.
cudaEvent_t slot_release(lst_ctx* c, int n) {
  return c->release_at_deq ? c->ev_deqg[(size_t)n * NCHUNK + NCHUNK - 1] : c->ev_free[n];
}

lst_status enqueue_copy(lst_ctx* c, int n) {
  const int j = c->rd_layer[n];
  NvtxRange nr("copy read %d (layer %d)", n, j);
  const ReadPlan& p = c->plan[n];
  if (p.wait_free >= 0) CK(cudaStreamWaitEvent(c->copy_stream, slot_release(c, p.wait_free), 0));
  ProfScope ps(c, c->copy_stream, PC_COPY);
  TRY(tl_record(c, n, lst_ctx::TL_COPY0, c->copy_stream));
  int64_t bytes = 0;
  TRY(copy_layer(c, p.slot, j, &c->ev_chunk[(size_t)n * NCHUNK], &bytes));
  TRY(tl_record(c, n, lst_ctx::TL_COPY1, c->copy_stream));
  c->st.layer_reads_last_step += 1;
  c->st.h2d_bytes_last_step += bytes;
  return LST_OK;
}

// The next step's first read, copied ahead into the slot plan_pre names once the read that last
// computes from it has finished; counted as a read of the next step, which finds it in place.
lst_status enqueue_prefetch(lst_ctx* c) {
  const int slot = c->plan_pre[0], wait = c->plan_pre[1], j = c->rd_layer[0];
  NvtxRange nr("prefetch into slot %d (layer %d)", slot, j);
  if (wait >= 0) CK(cudaStreamWaitEvent(c->copy_stream, slot_release(c, wait), 0));
  ProfScope ps(c, c->copy_stream, PC_COPY);
  int64_t bytes = 0;
  TRY(copy_layer(c, slot, j, nullptr, &bytes));
  CK(cudaEventRecord(c->ev_pre, c->copy_stream));
  c->pre_issued = true;
  c->pre_bytes = bytes;
  return LST_OK;
}

// Enqueue, in read order, every planned copy whose slot is released by a read <= done.
lst_status issue_copies(lst_ctx* c, int done, int& next) {
  const int R = (int)c->rd_layer.size();
  while (next < R) {
    const ReadPlan& p = c->plan[next];
    if (p.copy) {
      if (p.wait_free > done) break;
      TRY(enqueue_copy(c, next));
    }
    ++next;
  }
  return LST_OK;
}

void build_reads(lst_ctx* c, HeadMode mode) {
  const int L = c->L;
  c->rd_layer.clear();
  c->rd_kind.clear();
  if (mode == HEAD_DPO) {
    for (int i = 0; i < L; ++i) {
      c->rd_layer.push_back(i);
      c->rd_kind.push_back(RD_REF);
    }
  }
  for (int i = 0; i < L; ++i) {
    c->rd_layer.push_back(i);
    c->rd_kind.push_back(RD_FWD);
  }
  for (int i = L - 1; i >= 0; --i) {
    c->rd_layer.push_back(i);
    c->rd_kind.push_back(RD_BWD);
  }
}

lst_status head_after(lst_ctx* c, int kind, HeadMode mode) {
  if (kind == RD_REF) return head_ref(c);
  if (mode == HEAD_DPO) return head_dpo(c);
  if (mode == HEAD_SFT) return head_fwd_bwd(c);
  const int64_t T = c->curT;
  const float* xL = c->xs + (int64_t)c->L * c->Tmax * c->d;
  ProfScope ps(c, c->stream, PC_OTHER);
  CK(dot_fixed(xL, c->gbuf, T * c->d, c->dot_part, c->loss_dev, c->stream));
  CK(cudaMemcpyAsync(c->dout_b, c->gbuf, T * c->d * 2, cudaMemcpyDeviceToDevice, c->stream));
  CK(bf16_to_f32(c->gbuf, T * c->d, c->ga, c->stream));
  return LST_OK;
}

lst_status run_layers(lst_ctx* c, HeadMode mode) {
  const int L = c->L;
  const bool streamed = c->cfg.streamed != 0;
  const bool nf4 = c->cfg.base_format != LST_BASE_BF16;
  build_reads(c, mode);
  const int R = (int)c->rd_layer.size();
  auto blob_of = [&](int n) -> const uint8_t* {
    return streamed ? c->pool[c->plan[n].slot] : c->resident + (int64_t)c->rd_layer[n] * c->lay.total;
  };
  plan_reads(c);
  c->release_at_deq = streamed && nf4 && !c->cfg.reuse && c->whdr[0] != nullptr;
  for (int g = 0; g < NCHUNK; ++g) c->release_at_deq = c->release_at_deq && !fused_group(c, g);
  // the slots' and scratches' contents are only trusted again once this step has completed
  c->slot_layer[0] = c->slot_layer[1] = -1;
  c->w_layer[0] = c->w_layer[1] = -1;
  if (streamed && !c->cfg.reuse && !c->plan[0].copy) {  // the last step copied this first read
    c->st.layer_reads_last_step += 1;
    c->st.h2d_bytes_last_step += c->pre_bytes;
  }
  c->pre_slot = c->pre_layer = -1;
  c->pre_issued = false;
  // copies and dequants of this step start after everything already on the compute stream (e.g. a
  // step that returned early with work in flight)
  CK(cudaEventRecord(c->ev_start, c->stream));
  CK(cudaStreamWaitEvent(c->copy_stream, c->ev_start, 0));
  CK(cudaStreamWaitEvent(c->prep_stream, c->ev_start, 0));
  CK(cudaStreamWaitEvent(c->d2h_stream, c->ev_start, 0));
  int next_copy = 0;
  if (streamed) TRY(issue_copies(c, -1, next_copy));
  // dequant of read m on the prep stream, chunk by chunk as the copy lands; every event it waits on
  // is already recorded
  auto enqueue_deq = [&](int m) -> lst_status {
    if (m >= R || !c->plan[m].deq) return LST_OK;
    const ReadPlan& p = c->plan[m];
    if (p.wwait >= 0) CK(cudaStreamWaitEvent(c->prep_stream, c->ev_free[p.wwait], 0));
    bool started = false;
    for (int g = 0; g < NCHUNK; ++g) {
      if (fused_group(c, g)) continue;  // dequantised inside the GEMMs
      if (streamed && p.loaded_by >= 0)
        CK(cudaStreamWaitEvent(c->prep_stream, c->ev_chunk[p.loaded_by * NCHUNK + g], 0));
      if (!started) TRY(tl_record(c, m, lst_ctx::TL_DEQ0, c->prep_stream));
      if (g == 0 && c->release_at_deq)  // the header lies in chunk 0
        CK(copy16(blob_of(m), c->whdr[p.wslot], c->hdr_bytes, c->prep_stream));
      started = true;
      TRY(dequant_chunk(c, blob_of(m), c->wscr[p.wslot], g, c->prep_stream));
      CK(cudaEventRecord(c->ev_deqg[m * NCHUNK + g], c->prep_stream));
    }
    if (started) TRY(tl_record(c, m, lst_ctx::TL_DEQ1, c->prep_stream));
    return LST_OK;
  };
  TRY(enqueue_deq(0));
  static const char* kRangeName[3] = {"reference forward read %d (layer %d)", "forward read %d (layer %d)",
                                       "backward read %d (layer %d)"};
  for (int n = 0; n < R; ++n) {
    const int j = c->rd_layer[n], kind = c->rd_kind[n];
    const ReadPlan& p = c->plan[n];
    NvtxRange nr(kRangeName[kind], n, j);
    TRY(enqueue_deq(n + 1));
    const uint8_t* blob = blob_of(n);
    // the compute of chunk g waits for the copy that filled the slot and, for an NF4 base, the
    // dequant that filled the weight scratch, when they belong to this step (the slot and the
    // scratch may have been filled by different reads when layers are reused)
    for (int g = 0; g < NCHUNK; ++g) {
      c->cur_wait[g][0] = streamed && p.loaded_by >= 0 ? c->ev_chunk[p.loaded_by * NCHUNK + g] : nullptr;
      c->cur_wait[g][1] =
          nf4 && p.wfilled_by >= 0 && !fused_group(c, g) ? c->ev_deqg[p.wfilled_by * NCHUNK + g] : nullptr;
    }
    const __nv_bfloat16* W =
        nf4 ? c->wscr[p.wslot] : reinterpret_cast<const __nv_bfloat16*>(blob + c->lay.w16);
    const uint8_t* hdr = c->release_at_deq ? c->whdr[p.wslot] : blob;
    if (c->profiling) {  // the read's compute starts once its first weight group is in place
      TRY(wait_chunk(c, 0));
      TRY(tl_record(c, n, lst_ctx::TL_COMP0, c->stream));
    }
    if (kind == RD_REF) {
      c->adapters_off = true;
      const lst_status st = layer_fwd(c, j, blob, hdr, W, false);
      c->adapters_off = false;
      TRY(st);
    } else if (kind == RD_FWD) {
      TRY(layer_fwd(c, j, blob, hdr, W, false));
    } else {
      TRY(layer_fwd(c, j, blob, hdr, W, true));
      TRY(layer_bwd(c, j, blob, hdr, W));
    }
    CK(cudaEventRecord(c->ev_free[n], c->stream));
    TRY(tl_record(c, n, lst_ctx::TL_COMP1, c->stream));
    if (kind == RD_BWD && c->grads_host) {
      // this layer's gradients are final: send them while the layers below compute
      const int64_t o0 = c->offA[j * NPROJ], o1 = j + 1 < L ? c->offA[(j + 1) * NPROJ] : c->lora_numel;
      CK(cudaStreamWaitEvent(c->d2h_stream, c->ev_free[n], 0));
      CK(cudaMemcpyAsync(c->grads_host + o0, c->grads + o0, (o1 - o0) * 4, cudaMemcpyDeviceToHost, c->d2h_stream));
    }
    if (kind != RD_BWD && (n + 1 == R || c->rd_kind[n + 1] != kind)) TRY(head_after(c, kind, mode));
    if (streamed) TRY(issue_copies(c, n, next_copy));
  }
  if (streamed && c->plan_pre[0] >= 0) TRY(enqueue_prefetch(c));
  return LST_OK;
}

lst_status finish_step(lst_ctx* c, float* loss, float* grads_out) {
  if (c->grads_host) {
    // sent layer by layer during the backward (run_layers); the step ends when they have arrived
    CK(cudaEventRecord(c->ev_d2h, c->d2h_stream));
    CK(cudaStreamWaitEvent(c->stream, c->ev_d2h, 0));
  } else if (grads_out) {
    const bool dev = is_device_ptr(grads_out);
    CK(cudaMemcpyAsync(grads_out, c->grads, c->lora_numel * 4, dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                       c->stream));
  }
  if (c->pre_issued) CK(cudaStreamWaitEvent(c->stream, c->ev_pre, 0));  // the next step's first read landed
  CK(cudaMemcpyAsync(c->host_loss, c->loss_dev, 4, cudaMemcpyDeviceToHost, c->stream));
  if (c->profiling) CK(cudaEventRecord(c->prof_step1, c->stream));
  CK(cudaEventRecord(c->ev_done, c->stream));
  const int tmo = c->cfg.timeout_ms > 0 ? c->cfg.timeout_ms : 600000;
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    cudaError_t q = cudaEventQuery(c->ev_done);
    if (q == cudaSuccess) break;
    if (q != cudaErrorNotReady) return cuda_fail(c, q, "step");
    if (c->faults.timeout ||
        std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count() > tmo)
      return fail(c, LST_ERR_TIMEOUT, "step did not finish within timeout_ms");
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
  if (c->faults.timeout) return fail(c, LST_ERR_TIMEOUT, "step did not finish within timeout_ms (injected)");
  int derr = 0;
  CK(cudaMemcpyFromSymbol(&derr, g_lst_dev_error, sizeof(int)));
  if (derr) {
    int zero = 0;
    cudaMemcpyToSymbol(g_lst_dev_error, &zero, sizeof(int));
    return fail(c, LST_ERR_DEVICE, "device code reported error " + std::to_string(derr));
  }
  *loss = *c->host_loss;
  if (c->check_guards) TRY(check_guards(c));
  if (c->cfg.streamed) {
    c->slot_layer[0] = c->plan_held[0];
    c->slot_layer[1] = c->plan_held[1];
    if (c->pre_issued) {
      c->pre_slot = c->plan_pre[0];
      c->pre_layer = c->rd_layer[0];
    }
  }
  c->w_layer[0] = c->plan_wheld[0];
  c->w_layer[1] = c->plan_wheld[1];
  c->st.steps += 1;
  c->st.launches_last_step = g_launch_count.load() - c->launches_at_step_start;
  if (c->profiling) {
    double ms[PC_N] = {};
    int64_t cnt[PC_N] = {};
    double flops = 0;
    for (auto& r : c->prof_recs) {
      float t = 0.f;
      cudaEventElapsedTime(&t, r.a, r.b);
      ms[r.cls] += t;
      cnt[r.cls] += 1;
      if (r.cls == PC_GEMM) flops += r.flops;
    }
    float step = 0.f;
    cudaEventElapsedTime(&step, c->prof_step0, c->prof_step1);
    c->st.gemm_ms = ms[PC_GEMM];
    c->st.attention_ms = ms[PC_ATTN];
    c->st.dequant_ms = ms[PC_DEQ];
    c->st.other_ms = ms[PC_OTHER];
    c->st.copy_ms = ms[PC_COPY];
    c->st.gemm_launches = cnt[PC_GEMM];
    c->st.attention_launches = cnt[PC_ATTN];
    c->st.dequant_launches = cnt[PC_DEQ];
    c->st.copy_count = cnt[PC_COPY];
    c->st.lora_ms = ms[PC_LORA];
    c->st.lora_launches = cnt[PC_LORA];
    c->st.gemm_flops = flops;
    c->st.step_ms = step;
    c->tl_reads = (int)c->rd_layer.size();
    c->tl_ms.assign((size_t)c->tl_reads * lst_ctx::TL_N, -1.f);
    for (size_t i = 0; i < c->tl_ms.size(); ++i) {
      float t = -1.f;
      if (c->tl_set[i] && cudaEventElapsedTime(&t, c->prof_step0, c->tl_ev[i]) == cudaSuccess) c->tl_ms[i] = t;
    }
    cudaGetLastError();
  }
  return LST_OK;
}

// Pinned host gradient buffers are filled layer by layer during the backward; any other
// destination gets one copy at the end of the step.
void set_grads_dest(lst_ctx* c, float* grads) { c->grads_host = grads && is_pinned_host_ptr(grads) ? grads : nullptr; }

lst_status begin_step(lst_ctx* c, int32_t batch, int32_t seq) {
  for (int i = 0; i < c->L; ++i)
    if (!c->registered[i]) return fail(c, LST_ERR_STATE, "layer " + std::to_string(i) + " is not registered");
  if (batch <= 0 || seq <= 0 || batch > c->cfg.max_batch || seq > c->cfg.max_seq)
    return fail(c, LST_ERR_ARG, "batch/seq outside (0, max]");
  c->curB = batch;
  c->curS = seq;
  c->curT = (int64_t)batch * seq;
  c->st.layer_reads_last_step = 0;
  c->st.h2d_bytes_last_step = 0;
  c->prof_used = 0;
  c->prof_recs.clear();
  if (c->profiling) {
    const size_t need = (size_t)3 * c->L * lst_ctx::TL_N;
    while (c->tl_ev.size() < need) {
      cudaEvent_t e;
      CK(cudaEventCreate(&e));
      c->tl_ev.push_back(e);
    }
    c->tl_set.assign(need, 0);
  }
  c->launches_at_step_start = g_launch_count.load();
  if (c->profiling) CK(cudaEventRecord(c->prof_step0, c->stream));
  return LST_OK;
}

lst_status copy_in(lst_ctx* c, void* dst, const void* src, int64_t bytes) {
  CK(cudaMemcpyAsync(dst, src, bytes, is_device_ptr(src) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                     c->stream));
  return LST_OK;
}

// fp32 host/device tensor -> bf16 device buffer
lst_status upload_bf16(lst_ctx* c, __nv_bfloat16* dst, const float* src, int64_t n) {
  if (is_device_ptr(src)) {
    CK(f32_to_bf16(src, n, dst, c->stream));
    return LST_OK;
  }
  const int64_t chunk = 1 << 24;
  float* tmp = nullptr;
  CK(cudaMalloc(&tmp, chunk * 4));
  for (int64_t i = 0; i < n; i += chunk) {
    const int64_t k = std::min(chunk, n - i);
    cudaError_t e = cudaMemcpyAsync(tmp, src + i, k * 4, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess) e = f32_to_bf16(tmp, k, dst + i, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    if (e != cudaSuccess) {
      cudaFree(tmp);
      return cuda_fail(c, e, "upload_bf16");
    }
  }
  cudaFree(tmp);
  return LST_OK;
}

lst_status create_impl(lst_ctx* c, const float* embed, const float* final_norm, const float* lm_head,
                       void* stream) {
  const lst_config& k = c->cfg;
  CK(cudaGetDevice(&c->dev));
  c->d = k.d_model;
  c->hq = k.n_heads;
  c->hkv = k.n_kv_heads;
  c->hd = k.head_dim;
  c->F = k.ffn;
  c->V = k.vocab;
  c->L = k.n_layers;
  c->r = k.lora_rank;
  c->s = k.lora_alpha / (float)k.lora_rank;
  c->dq = (int64_t)c->hq * c->hd;
  c->dkv = (int64_t)c->hkv * c->hd;
  c->dqkv = c->dq + 2 * c->dkv;
  c->Tmax = (int64_t)k.max_batch * k.max_seq;
  c->lay = make_layout(k);
  auto setg = [&](int g, int nseg, std::initializer_list<int> pr, int in, std::initializer_list<int> bnd) {
    Group& G = c->grp[g];
    G.nseg = nseg;
    int i = 0;
    for (int p : pr) G.proj[i++] = p;
    G.in = in;
    i = 0;
    for (int b : bnd) G.bounds[i++] = b;
    G.out = G.bounds[nseg];
    G.R = nseg * c->r;
    G.RS = (G.R + 7) / 8 * 8;
    G.KP = (3 * G.RS + 63) / 64 * 64;
    G.woff = c->lay.woff[G.proj[0]];
  };
  setg(G_QKV, 3, {0, 1, 2}, c->d, {0, (int)c->dq, (int)(c->dq + c->dkv), (int)c->dqkv});
  setg(G_O, 1, {3}, (int)c->dq, {0, c->d});
  setg(G_GU, 2, {4, 5}, c->d, {0, c->F, 2 * c->F});
  setg(G_DOWN, 1, {6}, c->F, {0, c->d});
  for (int g = 0; g < NGROUP; ++g) c->fuse_ok[g] = k.base_format == LST_BASE_NF4 && c->grp[g].in % 64 == 0;

  int prio_low = 0, prio_high = 0;
  CK(cudaDeviceGetStreamPriorityRange(&prio_low, &prio_high));
  if (stream) {
    c->stream = static_cast<cudaStream_t>(stream);
  } else {
    CK(cudaStreamCreateWithPriority(&c->stream, cudaStreamNonBlocking, prio_high));
    c->own_stream = true;
  }
  CK(cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking));
  // lowest priority: the next read's dequant takes the SM slots the compute stream leaves free
  CK(cudaStreamCreateWithPriority(&c->prep_stream, cudaStreamNonBlocking, prio_low));
  CK(cudaStreamCreateWithFlags(&c->d2h_stream, cudaStreamNonBlocking));

  // LoRA parameter / gradient layout
  c->offA.resize(c->L * NPROJ);
  c->offB.resize(c->L * NPROJ);
  int64_t off = 0;
  for (int l = 0; l < c->L; ++l)
    for (int p = 0; p < NPROJ; ++p) {
      c->offA[l * NPROJ + p] = off;
      off += (int64_t)c->r * c->lay.ind[p];
      c->offB[l * NPROJ + p] = off;
      off += c->lay.outd[p] * c->r;
    }
  c->lora_numel = off;
  TRY(dalloc(c, &c->lora, off, true));
  TRY(dalloc(c, &c->grads, off, true));
  c->der.resize(c->L * NGROUP);
  for (int l = 0; l < c->L; ++l)
    for (int g = 0; g < NGROUP; ++g) {
      auto& D = c->der[l * NGROUP + g];
      const Group& G = c->grp[g];
      TRY(dalloc(c, &D.Acat16, (int64_t)G.KP * G.in, true));
      TRY(dalloc(c, &D.Bexp16, (int64_t)G.out * G.KP, true));
    }
  {
    // table of every adapter tensor for the fused AdamW pass (and where its bf16 copy lives)
    std::vector<AdamTensor> tab;
    for (int l = 0; l < c->L; ++l)
      for (int g = 0; g < NGROUP; ++g) {
        const Group& G = c->grp[g];
        const auto& D = c->der[l * NGROUP + g];
        for (int k = 0; k < G.nseg; ++k) {
          const int p = G.proj[k];
          AdamTensor a{c->offA[l * NPROJ + p], (int64_t)c->r * G.in, c->r, G.in, D.Acat16, G.in, k * c->r, 0,
                       (int64_t)G.RS * G.in};
          const int outp = G.bounds[k + 1] - G.bounds[k];
          AdamTensor b{c->offB[l * NPROJ + p], (int64_t)outp * c->r, outp, c->r, D.Bexp16, G.KP, G.bounds[k],
                       k * c->r, (int64_t)G.RS};
          tab.push_back(a);
          tab.push_back(b);
          c->opt_maxn = std::max(c->opt_maxn, std::max(a.n, b.n));
        }
      }
    c->opt_ntab = (int)tab.size();
    TRY(dalloc(c, &c->opt_tab, (int64_t)tab.size()));
    CK(cudaMemcpy(c->opt_tab, tab.data(), tab.size() * sizeof(AdamTensor), cudaMemcpyHostToDevice));
  }

  // base storage
  const int64_t blob = c->lay.total;
  if (k.streamed) {
    if (c->faults.fail_pinned()) return fail(c, LST_ERR_OOM, "pinned host allocation failed (injected)");
    void* a = nullptr;
    cudaError_t e = cudaHostAlloc(&a, (size_t)blob * c->L, cudaHostAllocDefault);
    if (e != cudaSuccess) return cuda_fail(c, e, "cudaHostAlloc(arena)");
    c->arena = static_cast<uint8_t*>(a);
    TRY(dalloc(c, &c->pool[0], blob + kGuardBytes));
    TRY(dalloc(c, &c->pool[1], blob + kGuardBytes));
    TRY(add_guard(c, c->pool[0] + blob));
    TRY(add_guard(c, c->pool[1] + blob));
    c->pool_bytes = blob;
    c->st.arena_bytes = blob * c->L;
  } else {
    TRY(dalloc(c, &c->resident, blob * c->L));
    c->st.arena_bytes = blob * c->L;
  }
  c->st.blob_bytes = blob;
  c->registered.assign(c->L, 0);
  if (k.base_format == LST_BASE_NF4) {
    TRY(dalloc(c, &c->wscr[0], c->lay.P + kGuardBytes / 2));
    TRY(dalloc(c, &c->wscr[1], c->lay.P + kGuardBytes / 2));
    TRY(add_guard(c, reinterpret_cast<uint8_t*>(c->wscr[0] + c->lay.P)));
    TRY(add_guard(c, reinterpret_cast<uint8_t*>(c->wscr[1] + c->lay.P)));
    c->hdr_bytes = c->lay.packed[0];  // means, norm gains and bias come first
    if (k.streamed) {
      TRY(dalloc(c, &c->whdr[0], c->hdr_bytes));
      TRY(dalloc(c, &c->whdr[1], c->hdr_bytes));
    }
  }

  // activations
  const int64_t T = c->Tmax, d = c->d;
  TRY(dalloc(c, &c->xs, (int64_t)(c->L + 1) * T * d));
  TRY(dalloc(c, &c->n1, T * d));
  TRY(dalloc(c, &c->qkv, T * c->dqkv));
  TRY(dalloc(c, &c->o, T * c->dq));
  TRY(dalloc(c, &c->h, T * d));
  TRY(dalloc(c, &c->n2, T * d));
  TRY(dalloc(c, &c->gu, T * 2 * c->F));
  TRY(dalloc(c, &c->m, T * c->F));
  TRY(dalloc(c, &c->rstd1, T));
  TRY(dalloc(c, &c->rstd2, T));
  TRY(dalloc(c, &c->lse, T * c->hq));
  TRY(dalloc(c, &c->o32, T * c->dq));
  TRY(dalloc(c, &c->Dbuf, T * c->hq));
  for (int g = 0; g < NGROUP; ++g) {
    const Group& G = c->grp[g];
    TRY(dalloc(c, &c->Us[g], T * G.KP, true));
    TRY(dalloc(c, &c->Vs[g], T * G.KP, true));
  }
  TRY(dalloc(c, &c->ga, T * d));
  TRY(dalloc(c, &c->gb, T * d));
  TRY(dalloc(c, &c->dn, T * d));
  TRY(dalloc(c, &c->dm, T * c->F));
  TRY(dalloc(c, &c->dout_b, T * d));
  TRY(dalloc(c, &c->dh_b, T * d));
  TRY(dalloc(c, &c->do_b, T * c->dq));
  TRY(dalloc(c, &c->dqkvb, T * c->dqkv));
  TRY(dalloc(c, &c->dgu, T * 2 * c->F));
  TRY(dalloc(c, &c->loss_dev, 1, true));
  TRY(dalloc(c, &c->dot_part, 1024));
  TRY(dalloc(c, &c->cos_t, (int64_t)k.max_seq * c->hd / 2));
  TRY(dalloc(c, &c->sin_t, (int64_t)k.max_seq * c->hd / 2));
  CK(rope_tables(k.max_seq, c->hd, (double)k.rope_theta, c->cos_t, c->sin_t, c->stream));
  {
    void* hl = nullptr;
    CK(cudaHostAlloc(&hl, 64, cudaHostAllocDefault));
    c->host_loss = static_cast<float*>(hl);
  }
  if (c->V > 0) {
    const int64_t Vd = (int64_t)c->V * d;
    TRY(dalloc(c, &c->E, Vd));
    TRY(dalloc(c, &c->H, Vd));
    TRY(dalloc(c, &c->gf, d));
    TRY(upload_bf16(c, c->E, embed, Vd));
    TRY(upload_bf16(c, c->H, lm_head, Vd));
    TRY(copy_in(c, c->gf, final_norm, d * 4));
    TRY(dalloc(c, &c->nf, T * d));
    TRY(dalloc(c, &c->rstdf, T));
    c->head_rows = k.head_chunk > 0 ? std::min<int64_t>(k.head_chunk, T) : T;
    TRY(dalloc(c, &c->logits, c->head_rows * c->V));
    TRY(dalloc(c, &c->dlog, c->head_rows * c->V));
    TRY(dalloc(c, &c->loss_rows, T));
    TRY(dalloc(c, &c->lse_rows, T));
    TRY(dalloc(c, &c->mask_dev, T));
    TRY(dalloc(c, &c->seq_pi, k.max_batch));
    TRY(dalloc(c, &c->seq_ref, k.max_batch));
    TRY(dalloc(c, &c->w_seq, k.max_batch));
    TRY(dalloc(c, &c->tok, T));
    TRY(dalloc(c, &c->tgt, T));
  } else {
    TRY(dalloc(c, &c->gbuf, T * d));
  }
  c->ev_free.resize(3 * c->L);  // up to 3L reads per step (DPO)
  c->ev_chunk.resize(3 * c->L * NCHUNK);
  c->ev_deqg.resize(3 * c->L * NCHUNK);
  for (auto& e : c->ev_free) CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  for (auto& e : c->ev_chunk) CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  for (auto& e : c->ev_deqg) CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  CK(cudaEventCreateWithFlags(&c->ev_done, cudaEventDisableTiming));
  CK(cudaEventCreateWithFlags(&c->ev_start, cudaEventDisableTiming));
  CK(cudaEventCreateWithFlags(&c->ev_d2h, cudaEventDisableTiming));
  CK(cudaEventCreateWithFlags(&c->ev_pre, cudaEventDisableTiming));
  CK(cudaEventCreate(&c->prof_step0));
  CK(cudaEventCreate(&c->prof_step1));
  CK(cudaStreamSynchronize(c->stream));
  c->st.device_bytes = c->dev_bytes;
  return LST_OK;
}

void free_all(lst_ctx* c) {
  if (c->stream) cudaStreamSynchronize(c->stream);
  if (c->nccl_comm) {
    if (c->copy_stream) cudaStreamSynchronize(c->copy_stream);
    nccl().comm_destroy(c->nccl_comm);
    c->nccl_comm = nullptr;
  }
  if (c->copy_stream) cudaStreamSynchronize(c->copy_stream);
  if (c->prep_stream) cudaStreamSynchronize(c->prep_stream);
  if (c->d2h_stream) cudaStreamSynchronize(c->d2h_stream);
  for (void* p : c->dev_allocs) cudaFree(p);
  c->dev_allocs.clear();
  if (c->stage_w) cudaFree(c->stage_w);
  if (c->stage_blob) cudaFree(c->stage_blob);
  if (c->stage_absmax) cudaFree(c->stage_absmax);
  if (c->stage_gsum) cudaFree(c->stage_gsum);
  if (c->arena) cudaFreeHost(c->arena);
  if (c->host_loss) cudaFreeHost(c->host_loss);
  for (auto e : c->ev_chunk) cudaEventDestroy(e);
  for (auto e : c->ev_free) cudaEventDestroy(e);
  for (auto e : c->ev_deqg) cudaEventDestroy(e);
  for (auto e : c->prof_pool) cudaEventDestroy(e);
  for (auto e : c->tl_ev) cudaEventDestroy(e);
  if (c->ev_done) cudaEventDestroy(c->ev_done);
  if (c->ev_start) cudaEventDestroy(c->ev_start);
  if (c->ev_d2h) cudaEventDestroy(c->ev_d2h);
  if (c->ev_pre) cudaEventDestroy(c->ev_pre);
  if (c->prof_step0) cudaEventDestroy(c->prof_step0);
  if (c->prof_step1) cudaEventDestroy(c->prof_step1);
  if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
  if (c->prep_stream) cudaStreamDestroy(c->prep_stream);
  if (c->d2h_stream) cudaStreamDestroy(c->d2h_stream);
  if (c->own_stream && c->stream) cudaStreamDestroy(c->stream);
  cudaGetLastError();
}

lst_status ensure_staging(lst_ctx* c) {
  if (c->stage_blob) return LST_OK;
  int64_t maxn = 0;
  for (int p = 0; p < NPROJ; ++p) maxn = std::max(maxn, c->lay.n[p]);
  CK(cudaMalloc(&c->stage_w, maxn * 4));
  CK(cudaMalloc(&c->stage_blob, c->lay.total));
  CK(cudaMalloc(&c->stage_absmax, (maxn / 64) * 4));
  CK(cudaMalloc(&c->stage_gsum, ((maxn / 64 + 255) / 256) * 8));
  return LST_OK;
}

void release_staging(lst_ctx* c) {
  cudaStreamSynchronize(c->stream);
  cudaFree(c->stage_w);
  cudaFree(c->stage_blob);
  cudaFree(c->stage_absmax);
  cudaFree(c->stage_gsum);
  c->stage_w = nullptr;
  c->stage_blob = nullptr;
  c->stage_absmax = nullptr;
  c->stage_gsum = nullptr;
}

lst_status register_impl(lst_ctx* c, int layer, const lst_layer_weights* w) {
  const lst_config& k = c->cfg;
  for (int p = 0; p < NPROJ; ++p)
    if (!w->w[p] || !w->lora_a[p] || !w->lora_b[p]) return fail(c, LST_ERR_ARG, "null weight pointer");
  if (!w->attn_norm || !w->mlp_norm) return fail(c, LST_ERR_ARG, "null norm pointer");
  if (k.qkv_bias && (!w->bias[0] || !w->bias[1] || !w->bias[2])) return fail(c, LST_ERR_ARG, "qkv_bias needs 3 biases");
  TRY(ensure_staging(c));
  CK(cudaMemsetAsync(c->stage_blob, 0, c->lay.total, c->stream));
  for (int p = 0; p < NPROJ; ++p) {
    const int64_t n = c->lay.n[p];
    const float* src = w->w[p];
    if (!is_device_ptr(src)) {
      CK(cudaMemcpyAsync(c->stage_w, src, n * 4, cudaMemcpyHostToDevice, c->stream));
      src = c->stage_w;
    }
    if (k.base_format == LST_BASE_NF4) {
      Nf4Out o;
      o.packed = c->stage_blob + c->lay.packed[p];
      o.qabs = reinterpret_cast<int8_t*>(c->stage_blob + c->lay.qabs[p]);
      o.gscale = reinterpret_cast<float*>(c->stage_blob + c->lay.gscale[p]);
      o.mean = reinterpret_cast<float*>(c->stage_blob + c->lay.means) + p;
      CK(nf4_quantize(src, n, o, c->stage_absmax, c->stage_gsum, c->stream));
    } else {
      CK(f32_to_bf16(src, n, reinterpret_cast<__nv_bfloat16*>(c->stage_blob + c->lay.w16) + c->lay.woff[p],
                     c->stream));
    }
    CK(cudaStreamSynchronize(c->stream));  // stage_w is reused by the next projection
  }
  TRY(copy_in(c, c->stage_blob + c->lay.norms, w->attn_norm, c->d * 4));
  TRY(copy_in(c, c->stage_blob + c->lay.norms + c->d * 4, w->mlp_norm, c->d * 4));
  if (k.qkv_bias) {
    float* b = reinterpret_cast<float*>(c->stage_blob + c->lay.bias);
    TRY(copy_in(c, b, w->bias[0], c->dq * 4));
    TRY(copy_in(c, b + c->dq, w->bias[1], c->dkv * 4));
    TRY(copy_in(c, b + c->dq + c->dkv, w->bias[2], c->dkv * 4));
  }
  if (k.streamed) {
    CK(cudaMemcpyAsync(c->arena + (int64_t)layer * c->lay.total, c->stage_blob, c->lay.total,
                       cudaMemcpyDeviceToHost, c->stream));
  } else {
    CK(cudaMemcpyAsync(c->resident + (int64_t)layer * c->lay.total, c->stage_blob, c->lay.total,
                       cudaMemcpyDeviceToDevice, c->stream));
  }
  for (int p = 0; p < NPROJ; ++p) {
    TRY(copy_in(c, c->lora + c->offA[layer * NPROJ + p], w->lora_a[p], (int64_t)c->r * c->lay.ind[p] * 4));
    TRY(copy_in(c, c->lora + c->offB[layer * NPROJ + p], w->lora_b[p], c->lay.outd[p] * c->r * 4));
  }
  TRY(prep_lora(c, layer));
  CK(cudaStreamSynchronize(c->stream));
  int derr = 0;
  CK(cudaMemcpyFromSymbol(&derr, g_lst_dev_error, sizeof(int)));
  if (derr) return fail(c, LST_ERR_DEVICE, "device error during registration");
  c->registered[layer] = 1;
  bool all = true;
  for (int i = 0; i < c->L; ++i) all = all && c->registered[i];
  if (all) release_staging(c);
  return LST_OK;
}

}  // namespace

namespace lst {
void note_launch(int n) { g_launch_count.fetch_add(n, std::memory_order_relaxed); }

int device_sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev].load() > 0) return cached[dev].load();
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  if (dev >= 0 && dev < 64) cached[dev].store(n);
  return n;
}

static unsigned long long device_bit() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
}
bool done_on_device(const std::atomic<unsigned long long>& mask) {
  const unsigned long long bit = device_bit();
  return bit && (mask.load() & bit);
}
void mark_done_on_device(std::atomic<unsigned long long>& mask) { mask.fetch_or(device_bit()); }
}  // namespace lst

// Makes the context's device current for the duration of an API call and restores the caller's
// device afterwards (a thread may drive contexts on several GPUs).
struct DeviceScope {
  int prev = -1;
  explicit DeviceScope(const lst_ctx* c) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    if (cur != c->dev && cudaSetDevice(c->dev) == cudaSuccess) prev = cur;
  }
  ~DeviceScope() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// =========================================================================== C ABI
extern "C" {

lst_status lst_create(const lst_config* cfg, const float* embed, const float* final_norm, const float* lm_head,
                      void* cuda_stream, lst_ctx** out) {
  if (!out) return LST_ERR_ARG;
  *out = nullptr;
  std::string why;
  if (!valid_config(cfg, &why)) return LST_ERR_ARG;
  if ((cfg->vocab > 0) != (embed && final_norm && lm_head)) return LST_ERR_ARG;
  if (cfg->vocab == 0 && (embed || final_norm || lm_head)) return LST_ERR_ARG;
  lst_ctx* c = new lst_ctx();
  c->cfg = *cfg;
  lst_status s = create_impl(c, embed, final_norm, lm_head, cuda_stream);
  if (s != LST_OK) {
    free_all(c);
    delete c;
    return s;
  }
  *out = c;
  return LST_OK;
}

lst_status lst_register_layer(lst_ctx* c, int32_t layer, const lst_layer_weights* w) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!w || layer < 0 || layer >= c->L) return fail(c, LST_ERR_ARG, "bad layer index or null weights");
  // the layer's bytes change: nothing kept in the pool or the weight scratch is trusted any more,
  // and no copy from the arena may still be running (a prefetch of the next step's first read)
  CK(cudaStreamSynchronize(c->copy_stream));
  c->slot_layer[0] = c->slot_layer[1] = -1;
  c->w_layer[0] = c->w_layer[1] = -1;
  c->pre_slot = c->pre_layer = -1;
  return register_impl(c, layer, w);
}

lst_status lst_set_lora(lst_ctx* c, int32_t layer, int32_t proj, const float* a, const float* b) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (layer < 0 || layer >= c->L || proj < 0 || proj >= NPROJ || !a || !b)
    return fail(c, LST_ERR_ARG, "bad layer/projection or null pointer");
  TRY(copy_in(c, c->lora + c->offA[layer * NPROJ + proj], a, (int64_t)c->r * c->lay.ind[proj] * 4));
  TRY(copy_in(c, c->lora + c->offB[layer * NPROJ + proj], b, c->lay.outd[proj] * c->r * 4));
  TRY(prep_lora(c, layer));
  CK(cudaStreamSynchronize(c->stream));
  return LST_OK;
}

int64_t lst_lora_numel(const lst_ctx* c) { return c ? c->lora_numel : 0; }

// One AdamW update of every adapter with the gradient g (device), refreshing the bf16 operands.
static lst_status adamw_apply(lst_ctx* c, const float* g) {
  c->opt_t += 1;
  const double t = (double)c->opt_t;
  AdamHyper h;
  h.lr = c->opt.lr;
  h.b1 = c->opt.beta1;
  h.b2 = c->opt.beta2;
  h.eps = c->opt.eps;
  h.wd = c->opt.weight_decay;
  h.step_size = (float)(c->opt.lr / (1.0 - std::pow((double)c->opt.beta1, t)));
  h.sqrt_bc2 = (float)std::sqrt(1.0 - std::pow((double)c->opt.beta2, t));
  ProfScope ps(c, c->stream, PC_OTHER);
  CK(adamw_update(c->opt_tab, c->opt_ntab, c->opt_maxn, c->lora, g, c->opt_m, c->opt_v, h, c->stream));
  return LST_OK;
}

// The in-step update (optimizer on and not deferred) with the step's own gradients.
static lst_status optimizer_update(lst_ctx* c) {
  if (!c->opt_on || c->opt.deferred) return LST_OK;
  return adamw_apply(c, c->grads);
}

lst_status lst_step(lst_ctx* c, const int32_t* tokens, const int32_t* targets, int32_t batch, int32_t seq,
                    float* loss, float* grads) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!tokens || !targets || !loss) return fail(c, LST_ERR_ARG, "null tokens/targets/loss");
  if (c->V <= 0) return fail(c, LST_ERR_STATE, "lst_step needs a head (vocab > 0); use lst_step_hidden");
  TRY(begin_step(c, batch, seq));
  TRY(copy_in(c, c->tok, tokens, c->curT * 4));
  TRY(copy_in(c, c->tgt, targets, c->curT * 4));
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(embed(c->tok, c->E, c->curT, c->d, c->V, c->xs, c->stream));
  }
  set_grads_dest(c, grads);
  TRY(run_layers(c, HEAD_SFT));
  TRY(optimizer_update(c));
  c->have_logits = true;
  return finish_step(c, loss, grads);
}

lst_status lst_step_hidden(lst_ctx* c, const uint16_t* x, const uint16_t* g, int32_t batch, int32_t seq,
                           float* loss, float* grads) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!x || !g || !loss) return fail(c, LST_ERR_ARG, "null x/g/loss");
  if (c->V != 0) return fail(c, LST_ERR_STATE, "lst_step_hidden needs a headless config (vocab == 0)");
  TRY(begin_step(c, batch, seq));
  TRY(copy_in(c, c->dout_b, x, c->curT * c->d * 2));  // bf16 input staged, widened to fp32
  CK(bf16_to_f32(c->dout_b, c->curT * c->d, c->xs, c->stream));
  TRY(copy_in(c, c->gbuf, g, c->curT * c->d * 2));
  set_grads_dest(c, grads);
  TRY(run_layers(c, HEAD_HIDDEN));
  TRY(optimizer_update(c));
  c->have_logits = false;
  return finish_step(c, loss, grads);
}

lst_status lst_step_dpo(lst_ctx* c, const int32_t* tokens, const int32_t* targets, const int32_t* mask,
                        int32_t n_pairs, int32_t seq, float beta, float* loss, float* grads) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!tokens || !targets || !loss) return fail(c, LST_ERR_ARG, "null tokens/targets/loss");
  if (c->V <= 0) return fail(c, LST_ERR_STATE, "lst_step_dpo needs a head (vocab > 0)");
  if (n_pairs <= 0 || !(beta > 0.f) || !std::isfinite(beta)) return fail(c, LST_ERR_ARG, "n_pairs <= 0 or beta not > 0");
  if ((int64_t)2 * n_pairs > c->cfg.max_batch) return fail(c, LST_ERR_ARG, "2 * n_pairs above max_batch");
  TRY(begin_step(c, 2 * n_pairs, seq));
  TRY(copy_in(c, c->tok, tokens, c->curT * 4));
  TRY(copy_in(c, c->tgt, targets, c->curT * 4));
  c->have_mask = mask != nullptr;
  if (mask) TRY(copy_in(c, c->mask_dev, mask, c->curT * 4));
  c->dpo_beta = beta;
  {
    ProfScope ps(c, c->stream, PC_OTHER);
    CK(embed(c->tok, c->E, c->curT, c->d, c->V, c->xs, c->stream));
  }
  set_grads_dest(c, grads);
  TRY(run_layers(c, HEAD_DPO));
  TRY(optimizer_update(c));
  c->have_logits = false;
  return finish_step(c, loss, grads);
}

lst_status lst_get_logits(lst_ctx* c, float* dst) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!dst) return fail(c, LST_ERR_ARG, "null dst");
  if (!c->have_logits) return fail(c, LST_ERR_STATE, "no logits: run lst_step first");
  if (!c->logits_whole) return fail(c, LST_ERR_STATE, "the head ran in passes (head_chunk): logits are not kept whole");
  const bool dev = is_device_ptr(dst);
  CK(cudaMemcpyAsync(dst, c->logits, c->curT * c->V * 4, dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                     c->stream));
  CK(cudaStreamSynchronize(c->stream));
  return LST_OK;
}

lst_status lst_get_activation(lst_ctx* c, int32_t which, int32_t layer, void* dst) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!dst) return fail(c, LST_ERR_ARG, "null dst");
  if (c->st.steps == 0) return fail(c, LST_ERR_STATE, "no step has run");
  const int64_t T = c->curT, d = c->d;
  const void* src = nullptr;
  int64_t bytes = 0;
  if (which == LST_ACT_X) {
    if (layer < 0 || layer > c->L) return fail(c, LST_ERR_ARG, "layer outside [0, L]");
    src = c->xs + (int64_t)layer * c->Tmax * d;
    bytes = T * d * 4;
  } else {
    if (layer != 0) return fail(c, LST_ERR_ARG, "intermediates are kept for layer 0 only");
    switch (which) {
      case LST_ACT_N1: src = c->n1; bytes = T * d * 2; break;
      case LST_ACT_QKV: src = c->qkv; bytes = T * c->dqkv * 2; break;
      case LST_ACT_O: src = c->o; bytes = T * c->dq * 2; break;
      case LST_ACT_H: src = c->h; bytes = T * d * 4; break;
      case LST_ACT_N2: src = c->n2; bytes = T * d * 2; break;
      case LST_ACT_GU: src = c->gu; bytes = T * 2 * c->F * 2; break;
      case LST_ACT_M: src = c->m; bytes = T * c->F * 2; break;
      default: return fail(c, LST_ERR_ARG, "unknown activation");
    }
  }
  CK(cudaMemcpyAsync(dst, src, bytes, is_device_ptr(dst) ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                     c->stream));
  CK(cudaStreamSynchronize(c->stream));
  return LST_OK;
}

lst_status lst_set_optimizer(lst_ctx* c, const lst_adamw* cfg) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!cfg) {
    c->opt_on = false;
    return LST_OK;
  }
  if (!(cfg->lr >= 0.f) || !(cfg->beta1 >= 0.f && cfg->beta1 < 1.f) || !(cfg->beta2 >= 0.f && cfg->beta2 < 1.f) ||
      !(cfg->eps > 0.f) || !(cfg->weight_decay >= 0.f))
    return fail(c, LST_ERR_ARG, "bad AdamW hyper-parameters");
  if (!c->opt_m) {
    TRY(dalloc(c, &c->opt_m, c->lora_numel, true));
    TRY(dalloc(c, &c->opt_v, c->lora_numel, true));
  } else {
    CK(cudaMemsetAsync(c->opt_m, 0, c->lora_numel * 4, c->stream));
    CK(cudaMemsetAsync(c->opt_v, 0, c->lora_numel * 4, c->stream));
    CK(cudaStreamSynchronize(c->stream));
  }
  c->opt = *cfg;
  c->opt_t = 0;
  c->opt_on = true;
  return LST_OK;
}

lst_status lst_apply_optimizer(lst_ctx* c, const float* g) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!g) return fail(c, LST_ERR_ARG, "null gradient");
  if (!c->opt_on || !c->opt.deferred) return fail(c, LST_ERR_STATE, "set the optimizer with deferred = 1 first");
  const float* src = g;
  if (!is_device_ptr(g)) {  // host gradient: staged through the context's gradient buffer
    TRY(copy_in(c, c->grads, g, c->lora_numel * 4));
    src = c->grads;
  }
  TRY(adamw_apply(c, src));
  CK(cudaStreamSynchronize(c->stream));
  return LST_OK;
}

lst_status lst_get_lora(lst_ctx* c, float* dst) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (!dst) return fail(c, LST_ERR_ARG, "null dst");
  const bool dev = is_device_ptr(dst);
  CK(cudaMemcpyAsync(dst, c->lora, c->lora_numel * 4, dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                     c->stream));
  CK(cudaStreamSynchronize(c->stream));
  return LST_OK;
}

lst_status lst_set_profiling(lst_ctx* c, int32_t on) {
  if (!c) return LST_ERR_ARG;
  c->profiling = on != 0;
  return LST_OK;
}

lst_status lst_split_plan(int64_t blob_bytes, int32_t world, int32_t rank, int64_t* offset, int64_t* bytes,
                          int64_t* count) {
  if (blob_bytes <= 0 || world < 1 || rank < 0 || rank >= world || !offset || !bytes || !count) return LST_ERR_ARG;
  split_plan(blob_bytes, world, rank, offset, bytes, count);
  return LST_OK;
}

lst_status lst_nccl_unique_id(void* out) {
  if (!out) return LST_ERR_ARG;
  if (!nccl().ok) return LST_ERR_STATE;
  NcclUid id;
  if (nccl().get_unique_id(&id) != 0) return LST_ERR_CUDA;
  std::memcpy(out, &id, sizeof(id));
  return LST_OK;
}

lst_status lst_set_split_copy(lst_ctx* c, int32_t rank, int32_t world, const void* unique_id) {
  if (!c) return LST_ERR_ARG;
  DeviceScope ds(c);
  if (world < 1 || rank < 0 || rank >= world || !unique_id) return fail(c, LST_ERR_ARG, "bad rank / world or null unique id");
  if (!c->cfg.streamed) return fail(c, LST_ERR_STATE, "split copies need a streamed context");
  if (c->nccl_comm) return fail(c, LST_ERR_STATE, "split copies are already set");
  if (!nccl().ok) return fail(c, LST_ERR_STATE, "libnccl.so.2 could not be loaded");
  int64_t off = 0, bytes = 0, count = 0;
  split_plan(c->lay.total, world, rank, &off, &bytes, &count);
  if (world * count > c->pool_bytes) {
    // the all-gather fills world * count bytes: grow both slots (new guards after them)
    CK(cudaStreamSynchronize(c->stream));
    CK(cudaStreamSynchronize(c->copy_stream));
    for (int k = 0; k < 2; ++k) {
      uint8_t* q = nullptr;
      TRY(dalloc(c, &q, world * count + kGuardBytes));
      TRY(add_guard(c, q + world * count));
      c->pool[k] = q;  // the old slot stays in dev_allocs and is freed with the context
    }
    c->pool_bytes = world * count;
    c->slot_layer[0] = c->slot_layer[1] = -1;
    c->pre_slot = c->pre_layer = -1;
  }
  NcclUid id;
  std::memcpy(&id, unique_id, sizeof(id));
  NcclCommT comm = nullptr;
  const int r = nccl().comm_init_rank(&comm, world, id, rank);
  if (r != 0) return fail(c, LST_ERR_CUDA, std::string("ncclCommInitRank: ") + nccl().error_string(r));
  c->nccl_comm = comm;
  c->split_world = world;
  c->split_rank = rank;
  return LST_OK;
}

lst_status lst_get_read_timeline(const lst_ctx* c, float* out, int32_t max_reads, int32_t* n_reads) {
  if (!c || !n_reads) return LST_ERR_ARG;
  *n_reads = c->tl_reads;
  if (c->tl_reads == 0) return LST_ERR_STATE;
  if (!out || max_reads < c->tl_reads) return LST_ERR_ARG;
  for (int n = 0; n < c->tl_reads; ++n) {
    const int j = c->rd_layer[n], kind = c->rd_kind[n];
    float* row = out + (int64_t)n * 8;
    row[0] = (float)j;
    row[1] = (float)kind;
    for (int k = 0; k < lst_ctx::TL_N; ++k) row[2 + k] = c->tl_ms[(size_t)n * lst_ctx::TL_N + k];
  }
  return LST_OK;
}

lst_status lst_plan_reads(const int32_t* reads, int32_t n_reads, int32_t reuse, int32_t nf4, int32_t* held,
                          int32_t* wheld, int32_t* prefetch, int32_t* out) {
  if (!reads || n_reads <= 0 || !held || !wheld || !out) return LST_ERR_ARG;
  std::vector<int> layers(reads, reads + n_reads);
  for (int v : layers)
    if (v < 0) return LST_ERR_ARG;
  if (prefetch && (prefetch[0] < -1 || prefetch[0] > 1)) return LST_ERR_ARG;
  int h[2] = {held[0], held[1]}, w[2] = {wheld[0], wheld[1]};
  int pre[2] = {prefetch ? prefetch[0] : -1, -1};
  std::vector<ReadPlan> plan;
  plan_schedule(layers, reuse != 0, nf4 != 0, h, w, plan, prefetch ? pre : nullptr);
  if (prefetch) {
    prefetch[0] = pre[0];
    prefetch[1] = pre[1];
  }
  for (int n = 0; n < n_reads; ++n) {
    const ReadPlan& p = plan[n];
    const int32_t row[8] = {p.slot, p.copy ? 1 : 0, p.wait_free, p.loaded_by,
                            nf4 ? p.wslot : -1, p.deq ? 1 : 0, p.wwait, p.wfilled_by};
    std::memcpy(out + 8 * (int64_t)n, row, sizeof(row));
  }
  held[0] = h[0];
  held[1] = h[1];
  wheld[0] = w[0];
  wheld[1] = w[1];
  return LST_OK;
}

lst_status lst_set_dequant_mode(lst_ctx* c, int32_t mode) {
  if (!c) return LST_ERR_ARG;
  if (mode != 0 && mode != 1) return fail(c, LST_ERR_ARG, "dequant mode must be 0 or 1");
  if (mode != c->deq_mode) {
    c->deq_mode = mode;
    c->w_layer[0] = c->w_layer[1] = -1;  // the scratches may lack the groups the GEMMs dequantised
  }
  return LST_OK;
}

lst_status lst_set_reuse(lst_ctx* c, int32_t reuse) {
  if (!c) return LST_ERR_ARG;
  c->cfg.reuse = reuse != 0;
  return LST_OK;
}

lst_status lst_set_prefetch(lst_ctx* c, int32_t on) {
  if (!c) return LST_ERR_ARG;
  c->prefetch_on = on != 0;
  if (!c->prefetch_on) c->pre_slot = c->pre_layer = -1;
  return LST_OK;
}

lst_status lst_get_stats(const lst_ctx* c, lst_stats* out) {
  if (!c || !out) return LST_ERR_ARG;
  *out = c->st;
  out->device_bytes = c->dev_bytes;
  return LST_OK;
}

const char* lst_last_error(const lst_ctx* c) { return c ? c->err.c_str() : "null context"; }

void lst_destroy(lst_ctx* c) {
  if (!c) return;
  {
    DeviceScope ds(c);
    free_all(c);
  }
  delete c;
}

lst_status lst_nf4_codebook(float out[16]) {
  if (!out) return LST_ERR_ARG;
  nf4_codebook(out);
  return LST_OK;
}

int64_t lst_blob_bytes(const lst_config* cfg) {
  std::string why;
  if (!valid_config(cfg, &why)) return -1;
  return make_layout(*cfg).total;
}

}  // extern "C"

extern "C" int32_t lst_k_device_error(void) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (cudaMemcpyFromSymbol(&v, lst::g_lst_dev_error, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (v) {
    int zero = 0;
    cudaMemcpyToSymbol(lst::g_lst_dev_error, &zero, sizeof(int));
  }
  return v;
}
