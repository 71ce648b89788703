/*
 * moeq.h -- C ABI of libmoeq: one decoder layer's Mixture-of-Experts FFN over
 * 4-bit and 2-bit affine group-quantised experts, on one NVIDIA B200 (sm_100a).
 *
 * The operation (pages cited by title and section):
 *   [FlashMoE] "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres
 *              sur un ordinateur portable" (fr.news.hada.io, topic 27758)
 *   [PagedMoE] "Qwen3.5-397B MoE fonctionne avec 14 Go de RAM via un
 *              chargement d'expert paginé sur M1 Ultra" (openclawradar.com)
 *   [Slotstream] "104 Go de modèle sur un Mac de 48 Go" (veilletech.fr)
 *
 *   router  : logits = W_r xhat, softmax, top-k experts, weights renormalised
 *             over the k selected ([PagedMoE] opening paragraph: 512 experts,
 *             top-10 routing; [FlashMoE] "Architecture du modèle": K active
 *             experts per token, one of them shared).
 *   experts : per selected expert, gate/up mat-vecs over quantised weights
 *             w = code*scale + bias ([FlashMoE] "Noyau de déquantification
 *             optimisé FMA"), h = silu(gate) * up, then the down mat-vec
 *             ([FlashMoE] "Shaders de calcul Metal": 4-bit/2-bit dequantising
 *             mat-vecs, SwiGLU).
 *   combine : out = residual + sum_i w_i y_i + gamma * y_shared
 *             ([FlashMoE] "Shaders de calcul Metal": MoE combine + residual +
 *             gate; "Deferred GPU Expert Compute": combine and residual done on
 *             the GPU and handed to the next layer).  gamma = sigmoid(g_s . xhat)
 *             when a shared-expert gate vector is given, else 1.
 *
 * Conventions (where the pages are silent):
 *   - codes: uint32 words, little endian, low bits first; a row of `cols`
 *     codes is cols*bits/32 words; rows are contiguous.
 *   - scale, bias: bf16, [rows][cols/64] (group of 64 consecutive codes).
 *   - gate and up are [inter][hidden]; down is [hidden][inter].
 *   - top-k order: descending logit, ties to the lower expert id.
 *
 * Memory and ownership: every array argument is a DEVICE pointer owned by the
 * caller unless marked "host".  The library allocates no device or host
 * memory and keeps no state between calls other than per-device attributes;
 * scratch lives in a caller-provided workspace (moe_workspace_size).
 * Kernels start early with programmatic dependent launch and read the router
 * matrix, the slot table and the expert weights before waiting on the kernel
 * queued before them: those (model weights) must not be written by the
 * kernel that immediately precedes the call on `stream`.  Activations,
 * residuals and id/weight arrays may come from it.
 *
 * Errors: every call validates its arguments on the host before launching
 * anything; on failure it launches nothing, returns a non-zero moe_status and
 * sets a thread-local message (moe_last_error).  Calls are asynchronous on
 * `stream`.  Problems only the device can see (an expert id outside the slot
 * table, a NULL or misaligned slot pointer, a non-finite logit, a bounded wait that ran out)
 * set bits of a status word inside the workspace; the affected expert
 * contributes zero and the kernels return normally.  Read and clear that word
 * with moe_get_device_status.  Nothing in this library traps, asserts or
 * exits.
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st *moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or size     */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. group!=64) */
    MOE_ERR_CUDA = 3,         /* a CUDA runtime call failed                  */
    MOE_ERR_DEVICE_FAULT = 4, /* the device status word reports a problem    */
    MOE_ERR_TIMEOUT = 5       /* a bounded device wait gave up               */
} moe_status;

/* Device status word bits (moe_get_device_status). */
#define MOE_DEV_BAD_EXPERT_ID 0x1 /* routed id < 0 or >= n_slots            */
#define MOE_DEV_BAD_SLOT 0x2      /* selected expert: NULL or misaligned    */
#define MOE_DEV_NONFINITE 0x4     /* a router logit was NaN or infinite     */
#define MOE_DEV_TIMEOUT 0x8       /* a bounded device wait ran out          */

/* Layer shape.  hidden, inter: multiples of 64; group_size must be 64; bits 4
 * or 2; 1 <= top_k <= min(n_experts, 32); n_experts <= 1024; has_shared 0/1. */
typedef struct {
    int32_t hidden;     /* H */
    int32_t inter;      /* I (expert intermediate size) */
    int32_t n_experts;  /* E (routed experts) */
    int32_t top_k;      /* k */
    int32_t group_size; /* G, must be 64 */
    int32_t bits;       /* 4 or 2 */
    int32_t has_shared; /* 1: one always-on shared expert */
} moe_layer_desc;

/* One quantised matrix [rows][cols]: codes (16-byte aligned), scale, bias. */
typedef struct {
    const void *codes; /* uint32 [rows][cols*bits/32] */
    const void *scale; /* bf16 [rows][cols/64]        */
    const void *bias;  /* bf16 [rows][cols/64]        */
} moe_qmat;

/* One expert: gate, up [I][H]; down [H][I]. */
typedef struct {
    moe_qmat gate, up, down;
} moe_qexpert;

/* Expert slot table: a DEVICE array of n_slots moe_qexpert, indexed by expert
 * id, resident in HBM ([Slotstream] "Ce qui se passe": experts kept in memory
 * slots; [PagedMoE]: experts held in memory and looked up by the router's
 * choice).  n_slots must be >= n_experts. */
typedef struct {
    const moe_qexpert *slots; /* device array */
    int32_t n_slots;
} moe_slot_table;

typedef enum { MOE_DT_BF16 = 0, MOE_DT_F32 = 1 } moe_dtype;

/* Bytes of workspace needed for up to max_tokens tokens of this layer shape.
 * Returns 0 for an invalid desc. */
size_t moe_workspace_size(const moe_layer_desc *desc, int32_t max_tokens);

/* Zero-fill a workspace (cudaMemsetAsync on stream).  A workspace must be
 * zero-filled once before its first use; the kernels leave their
 * synchronisation counters at zero when they finish, so later calls need no
 * re-initialisation.  Calls sharing one workspace must not overlap in time
 * (same stream, or ordered by events). */
moe_status moe_workspace_init(void *ws, size_t bytes, moe_stream_t stream);

/*
 * moe_route -- router logits, softmax, top-k, renormalised weights.
 *   x          bf16 [T][H], the normalised layer input (16-byte aligned)
 *   w_router   [E][H], bf16 or fp32 per router_dtype (16-byte aligned)
 *   logit_bias NULL or fp32 [T][E] added to the logits (test/benchmark hook
 *              for skewed routing; not part of the method; pass NULL)
 *   topk_idx   out int32 [T][k]; topk_w out fp32 [T][k] (sum to 1 per token)
 *   ws         workspace of moe_workspace_size(desc, >= T) bytes
 * Logits are accumulated in fp64 from exact products, so the selection equals
 * that of an fp64 evaluation except for logits equal to within rounding.
 * Below 64 tokens each token is routed by its own CTAs; from 64 tokens on the
 * logits are one tiled GEMM on the fp64 tensor cores, followed by one top-k
 * CTA per token (same selection rule, sums in another order).
 */
moe_status moe_route(const moe_layer_desc *desc, const void *x, int32_t T,
                     const void *w_router, moe_dtype router_dtype, const float *logit_bias,
                     int32_t *topk_idx, float *topk_w, void *ws, moe_stream_t stream);

/*
 * moe_expert_ffn_q4 / moe_expert_ffn_q2 -- the selected experts' FFNs and
 * their routing-weighted sum, without residual.
 *   desc->bits must be 4 (q4) or 2 (q2).
 *   x          bf16 [T][H]
 *   slots      host pointer to the slot table descriptor (table on device)
 *   shared     host pointer to the shared expert (device pointers inside), or
 *              NULL; required iff desc->has_shared
 *   topk_idx   int32 [T][k] expert ids; topk_w fp32 [T][k] weights
 *   y          out fp32 [T][2][H]: y[t][0] = sum_i w_i y_{idx_i};
 *              y[t][1] = y_shared (zeros without a shared expert)
 */
moe_status moe_expert_ffn_q4(const moe_layer_desc *desc, const void *x, int32_t T,
                             const moe_slot_table *slots, const moe_qexpert *shared,
                             const int32_t *topk_idx, const float *topk_w,
                             float *y, void *ws, moe_stream_t stream);
moe_status moe_expert_ffn_q2(const moe_layer_desc *desc, const void *x, int32_t T,
                             const moe_slot_table *slots, const moe_qexpert *shared,
                             const int32_t *topk_idx, const float *topk_w,
                             float *y, void *ws, moe_stream_t stream);

/*
 * moe_combine_residual -- out = residual + y[t][0] + gamma * y[t][1], rounded
 * to bf16 (nearest even).  gamma = sigmoid(shared_gate . x[t]) if shared_gate
 * is given (bf16 [H]), else 1.
 *   y fp32 [T][2][H] as written by moe_expert_ffn_*; residual, x bf16 [T][H];
 *   out bf16 [T][H] (may be the residual buffer).
 */
moe_status moe_combine_residual(const moe_layer_desc *desc, const float *y, const void *residual,
                                const void *shared_gate, const void *x, int32_t T,
                                void *out, moe_stream_t stream);

/*
 * moe_rmsnorm -- out[t] = x[t] / sqrt(mean_j x[t][j]^2 + eps) with unit
 * weight, rounded to bf16 (nearest even): the input normalisation of a
 * decoder layer.  The pages: "Flash-MoE - Exécuter un modèle de 397 milliards
 * de paramètres sur un ordinateur portable", "Shaders de calcul Metal" (RMS
 * normalisation) and "Deferred GPU Expert Compute" (norm + residual handed to
 * the next layer); the unit weight and eps are this library's reading.
 *   x, out bf16 [T][H] (device; out may be x); H a multiple of 8 in
 *   [8, 8192]; eps >= 0.  The sum of squares runs in fp64.
 * Errors: MOE_ERR_INVALID_ARG for NULL / misaligned (16 bytes) pointers or
 * bad sizes.
 */
moe_status moe_rmsnorm(const void *x, int32_t T, int32_t H, float eps, void *out, moe_stream_t stream);

/*
 * moe_layer_forward -- the whole layer: route, expert FFNs, combine, residual.
 *   x bf16 [T][H] normalised input; residual bf16 [T][H] (may equal x);
 *   out bf16 [T][H] must not overlap x (it may equal residual when residual
 *   is not x).  topk_idx_out / topk_w_out: NULL or int32/fp32 [T][k].
 *   Other arguments as in moe_route / moe_expert_ffn_*.
 * Below 64 tokens (and for 2-bit layers, or hidden / inter not multiples of
 * 128): the decode path, three kernels (route; gate/up + SwiGLU with the
 * top-k; down + combine + residual); only h passes through the workspace.
 * From 64 tokens on (4-bit, hidden and inter multiples of 128): the (token,
 * expert) pairs are sorted by expert and each expert's tokens go through
 * dequant-fused GEMMs on the tensor cores (fp16 operands, fp32 accumulation),
 * with sorted rows of x, h and y in the workspace's prefill area.  Both paths
 * give the same routing and agree within the output tolerance.
 */
moe_status moe_layer_forward(const moe_layer_desc *desc, const void *x, const void *residual,
                             int32_t T, const void *w_router, moe_dtype router_dtype,
                             const float *logit_bias, const moe_slot_table *slots,
                             const moe_qexpert *shared, const void *shared_gate, void *out,
                             int32_t *topk_idx_out, float *topk_w_out, void *ws,
                             moe_stream_t stream);

/*
 * moe_layer_forward_normed -- one layer of a stack fed by its hidden state:
 * x-hat = rmsnorm(h) (as moe_rmsnorm: unit weight, eps, bf16, bit-equal to
 * it), then out = h + MoE(x-hat) exactly as moe_layer_forward with
 * x = x-hat and residual = h.  The pages: "Flash-MoE - Exécuter un modèle de
 * 397 milliards de paramètres sur un ordinateur portable", "Deferred GPU
 * Expert Compute" (the combined output and residual feed the next layer's
 * normalisation) and "Shaders de calcul Metal" (RMS normalisation).  At
 * decode sizes the normalisation runs inside the router kernel (no extra
 * launch); from 64 tokens on (4-bit layers) it is a kernel of its own.
 *   h bf16 [T][H] (device, 16-byte aligned); out bf16 [T][H] (may be h,
 *   otherwise must not overlap it); xhat_out NULL or bf16 [T][H] (16-byte
 *   aligned, overlapping neither h nor out) receives x-hat; eps >= 0.
 *   Other arguments as in moe_layer_forward.
 * Errors: as moe_layer_forward; MOE_ERR_INVALID_ARG for eps < 0.
 */
moe_status moe_layer_forward_normed(const moe_layer_desc *desc, const void *h, int32_t T, float eps,
                                    const void *w_router, moe_dtype router_dtype,
                                    const float *logit_bias, const moe_slot_table *slots,
                                    const moe_qexpert *shared, const void *shared_gate, void *out,
                                    void *xhat_out, int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                    moe_stream_t stream);

/*
 * moe_layer_forward_noalloc -- moe_layer_forward without a workspace
 * argument, for callers that cannot allocate device memory at all.  The
 * pages describe no such call; it exists for this library's users.
 *
 * Who needs it: code that runs where a device allocation is not allowed or
 * not safe -- an inference engine's plugin or operator hook that must not
 * allocate while it enqueues work, a serving loop whose device memory is
 * fully planned up front, or a process whose memory is held by a caching
 * allocator so that a fresh cudaMalloc could fail or stall the device.  Such
 * a caller still owns x, residual, out and the other inputs and outputs, but
 * cannot provide the scratch workspace that moe_layer_forward takes.
 *
 * Scratch: a fixed array inside the library's device image,
 * MOE_NOALLOC_SCRATCH_BYTES (4 MiB) on every GPU that loads the library, kept
 * until the process exits.  A call whose scratch need
 * (moe_workspace_size(desc, T)) exceeds it is rejected with
 * MOE_ERR_INVALID_ARG; the decode layer hidden 4096 / inter 1024 / top-10 +
 * shared fits up to 49 tokens.  The call allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine).
 *
 * The first call on a device looks the array's device address up (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call clears the array's status word and arrival counters
 * on `stream` before launching, so it does not depend on what an earlier
 * call left behind.  All calls share the one array: calls that can overlap on
 * the GPU (other streams, other host threads) race and corrupt each other's
 * results, so order them.  The device status word is not readable through
 * this call; use moe_layer_forward with a workspace to inspect it.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
moe_status moe_layer_forward_noalloc(const moe_layer_desc *desc, const void *x, const void *residual,
                                     int32_t T, const void *w_router, moe_dtype router_dtype,
                                     const float *logit_bias, const moe_slot_table *slots,
                                     const moe_qexpert *shared, const void *shared_gate, void *out,
                                     int32_t *topk_idx_out, float *topk_w_out, moe_stream_t stream);

/* Synchronise `stream`, read the workspace's device status word into *st
 * (host), clear it.  Returns MOE_ERR_DEVICE_FAULT when *st != 0 (
 * MOE_ERR_TIMEOUT when only the timeout bit is set), MOE_OK otherwise. */
moe_status moe_get_device_status(void *ws, moe_stream_t stream, int32_t *st);

/* moe_set_kernel_events -- profiling aid; the pages have no counterpart.
 * With events set, every moe_layer_forward made on this host thread records,
 * on its stream, events[0] before the router kernel, events[1] between the
 * router and gate/up kernels, events[2] between the gate/up and down kernels
 * and events[3] after the down kernel, so cudaEventElapsedTime gives each
 * kernel's device time.  events: n = 4 cudaEvent_t handles (passed as
 * void *), created by the caller with timing enabled, owned by the caller;
 * events = NULL with n = 0 turns it off.  The setting belongs to the calling
 * host thread.  A recorded event between two kernels keeps the second from
 * starting before the first ends, so timed calls run slightly slower.
 * Errors: MOE_ERR_INVALID_ARG for any other n or a NULL handle. */
moe_status moe_set_kernel_events(void *const *events, int32_t n);

/*
 * Expert residency cache (host policy).  The pages keep only the experts a
 * token needs close to the compute and stream the rest in from slower memory
 * ("Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur un
 * ordinateur portable", "SSD Expert Streaming"; "104 Go de modèle sur un Mac
 * de 48 Go", expert slots), relying on the reuse of experts between
 * consecutive tokens.  This object decides, for a bounded number of slots,
 * which slot holds each expert a token routes to and which experts must be
 * copied in: least recently used slots are refilled first, and an expert
 * needed by the current token is never evicted for it.  It moves no data:
 * the caller copies each listed expert into its slot (e.g. cudaMemcpyAsync
 * from pinned host memory) and points its slot table at the slots.  Host
 * only; one object per layer; not thread-safe.
 *
 * moe_cache_create: n_experts >= 1 ids, n_slots in [1, n_experts]; *out
 *   receives the object (free with moe_cache_destroy).
 * moe_cache_plan: ids = the k expert ids of one token (host int32, distinct,
 *   each in [0, n_experts)), 1 <= k <= n_slots.  Writes slot_of[i] (host
 *   int32 [k]): the slot holding ids[i] after the call; fill_ids / fill_slots
 *   (host int32 [k]): the experts to copy and their slots, *n_fill of them, in
 *   the order of ids.  Counts hits and misses.
 * moe_cache_stats: hits and misses so far (either pointer may be NULL).
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, sizes out of range, an id
 * out of range or repeated within one call.
 */
typedef struct moe_expert_cache moe_expert_cache;
moe_status moe_cache_create(int32_t n_experts, int32_t n_slots, moe_expert_cache **out);
void moe_cache_destroy(moe_expert_cache *cache);
moe_status moe_cache_plan(moe_expert_cache *cache, const int32_t *ids, int32_t k, int32_t *slot_of,
                          int32_t *fill_ids, int32_t *fill_slots, int32_t *n_fill);
moe_status moe_cache_stats(const moe_expert_cache *cache, int64_t *hits, int64_t *misses);

/* Thread-local message for the last failed call on this thread ("" if none). */
const char *moe_last_error(void);

/* Library version string. */
const char *moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOEQ_H */
