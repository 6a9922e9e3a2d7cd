/*
 * moe.h -- C ABI of libmoe: one mixed-precision routed-expert (MoE) layer on a
 * B200 (sm_100a).
 *
 * The layer follows "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
 * Inference" (arXiv 2608.15383): the router's top-k rule is kept unchanged
 * (Section 3.1 routing equation), tokens are grouped by selected expert
 * (Figure 1), every selected expert runs as grouped gate/up and down GEMMs
 * (Section 3.4) on weights whose dequantised values define the operations
 * (Section 3.1), and expert outputs are summed with the router weights
 * (Section 3.4).  Each expert carries its own precision -- BF16, INT8 or
 * symmetric group-128 INT4 (Section 3.2) -- so one grouped launch serves GEMMs
 * of different precisions ("Mixed-precision GroupGEMM" idea of MxMoE,
 * arXiv 2505.05799, abstract).  Precision changes swap an expert's handle only
 * once the new version is complete ("stable expert handles", DynaExq,
 * arXiv 2511.15015, abstract).
 *
 * Conventions for every entry point
 *   - Returns MOE_OK (0) or a negative moe_status_t; never throws; on error
 *     moe_last_error() returns a message for the calling thread.
 *   - Pointers named *device* (all tensor arguments) are CUDA device pointers
 *     owned by the caller; the library never frees or retains them beyond what
 *     a function documents.  Host pointers are marked "host".
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronises the host, except functions marked
 *     "synchronising".
 *   - bf16 tensors are raw 16-bit bfloat16 bit patterns; fp16 scales are raw
 *     IEEE binary16 bit patterns.  Row-major throughout.
 *   - Shapes: H (hidden) and I (expert intermediate) multiples of 128,
 *     1 <= E <= 512 experts, 1 <= k <= min(E, 16), T >= 0 tokens.
 *
 * Expert storage format (per expert; K = reduction length of the matrix)
 *   w13  gate/up projection, 2I rows x K = H; rows 0..I-1 gate (W_g),
 *        rows I..2I-1 up (W_u).
 *   w2   down projection, H rows x K = I (W_d).
 *   BF16 : bf16 [rows][K].
 *   INT8 : int8 two's complement [rows][K], scales fp16 [K/128][rows].
 *   INT4 : uint8 [rows][K/2]; element k of a row sits in byte k/2, even k in
 *          the low nibble, stored offset-binary u = q + 8 (q in [-8, 7]);
 *          scales fp16 [K/128][rows].
 *   Scales are group-major: the scale of row r, K-group g (elements
 *   128g..128g+127) is scales[g * rows + r].  Dequantised weight = q * scale.
 *   Alignment: weight and scale buffers 16-byte aligned.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,      /* null pointer, bad size, bad id */
  MOE_ERR_UNSUPPORTED = -2,      /* shape or alignment outside the supported set */
  MOE_ERR_NOT_MATERIALIZED = -3, /* an expert of the layer has no weights set */
  MOE_ERR_CUDA = -4,             /* a CUDA runtime/driver call failed */
  MOE_ERR_TIMEOUT = -5,          /* a bounded device wait expired (see status) */
  MOE_ERR_DEVICE_STATUS = -6     /* device-side checks flagged bad input */
} moe_status_t;

typedef enum { MOE_BF16 = 0, MOE_INT8 = 1, MOE_INT4 = 2 } moe_precision_t;

/* Bits of the per-device status word (moe_get_device_status). */
#define MOE_STATUS_BAD_EXPERT_ID 0x1u  /* topk id outside [0,E) or repeated in a token */
#define MOE_STATUS_NONFINITE_LOGIT 0x2u /* a NaN logit (ordered as -inf) */
#define MOE_STATUS_WAIT_TIMEOUT 0x4u   /* a kernel gave up a bounded wait */
#define MOE_STATUS_UNSET_EXPERT 0x8u   /* FFN met an expert without weights */
#define MOE_STATUS_BAD_ROW_INDEX 0x10u /* expert_offsets or dest_row outside [0, rows) */

typedef struct moe_layer* moe_layer_t;

/* Device buffers of one expert, in the storage format above.  The scale
 * pointers are ignored (may be NULL) for MOE_BF16. */
typedef struct {
  const void* w13;
  const void* s13;
  const void* w2;
  const void* s2;
} moe_expert_weights;

/* Message describing the last error on the calling thread ("" if none). */
const char* moe_last_error(void);

/* ABI version of this header (incremented on incompatible change). */
int moe_abi_version(void);

/* Create a layer object on the current device: H, I multiples of 128,
 * 1 <= E <= 512, 1 <= k <= min(E, 16).  The layer owns a device table of E
 * expert descriptors (all initially unset).  *out receives the handle. */
int moe_layer_create(int H, int I, int E, int k, moe_layer_t* out);

/* Destroy a layer.  Synchronising (waits for the device) so that no enqueued
 * work can still read the descriptor table. */
int moe_layer_destroy(moe_layer_t layer);

/* Install or replace expert `expert`'s weights and precision (the "stable
 * handle" swap of the DynaExq abstract).  Stream-ordered: forwards enqueued on
 * `stream` after this call use the new version, earlier ones the old.  The
 * weights are not copied: the caller keeps the buffers alive, and keeps the old
 * buffers alive until an event recorded after the last forward that used them
 * has completed.  `w` is a host pointer, read during the call only. */
int moe_set_expert_precision(moe_layer_t layer, int expert, moe_precision_t precision,
                             const moe_expert_weights* w, void* stream);

/* Host-side view of the precision last installed for `expert` (-1 if unset). */
int moe_get_expert_precision(moe_layer_t layer, int expert, int* precision);

/* Top-k routing (ExactMoE Section 3.1 routing equation).
 *   logits   device fp32 [T][E]
 *   topk_idx device int32 [T][k]: experts by descending logit, ties broken by
 *            the lower expert id, -0.0 == +0.0; NaN is ordered as -inf and
 *            flags MOE_STATUS_NONFINITE_LOGIT.
 *   topk_w   device fp32 [T][k]: renormalize != 0 -> softmax over the k
 *            selected logits (sums to 1); renormalize == 0 -> the softmax over
 *            all E logits evaluated at the selected experts. */
int moe_route_topk(const float* logits, int T, int E, int k, int renormalize,
                   int32_t* topk_idx, float* topk_w, void* stream);

/* Router projection fused with top-k routing (ExactMoE Section 3.1 routing
 * equation z_t = W_r h_t, S_t = TopK(z_t, k); the router stays in BF16,
 * Abstract):
 *   h          device bf16 [T][H], the layer's input hidden states, row-major
 *   w_router   device bf16 [E][H], row e = expert e's router weights
 *   logits     device fp32 [T][E] or NULL: z in fp32 (bf16 products summed in
 *              fp32 on the tensor cores; the K split is summed in a fixed
 *              order, so results are deterministic)
 *   topk_idx, topk_w: as moe_route_topk, computed from those fp32 logits with
 *              the same rule (identical to moe_route_topk on `logits`)
 * H a multiple of 64, 1 <= E <= 512, 1 <= k <= min(E, 16); h and w_router
 * 16-byte aligned.  One launch: a thread-block cluster splits each tile of
 * tokens' K range over up to 8 CTAs, reduces the partial logits through
 * distributed shared memory and routes the tile's tokens. */
int moe_router_topk(const void* h, const void* w_router, int T, int H, int E, int k,
                    int renormalize, float* logits, int32_t* topk_idx, float* topk_w,
                    void* stream);

/* Group the T*k (token, slot) pairs by expert (ExactMoE Figure 1), experts in
 * id order, ascending token inside each expert; no pair is dropped.
 *   topk_idx       device int32 [T][k]; ids must lie in [0,E) and be distinct
 *                  within a token; a violating pair is left out (dest_row -1)
 *                  and flags MOE_STATUS_BAD_EXPERT_ID.
 *   x              device bf16 [T][H]
 *   expert_offsets device int32 [E+1]: rows of expert e are
 *                  [offsets[e], offsets[e+1]); offsets[E] = number of pairs kept.
 *   perm_token     device int32 [T*k]: row -> token (rows >= offsets[E] unset)
 *   dest_row       device int32 [T][k]: pair -> row, or -1
 *   x_perm         device bf16 [T*k][H]: x_perm[r] = x[perm_token[r]]
 * Deterministic: no atomic decides any order.  For T > 512 the grouping is
 * split over CTAs of 256 tokens (a count pass, then the ranking pass); the
 * per-CTA counts are kept in x_perm until the row gather overwrites it, so
 * x_perm is also written before the gather (it is an output either way). */
int moe_permute(const int32_t* topk_idx, const void* x, int T, int E, int k, int H,
                int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row,
                void* x_perm, void* stream);

/* Bytes of workspace moe_grouped_ffn_mixed needs for `rows` permuted rows. */
int moe_ffn_workspace_bytes(moe_layer_t layer, int rows, size_t* bytes);

/* Grouped SwiGLU expert FFN over the permuted rows (ExactMoE Section 3.4: one
 * fused gate/up grouped GEMM and one down grouped GEMM), each expert at its
 * own precision, INT8/INT4 weights dequantised to bf16 inside the GEMM
 * mainloop, fp32 accumulation on the tensor cores:
 *   h_r = silu(x_r W_g,e^T) * (x_r W_u,e^T)   (rounded to bf16)
 *   y_r = h_r W_d,e^T                        (rounded to bf16)
 * for every row r of expert e.
 *   x_perm         device bf16 [rows][H] (16-byte aligned)
 *   expert_offsets device int32 [E+1] as written by moe_permute
 *   rows           T*k, the row capacity of x_perm / y_perm
 *   y_perm         device bf16 [rows][H]; rows >= offsets[E] are not written
 *   workspace      device, >= moe_ffn_workspace_bytes(rows) bytes, 256-byte
 *                  aligned; holds h and the tile scheduler's counters (zeroed
 *                  by the call itself).
 * Fails with MOE_ERR_NOT_MATERIALIZED if any expert was never set.  An expert
 * whose rows [offsets[e], offsets[e+1]) do not lie inside [0, rows) is left
 * out (nothing of it is read or written) and flags MOE_STATUS_BAD_ROW_INDEX.
 * Calls that share a workspace must not overlap on the device. */
int moe_grouped_ffn_mixed(moe_layer_t layer, const void* x_perm,
                          const int32_t* expert_offsets, int rows, void* y_perm,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Allocation-free variant of moe_grouped_ffn_mixed (no counterpart on the
 * pages; it is an interface convenience).  Some callers cannot hand the library
 * a workspace: code running inside another framework's operator that has no
 * handle on that framework's allocator, or a latency-critical loop that must not
 * call cudaMalloc (which may synchronise the device and take milliseconds).
 * This entry point uses a fixed scratch array that the library keeps in device
 * memory instead (moe_ffn_noalloc_max_bytes() bytes, 8 MiB, held on every GPU
 * that loads the library until the process exits) and allocates nothing.
 *   Same arguments and results as moe_grouped_ffn_mixed, minus the workspace.
 *   Limit: moe_ffn_workspace_bytes(rows) must not exceed the scratch size, i.e.
 *   rows * I * 2 + 8192 <= 8 MiB; larger calls fail with MOE_ERR_UNSUPPORTED.
 *   The first call on a device looks up the scratch's device address (a
 *   cudaGetSymbolAddress with that device current); make that first call
 *   before any stream capture.  The address is cached per device index for
 *   the life of the process: after cudaDeviceReset (or with another context
 *   made current on that device) call moe_ffn_noalloc_reset() before the next
 *   call, so the address is looked up again.
 *   All calls on a device share the one scratch array, which keeps the last
 *   call's contents (the call zeroes the counters it needs): calls that
 *   overlap on the GPU (different streams, or several layers in flight) race
 *   and must not be issued. */
int moe_grouped_ffn_mixed_noalloc(moe_layer_t layer, const void* x_perm,
                                  const int32_t* expert_offsets, int rows, void* y_perm,
                                  void* stream);

/* Size in bytes of the scratch array behind moe_grouped_ffn_mixed_noalloc. */
int moe_ffn_noalloc_max_bytes(size_t* bytes);

/* Forget the cached scratch address of the current device (see above); the
 * next moe_grouped_ffn_mixed_noalloc call on it looks the address up again. */
int moe_ffn_noalloc_reset(void);

/* Weighted combine back to token order (ExactMoE Section 3.4; weights are not
 * renormalised): out[t] = sum_j topk_w[t][j] * y_perm[dest_row[t][j]] in fp32,
 * j in order 0..k-1, pairs with dest_row < 0 skipped, one rounding to bf16.
 *   y_perm device bf16 [rows][H] with rows = T*k; dest_row device int32
 *   [T][k]; topk_w device fp32 [T][k]; out device bf16 [T][H].
 * A dest_row >= T*k is skipped and flags MOE_STATUS_BAD_ROW_INDEX (no read
 * outside y_perm). */
int moe_combine(const void* y_perm, const int32_t* dest_row, const float* topk_w,
                int T, int k, int H, void* out, void* stream);

/* The whole layer in one call: moe_route_topk -> moe_permute ->
 * moe_grouped_ffn_mixed -> moe_combine on `stream`, with the layer's k and
 * H.  Every buffer is caller-owned device memory sized as for the four calls
 * (rows = T*k):
 *   logits fp32 [T][E], x bf16 [T][H] -> out bf16 [T][H];
 *   scratch: topk_idx int32 [T][k], topk_w fp32 [T][k], expert_offsets int32
 *   [E+1], perm_token int32 [T*k], dest_row int32 [T][k], x_perm bf16
 *   [T*k][H], y_perm bf16 [T*k][H], workspace (moe_ffn_workspace_bytes).
 * For T <= 128 routing, grouping and the row gather run as one kernel (each
 * CTA routes all T tokens in shared memory, then copies its share of x_perm
 * rows); the outputs are identical to the separate calls.  The launches use
 * programmatic dependent launch: each kernel may start while the previous one
 * drains and waits (griddepcontrol.wait) before reading its inputs. */
int moe_layer_forward(moe_layer_t layer, const float* logits, const void* x, int T,
                      int renormalize, int32_t* topk_idx, float* topk_w,
                      int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row,
                      void* x_perm, void* y_perm, void* workspace, size_t workspace_bytes,
                      void* out, void* stream);

/* The whole layer from the hidden states: z = W_r x (moe_router_topk) ->
 * top-k -> moe_permute -> moe_grouped_ffn_mixed -> moe_combine, the same
 * buffers as moe_layer_forward except that `logits` (fp32 [T][E]) is written
 * (the router's output) instead of read, and w_router (bf16 [E][H], the
 * layer's H and E) is added.  The outputs equal moe_layer_forward's on the
 * logits this call writes.  For T <= 128 the router kernel writes the logits
 * and the small-batch kernel routes them; above, the router kernel also takes
 * the top-k. */
int moe_layer_forward_hidden(moe_layer_t layer, const void* x, const void* w_router, int T,
                             int renormalize, float* logits, int32_t* topk_idx, float* topk_w,
                             int32_t* expert_offsets, int32_t* perm_token, int32_t* dest_row,
                             void* x_perm, void* y_perm, void* workspace, size_t workspace_bytes,
                             void* out, void* stream);

/* Symmetric group-128 quantiser (ExactMoE Section 3.2; INT8 by analogy with
 * Q = 127): for each row and K-group g, s = fp16_rne(max|W| / Q) with the
 * quotient in fp32, q = clip(rint_even(W / s), -Q-1, Q) using the rounded
 * scale (q = 0 where s = 0); Q = 7 for INT4, 127 for INT8.
 *   w_bf16 device bf16 [rows][K], K a multiple of 128
 *   q_out  device, storage format of `precision` (INT8 or INT4)
 *   scales device fp16 [K/128][rows] */
int moe_quantize_weights(const void* w_bf16, int rows, int K, moe_precision_t precision,
                         void* q_out, void* scales, void* stream);

/* ---- Device-side precision management (DynaExq, arXiv 2511.15015, abstract:
 * expert hotness estimated from router traces, a budget-feasible per-layer hot
 * set, asynchronous promotion and demotion by swapping stable expert handles
 * to fully materialised versions).  The counts, the selection and the handle
 * swap all run on the device, stream-ordered, so no host synchronisation is
 * needed between routing a batch and promoting its hot experts; only the
 * host->device copies of newly promoted experts' BF16 weights are issued by
 * the host (into slots registered below), from any stream. */

/* Register (or, with NULL, unregister) a hotness counter: device uint32 [E].
 * Every later moe_layer_forward of the layer adds, for each expert, the number
 * of (token, slot) pairs routed to it in that forward (integer atomics: the
 * totals do not depend on timing).  The caller owns and zeroes the buffer
 * (moe_select_hot_experts can clear it). */
int moe_layer_set_hotness_counter(moe_layer_t layer, unsigned int* counts);

/* Size of the hot set that a memory budget allows: *n_hot = min(E,
 * budget_bytes / (bytes of a BF16 expert - bytes of the same expert at
 * `low`)), the bytes being the stored weights plus fp16 group-128 scales of
 * the storage format above (ExactMoE Section 3.2 memory formula).  `low` is
 * MOE_INT8 or MOE_INT4, the precision the cold experts stay at. */
int moe_hot_set_size(moe_layer_t layer, size_t budget_bytes, moe_precision_t low, int* n_hot);

/* Hot-set selection on the device: the n_hot experts with the highest counts,
 * ties to the lower expert id, written to hot_ids (device int32 [n_hot]) in
 * ascending id order.  counts: device uint32 [E], E <= 512; zero_counts != 0
 * clears them afterwards (a new counting window starts).  Stream-ordered. */
int moe_select_hot_experts(unsigned int* counts, int E, int n_hot, int zero_counts,
                           int32_t* hot_ids, void* stream);

/* Register the BF16 promotion slots: n_slots device buffers, each one
 * expert's BF16 weights in the storage format above (slots[i].w13 bf16
 * [2I][H], slots[i].w2 bf16 [H][I]; scales ignored), host array of n_slots.
 * The library encodes one descriptor per slot; the caller keeps the buffers
 * alive.  Synchronising (waits for the device, since forwards may read the
 * slots it replaces); re-registering invalidates every promotion made from
 * the old slots: apply a hot set again afterwards. */
int moe_layer_set_bf16_slots(moe_layer_t layer, int n_slots, const moe_expert_weights* slots);

/* Stream-ordered handle swap to a hot set: expert hot_ids[i] (device int32
 * [n_hot], ascending, distinct, < E) now uses BF16 slot slot_base + i, and
 * every other expert its base version (the one last installed by
 * moe_set_expert_precision, which also replaces the expert's current handle).
 * The slots' weights must be complete before the swap runs (record an event
 * after their copies and make `stream` wait on it); forwards enqueued earlier
 * keep the previous handles.  Fails with MOE_ERR_NOT_MATERIALIZED if an expert
 * has no base version, MOE_ERR_INVALID_ARG if the slots are not registered. */
int moe_apply_hot_set(moe_layer_t layer, const int32_t* hot_ids, int n_hot, int slot_base,
                      void* stream);

/* Read and clear the current device's status word (MOE_STATUS_* bits).
 * Synchronising. */
int moe_get_device_status(unsigned int* status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
