/*
 * fp8_moe — forward pass of one mixture-of-experts layer at inference on NVIDIA B200 (sm_100a):
 * router GEMM, softmax, top-k with renormalised weights, stable permutation of the routed rows
 * by expert, W8A8 FP8 (e4m3) grouped expert FFN (gate/up GEMM, SwiGLU, per-row requantisation,
 * down GEMM) and the routing-weighted combine that restores token order.
 *
 * Sources of the operations (pages describing the method):
 *   - "Routage MoE entre GPU" (viite.ai blog): the router scores every expert from a token's
 *     hidden state and keeps the top-k with one routing weight each; only the selected experts
 *     process the token; the selected outputs are weighted, summed and put back in token order.
 *   - "La nouvelle bibliotheque megakernel d'Aleph Alpha ..." (seventnews.com), W8A8 paragraph
 *     and section "Comment fonctionne le megakernel": 8-bit FP8 weights and activations; routing,
 *     gating, expert compute and combine fused into as few persistent kernels as possible.
 *   - "MoE-Prism" (gist.science), sections 2B and 5: the routing budget k as a per-request
 *     runtime knob (here: an optional per-token k array).
 *   - "ELDR" (aiweekly.co), first and third paragraphs: decode cost is the weight bytes of the
 *     distinct experts a batch activates; outputs are those of standard top-k.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd, or torch CUDA tensors) unless the
 *     argument says otherwise; layouts are dense row-major with the last index contiguous.
 *   - bf16 tensors are passed as uint16_t bit patterns; e4m3 tensors as uint8_t codes (OCP FP8
 *     e4m3fn: bias 7, 3 mantissa bits, max 448, 0x7F/0xFF NaN).
 *   - hidden, router_w, w13, w2 (and the shared expert's weights), y and every fp32 output read
 *     or written with 128-bit accesses must be 16-byte aligned (torch allocations are).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every call is
 *     asynchronous on that stream and never synchronises it, except moe_device_status.
 *   - Ownership: the caller allocates and frees every buffer, including the workspace `ws`
 *     (at least moe_workspace_bytes(dims) bytes, 256-byte aligned). The library allocates no
 *     device memory and keeps no per-call state; calls on different streams are independent
 *     when they use different workspaces.
 *   - Errors: a negative moe_status is returned synchronously for anything the host can check
 *     (shapes, NULL pointers, alignment, workspace size, unsupported device) and nothing is
 *     launched. MOE_ERR_CUDA reports a failed launch. Errors detected on the device (an index out
 *     of range in caller-provided routing data, a bounded wait that expired) are recorded in a
 *     status word inside `ws` and read with moe_device_status; the kernels never trap.
 *   - T == 0 is valid and launches nothing.
 */
#ifndef FP8_MOE_H
#define FP8_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,    /* bad shape, NULL pointer, misaligned pointer, k out of range */
  MOE_ERR_UNSUPPORTED = -2,    /* device is not sm_100, or a size outside the supported range */
  MOE_ERR_WORKSPACE = -3,      /* ws is NULL or smaller than moe_workspace_bytes(dims) */
  MOE_ERR_CUDA = -4,           /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE_TIMEOUT = -5, /* (device) a bounded wait inside a kernel expired */
  MOE_ERR_DEVICE_CHECK = -6    /* (device) caller data out of range: expert id, k_t, offsets */
} moe_status;

/* Layer sizes. T tokens, hidden size d, E routed experts with FFN width F, at most k_max experts
 * per token (1..32), F_shared = FFN width of one always-on shared expert (0 = none; otherwise it
 * must equal F). d and F must be multiples of 16; E <= 1024. */
typedef struct moe_dims {
  int32_t T, d, E, F, k_max, F_shared;
} moe_dims;

/* Optional outputs of moe_forward, for inspection and profiling. Every member may be NULL.
 *   topk_ids [T, k_max] int32, topk_w [T, k_max] fp32: the routing decision;
 *   expert_offsets [E+1] int32, perm_token [T*k_max] int32, inv_row [T, k_max] int32: grouping;
 *   y_f32 [T, d] fp32: the combined output before its rounding to bf16;
 *   stage_events: MOE_NUM_STAGES + 1 cudaEvent_t (host array of handles created by the caller);
 *     event i is recorded on `stream` just before stage i's kernel, the last one after the last
 *     stage. Stages: 0 router logits, 1 top-k + activation quantisation, 2 permutation,
 *     3 row gather, 4 gate/up GEMM + SwiGLU, 5 intermediate requantisation, 6 down GEMM,
 *     7 combine. A stage computed by another stage's kernel brackets nothing: stage 1 when one
 *     kernel routes and quantises (E <= 32, or decode batches of T <= 8), and stage 3 always
 *     (the gate/up GEMM fetches the token rows through the permutation itself). */
#define MOE_NUM_STAGES 8
typedef struct moe_debug_out {
  int32_t* topk_ids;
  float* topk_w;
  int32_t* expert_offsets;
  int32_t* perm_token;
  int32_t* inv_row;
  float* y_f32;
  void* const* stage_events;
} moe_debug_out;

/* Host only, pure. Bytes of workspace any entry point needs for `dims` (0 if dims is invalid). */
size_t moe_workspace_bytes(const moe_dims* dims);

/* Host only, pure. A static English description of a moe_status value. */
const char* moe_status_string(int status);

/* Host only. The number of kernels this library has launched in this process so far (every
 * device, every host thread), for benchmarks and profiling: its difference across a region of
 * calls counts the library's launches in that region. Reads a relaxed atomic counter. */
uint64_t moe_kernel_launch_count(void);

/* Clears the device status word kept at the start of `ws` (16 bytes: error code, where-code,
 * detail, and the completion counter of the one-kernel decode router), async on `stream`.
 * moe_forward clears it itself; callers of the split entry points clear it once after
 * allocating `ws`. */
int moe_clear_status(void* ws, void* stream);

/* Reads the device status word of `ws` into *out_status (MOE_OK or a MOE_ERR_DEVICE_* code).
 * Synchronises `stream`. Returns MOE_ERR_CUDA if the copy or the synchronisation fails. */
int moe_device_status(const void* ws, void* stream, int32_t* out_status);

/* Router: logits l[t,e] = sum_d hidden[t,d] * router_w[e,d] (+ router_bias[e]), softmax over the
 * E experts, the k_t largest (descending; exact ties to the lower expert id) and their
 * probabilities renormalised to sum to 1 ("Routage MoE entre GPU", router paragraph). The logits
 * that decide the selection are summed in fp64 (each bf16 x fp32 product is exact there), so the
 * ids and their order are those of an fp64 evaluation unless two logits lie within ~1e-12; the
 * weights are computed in fp64 and rounded once to fp32.
 *   hidden [T, d] bf16; router_w [E, d] fp32; router_bias [E] fp32 or NULL;
 *   k: experts per token when k_per_token is NULL (1 <= k <= min(E, k_max));
 *   k_per_token [T] int32 or NULL: per-token k_t in [1, k_max] (MoE-Prism's elastic k);
 *   out topk_ids [T, k_max] int32 and topk_w [T, k_max] fp32; slots j >= k_t hold -1 and 0.
 * A k_t outside [1, min(E, k_max)] is clamped and flags MOE_ERR_DEVICE_CHECK. */
int moe_route_topk(const moe_dims* dims, const uint16_t* hidden, const float* router_w,
                   const float* router_bias, int32_t k, const int32_t* k_per_token,
                   int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Grouping by expert: histogram of the routed (token, slot) pairs, exclusive prefix sum, and a
 * stable scatter so that routed rows are ordered by (expert ascending, token ascending)
 * ("Routage MoE entre GPU": only the selected experts process a token).
 *   topk_ids [T, k_max] int32 (slots with id -1 or j >= k_t are skipped);
 *   out expert_offsets [E+1] int32 (offsets[E] = R = number of routed rows),
 *       perm_token [T*k_max] int32 (token of routed row r, r < R),
 *       inv_row [T, k_max] int32 (routed row of (t, j); -1 for unused slots).
 * An id of -1 marks an unused slot (as the expert-parallel receiver pads its rows); any other
 * expert id outside [0, E) is skipped and flags MOE_ERR_DEVICE_CHECK. */
int moe_permute(const moe_dims* dims, const int32_t* topk_ids, int32_t k,
                const int32_t* k_per_token, int32_t* expert_offsets, int32_t* perm_token,
                int32_t* inv_row, void* ws, size_t ws_bytes, void* stream);

/* Grouped W8A8 FP8 expert FFN over the routed rows (megakernel page: W8A8 FP8 expert compute).
 * For every routed row r < R of expert e (expert_offsets[e] <= r < expert_offsets[e+1]) with
 * token t = perm_token[r]:
 *   s_t = amax_d |hidden[t,:]| / 448 (fp32; 1 if 0),  xq = e4m3(hidden[t,:] / s_t)
 *   h[j] = s_t * w13_scale[e,j] * sum_d xq[d] * w13[e,j,d]           j in [0, 2F)
 *   act[f] = silu(h[f]) * h[F+f]                                    (rows [0,F) gate, [F,2F) up)
 *   s2 = amax_f |act| / 448 (fp32; 1 if 0),  aq = e4m3(act / s2)
 *   expert_out[r,i] = s2 * w2_scale[e,i] * sum_f aq[f] * w2[e,i,f]
 *   hidden [T, d] bf16; w13 [E, 2F, d] e4m3; w13_scale [E, 2F] fp32; w2 [E, d, F] e4m3;
 *   w2_scale [E, d] fp32; expert_offsets [E+1]; perm_token [R];
 *   out expert_out [T*k_max, d] fp32 (rows >= R untouched); act_scale_out [T] fp32 or NULL (s_t).
 * w13 and w2 must be 16-byte aligned. Offsets that are not non-decreasing or exceed T*k_max
 * flag MOE_ERR_DEVICE_CHECK and nothing is computed. */
int moe_grouped_ffn_fp8(const moe_dims* dims, const uint16_t* hidden, const uint8_t* w13,
                        const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                        const int32_t* expert_offsets, const int32_t* perm_token,
                        float* expert_out, float* act_scale_out, void* ws, size_t ws_bytes,
                        void* stream);

/* Weighted combine in token order ("Routage MoE entre GPU": outputs multiplied by their routing
 * weights, summed, original token order restored):
 *   y[t,i] = bf16_rne( sum_{j: inv_row[t,j] >= 0} topk_w[t,j] * expert_out[inv_row[t,j], i]
 *                      + shared_out[t,i] )
 *   expert_out [T*k_max, d] fp32; topk_w, inv_row [T, k_max]; shared_out [T, d] fp32 or NULL;
 *   out y [T, d] bf16; y_f32 [T, d] fp32 or NULL (the sum before rounding). */
int moe_combine(const moe_dims* dims, const float* expert_out, const float* topk_w,
                const int32_t* inv_row, const float* shared_out, uint16_t* y, float* y_f32,
                void* stream);

/* The whole layer in one call: router, top-k, activation quantisation, permutation, grouped FP8
 * FFN (plus the shared expert with weight 1.0 when dims->F_shared > 0), combine. Arguments as in
 * the split entry points; w13_shared [2F, d], w13s_scale [2F], w2_shared [d, F], w2s_scale [d]
 * are required iff F_shared > 0. out y [T, d] bf16. dbg may be NULL. */
int moe_forward(const moe_dims* dims, const uint16_t* hidden, const float* router_w,
                const float* router_bias, int32_t k, const int32_t* k_per_token,
                const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                const float* w2_scale, const uint8_t* w13_shared, const float* w13s_scale,
                const uint8_t* w2_shared, const float* w2s_scale, uint16_t* y, void* ws,
                size_t ws_bytes, void* stream, const moe_debug_out* dbg);

/* Router top-k without a workspace, for callers that cannot allocate device memory: an engine
 * that has already handed all device memory to its own pools, or a step that runs where
 * allocating is not allowed. The pages describing the method have no counterpart to this entry
 * point; it returns the same routing decision as moe_route_topk (same arguments, minus the
 * workspace), computed with the CUDA-core router.
 *   Scratch: one fixed device array of MOE_NOALLOC_SCRATCH_BYTES owned by this library, which
 *   every GPU that loads the library keeps until the process exits. It holds the fp64 partial
 *   router logits, 8 * T * E * splits bytes (splits = the number of pieces d is cut into so that the
 *   logits kernel fills the GPU; none at all for E <= 32); a larger shape returns
 *   MOE_ERR_UNSUPPORTED and launches nothing.
 *   The first call on a device looks up the array's device address (with that device current);
 *   make that first call before any stream capture.
 *   Every call uses the same array, and each call overwrites the partial logits it reads, so
 *   nothing in it needs clearing. Calls that overlap on one GPU (on different streams, or from
 *   several host threads) race for it and can return wrong results: serialise them.
 *   A k_t outside [1, min(E, k_max)] is clamped without a report (there is no status word). */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
int moe_route_topk_noalloc(const moe_dims* dims, const uint16_t* hidden, const float* router_w,
                           const float* router_bias, int32_t k, const int32_t* k_per_token,
                           int32_t* topk_ids, float* topk_w, void* stream);

/* Expert-parallel dispatch ("Routage MoE entre GPU": a token's activations are sent to the GPUs
 * that hold its selected experts and the results are sent back; "Semantic Parallelism", section 1:
 * the all-to-all exchange of expert parallelism). The E experts are split over n_ranks GPUs in
 * contiguous blocks of E_local = E / n_ranks: rank r holds experts [r * E_local, (r+1) * E_local).
 * For every token t and every rank r that holds at least one of t's selected experts, one send
 * row is written; the rows are ordered by (rank ascending, token ascending), so the rows for rank
 * r are one contiguous segment of send_counts[r] rows. With kl = min(k_max, E_local):
 *   dims: T, d, E, k_max as for moe_route_topk (F must be valid; F_shared is ignored);
 *   n_ranks in [1, 32], dividing E;
 *   hidden [T, d] bf16; topk_ids, topk_w [T, k_max] (the output of moe_route_topk); k /
 *   k_per_token as in moe_permute;
 *   out send_hidden [T * min(n_ranks, k_max), d] bf16 (capacity; rows >= sum(send_counts) are
 *       untouched): send row i holds the hidden row of its token;
 *       send_ids [same rows, kl] int32: the local ids (e - r * E_local) of the token's experts on
 *       rank r in slot order, then -1;  send_w [same rows, kl] fp32: their routing weights, then 0;
 *       send_counts [n_ranks] int32: rows for each rank (also written when T == 0);
 *       slot_of [T, n_ranks] int32: the send row of (t, r), or -1;
 *       slot_w [T, n_ranks] fp32: 1 where slot_of >= 0, else 0.
 * On rank r the segment it receives from every source is a batch of tokens with kl local experts
 * each (-1 = unused slot): moe_permute, moe_grouped_ffn_fp8 and moe_combine (its y_f32 output,
 * E = E_local, k_max = kl) give the partial outputs, which go back to the sources in the same row
 * order; there moe_combine with k_max = n_ranks, inv_row = slot_of, topk_w = slot_w and the shared
 * expert's output as shared_out sums them into y. hidden and send_hidden must be 16-byte aligned;
 * ws: at least moe_workspace_bytes(dims) bytes, as for the other entry points (only its status
 * word is used). An expert id >= E, a k_t outside [0, k_max] or an expert selected twice for one
 * token flags MOE_ERR_DEVICE_CHECK; such ids are left out of the plan. */
int moe_ep_dispatch(const moe_dims* dims, int32_t n_ranks, const uint16_t* hidden,
                    const int32_t* topk_ids, const float* topk_w, int32_t k,
                    const int32_t* k_per_token, uint16_t* send_hidden, int32_t* send_ids,
                    float* send_w, int32_t* send_counts, int32_t* slot_of, float* slot_w,
                    void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8_MOE_H */
