/*
 * fp8_expert_ffn_b200 — forward pass of one fine-grained-FP8 Mixture-of-Experts
 * layer (dots3-note preview shape) on a B200 (sm_100a).
 *
 * The layer (transformers docs page "Dots 3 Note Preview", Dots3NoteTextConfig;
 * model card dots-studio/dots3-note-prev, "Model Overview"): hidden size H,
 * E routed SwiGLU experts plus 1 shared expert, top-K routing with the K
 * weights renormalised (norm_topk_prob), expert FFN width F, no biases.
 * Weights are a fine-grained FP8 checkpoint (transformers PR #47844, "What
 * does this PR do?"): E4M3 codes with one fp32 scale per 128 x 128 block;
 * activations are quantised at run time per token per 128 channels.
 *
 * Readings taken where the pages are silent (all fixed here):
 *   - router logits are FP32; top-K by logit (equivalently by softmax
 *     probability), ties to the lower expert id; the K weights are the
 *     softmax over the K selected logits (= softmax over all E experts
 *     renormalised over the selection), times routed_scaling; the router
 *     variants of the config schema (n_group / topk_group, norm_topk_prob
 *     off, a selection-only bias) are described at moe_route;
 *   - the K slots of a token are listed in ascending expert id;
 *   - E4M3 is the OCP "FN" flavour (max 448, no infinities); quantisation
 *     is s = fp32(amax)/448 (IEEE fp32 divide), q = E4M3_RNE_satfinite(v/s)
 *     (IEEE fp32 divide); an all-zero group gives s = 0 and q = 0;
 *   - scales are dequantisation multipliers: value ~ decode(q) * s;
 *   - the SwiGLU output h is quantised the same way from fp32, per row per
 *     128 channels, before the down projection;
 *   - the shared expert (index E in every weight array) is added with
 *     weight 1; its rows follow the routed rows in token order.
 *
 * Conventions for every call:
 *   - all data pointers are DEVICE pointers owned by the caller; the library
 *     never allocates after moe_layer_create, which allocates, per handle:
 *     a 4-byte device status word; the router weight's three-term bf16
 *     split, 3*E*H*2 bytes; the split-K partials of the down GEMM,
 *     8*256*H*4 bytes (42 MB at H = 5120); and, when a router bias is
 *     given, an E*4-byte copy of it. Nothing else is allocated (the one
 *     file-scope array of moe_permute_noalloc, below, is part of the
 *     library image, not an allocation), except by moe_ep_comm_create,
 *     which allocates the expert-parallel exchange buffers it describes;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default);
 *     calls are asynchronous on that stream and never synchronise the host;
 *     the kernels are chained with programmatic dependent launch (each one's
 *     set-up overlaps the previous kernel's tail; stream order is kept);
 *   - bf16 tensors are passed as uint16_t bit patterns;
 *   - row strides (ld*) are in elements; every byte stride must be a
 *     multiple of 16 and every base pointer 16-byte aligned, else
 *     MOE_ERR_MISALIGNED;
 *   - T = 0 is a no-op that returns MOE_OK;
 *   - inputs must be finite; NaN/Inf inputs give unspecified results;
 *   - errors found by the host are returned before anything is launched;
 *     errors found on the device (an expert id out of range, a repeated
 *     expert in one token's slots, a pipeline wait that timed out) set the
 *     layer's device status word, skip the offending work and are read back
 *     with moe_get_device_status.
 *
 * Row count: R = T*K routed rows plus T*S shared rows (S = n_shared, 0 or 1),
 * rows = T*(K+S). A layer with n_shared = 0 has no group-E rows; one with
 * n_routed = 1, top_k = 1, n_shared = 0 is a dense FP8 FFN (weight 1).
 */
#ifndef FP8_EXPERT_FFN_MOE_H
#define FP8_EXPERT_FFN_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size or count */
  MOE_ERR_MISALIGNED = 2,   /* pointer or byte stride not 16-byte aligned */
  MOE_ERR_UNSUPPORTED = 3,  /* a layer shape this build does not handle */
  MOE_ERR_WORKSPACE = 4,    /* workspace smaller than moe_workspace_size */
  MOE_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE = 6        /* a kernel reported bad data or a timed-out wait */
} moe_status;

/* Layer description; mirrors Dots3NoteTextConfig (transformers docs page
 * "Dots 3 Note Preview"): hidden_size, n_routed_experts, n_shared_experts,
 * num_experts_per_tok, moe_intermediate_size, shared_experts_intermediate_size,
 * routed_scaling_factor, norm_topk_prob, n_group, topk_group; block = the
 * 128 x 128 weight block edge of transformers PR #47844. This build requires:
 * hidden % 128 == 0, 128 <= hidden <= 16384, 1 <= n_routed <= 256, n_shared
 * 0 or 1, 1 <= top_k <= min(8, n_routed), 1 <= ffn <= 16384, shared_ffn ==
 * ffn when n_shared = 1, block == 128, norm_topk 0 or 1, 1 <= n_group <= 32
 * with n_routed % n_group == 0, 1 <= topk_group <= n_group and top_k <=
 * topk_group * n_routed / n_group; otherwise MOE_ERR_UNSUPPORTED. */
typedef struct {
  int hidden;           /* H */
  int n_routed;         /* E */
  int n_shared;         /* S: 0 or 1 */
  int top_k;            /* K */
  int ffn;              /* F */
  int shared_ffn;       /* must equal ffn when n_shared = 1 */
  int block;            /* must be 128 */
  float routed_scaling; /* multiplies the routed weights */
  int norm_topk;        /* 1: the K weights are renormalised to sum 1 */
  int n_group;          /* experts e of group e / (E / n_group); 1 = ungrouped */
  int topk_group;       /* groups a token may draw its K experts from */
} moe_layer_desc;

/* Caller-owned device weights; they must outlive the layer handle. Expert
 * index E is the shared expert (present when n_shared = 1; S = n_shared).
 * Codes are E4M3 bytes; scales are fp32 dequantisation multipliers, one per
 * 128 x 128 block (edge blocks cover the real rows/columns only):
 *   w_gate, w_up : [E+S][F][ld_h]   bytes, ld_h >= H, ld_h % 16 == 0
 *   s_gate, s_up : [E+S][ceil(F/128)][H/128]
 *   w_down       : [E+S][H][ld_f]   bytes, ld_f >= F, ld_f % 16 == 0
 *   s_down       : [E+S][H/128][ceil(F/128)]
 *   router_w     : [E][H] fp32, row-major
 *   router_bias  : [E] fp32 or NULL; selection-only bias of routers balanced
 *                  by a bias instead of an auxiliary loss (added to the
 *                  softmax probabilities to choose experts, not to weigh them)
 * The six expert arrays may all be NULL (then ld_h/ld_f are ignored): a
 * routing-only handle for route, permute and combine, as the source side of
 * expert parallelism uses (see moe_ep_regroup). */
typedef struct {
  const uint8_t* w_gate;
  const uint8_t* w_up;
  const uint8_t* w_down;
  const float* s_gate;
  const float* s_up;
  const float* s_down;
  const float* router_w;
  int ld_h;
  int ld_f;
  const float* router_bias;
} moe_weights;

typedef struct moe_layer_s* moe_layer_t;

/* Static description of a status code (never NULL). Library plumbing: no
 * counterpart on the pages. */
const char* moe_status_string(moe_status s);

/* Creates the handle of one MoE layer of the shape moe_layer_desc describes
 * (Dots3NoteTextConfig, transformers docs page "Dots 3 Note Preview").
 * Validates desc/weights, queries the current device (must be sm_100),
 * encodes the weights' TMA descriptors once, allocates the 4-byte device
 * status word and writes the router weight as three bf16 terms
 * (hi + mid + lo == router_w exactly; the tensor-core router multiplies the
 * bf16 input by each term) and copies router_bias when given. It also
 * allocates 8 x 256 x H fp32 of split-K partials (8 MB per 1024 of H): when a
 * batch gives the down GEMM fewer output tiles than half the SMs (a layer
 * with one or two groups at up to 256 rows), its K blocks are split over
 * CTAs and a second kernel adds the partials in a fixed order, so calls on
 * one handle must not overlap on the GPU. Synchronises the device once. On
 * error *out is NULL. The router weight and bias are read only here: a later
 * change to either needs a new handle. */
moe_status moe_layer_create(const moe_layer_desc* desc, const moe_weights* w, moe_layer_t* out);

/* Frees the handle (not the caller's weights). NULL is accepted. Library
 * plumbing: no counterpart on the pages. */
moe_status moe_layer_destroy(moe_layer_t layer);

/* Bytes of workspace that moe_layer_forward needs for T tokens; it also
 * covers the scratch of moe_route, moe_permute, moe_expert_ffn and the
 * expert-parallel calls. For a routing-only handle it is the route and
 * permutation scratch alone (a few bytes per token per expert). 0 on bad
 * input. Library plumbing: no counterpart on the pages. */
size_t moe_workspace_size(moe_layer_t layer, int T);

/* Router: logits = x . router_w^T in FP32, p = softmax over the E experts,
 * selection score s = p + router_bias (s orders like the logits when there
 * is no bias); with n_group > 1 only the topk_group groups with the best
 * member s (ties to the lower group) are eligible; top-K eligible experts by
 * s (ties to the lower id, slots in ascending id); weights = the selected p
 * (renormalised to sum 1 when norm_topk) times routed_scaling. Dots3NoteTextConfig
 * n_group / topk_group / norm_topk_prob / routed_scaling_factor; the pages
 * give no group-scoring rule, a group is scored by its best member.
 *   x             [T][ldx] bf16, ldx >= H
 *   topk_idx      [T][K] int32 (out)
 *   topk_w        [T][K] fp32  (out)
 *   router_logits [T][E] fp32  (out, may be NULL)
 *   ws, ws_bytes  scratch, at least moe_workspace_size(layer, T) bytes    */
moe_status moe_route(moe_layer_t layer, const uint16_t* x, int T, int ldx, int32_t* topk_idx, float* topk_w,
                     float* router_logits, void* ws, size_t ws_bytes, void* stream);

/* Token permutation by expert with fused activation quantisation.
 * On one GPU this is the "dispatch" of the DeepEP transport that the SGLang
 * cookbook "Dots3-Note" names for the MoE layer ("2. Configuration Tips");
 * the activations are quantised dynamically, per token per 128 channels, to
 * E4M3 (transformers PR #47844, "What does this PR do?").
 * Counting sort of the T*K (token, slot) pairs by expert id, stable in token
 * order; with n_shared = 1, group E (shared expert) holds rows [T*K, T*K+T)
 * in token order (with n_shared = 0 it is empty).
 *   topk_idx  [T][K] int32 (in); ids outside [0,E) or repeated within a
 *             token set MOE_ERR_DEVICE and are skipped
 *   offsets   [E+2] int32 (out): group g is rows [offsets[g], offsets[g+1])
 *   perm      [rows] int32 (out): row -> token
 *   inv       [T][K] int32 (out): (token, slot) -> row
 *   xq        [rows][H] E4M3 bytes (out): x of the row's token, quantised
 *             per 128 channels
 *   xs        [H/128][rows] fp32 (out, group-major): the row's scales      */
moe_status moe_permute(moe_layer_t layer, const uint16_t* x, int T, int ldx, const int32_t* topk_idx,
                       int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs, void* ws,
                       size_t ws_bytes, void* stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: a serving runtime that has handed all free HBM to its own pools
 * (KV cache, weights) and owns no spare buffer to lend, a caller that is
 * capturing a stream into a CUDA graph in a mode where cudaMalloc is not
 * permitted, or a latency-critical path where cudaMalloc's implicit device
 * synchronisation is not acceptable. The pages describe no such call; it
 * exists only for those callers.
 *   Arguments and outputs are those of moe_permute (minus ws/ws_bytes).
 *   T must be <= MOE_NOALLOC_MAX_TOKENS; larger T returns
 *   MOE_ERR_UNSUPPORTED before anything is launched (use moe_permute).
 *   The scratch is one library-owned device array per GPU (about 257 KB,
 *   held until the process exits), found with cudaGetSymbolAddress on the
 *   first call made on each device: make that first call before capturing
 *   any stream. Every call on a device shares that array and it keeps the
 *   last call's contents (each call clears what must start at zero), so
 *   calls whose kernels overlap on the GPU (other streams, other host
 *   threads) race on it and must be serialised by the caller.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define MOE_NOALLOC_MAX_TOKENS 4096
moe_status moe_permute_noalloc(moe_layer_t layer, const uint16_t* x, int T, int ldx, const int32_t* topk_idx,
                               int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs,
                               void* stream);

/* Grouped expert FFN over the permuted rows. The experts are SwiGLU FFNs
 * (Dots3NoteTextConfig of the transformers docs page "Dots 3 Note Preview":
 * hidden_act silu, mlp_bias False, moe_intermediate_size 1536; model card
 * dots-studio/dots3-note-prev, "Model Overview": FFN 1536 per expert) with
 * fine-grained FP8 weights (transformers PR #47844, "What does this PR do?":
 * E4M3, one scale per 128 x 128 block, dynamic activations). For each group
 * g and row r in it, h = silu(xq Wg_g^T) * (xq Wu_g^T) with per-128-K-block scale promotion,
 * h quantised per 128 channels (E4M3, fp32 scale), y = h Wd_g^T in FP32,
 * rounded to bf16.
 *   xq, xs, offsets as written by moe_permute for the same T
 *   y         [rows][H] bf16 (out)                                         */
moe_status moe_expert_ffn(moe_layer_t layer, const uint8_t* xq, const float* xs, const int32_t* offsets, int T,
                          uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* The two halves of moe_expert_ffn, for callers that keep h themselves
 * (SwiGLU experts of Dots3NoteTextConfig with the fine-grained FP8 weights
 * of transformers PR #47844, as cited at moe_expert_ffn).
 * moe_gate_up: h = quantise(silu(xq Wg^T) * (xq Wu^T)) per row per 128
 * channels.
 *   h   [rows][ceil(F/128)*128] E4M3 bytes (out); channels >= F are zero
 *   hs  [ceil(F/128)][rows] fp32 (out, group-major)
 * moe_down: y = h Wd^T (FP32 with block-scale promotion) rounded to bf16.
 *   y   [rows][H] bf16 (out)
 * Neither needs a workspace; both read the groups from the device-side
 * offsets written by moe_permute. */
moe_status moe_gate_up(moe_layer_t layer, const uint8_t* xq, const float* xs, const int32_t* offsets, int T,
                       uint8_t* h, float* hs, void* stream);
moe_status moe_down(moe_layer_t layer, const uint8_t* h, const float* hs, const int32_t* offsets, int T,
                    uint16_t* y, void* stream);

/* moe_gate_up / moe_down over an explicit row count instead of T (the rows
 * of an expert-parallel owner: the routed rows it received plus its own
 * shared rows; see moe_ep_regroup). The SwiGLU experts of
 * Dots3NoteTextConfig with the fine-grained FP8 weights of transformers
 * PR #47844, as cited at moe_expert_ffn.
 *   rows     the permuted row count: xq/h have `rows` rows and the scale
 *            arrays are group-major with group stride `rows`
 *   offsets  [E+2] group offsets over those rows (group E: shared rows) */
moe_status moe_grouped_gate_up(moe_layer_t layer, const uint8_t* xq, const float* xs, const int32_t* offsets,
                               int rows, uint8_t* h, float* hs, void* stream);
moe_status moe_grouped_down(moe_layer_t layer, const uint8_t* h, const float* hs, const int32_t* offsets, int rows,
                            uint16_t* y, void* stream);

/* Expert parallelism (SGLang cookbook "Dots3-Note", "2. Configuration
 * Tips": the MoE layer served with expert parallelism across the GPUs of a
 * node, DeepEP carrying the dispatch and combine all-to-alls). The routed
 * experts are split into `ranks` contiguous blocks of El experts (rank p
 * owns experts [p*El, (p+1)*El)); the shared expert and the router are on
 * every rank. A source rank routes and permutes its own tokens with a
 * routing-only handle (moe_layer_create with all six expert arrays NULL:
 * route, permute and combine work, the GEMM calls return
 * MOE_ERR_INVALID_ARG); its rows for rank p are then one contiguous range.
 * An owner rank runs the GEMMs with a handle of its El experts plus the
 * shared expert (n_routed = El). These three calls move rows around the two
 * exchanges (which the caller performs, e.g. NCCL all-to-all); with
 * seg_counts[s*El + e] = the rows sender s sent for local expert e and
 * n_recv = their sum:
 * moe_ep_pack_scales (source side, route handle): xs_rows [T*K][H/128] fp32
 *   = the routed rows' scales of xs [H/128][T*(K+S)] made row-major, so a
 *   destination's rows and their scales are contiguous.
 * moe_ep_regroup (owner side, expert handle): recv_q [n_recv][H] bytes and
 *   recv_s [n_recv][H/128] fp32 in sender-major order (sender 0's rows for
 *   local experts 0..El-1, then sender 1's, ...), plus the owner's own
 *   shared rows (own_q/own_s: its moe_permute outputs for T tokens, rows
 *   [T*K, T*K + T*S)) -> out_q [n_recv + T*S][H] expert-major with the shared
 *   rows last, out_s [H/128][n_recv + T*S] group-major, out_offsets [El+2]
 *   (for moe_grouped_gate_up / moe_grouped_down with rows = n_recv + T*S).
 * moe_ep_unregroup (owner side, expert handle): y_g [n_recv + T*S][H] bf16
 *   (the grouped GEMM output) -> y_send [n_recv][H] in the sender-major
 *   order of recv_q (for the return exchange) and the shared rows into
 *   y_own rows [T*K, T*K + T*S) (the owner's own moe_combine input).
 * seg_counts is a device array; ranks * El <= 2048. */
moe_status moe_ep_pack_scales(moe_layer_t route_layer, const float* xs, int T, float* xs_rows, void* stream);
moe_status moe_ep_regroup(moe_layer_t expert_layer, int ranks, const int32_t* seg_counts, int n_recv,
                          const uint8_t* recv_q, const float* recv_s, const uint8_t* own_q, const float* own_s, int T,
                          uint8_t* out_q, float* out_s, int32_t* out_offsets, void* stream);
moe_status moe_ep_unregroup(moe_layer_t expert_layer, int ranks, const int32_t* seg_counts, int n_recv,
                            const uint16_t* y_g, int T, uint16_t* y_send, uint16_t* y_own, void* stream);

/* Expert parallelism over peer memory: the dispatch and combine of the
 * DeepEP transport (SGLang cookbook "Dots3-Note", "2. Configuration Tips")
 * done by the library's own kernels, with no all-to-all of rows. The
 * dispatch kernel quantises each routed row and stores it straight into
 * the receive buffer of its expert's owner (a peer GPU's memory over
 * NVLink, through a CUDA IPC mapping), at the row the owner's grouped GEMMs
 * read it from; the combine kernel reads the owners' output rows back the
 * same way. The caller exchanges only the E+2 offsets of every rank (an
 * all-gather) and orders the phases with two barriers (a kernel never waits
 * on another rank). Per forward, on every rank r of P:
 *   1. moe_route (route handle), then moe_ep_plan -> offsets [E+2];
 *   2. all-gather the offsets -> all_offsets [P][E+2] (rank order);
 *   3. moe_ep_dispatch -> rows into the owners' buffers, inv_ep, and this
 *      rank's group_offsets [El+2] as an owner;
 *   4. barrier (every rank's dispatch complete);
 *   5. moe_grouped_gate_up / moe_grouped_down (expert handle) on this
 *      rank's buffers (moe_ep_comm_buffers) with group_offsets and
 *      rows = capacity;
 *   6. barrier (every owner's y complete);
 *   7. moe_ep_combine -> out [T][H].
 * The next forward's step 2 keeps a rank from overwriting buffers that a
 * slower rank still reads.
 *
 * Owner p's buffer holds, for its local experts e = 0..El-1 in turn, the
 * rows from sender 0, 1, ..., P-1 (each sender's in token order), then its
 * own T*S shared rows: the rows a single-GPU forward would give those
 * experts, regrouped. `capacity` rows bound every owner's total; a forward
 * whose rows for some owner exceed it dispatches nothing on any rank, sets
 * MOE_STATUS_EP_OVERFLOW and writes zero group offsets. */
typedef struct moe_ep_comm_s* moe_ep_comm_t;

#define MOE_EP_HANDLE_BYTES 64   /* one rank's exported buffer handle */

/* Allocates this rank's exchange buffers on the current device (one
 * allocation: codes [capacity][H] u8, scales [H/128][capacity] fp32, output
 * rows [capacity][H] bf16) and the device tables of the P ranks' buffers.
 * `layer` gives H (any handle of the layer). 1 <= ranks <= 64,
 * 0 <= rank < ranks, 1 <= capacity <= 2^20. Library plumbing: no
 * counterpart on the pages. */
moe_status moe_ep_comm_create(moe_layer_t layer, int rank, int ranks, int capacity, moe_ep_comm_t* out);
/* The handle another process passes to moe_ep_comm_connect to map this
 * rank's buffers (cudaIpcGetMemHandle of the allocation). Library
 * plumbing: no counterpart on the pages. */
moe_status moe_ep_comm_export(moe_ep_comm_t comm, unsigned char handle[MOE_EP_HANDLE_BYTES]);
/* Maps every other rank's buffers from `handles` ([ranks][MOE_EP_HANDLE_BYTES],
 * in rank order; this rank's own entry is not used) and fills the tables.
 * Peers must have been created with the same ranks, capacity and H.
 * Library plumbing: no counterpart on the pages. */
moe_status moe_ep_comm_connect(moe_ep_comm_t comm, const unsigned char* handles);
/* Emulated ranks in one process on one device: comms[0..ranks) (rank i at
 * index i) use one another's buffers directly. Library plumbing: no
 * counterpart on the pages. */
moe_status moe_ep_comm_connect_local(moe_ep_comm_t* comms, int ranks);
/* This rank's own buffers (device pointers): codes, scales, output rows.
 * Library plumbing: no counterpart on the pages. */
moe_status moe_ep_comm_buffers(moe_ep_comm_t comm, uint8_t** recv_q, float** recv_s, uint16_t** y);
/* Unmaps the peers' buffers and frees this rank's (synchronises the device;
 * call it on every rank together, after the last forward). Library
 * plumbing: no counterpart on the pages. */
moe_status moe_ep_comm_destroy(moe_ep_comm_t comm);

/* Step 1 of the expert-parallel forward of the SGLang cookbook
 * "Dots3-Note" ("2. Configuration Tips"): the plan of the permutation of
 * this rank's T tokens (route handle): offsets [E+2] as moe_permute gives
 * them (offsets[E] = T*K routed rows, offsets[E+1] = offsets[E] + T*S),
 * and the token bitmap and
 * its prefixes in `ws` (moe_workspace_size(route_layer, T) bytes), which
 * moe_ep_dispatch reads: pass it the same workspace, unchanged. T = 0 writes
 * zero offsets. */
moe_status moe_ep_plan(moe_layer_t route_layer, const int32_t* idx, int T, int32_t* offsets, void* ws,
                       size_t ws_bytes, void* stream);
/* Step 3, the DeepEP "dispatch" of the SGLang cookbook "Dots3-Note"
 * ("2. Configuration Tips") (route handle; comm connected; route_layer
 * n_routed divisible by the comm's ranks): quantises x [T][ldx] bf16 per
 * token per 128 channels (as moe_permute) and writes routed row (t, k)
 * into the buffer of expert
 * idx[t][k]'s owner and t's shared row into this rank's; inv_ep [T][K] =
 * the row in the owner's buffer (-1 for a skipped slot; the owner is
 * idx[t][k] / El); group_offsets [El+2] = this rank's offsets as an owner
 * (shared rows from group_offsets[El]). all_offsets [ranks][E+2] is every
 * rank's moe_ep_plan output. Runs with T = 0 too (it still writes
 * group_offsets). Offsets that are not ascending dispatch nothing (zero
 * group offsets, inv_ep all -1); rows of this rank beyond its own entry of
 * all_offsets are skipped (inv_ep -1); both set MOE_STATUS_BAD_PLAN. No
 * store leaves the owners' buffers. */
moe_status moe_ep_dispatch(moe_layer_t route_layer, moe_ep_comm_t comm, const uint16_t* x, int T, int ldx,
                           const int32_t* idx, const int32_t* all_offsets, int32_t* inv_ep, int32_t* group_offsets,
                           void* ws, size_t ws_bytes, void* stream);
/* Step 7, the DeepEP "combine" of the SGLang cookbook "Dots3-Note"
 * (route handle): out [T][ldo] bf16 = sum over slots k of w[t][k]
 * times row inv_ep[t][k] of the owner's output rows (slot order, FP32),
 * plus this rank's shared row group_offsets[El] + t, rounded once to bf16:
 * the same arithmetic as moe_combine. */
moe_status moe_ep_combine(moe_layer_t route_layer, moe_ep_comm_t comm, const int32_t* idx, const int32_t* inv_ep,
                          const float* w, const int32_t* group_offsets, int T, uint16_t* out, int ldo, void* stream);

/* Weighted combine of the routed experts' outputs plus the shared expert's
 * (Dots3NoteTextConfig: norm_topk_prob, routed_scaling_factor,
 * n_shared_experts 1), the "combine" of the DeepEP transport of the SGLang
 * cookbook "Dots3-Note" ("2. Configuration Tips") done as a gather on one GPU:
 * out[t] = bf16_RNE( sum_k topk_w[t,k] * y[inv[t,k]] + S * y[T*K + t] ), FP32
 * sum in slot order, shared row (when n_shared = 1) last.
 *   out [T][ldo] bf16, ldo >= H                                            */
moe_status moe_combine(moe_layer_t layer, const uint16_t* y, const int32_t* inv, const float* topk_w, int T,
                       uint16_t* out, int ldo, void* stream);

/* The whole MoE layer of the dots3-note language model (Dots3NoteTextConfig;
 * model card dots-studio/dots3-note-prev, "Model Overview": 256 routed + 1
 * shared experts, top-8):
 * moe_route -> moe_permute -> moe_expert_ffn -> moe_combine,
 * with every intermediate in the workspace. */
moe_status moe_layer_forward(moe_layer_t layer, const uint16_t* x, int T, int ldx, uint16_t* out, int ldo,
                             void* ws, size_t ws_bytes, void* stream);

/* Bits of the device status word (moe_get_device_status's `detail`). */
#define MOE_STATUS_BAD_EXPERT 0x1u   /* an expert id outside [0, E) was skipped */
#define MOE_STATUS_DUP_EXPERT 0x2u   /* an expert repeated in one token's slots */
#define MOE_STATUS_WAIT_TIMEOUT 0x4u /* a pipeline wait gave up; that launch's outputs are incomplete */
#define MOE_STATUS_BAD_PLAN 0x8u     /* group offsets not ascending within [0, rows]; no GEMM work done */
#define MOE_STATUS_EP_OVERFLOW 0x10u /* an owner's rows exceed its exchange buffer; nothing dispatched */
#define MOE_STATUS_BOUNDS 0x20u      /* bounds-checked build only: a row index taken from the inputs
                                      (inv, offsets, segment counts) fell outside its buffer; the
                                      access was skipped */

/* Synchronises `stream`, returns MOE_ERR_DEVICE if any kernel of this layer
 * flagged an error since the last call (and clears the flag), else MOE_OK.
 * If `detail` is not NULL it receives the raw status bits (MOE_STATUS_*).
 * Library plumbing: no counterpart on the pages. */
moe_status moe_get_device_status(moe_layer_t layer, void* stream, uint32_t* detail);

/* Number of kernels moe_layer_forward launches for T tokens (route 2,
 * permute 2 when the E x ceil(T/32)-word token bitmap fits in 8192 words,
 * else 4, gate/up 1, down 1 plus 1 when its K blocks are split, combine 1);
 * 0 for T = 0 or bad arguments. Library plumbing: no counterpart on the
 * pages. */
int moe_kernels_per_forward(moe_layer_t layer, int T);

/* Test hook for failure detection (library plumbing: no counterpart on the
 * pages). Arms a one-shot stall for the next grouped-GEMM launch on this
 * handle (moe_gate_up, moe_down, or those inside moe_expert_ffn and
 * moe_layer_forward): the first CTA's TMA producer skips its first pipeline
 * stage, so the MMA issuer's wait for it can never complete, and every
 * pipeline wait of that launch gives up after wait_limit_ns (> 0) instead of
 * the normal 1 s. The kernel then records MOE_STATUS_WAIT_TIMEOUT, every
 * role leaves its loop, the producer waits (bounded) for the copies it did
 * issue, and the TMEM is freed; that launch's outputs are incomplete, the
 * next launch runs normally. Nothing traps or hangs. */
moe_status moe_test_inject_stall(moe_layer_t layer, unsigned long long wait_limit_ns);

/* Test hook for the grouped FP8 GEMM with per-128-K-block promotion (the
 * 128 x 128 weight blocks and per-token activation scales of transformers
 * PR #47844, "What does this PR do?"): writes the promoted FP32 accumulators
 * instead of the fused epilogue.
 *   which = 0: gate/up GEMM; a = xq [rows][H], as = [H/128][rows];
 *              out [rows][2*ceil(F/128)*128] fp32, channel block c of the
 *              gate result at columns [256c, 256c+128), of the up result at
 *              [256c+128, 256c+256)
 *   which = 1: down GEMM; a = h [rows][ceil(F/128)*128] (bytes beyond F are
 *              ignored), as = [ceil(F/128)][rows]; out [rows][H] fp32
 * offsets gives the groups as in moe_permute; rows = T*(K+S). */
moe_status moe_test_grouped_gemm_f32(moe_layer_t layer, int which, const uint8_t* a, const float* as,
                                     const int32_t* offsets, int T, float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8_EXPERT_FFN_MOE_H */
