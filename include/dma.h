/*
 * dma.h -- C ABI of the Dynamic Mask Attention (DMA) hot path for NVIDIA B200 (sm_100a).
 *
 * The method is the one described on the page "Trainable Dynamic Mask Sparse Attention:
 * Bridging Efficiency and Effectiveness in Long-Context Language Models" (Hugging Face blog
 * "dmattn", arXiv 2508.02124).  Three steps run on the GPU:
 *
 *   1. gate       delta = exp(softplus(v Delta) * A)           (section "Dynamic Sparse Mask
 *                                                              Generation", delta equation)
 *   2. mask       m_t = f(top_w(delta + m_c^t))                (same section, m_t equation)
 *   3. attention  o_t = softmax(q_t k^T / sqrt(d) + m_t) v     (section "Efficient Sparse
 *                                                              Attention Computation", o_t
 *                                                              equation), forward and backward
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every call is asynchronous on the caller's CUDA stream (`stream` is a cudaStream_t passed
 *    as void*; NULL is the legacy default stream).  No call allocates device memory or keeps a
 *    pointer after its stream work completes, and none synchronises the host except
 *    dma_check_device_status, which reads the workspace status word back.  The library's only
 *    global state is a host-side record, per kernel and device, that the kernel's shared-memory
 *    limit has been raised (kept behind a mutex), and the fixed scratch array of
 *    dma_gate_bwd_noalloc.  Calls on different streams may run concurrently when their buffers
 *    (including workspaces) are distinct; dma_gate_bwd_noalloc calls must not overlap.
 *  - All pointers are device pointers, 16-byte aligned, to dense row-major (C-contiguous)
 *    tensors with the layouts given per argument.  The caller owns every buffer.
 *  - Arguments are validated before anything is launched.  On any error nothing is launched
 *    and no output is touched, except DMA_ERR_CUDA, which reports a failed launch (outputs are
 *    then unspecified).
 *  - Outputs are fully overwritten, never accumulated into.
 *  - Tensor names follow the page: Q, K, V, Delta (the sampling weights), A (per-head
 *    selective control), delta (the dynamic weights), O, LSE.
 *
 * Readings of points the page leaves open (also listed in the project design notes):
 *  - tau is softplus.  The value vector of key position j is the concatenation of its Hkv
 *    value heads (length Hkv*d); Delta is [Hkv*d, H]; delta has one value per query head.
 *  - The mask is ADDED to the scaled scores: a selected key j contributes +delta_j, any
 *    other key -inf.  The scale multiplies q k^T only.
 *  - top-w orders keys by delta descending and breaks ties toward the lower key index
 *    (-0.0 compares equal to +0.0).  A query at position t with t+1 <= w keeps all of its
 *    causal keys; the query's own key competes like any other.  NaN gate values are not
 *    supported (their selection is unspecified).
 *  - In the backward pass the selection is a constant: gradients reach delta only through
 *    the additive bias of selected pairs.  Masked pairs get exactly zero gradient (section
 *    "Theoretical Guarantees for Safe Computation Skipping").
 *  - LSE is the natural logarithm of the softmax denominator sum_j exp(s_tj).
 */
#ifndef DMA_H_
#define DMA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DMA_ABI_VERSION 2

/* Query rows per block of the mask encoding and of the attention kernels. */
#define DMA_BLOCK_Q 128

typedef enum {
  DMA_OK = 0,
  DMA_ERR_INVALID_ARG = 1, /* a NULL/misaligned pointer, an inconsistent or out-of-range size */
  DMA_ERR_UNSUPPORTED = 2, /* a valid request outside what the kernels implement (see limits) */
  DMA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than dma_workspace_size() */
  DMA_ERR_CUDA = 4,        /* a CUDA launch failed (cudaGetLastError after the launch) */
  DMA_ERR_TIMEOUT = 5      /* a device-side bounded wait gave up (see dma_check_device_status) */
} dma_status_t;

typedef enum {
  DMA_BF16 = 0, /* Q, K, V, Delta, dO, O, dQ, dK, dV stored as bfloat16 */
  DMA_F32 = 1   /* stored as float32 (the gate then runs on float32 values; the attention
                   kernels round Q, K, V to bfloat16 in their load stage) */
} dma_dtype_t;

/*
 * Problem description.
 *   B      batch
 *   H      query heads;  Hkv key/value heads, H % Hkv == 0 (grouped-query attention:
 *          query head h reads key/value head h / (H / Hkv))
 *   N      key length (sequence length, or cache length for decode)
 *   Nq     query rows, 1 <= Nq <= N; the queries are the last Nq positions, query row i at
 *          position N - Nq + i: Nq == N (prefill / training), Nq == 1 (decode), otherwise a
 *          chunk of queries over a longer cache (chunked prefill: the selection still runs over
 *          all N keys; the block lists and the attention cover the blocks from position N - Nq
 *          on; dma_attn_bwd needs Nq == N)
 *   d      head dimension, 64 or 128
 *   w      window of the top-w selection, w >= 1 (w >= N keeps every causal key)
 *   scale  multiplier of q k^T; a value <= 0 selects 1/sqrt(d)
 *   dtype  a dma_dtype_t
 *   flags  0, or DMA_FLAG_FORWARD_ONLY: a problem whose forward is not followed by a backward (inference
 *          prefill): dma_attn_fwd then keeps nothing for a backward in the workspace (see dma_attn_fwd)
 *          and dma_attn_bwd returns DMA_ERR_UNSUPPORTED.  Other bits are reserved (DMA_ERR_INVALID_ARG).
 *   w_heads  NULL (every head selects with window w), or a device array of H int32 windows, one per
 *          query head ("adaptive window sizing", section "Future Directions" of the page: the
 *          window adapted per head, here supplied by the caller): head h selects with window
 *          w_heads[h].  The kernels clamp each value to [1, w], so w must be the largest of them: it
 *          sizes the workspace.  Every row of head h then keeps min(t+1, w_heads[h]) keys; the mask
 *          encoding, the lists and the attention are otherwise unchanged.  The array is read on the
 *          device by dma_topk_mask, dma_topk_append and the decode attention, and must hold the
 *          same values for every call of one problem.
 *
 * Limits of this implementation (DMA_ERR_UNSUPPORTED beyond them): prefill/training
 * N <= 16384; decode N <= 1<<24 and min(w, N) <= 4096 * d; B*H <= 65535; d in {64, 128};
 * dma_gate, dma_gate_bwd and dma_gate_bwd_noalloc: H <= 64.
 */
#define DMA_FLAG_FORWARD_ONLY 1

typedef struct {
  int32_t B, H, Hkv, N, Nq, d, w;
  float scale;
  int32_t dtype;
  int32_t flags;
  const int32_t* w_heads;
} dma_params_t;

/*
 * Workspace layout.  The workspace is one caller-allocated device buffer of at least
 * dma_workspace_size() bytes, passed to every call of one problem.  Its leading regions are
 * part of the ABI so that callers and tests can read the mask encoding:
 *
 *   off_status  int32 device status word (0 = ok): kernels OR an error code into it (a bounded
 *               wait that gave up, an internal consistency check that failed).  Its content in a
 *               new workspace is undefined: clear it once with dma_clear_device_status.
 *   off_counts  int32 [B, H, n_blocks, 2]: per query block, (n_full, n_live) (with Nq < N only
 *               the blocks of pairs of blocks that hold a query row are written).
 *   off_lists   int32 [B, H, n_blocks, list_cap]: the live keys of each query block
 *               [t0, t1), t1 = min(t0 + DMA_BLOCK_Q, N): first the n_full "full" keys, selected
 *               by every row of the block (j <= t0 and e_j >= t1), then the partial ones (at
 *               most 2*DMA_BLOCK_Q); each group in ascending key order.  Entries past n_live
 *               are unspecified.
 *   off_sel     decode only: int32 [B, H, sel_len] selected keys of the query, ascending:
 *               sel_len = min(w, N), every row full; with w_heads, sel_len = w and row (b, h)
 *               holds min(w_heads[h], N) keys (the rest unspecified), so that the row stride
 *               stays the same as keys are appended.
 *   the rest    internal scratch.
 */
typedef struct {
  size_t bytes;
  size_t off_status;
  size_t off_counts;
  size_t off_lists;
  size_t off_sel;
  int32_t n_blocks;
  int32_t list_cap;
  int32_t sel_len;
  int32_t reserved;
} dma_ws_layout_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char* dma_status_string(dma_status_t status);

/* DMA_ABI_VERSION of the loaded library. */
int32_t dma_abi_version(void);

/* Bytes of workspace every call of problem `p` needs (covers all entry points). */
dma_status_t dma_workspace_size(const dma_params_t* p, size_t* bytes);

/* Offsets of the ABI-visible workspace regions for problem `p`. */
dma_status_t dma_workspace_layout(const dma_params_t* p, dma_ws_layout_t* layout);

/*
 * Gate (delta equation).
 *   V       [B, Hkv, N, d]   dtype
 *   Delta   [Hkv*d, H]       dtype
 *   A       [H]              float32
 *   delta   [B, H, N]        float32 out: exp(A_h * softplus(x)),  x[b,h,j] = sum_r v_j[r] Delta[r,h]
 *   x_save  [B, H, N]        float32 out, may be NULL: x, kept for dma_gate_bwd
 * x is accumulated in float32 (bf16 products are exact in float32).
 */
dma_status_t dma_gate(const dma_params_t* p, const void* V, const void* Delta, const float* A,
                      float* delta, float* x_save, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * Causal top-w mask (m_t equation), encoded exactly.
 *   delta  [B, H, N] float32 in
 *   evict  [B, H, N] int32 out (prefill/training): e_j = the first query position at which key
 *          j is no longer among the w best causal keys (N if never).  Query t selects key j
 *          iff j <= t < e_j; e_j == j means key j is never selected.  Because delta does not
 *          depend on the query, the queries selecting a key always form this interval.
 *          Also writes the per-block live-key lists and counts into the workspace, and beside
 *          each list entry the values the attention forward needs for that key (e_j and delta_j),
 *          so that its load stage reads them with contiguous loads instead of a gather.
 *          Decode (Nq == 1): `evict` must be NULL; the selected keys of the query at
 *          position N-1 are written to the workspace region off_sel.
 */
dma_status_t dma_topk_mask(const dma_params_t* p, const float* delta, int32_t* evict,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode selection after one key is appended to the cache (section "Unified Training-Inference
 * Architecture": the same selection at every decode step).  p: decode parameters (Nq == 1) with
 * N = L >= 2, the cache length including the new key at position L-1, whose gate value is in
 * delta [B, H, L] float32.  Because delta_j does not depend on the query, the best keys of [0, L)
 * are the best of those of [0, L-1) plus the new key: while fewer than w keys are selected it
 * joins; otherwise it replaces the worst selected key (smallest delta, the larger index among
 * equal ones) when its delta is strictly larger.  O(min(L, w)) work per (b, h) instead of a
 * selection over all L keys.  Writes to the workspace region off_sel exactly what dma_topk_mask
 * writes for N = L.  When L - 1 > w the region must already hold the selection over the first
 * L - 1 keys (dma_topk_mask or dma_topk_append with N = L - 1 and the same B, H, w, on the same
 * workspace); otherwise (every earlier key is selected) nothing is read from it.
 */
dma_status_t dma_topk_append(const dma_params_t* p, const float* delta, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Gate of the last key position only (the key just appended to a decode cache), "Dynamic Weight
 * Computation" equation: delta[b, h, N-1] = exp(A_h softplus(x)),
 * x = sum_{g,c} V[b, g, N-1, c] Delta[g*d + c, h]; x_save[b, h, N-1] = x when x_save is not NULL.
 * Other positions of delta and x_save are left as they are.  V [B, Hkv, N, d] dtype (the cache),
 * Delta [Hkv*d, H] dtype, A [H] float32.  Within the gate's float32 tolerance of dma_gate (the sum
 * runs in another order).  Needs no workspace.
 */
dma_status_t dma_gate_append(const dma_params_t* p, const void* V, const void* Delta, const float* A,
                             float* delta, float* x_save, void* stream);

/*
 * Masked attention forward (o_t equation), computing only on the live keys of each block
 * (masked pairs are skipped, section "Theoretical Guarantees for Safe Computation Skipping").
 *   Q      [B, H, Nq, d] dtype;  K, V [B, Hkv, N, d] dtype;  delta [B, H, N] float32
 *   evict  [B, H, N] int32 from dma_topk_mask (NULL for decode); the workspace must hold the
 *          lists (or selection) dma_topk_mask wrote for the same delta.  Prefill takes delta_j
 *          and e_j from the per-entry copies dma_topk_mask stored with the lists, and decode takes
 *          delta_j from the copy dma_topk_mask / dma_topk_append stored beside the selection, so a
 *          delta changed after the selection is not seen there: run the selection again.
 *   O      [B, H, Nq, d] dtype out;  LSE [B, H, Nq] float32 out
 * With bfloat16 storage and Nq == N (a problem the backward can take) the call also keeps, in the
 * workspace, the low-order part of every output, O - bf16(O), rounded to bfloat16, which
 * dma_attn_bwd reads back; DMA_FLAG_FORWARD_ONLY skips it.
 */
dma_status_t dma_attn_fwd(const dma_params_t* p, const void* Q, const void* K, const void* V,
                          const float* delta, const int32_t* evict, void* workspace,
                          size_t workspace_bytes, void* O, float* LSE, void* stream);

/*
 * Masked attention backward (prefill/training only), selection held constant.
 *   O, LSE from dma_attn_fwd, on the same workspace: with bfloat16 storage the row sums
 *   D_t = sum_c dO_tc O_tc use O plus the low-order part the forward kept there, so that D carries
 *   O to about 16 significant bits rather than bfloat16's 8; dO [B, H, N, d] dtype.
 *   dQ [B, H, N, d], dK, dV [B, Hkv, N, d] dtype out (dK, dV summed over the query heads of
 *   each group);  d_delta [B, H, N] float32 out (sum over queries of dS_tj).
 */
dma_status_t dma_attn_bwd(const dma_params_t* p, const void* Q, const void* K, const void* V,
                          const float* delta, const int32_t* evict, void* workspace,
                          size_t workspace_bytes, const void* O, const float* LSE,
                          const void* dO, void* dQ, void* dK, void* dV, float* d_delta,
                          void* stream);

/*
 * Gate backward (Delta and A are learnable; the method is trainable end to end, section
 * "Gradient Flow Integrity").  With gx = d_delta * delta * A * sigmoid(x):
 *   dDelta  [Hkv*d, H] float32 out:  sum_{b,j} v_j[r] gx[b,h,j]
 *   dA      [H] float32 out:         sum_{b,j} d_delta * delta * softplus(x)
 *   dV_gate [B, Hkv, N, d] float32 out: sum_h gx[b,h,j] Delta[g*d+c, h]  (the gate's share of
 *           dV; the caller adds it to dma_attn_bwd's dV)
 *   x_save, delta: from dma_gate on the same V, Delta, A (x_save must not be NULL).
 */
dma_status_t dma_gate_bwd(const dma_params_t* p, const void* V, const void* Delta,
                          const float* A, const float* x_save, const float* delta,
                          const float* d_delta, float* dDelta, float* dA, float* dV_gate,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Gate backward without a workspace, for callers that cannot allocate device memory: code that
 * runs where it may not call cudaMalloc (for example inside a host application or framework that
 * owns the GPU's allocator, or a plugin called from another runtime's graph).  The page has no
 * counterpart of this entry point; it exists for those callers only.
 *
 * Arguments and results are those of dma_gate_bwd (outputs within the same tolerance), except
 * that there is no workspace: the scratch (gx, the partial sums of dA and those of dDelta) lives in
 * a fixed array of DMA_NOALLOC_SCRATCH_BYTES that the library reserves on every GPU that loads it,
 * until the process exits.  With a(x) = x rounded up to a multiple of 256, a problem needs
 *     a(4*B*H*N) + a(4*B*H*ceil(N/1024)) + a(4*ceil(N/512)*B*Hkv*d*H)
 * bytes of it; one that needs more returns DMA_ERR_UNSUPPORTED before anything is launched.
 * The first call on a device (and the first after a device reset, which gives the device a new
 * context) looks the array's device address up (cudaGetSymbolAddress) with that device current,
 * so make that first call before any stream capture.  All calls share the one array: calls whose
 * GPU work overlaps (on different streams or from different host threads on one device) race on
 * it, so the caller must serialise them.  Every scratch element a call reads is written by that
 * call first.  Nothing is allocated or freed.
 */
#define DMA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
dma_status_t dma_gate_bwd_noalloc(const dma_params_t* p, const void* V, const void* Delta,
                                  const float* A, const float* x_save, const float* delta,
                                  const float* d_delta, float* dDelta, float* dA, float* dV_gate,
                                  void* stream);

/*
 * Context-parallel prefill: the sequence split into contiguous shards, one per rank (GPU), with one
 * exchange of each shard's best keys.  Reading of the m_t equation (section "Dynamic Sparse Mask
 * Generation"): a query keeps the best min(t+1, w) keys of [0, t] by delta, ties to the lower
 * position; the best keys of a union are among the best keys of its parts, so every query of shard r
 * selects within (the best keys of the prefix in front of the shard) + (the shard's own keys), and
 * the best keys of that prefix lie among the best keys of each earlier shard.  The page names no
 * multi-GPU scheme; this follows from the equation alone.
 *
 * Per rank r, with p the shard problem (N = the shard's length len, every other field as for the
 * whole sequence; w_heads allowed; Nq is ignored):
 *   1. dma_gate on the shard (delta is per position);
 *   2. dma_cp_candidates: the shard's candidate buffer (cand_bytes, the same on every rank);
 *   3. the exchange: every rank receives the candidate buffers of the ranks before it (an all-gather
 *      of the fixed-size buffers, e.g. NCCL);
 *   4. dma_cp_compact: from those n_prev buffers, the compacted sequence of P + len rows (P =
 *      prefix_rows = min(G w, prefix_len), prefix_len = the shard's first position);
 *   5. dma_topk_mask and dma_attn_fwd on the compacted sequence as a chunk of queries: N = P + len,
 *      Nq = len, K = Kc, V = Vc, delta = delta_c.  The shard's O and LSE equal the rows of the whole
 *      sequence's (selection bit for bit; attention within rounding).
 *
 * Layout of a candidate buffer (offsets from dma_cp_layout): pos int32 [B, H, w] (global positions,
 * ascending per row, -1 past the row's min(W_h, len) keys), delta float32 [B, H, w] (-inf past them),
 * K and V rows [B, H, w, d] in the storage dtype (zero past them; the rows of head h's KV head).
 * The workspace of both calls is ws_bytes long; its first int32 is a status word (0 = ok) that
 * dma_cp_compact ORs 0x20000000 into if a group's union exceeds its P rows (an internal consistency
 * check; the union holds at most min(G w, prefix_len) keys): clear it before the first call.
 * Limits: the shard problem's (len <= 16384), G w <= 16384, G <= 255, n_prev w < 2^24.
 */
typedef struct {
  size_t cand_bytes;   /* one shard's candidate buffer */
  size_t off_pos, off_delta, off_k, off_v;
  size_t ws_bytes;     /* workspace of dma_cp_candidates and dma_cp_compact */
  size_t off_status;   /* the workspace's status word */
  int32_t prefix_rows; /* P = min(G w, prefix_len) */
  int32_t reserved;
} dma_cp_layout_t;

/* Sizes and offsets for shard problem p with a prefix of prefix_len positions held by n_prev earlier
 * shards (both 0 for the first shard). */
dma_status_t dma_cp_layout(const dma_params_t* p, int32_t prefix_len, int32_t n_prev, dma_cp_layout_t* layout);

/* Candidate buffer of a shard starting at global position shard_start: delta [B, H, len] float32,
 * K, V [B, Hkv, len, d] dtype (the shard's rows). */
dma_status_t dma_cp_candidates(const dma_params_t* p, int32_t shard_start, const float* delta, const void* K,
                               const void* V, void* cand, size_t cand_bytes, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Compacted sequence of a shard from the candidate buffers of the n_prev shards before it (back to
 * back in shard order in `cands`, cand_bytes each), holding prefix_len positions together:
 *   delta_c [B, H, P + len] float32, Kc, Vc [B, Hkv, P + len, d] dtype, pos_c [B, Hkv, P + len] int32
 *   (the original position of every row, -1 for padding).  Rows [0, P): P - |U| padding rows (zero
 *   K, V; delta -inf), then the union U, ascending in position, over the heads of the group of each
 *   head's best min(W_h, prefix_len) keys of the prefix (delta -inf for a head that did not select the
 *   key); rows [P, P + len): the shard's own keys. */
dma_status_t dma_cp_compact(const dma_params_t* p, int32_t prefix_len, int32_t n_prev, const void* cands,
                            size_t cands_bytes, const float* delta, const void* K, const void* V, float* delta_c,
                            void* Kc, void* Vc, int32_t* pos_c, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * Reads the device status word of `workspace` (synchronises `stream`).  Returns DMA_OK or
 * DMA_ERR_TIMEOUT when a kernel's bounded wait gave up; *code receives the raw word.
 * dma_clear_device_status resets it (asynchronously on `stream`).
 */
dma_status_t dma_check_device_status(const dma_params_t* p, void* workspace, void* stream,
                                     int32_t* code);
dma_status_t dma_clear_device_status(const dma_params_t* p, void* workspace, void* stream);

/*
 * Check of the device-side failure path: launches one thread that waits on a barrier nothing
 * completes, with a limit of limit_cycles SM clocks (1 .. 2^34), after which it gives up, ORs
 * status bit 0x1 into the workspace status word and returns.  dma_check_device_status then reports
 * DMA_ERR_TIMEOUT; clear the word afterwards.  The same bounded wait guards every wait of the
 * tcgen05 kernels (there with a limit of about two seconds).
 */
dma_status_t dma_selftest_bounded_wait(const dma_params_t* p, void* workspace, size_t workspace_bytes,
                                       int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DMA_H_ */
