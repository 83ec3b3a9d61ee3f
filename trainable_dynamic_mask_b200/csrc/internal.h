// Internal interface between the C-ABI layer (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dma.h"

namespace dma {

constexpr int kBlockQ = DMA_BLOCK_Q;   // query rows per block of the mask encoding
constexpr int kPairQ = 2 * kBlockQ;    // query rows per attention-forward work item
constexpr int kTopwMaxN = 16384;      // prefill/training selection keeps a whole row in SMEM
constexpr int kDecodeSplit = 256;      // selected keys per decode split (one per thread)
constexpr int kGateSlice = 512;        // positions per partial sum of dDelta
constexpr int kGateMaxH = 64;          // query heads the gate kernels hold in one register tile

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Segment length of the top-w rank computation for a row of N keys: about 8 segments per row.
inline int topw_seg_len(int N) { return N <= 4096 ? 512 : N <= 8192 ? 1024 : 2048; }

// Attention-forward work schedule.  A work unit is one split of a pair of query blocks (b, h, kp):
// pairs with long live lists are split into S parts of their list (partial results merged by the
// unit that finishes last), so that a problem with few heavy pairs still spreads evenly over the
// SMs.  Units are enumerated group by group (a group = one kp, its S, every (b, h)), heaviest
// groups first; inside a group unit index = start + bh * S + s.
constexpr int kMaxPairs = (kTopwMaxN + 2 * DMA_BLOCK_Q - 1) / (2 * DMA_BLOCK_Q);
constexpr int kMaxSplits = 4;
struct FwdGroup {
  int kp, S, start, slot;   // slot: first partial-result slot of the group (-1 when S == 1)
};
struct FwdSchedule {
  int n_groups, n_units, n_slots, pad;
  FwdGroup g[kMaxPairs];
};

// Resolved problem and workspace plan.
struct Plan {
  int B, H, Hkv, N, Nq, d, w, G;
  const int32_t* w_heads;   // per-head windows (device, [H]) or nullptr: every head uses w
  float scale;
  bool bf16;      // storage dtype is bf16 (else f32)
  bool decode;    // Nq == 1 and N > 1 ... the single query sits at position N-1
  bool fwd_only;  // DMA_FLAG_FORWARD_ONLY: no backward follows the forward
  int q0;         // first query position, N - Nq: 0 (prefill), N - 1 (decode), else a chunk of a longer
                  // sequence (chunked prefill: the queries are the last Nq positions)
  int n_blocks;   // query blocks of kBlockQ rows (prefill)
  int list_cap;   // entries per block list
  int n_pairs;    // query blocks of kPairQ rows (attention forward work items)
  int pair_cap;   // entries per pair list (a multiple of 128; every list is padded to 128)
  int sel_len;    // decode: row stride of the selection, min(w, N) (w with per-head windows)
  int n_split;    // decode: splits per (b, h)
  int n_slices;   // gate backward: position slices of kGateSlice
  // byte offsets in the workspace
  size_t off_status, off_counts, off_lists, off_sel;
  size_t off_q16, off_k16, off_v16, off_do16;  // bf16 copies of f32 Q, K, V, dO (dtype f32 only)
  size_t off_dec_part;                 // decode partials: [B*H*n_split][d + 2] f32
  size_t off_seld;                     // decode: delta of each selected key, beside off_sel [B, H, sel_len] f32
  size_t off_rowD;                     // backward: D = rowsum(dO * O) [B, H, Nq] f32
  size_t off_olo;                      // bf16 prefill/training: O - bf16(O) as bf16, blocked
                                       // [B, H][n_blocks][d / 8][128 rows][8]; 0 if none
  // backward dK/dV: per-head key order [B, H, N] i32, item records [n_slots] int4 {qlo, steps, keys,
  // perm offset}, items by length [n_slots] + count i32, f32 partial dK_h, dV_h [2][B, H, N, d]
  size_t off_dkv_perm, off_dkv_slots, off_dkv_items, off_dkv_part;
  size_t off_tw_p, off_tw_rank;        // top-w: rank -> position, position -> rank [B, H, N] i32
  size_t off_tw_T;                     // top-w: threshold ranks [B, H, n_blocks + 1] i32
  size_t off_tw_keys;                  // top-w: sorted segments of composite keys [B, H, npad] u64
  // attention forward: live-key lists of query pairs of blocks (kPairQ rows), each entry with its
  // e_j - j (i32) and delta_j * log2(e) (f32); [B, H, n_pairs, pair_cap], counts [.., 2]
  size_t off_pcounts, off_plists, off_plen, off_pdl;
  // attention forward split units: partial O [slot][half][D][128] f32, (m, l) [slot][half][2][128]
  // f32, and per pair [arrivals, partials written] x 2 halves (i32, zeroed by the list kernel),
  // followed by the dynamic schedule's [next unit, CTAs done] (i32, zeroed likewise)
  size_t off_fpart, off_fml, off_fcnt;
  FwdSchedule sched;
  size_t off_gx;                       // gate backward: gx [B, H, N] f32
  size_t off_dA_part;                  // gate backward: [B*H][ceil(N/1024)] f32
  size_t off_dDelta_part;              // gate backward: [n_slices*B][Hkv*d][H] f32
  size_t bytes;
};

dma_status_t make_plan(const dma_params_t* p, Plan* plan);
void fwd_schedule(const Plan& P, FwdSchedule* S);

template <typename T> inline T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

// ---------------------------------------------------------------- host helpers (tmap.cu)
// 2-D view [rows, d] of a row-major bf16 tensor for TMA gather4: boxes of 64 columns x 1 row,
// 128-byte swizzle.  `map` must point to a CUtensorMap (128 bytes, 64-byte aligned).
bool make_row_map(void* map, const void* base, uint64_t rows, int d);
// 2-D view [rows, d] for TMA box loads: boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tile_map(void* map, const void* base, uint64_t rows, int d, int box_rows);
int sm_count();   // SMs of the current device

// ---------------------------------------------------------------- launchers (cudaError_t)
cudaError_t launch_gate_fwd(const Plan& P, const void* V, const void* Delta, const float* A,
                            float* delta, float* x_save, cudaStream_t s);
cudaError_t launch_topw_prefill(const Plan& P, const float* delta, int32_t* evict, void* ws,
                                cudaStream_t s);
cudaError_t launch_topw_decode(const Plan& P, const float* delta, void* ws, cudaStream_t s);
// Top-min(window, N) of each of `rows` rows of N values (delta desc, index asc), ascending indices into
// sel[row * sel_stride ..] and, when seld is not null, their values into seld at the same places; the
// row's window is w_heads[row % H] clamped to [1, w] (w when w_heads is null).
cudaError_t launch_topw_select_rows(const float* delta, int rows, int N, int w, const int32_t* w_heads, int H,
                                    int32_t* sel, float* seld, int sel_stride, cudaStream_t s);
cudaError_t launch_topw_append(const Plan& P, const float* delta, void* ws, cudaStream_t s);
cudaError_t launch_selftest_wait(const Plan& P, void* ws, long long limit_cycles, cudaStream_t s);
cudaError_t launch_gate_append(const Plan& P, const void* V, const void* Delta, const float* A, float* delta,
                               float* x_save, cudaStream_t s);
cudaError_t launch_convert_f32_to_bf16(const float* src, uint16_t* dst, size_t n, cudaStream_t s);
cudaError_t launch_attn_fwd(const Plan& P, const uint16_t* Q, const uint16_t* K,
                            const uint16_t* V, const float* delta, const int32_t* evict,
                            void* ws, void* O, float* LSE, cudaStream_t s);
cudaError_t launch_attn_fwd_tc(const Plan& P, const uint16_t* Q, const uint16_t* K,
                               const uint16_t* V, const float* delta, const int32_t* evict,
                               void* ws, void* O, float* LSE, cudaStream_t s);
cudaError_t launch_decode_attn(const Plan& P, const uint16_t* Q, const uint16_t* K,
                               const uint16_t* V, const float* delta, void* ws, void* O,
                               float* LSE, cudaStream_t s);
cudaError_t launch_attn_bwd(const Plan& P, const uint16_t* Q, const uint16_t* K,
                            const uint16_t* V, const float* delta, const int32_t* evict,
                            void* ws, const void* O, const float* LSE, const uint16_t* dO16,
                            void* dQ, void* dK, void* dV, float* d_delta, cudaStream_t s);
cudaError_t launch_bwd_dq_tc(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                             const float* LSE, const float* Drow, void* dQ, cudaStream_t s);
cudaError_t launch_bwd_dkv_tc(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                              const float* LSE, const float* Drow, void* dK, void* dV, float* d_delta,
                              cudaStream_t s);
cudaError_t launch_gate_bwd(const Plan& P, const void* V, const void* Delta, const float* A,
                            const float* x_save, const float* delta, const float* d_delta,
                            float* dDelta, float* dA, float* dV_gate, void* ws, cudaStream_t s);

}  // namespace dma
