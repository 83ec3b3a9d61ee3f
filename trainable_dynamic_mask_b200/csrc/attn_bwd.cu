// Masked attention backward with the selection held constant.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Theoretical Guarantees for
// Safe Computation Skipping" (masked pairs have exactly zero gradient with respect to q and k, so
// they are skipped) and section "Gradient Flow Integrity" (end-to-end trainable).
//
// With P the masked softmax: dP = dO V^T, D_t = sum_c dO_tc O_tc, dS = P (dP - D),
// dQ = scale dS K, dK_g = scale sum_{h in g} dS_h^T Q_h, dV_g = sum_{h in g} P_h^T dO_h,
// d delta_{h,j} = sum_t dS_tj (delta enters the scores additively, unscaled).
//
// Kernels here: rowdot (D) and the launch sequence.  dQ is query-major over each block's live-key
// list, like the forward, so it needs no atomics (the tcgen05 kernel of attn_bwd_tc.cu); dK, dV
// and d delta are key-major over tiles of keys with similar selection intervals (attn_bwd_dkv_tc.cu).
#include <limits.h>

#include "common.cuh"

namespace dma {
namespace {

// ---------------------------------------------------------------- D = rowsum(dO * O)
// One CTA per 128-row block of one (b, h), one thread per row: the thread walks its row in groups of
// 8 columns (16-byte loads of O and dO; the row's 128-byte lines stay in L1 across the groups), four
// groups' loads in flight together.  With Olo (bf16 storage) the row of O is O + Olo, the output plus
// the low-order part the forward kept in its blocked layout [128-row block][D / 8][128 rows][8], read
// by the 32 lanes of a warp as 512 contiguous bytes: D then carries O to about 16 significant bits.
// D_t weighs every dS of row t; with O rounded to bf16 its error alone moved the column sums of dS
// (d delta) of keys that the first rows select (large P and large |O|) by more than the parity
// tolerance.
DMA_DEVINL void load8_f32(const uint16_t* p, float (&v)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(u[k] << 16);
    v[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
  }
}
DMA_DEVINL void load8_f32(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kRowdotBlock = DMA_BLOCK_Q;   // rows per CTA (one per thread)
constexpr int kRowdotBatch = 4;             // column groups loaded together

template <int D, typename OT>
__global__ void __launch_bounds__(kRowdotBlock)
bwd_rowdot_kernel(const OT* __restrict__ O, const uint16_t* __restrict__ Olo, const uint16_t* __restrict__ dO,
                  float* __restrict__ Drow, int N) {
  constexpr int NG = D / 8;
  const int blk = blockIdx.x, bh = blockIdx.y, r = threadIdx.x;
  const int t = blk * kRowdotBlock + r;
  if (t >= N) return;
  const size_t row = (size_t)bh * N + t;
  const uint16_t* lo = Olo != nullptr
                           ? Olo + ((size_t)bh * gridDim.x + blk) * kRowdotBlock * D + (size_t)r * 8
                           : nullptr;
  float acc = 0.f;
#pragma unroll
  for (int g0 = 0; g0 < NG; g0 += kRowdotBatch) {
    float o[kRowdotBatch][8], g[kRowdotBatch][8], l[kRowdotBatch][8];
#pragma unroll
    for (int k = 0; k < kRowdotBatch; ++k) {
      load8_f32(O + row * D + (g0 + k) * 8, o[k]);
      load8_f32(dO + row * D + (g0 + k) * 8, g[k]);
      if (lo != nullptr) load8_f32(lo + (size_t)(g0 + k) * kRowdotBlock * 8, l[k]);
    }
#pragma unroll
    for (int k = 0; k < kRowdotBatch; ++k)
#pragma unroll
      for (int u = 0; u < 8; ++u) acc = fmaf(lo != nullptr ? o[k][u] + l[k][u] : o[k][u], g[k][u], acc);
  }
  Drow[row] = acc;
}

template <int D, typename OutT>
cudaError_t launch_bwd_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, const int32_t* evict, void* ws, const void* O,
                         const float* LSE, const uint16_t* dO, void* dQ, void* dK, void* dV,
                         float* d_delta, cudaStream_t s) {
  float* Drow = ws_ptr<float>(ws, P.off_rowD);
  const uint16_t* Olo = P.off_olo ? ws_ptr<uint16_t>(ws, P.off_olo) : nullptr;
  bwd_rowdot_kernel<D, OutT><<<dim3(P.n_blocks, P.B * P.H), kRowdotBlock, 0, s>>>((const OutT*)O, Olo, dO, Drow,
                                                                                  P.N);
  {
    cudaError_t e = launch_bwd_dq_tc(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dQ, s);
    if (e != cudaSuccess) return e;
  }
  return launch_bwd_dkv_tc(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dK, dV, d_delta, s);
}

}  // namespace

cudaError_t launch_attn_bwd(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            const float* delta, const int32_t* evict, void* ws, const void* O,
                            const float* LSE, const uint16_t* dO16, void* dQ, void* dK, void* dV,
                            float* d_delta, cudaStream_t s) {
  if (P.d == 128)
    return P.bf16 ? launch_bwd_t<128, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, dO16, dQ, dK, dV, d_delta, s)
                  : launch_bwd_t<128, float>(P, Q, K, V, delta, evict, ws, O, LSE, dO16, dQ, dK, dV, d_delta, s);
  return P.bf16 ? launch_bwd_t<64, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, dO16, dQ, dK, dV, d_delta, s)
                : launch_bwd_t<64, float>(P, Q, K, V, delta, evict, ws, O, LSE, dO16, dQ, dK, dV, d_delta, s);
}

}  // namespace dma
