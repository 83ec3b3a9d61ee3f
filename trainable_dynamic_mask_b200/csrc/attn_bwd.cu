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
// One warp per kRowdotRows rows; each lane reads 4 consecutive elements of O and of dO per row (8- or
// 16-byte loads), the loads of all the warp's rows issued before the sums.
DMA_DEVINL void load4_f32(const uint16_t* p, float (&v)[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(w.x << 16);
  v[1] = __uint_as_float(w.x & 0xffff0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xffff0000u);
}
DMA_DEVINL void load4_f32(const float* p, float (&v)[4]) {
  const float4 w = *reinterpret_cast<const float4*>(p);
  v[0] = w.x;
  v[1] = w.y;
  v[2] = w.z;
  v[3] = w.w;
}

constexpr int kRowdotRows = 4;   // rows per warp, loaded together

template <typename OT>
__global__ void bwd_rowdot_kernel(const OT* __restrict__ O, const uint16_t* __restrict__ dO,
                                  float* __restrict__ Drow, size_t rows, int D) {
  const size_t r0 = ((size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * kRowdotRows;
  const int lane = threadIdx.x & 31;
  if (r0 >= rows) return;
  float acc[kRowdotRows];
  for (int c = lane * 4; c < D; c += 128) {
    float o[kRowdotRows][4], g[kRowdotRows][4];
#pragma unroll
    for (int k = 0; k < kRowdotRows; ++k) {
      const size_t r = r0 + k < rows ? r0 + k : r0;
      load4_f32(O + r * D + c, o[k]);
      load4_f32(dO + r * D + c, g[k]);
    }
#pragma unroll
    for (int k = 0; k < kRowdotRows; ++k)
      acc[k] = fmaf(o[k][0], g[k][0], fmaf(o[k][1], g[k][1], fmaf(o[k][2], g[k][2],
                    fmaf(o[k][3], g[k][3], c == lane * 4 ? 0.f : acc[k]))));
  }
#pragma unroll
  for (int k = 0; k < kRowdotRows; ++k) {
    float v = lane * 4 < D ? acc[k] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && r0 + k < rows) Drow[r0 + k] = v;
  }
}

template <int D, typename OutT>
cudaError_t launch_bwd_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, const int32_t* evict, void* ws, const void* O,
                         const float* LSE, const uint16_t* dO, void* dQ, void* dK, void* dV,
                         float* d_delta, cudaStream_t s) {
  float* Drow = ws_ptr<float>(ws, P.off_rowD);
  const size_t rows = (size_t)P.B * P.H * P.N;
  const size_t per_block = 8 * kRowdotRows;
  bwd_rowdot_kernel<OutT><<<(unsigned)((rows + per_block - 1) / per_block), 256, 0, s>>>((const OutT*)O, dO, Drow,
                                                                                       rows, D);
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
