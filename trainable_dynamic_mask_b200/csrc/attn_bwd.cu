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
template <typename OT>
__global__ void bwd_rowdot_kernel(const OT* __restrict__ O, const uint16_t* __restrict__ dO,
                                  float* __restrict__ Drow, size_t rows, int D) {
  const size_t r = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < D; c += 32)
    acc = fmaf(load_as_f32(O + r * D + c), bf16_to_f32(dO[r * D + c]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) Drow[r] = acc;
}

template <int D, typename OutT>
cudaError_t launch_bwd_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, const int32_t* evict, void* ws, const void* O,
                         const float* LSE, const uint16_t* dO, void* dQ, void* dK, void* dV,
                         float* d_delta, cudaStream_t s) {
  float* Drow = ws_ptr<float>(ws, P.off_rowD);
  const size_t rows = (size_t)P.B * P.H * P.N;
  bwd_rowdot_kernel<OutT><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const OutT*)O, dO, Drow, rows, D);
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
