// Single-query decode attention over the selected keys of the last position.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient Sparse Attention
// Computation", o_t equation (only the w selected keys carry weight) and section "Hardware-Optimized
// Implementation" (O(w d) work per query instead of O(n d)).
//
// s_j = q . k_j * scale + delta_j for the selected j; o = softmax(s) V; LSE = ln sum_j exp(s_j).
// Split-K: each CTA folds kDecodeSplit selected keys into an unnormalised partial (m in log2 units,
// l, o[D]); a second kernel combines the splits.  The prefill forward is the tensor-core kernel of
// attn_fwd_tc.cu.
#include <limits.h>

#include "common.cuh"

namespace dma {
namespace {

// ---------------------------------------------------------------- decode

constexpr int kDecThreads = 128;

// One CTA per (split of kDecodeSplit selected keys, b*H + h).  Each warp holds four lane groups of
// eight lanes, one key row per group at a time, each lane owning D/8 channels.  Writes an unnormalised partial
// (m in log2 units, l, o[D]) per split.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                    const uint16_t* __restrict__ V, const float* __restrict__ delta,
                    const int32_t* __restrict__ sel, float* __restrict__ part, int H, int G, int N,
                    int sel_len, int n_split, float scale_log2) {
  constexpr int PL = D / 8;   // channels per lane
  __shared__ float red_m[kDecThreads / 32], red_l[kDecThreads / 32];
  __shared__ float red_o[kDecThreads / 32][D];
  const int s = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh % H, g = h / G, Hkv = H / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 3, sub = lane & 7;
  const uint16_t* Kg = K + (size_t)(b * Hkv + g) * N * D;
  const uint16_t* Vg = V + (size_t)(b * Hkv + g) * N * D;
  const float* drow = delta + (size_t)bh * N;
  const int32_t* srow = sel + (size_t)bh * sel_len;
  float q[PL];
  {
    const uint16_t* qp = Q + (size_t)bh * D + sub * PL;
#pragma unroll
    for (int c = 0; c < PL; c += 8) {
      uint4 v = *reinterpret_cast<const uint4*>(qp + c);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        q[c + 2 * u] = __uint_as_float(w4[u] << 16);
        q[c + 2 * u + 1] = __uint_as_float(w4[u] & 0xffff0000u);
      }
    }
  }
  float m = -INFINITY, l = 0.f, acc[PL];
#pragma unroll
  for (int c = 0; c < PL; ++c) acc[c] = 0.f;
  const int k0 = s * kDecodeSplit, k1 = min(sel_len, k0 + kDecodeSplit);
  // This lane group's keys: kk = k0 + warp * 4 + grp + it * kStride.  All their indices are loaded
  // first; then the K and V rows of kChunk keys at a time are loaded together before any is used,
  // so that each lane keeps 4 KB of row loads of its warp in flight.
  constexpr int kStride = kDecThreads / 8;
  constexpr int kMaxIt = (kDecodeSplit + kStride - 1) / kStride;
  constexpr int kChunk = 2;
  static_assert(kMaxIt % kChunk == 0, "chunks of keys per lane group");
  const int kfirst = k0 + warp * 4 + grp;
  int jl[kMaxIt];
#pragma unroll
  for (int it = 0; it < kMaxIt; ++it) {
    const int kk = kfirst + it * kStride;
    jl[it] = kk < k1 ? srow[kk] : -1;
  }
#pragma unroll
  for (int it0 = 0; it0 < kMaxIt; it0 += kChunk) {
    // the shuffles below involve the whole warp: stop only when no lane group has a key left
    if (!__any_sync(0xffffffffu, jl[it0] >= 0)) break;
    uint4 kr[kChunk][PL / 8], vr[kChunk][PL / 8];
    float dl[kChunk];
#pragma unroll
    for (int c4 = 0; c4 < kChunk; ++c4) {
      const int j = jl[it0 + c4];
#pragma unroll
      for (int c = 0; c < PL / 8; ++c) {
        kr[c4][c] = j >= 0 ? *reinterpret_cast<const uint4*>(Kg + (size_t)j * D + sub * PL + c * 8) : make_uint4(0, 0, 0, 0);
        vr[c4][c] = j >= 0 ? *reinterpret_cast<const uint4*>(Vg + (size_t)j * D + sub * PL + c * 8) : make_uint4(0, 0, 0, 0);
      }
      dl[c4] = j >= 0 ? drow[j] * kLog2e : 0.f;
    }
#pragma unroll
    for (int c4 = 0; c4 < kChunk; ++c4) {
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < PL / 8; ++c) {
        const uint32_t w4[4] = {kr[c4][c].x, kr[c4][c].y, kr[c4][c].z, kr[c4][c].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          dot = fmaf(q[c * 8 + 2 * u], __uint_as_float(w4[u] << 16), dot);
          dot = fmaf(q[c * 8 + 2 * u + 1], __uint_as_float(w4[u] & 0xffff0000u), dot);
        }
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      if (jl[it0 + c4] < 0) continue;
      const float x = fmaf(dot, scale_log2, dl[c4]);
      const float mn = fmaxf(m, x);
      const float a = fast_exp2(m - mn), p = fast_exp2(x - mn);
      m = mn;
      l = l * a + p;
#pragma unroll
      for (int c = 0; c < PL / 8; ++c) {
        const uint32_t w4[4] = {vr[c4][c].x, vr[c4][c].y, vr[c4][c].z, vr[c4][c].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc[c * 8 + 2 * u] = fmaf(p, __uint_as_float(w4[u] << 16), acc[c * 8 + 2 * u] * a);
          acc[c * 8 + 2 * u + 1] = fmaf(p, __uint_as_float(w4[u] & 0xffff0000u), acc[c * 8 + 2 * u + 1] * a);
        }
      }
    }
  }
  // merge the four key groups of the warp (lanes sub, sub+8, sub+16, sub+24 share channels)
#pragma unroll
  for (int o = 8; o <= 16; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mn = fmaxf(m, m2);
    const float base = mn == -INFINITY ? 0.f : mn;
    const float a = fast_exp2(m - base), a2 = fast_exp2(m2 - base);
    l = l * a + l2 * a2;
#pragma unroll
    for (int c = 0; c < PL; ++c) {
      const float v2 = __shfl_xor_sync(0xffffffffu, acc[c], o);
      acc[c] = acc[c] * a + v2 * a2;
    }
    m = mn;
  }
  if (grp == 0) {
#pragma unroll
    for (int c = 0; c < PL; ++c) red_o[warp][sub * PL + c] = acc[c];
    if (sub == 0) { red_m[warp] = m; red_l[warp] = l; }
  }
  __syncthreads();
  float* out = part + ((size_t)bh * n_split + s) * (D + 2);
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kDecThreads / 32; ++w) M = fmaxf(M, red_m[w]);
  const float base = M == -INFINITY ? 0.f : M;
  for (int c = tid; c < D; c += kDecThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) v += red_o[w][c] * fast_exp2(red_m[w] - base);
    out[2 + c] = v;
  }
  if (tid == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) L += red_l[w] * fast_exp2(red_m[w] - base);
    out[0] = M;
    out[1] = L;
  }
}

template <int D, typename OutT>
__global__ void decode_combine_kernel(const float* __restrict__ part, OutT* __restrict__ O,
                                      float* __restrict__ LSE, int n_split) {
  const int bh = blockIdx.x;
  const float* pr = part + (size_t)bh * n_split * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, pr[(size_t)s * (D + 2)]);
  const float base = M == -INFINITY ? 0.f : M;
  float L = 0.f;
  for (int s = 0; s < n_split; ++s) L += pr[(size_t)s * (D + 2) + 1] * fast_exp2(pr[(size_t)s * (D + 2)] - base);
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < n_split; ++s)
      v += pr[(size_t)s * (D + 2) + 2 + c] * fast_exp2(pr[(size_t)s * (D + 2)] - base);
    store_from_f32(O + (size_t)bh * D + c, v / L);
  }
  if (threadIdx.x == 0) LSE[bh] = (M + __log2f(L)) * kLn2;
}

template <int D, typename OutT>
cudaError_t launch_dec_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, void* ws, void* O, float* LSE, cudaStream_t s) {
  float* part = ws_ptr<float>(ws, P.off_dec_part);
  decode_split_kernel<D><<<dim3(P.n_split, P.B * P.H), kDecThreads, 0, s>>>(
      Q, K, V, delta, ws_ptr<int32_t>(ws, P.off_sel), part, P.H, P.G, P.N, P.sel_len, P.n_split,
      P.scale * kLog2e);
  decode_combine_kernel<D, OutT><<<P.B * P.H, D, 0, s>>>(part, (OutT*)O, LSE, P.n_split);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                            cudaStream_t s) {
  return launch_attn_fwd_tc(P, Q, K, V, delta, evict, ws, O, LSE, s);
}

cudaError_t launch_decode_attn(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               const float* delta, void* ws, void* O, float* LSE, cudaStream_t s) {
  if (P.d == 128)
    return P.bf16 ? launch_dec_t<128, uint16_t>(P, Q, K, V, delta, ws, O, LSE, s)
                  : launch_dec_t<128, float>(P, Q, K, V, delta, ws, O, LSE, s);
  return P.bf16 ? launch_dec_t<64, uint16_t>(P, Q, K, V, delta, ws, O, LSE, s)
                : launch_dec_t<64, float>(P, Q, K, V, delta, ws, O, LSE, s);
}

}  // namespace dma
