// Single-query decode attention over the selected keys of the last position.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient Sparse Attention
// Computation", o_t equation (only the w selected keys carry weight) and section "Hardware-Optimized
// Implementation" (O(w d) work per query instead of O(n d)).
//
// s_j = q . k_j * scale + delta_j for the selected j; o = softmax(s) V; LSE = ln sum_j exp(s_j).
// Split-K: each CTA reduces kDecodeSplit selected keys to an unnormalised partial (m in log2 units,
// l, o[D]); a second kernel combines the splits.  The prefill forward is the tensor-core kernel of
// attn_fwd_tc.cu.
#include <limits.h>

#include "tc_ops.cuh"

namespace dma {
namespace {

// ---------------------------------------------------------------- decode

constexpr int kDecThreads = 256;

// One CTA per (split of kDecodeSplit selected keys, b * H + h), one key per thread.  The split's K
// rows are copied into shared memory (16-byte cp.async, each row read as one contiguous 256-byte
// run, chunks XOR-swizzled by row so that the row-per-thread reads below are conflict-free); each
// thread then forms its key's score, the CTA takes the exact max and the weights of the split, and
// the V rows replace the K rows in the same buffer while the weight sum is formed.  The weighted V
// sum is split over (16-byte chunk, key group) threads and reduced through shared memory.  Writes
// an unnormalised partial (m in log2 units, l, o[D]) per split.  The whole split's loads are in
// flight at once, and several CTAs share an SM, so the selected rows stream at close to the
// random-row bandwidth of the memory.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                    const uint16_t* __restrict__ V, const float* __restrict__ seld,
                    const int32_t* __restrict__ sel, float* __restrict__ part, int H, int G, int N,
                    int sel_len, int n_split, float scale_log2, int w, const int32_t* __restrict__ w_heads) {
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int NG = kDecThreads / CH;      // key groups of the weighted V sum
  static_assert(kDecodeSplit == kDecThreads, "one key per thread");
  extern __shared__ __align__(16) unsigned char dec_sm[];
  uint4* rows = reinterpret_cast<uint4*>(dec_sm);                              // [kDecodeSplit][CH]
  float* qs = reinterpret_cast<float*>(dec_sm + kDecodeSplit * D * 2);         // [D]
  float* wp = qs + D;                                                          // [kDecodeSplit]
  int32_t* idx = reinterpret_cast<int32_t*>(wp + kDecodeSplit);                // [kDecodeSplit]
  __shared__ float wred[2][kDecThreads / 32];
  const int s = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh % H, g = h / G, Hkv = H / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the combine kernel may be scheduled now: it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint16_t* Kg = K + (size_t)(b * Hkv + g) * N * D;
  const uint16_t* Vg = V + (size_t)(b * Hkv + g) * N * D;
  const int k0 = s * kDecodeSplit;
  // the row holds min(window, N) selected keys (sel_len is the row stride; with per-head windows a
  // row may hold fewer, and splits past its end reduce nothing: m = -inf, l = 0)
  const int n_row = min(row_window(w_heads, bh, H, w), N);
  const int nk = min(kDecodeSplit, n_row - k0);
  // the split's keys and their delta, stored beside each other by the selection (no gather of delta)
  const int j = tid < nk ? sel[(size_t)bh * sel_len + k0 + tid] : -1;
  idx[tid] = j;
  const float dl = j >= 0 ? seld[(size_t)bh * sel_len + k0 + tid] * kLog2e : 0.f;
  for (int c = tid; c < D; c += kDecThreads) qs[c] = bf16_to_f32(Q[(size_t)bh * D + c]);
  __syncthreads();
  // rows of the split: thread sweep over (row, chunk), consecutive threads along a row
  auto load_rows = [&](const uint16_t* src) {
#pragma unroll
    for (int i = 0; i < kDecodeSplit * CH / kDecThreads; ++i) {
      const int u = tid + i * kDecThreads, r = u / CH, c = u % CH;
      const int jr = idx[r];
      cp_async_16(smem_u32(rows + r * CH + (c ^ (r & (CH - 1)))), src + (size_t)(jr >= 0 ? jr : 0) * D + c * 8,
                  jr >= 0 ? 16 : 0);
    }
    cp_async_commit();
  };
  load_rows(Kg);
  cp_async_wait<0>();
  __syncthreads();
  // score of this thread's key (log2 units)
  float x = -INFINITY;
  {
    uint64_t acc2 = f2(0.f, 0.f);
#pragma unroll
    for (int cc = 0; cc < CH; ++cc) {
      const uint4 kv = rows[tid * CH + (cc ^ (tid & (CH - 1)))];
      const float4 qa = reinterpret_cast<const float4*>(qs)[2 * cc];
      const float4 qb = reinterpret_cast<const float4*>(qs)[2 * cc + 1];
      const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        acc2 = f2_fma(f2(__uint_as_float(w4[u] << 16), __uint_as_float(w4[u] & 0xffff0000u)),
                      f2(qv[2 * u], qv[2 * u + 1]), acc2);
    }
    float d0, d1;
    f2_split(acc2, d0, d1);
    if (j >= 0) x = fmaf(d0 + d1, scale_log2, dl);
  }
  float m = x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wred[0][warp] = m;
  __syncthreads();   // also: every K row has been read, so the buffer may take the V rows
  load_rows(Vg);
  float M = wred[0][0];
#pragma unroll
  for (int w = 1; w < kDecThreads / 32; ++w) M = fmaxf(M, wred[0][w]);
  const float base = M == -INFINITY ? 0.f : M;
  const float p = fast_exp2(x - base);   // 0 for empty slots (x = -inf)
  wp[tid] = p;
  float l = p;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) wred[1][warp] = l;
  cp_async_wait<0>();
  __syncthreads();
  // o = sum_k p_k V_k: thread = (chunk c, key group kg), keys kg, kg + NG, ...
  const int c = tid % CH, kg = tid / CH;
  float acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u] = 0.f;
  for (int kk = kg; kk < nk; kk += NG) {
    const float pk = wp[kk];
    const uint4 vv = rows[kk * CH + (c ^ (kk & (CH - 1)))];
    const uint32_t w4[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc[2 * u] = fmaf(pk, __uint_as_float(w4[u] << 16), acc[2 * u]);
      acc[2 * u + 1] = fmaf(pk, __uint_as_float(w4[u] & 0xffff0000u), acc[2 * u + 1]);
    }
  }
  __syncthreads();   // the V rows are no longer read: reuse the buffer for the group sums
  float* red = reinterpret_cast<float*>(dec_sm);   // [NG][D]
#pragma unroll
  for (int u = 0; u < 8; ++u) red[kg * D + c * 8 + u] = acc[u];
  __syncthreads();
  float* out = part + ((size_t)bh * n_split + s) * (D + 2);
  for (int ch = tid; ch < D; ch += kDecThreads) {
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < NG; ++q) v += red[q * D + ch];
    out[2 + ch] = v;
  }
  if (tid == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) L += wred[1][w];
    out[0] = M;
    out[1] = L;
  }
}

template <int D>
constexpr int decode_smem_bytes() {
  return kDecodeSplit * D * 2 + D * 4 + kDecodeSplit * 4 + kDecodeSplit * 4;
}

// One CTA per (b, h): o = sum_s 2^(m_s - M) o_s / L, L = sum_s 2^(m_s - M) l_s,
// LSE = (M + log2 L) ln 2.  The splits' (m, l) are loaded one per thread into shared memory and
// each channel's partials 16 at a time, so that the loads are in flight together.
template <int D, typename OutT>
__global__ void decode_combine_kernel(const float* __restrict__ part, OutT* __restrict__ O,
                                      float* __restrict__ LSE, int n_split) {
  extern __shared__ float cmb[];   // [n_split] m, then [n_split] l and later the weights
  float* sm_m = cmb;
  float* sm_w = cmb + n_split;
  const int bh = blockIdx.x, tid = threadIdx.x;
  // launched as a programmatic dependent of the split kernel: wait for its completion (a no-op when
  // launched in plain stream order)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* pr = part + (size_t)bh * n_split * (D + 2);
  for (int q = tid; q < n_split; q += blockDim.x) {
    sm_m[q] = pr[(size_t)q * (D + 2)];
    sm_w[q] = pr[(size_t)q * (D + 2) + 1];
  }
  __syncthreads();
  float M = -INFINITY;
  for (int q = 0; q < n_split; ++q) M = fmaxf(M, sm_m[q]);
  const float base = M == -INFINITY ? 0.f : M;
  float L = 0.f;
  for (int q = 0; q < n_split; ++q) L += sm_w[q] * fast_exp2(sm_m[q] - base);
  __syncthreads();
  for (int q = tid; q < n_split; q += blockDim.x) sm_w[q] = fast_exp2(sm_m[q] - base) / L;
  __syncthreads();
  for (int c = tid; c < D; c += blockDim.x) {
    float v = 0.f;
    for (int q0 = 0; q0 < n_split; q0 += 16) {
      float t[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) t[u] = q0 + u < n_split ? pr[(size_t)(q0 + u) * (D + 2) + 2 + c] : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) v += q0 + u < n_split ? t[u] * sm_w[q0 + u] : 0.f;
    }
    store_from_f32(O + (size_t)bh * D + c, v);
  }
  if (tid == 0) LSE[bh] = (M + __log2f(L)) * kLn2;
}

template <int D, typename OutT>
cudaError_t launch_dec_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, void* ws, void* O, float* LSE, cudaStream_t s) {
  float* part = ws_ptr<float>(ws, P.off_dec_part);
  {
    cudaError_t ea = ensure_smem_limit(decode_split_kernel<D>, decode_smem_bytes<D>());
    if (ea != cudaSuccess) return ea;
  }
  decode_split_kernel<D><<<dim3(P.n_split, P.B * P.H), kDecThreads, decode_smem_bytes<D>(), s>>>(
      Q, K, V, ws_ptr<float>(ws, P.off_seld), ws_ptr<int32_t>(ws, P.off_sel), part, P.H, P.G, P.N, P.sel_len, P.n_split,
      P.scale * kLog2e, P.w, P.w_heads);
  if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
  // the combine as a programmatic dependent launch: its CTAs are scheduled while the split kernel
  // finishes and wait on its completion inside (griddepcontrol.wait), hiding the launch gap
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.B * P.H);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 2 * P.n_split * sizeof(float);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, OutT>, (const float*)part, (OutT*)O, LSE, P.n_split);
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
