// Masked attention forward over the live keys of each query block, and single-query decode.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient Sparse Attention
// Computation", o_t equation; section "Theoretical Guarantees for Safe Computation Skipping"
// (a masked pair has weight exactly 0, so it is skipped); section "Hardware-Optimized
// Implementation" (block-wise, FlashAttention-style computation on tensor cores, O(n w d) work).
//
// s_tj = q_t . k_j * scale + delta_j for selected j, -inf otherwise; O_t = softmax(s_t) V;
// LSE_t = ln sum_j exp(s_tj).  The kernel works in the log2 domain: s2 = s * log2(e).
//
// Prefill kernel: one CTA per (b, h, query block of 128 rows), 8 warps x 16 rows.  The block's
// live-key list (full keys first) is consumed in tiles of 64 keys whose K and V rows are gathered
// with 16-byte cp.async into XOR-swizzled shared memory, double-buffered against the tensor-core
// work (mma.sync m16n8k16 bf16, fp32 accumulation).  Tiles made only of full keys skip the per-pair
// mask test; the others test j <= t < e_j.  Online softmax with fp32 row state.
#include <limits.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kFwdThreads = 256;
constexpr int kBK = 64;   // keys per tile

template <int D>
struct FwdSmem {
  static constexpr int kRowChunks = D / 8;                // 16-byte chunks per row
  static constexpr int kQBytes = kBlockQ * D * 2;
  static constexpr int kKVBytes = kBK * D * 2;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffMeta = kOffV + 2 * kKVBytes;   // 2 stages x {j, dl, e} x kBK
  static constexpr int kBytes = kOffMeta + 2 * 3 * kBK * 4;
};

template <int D>
DMA_DEVINL void fwd_load_tile(unsigned char* sm, int stage, int tile, const int32_t* list, int n_live,
                              const uint16_t* Kg, const uint16_t* Vg, const float* drow,
                              const int32_t* erow) {
  using S = FwdSmem<D>;
  constexpr int kChunksPerThread = kBK * S::kRowChunks / kFwdThreads;   // 4 (D=128) or 2 (D=64)
  const int tid = threadIdx.x;
  const int r = tid / (kFwdThreads / kBK);                              // 4 threads per row
  const int c0 = (tid % (kFwdThreads / kBK)) * kChunksPerThread;
  const int li = tile * kBK + r;
  const int j = li < n_live ? list[li] : -1;
  const uint32_t kbase = smem_u32(sm + S::kOffK + stage * S::kKVBytes);
  const uint32_t vbase = smem_u32(sm + S::kOffV + stage * S::kKVBytes);
  const uint16_t* ksrc = Kg + (size_t)(j < 0 ? 0 : j) * D;
  const uint16_t* vsrc = Vg + (size_t)(j < 0 ? 0 : j) * D;
  const int nbytes = j < 0 ? 0 : 16;
#pragma unroll
  for (int u = 0; u < kChunksPerThread; ++u) {
    const int c = c0 + u;
    cp_async_16(kbase + swz(r, c, S::kRowChunks), ksrc + c * 8, nbytes);
    cp_async_16(vbase + swz(r, c, S::kRowChunks), vsrc + c * 8, nbytes);
  }
  if (c0 == 0) {
    int32_t* mj = reinterpret_cast<int32_t*>(sm + S::kOffMeta) + stage * 3 * kBK;
    float* md = reinterpret_cast<float*>(mj + kBK);
    int32_t* me = mj + 2 * kBK;
    mj[r] = j < 0 ? INT_MAX : j;
    md[r] = j < 0 ? 0.f : drow[j] * kLog2e;
    me[r] = j < 0 ? 0 : erow[j];
  }
}

template <int D, typename OutT>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                const uint16_t* __restrict__ V, const float* __restrict__ delta,
                const int32_t* __restrict__ evict, const int32_t* __restrict__ counts,
                const int32_t* __restrict__ lists, OutT* __restrict__ O, float* __restrict__ LSE,
                int H, int G, int N, int n_blocks, int list_cap, float scale_log2) {
  using S = FwdSmem<D>;
  extern __shared__ __align__(128) unsigned char sm[];
  const int kb = n_blocks - 1 - (int)blockIdx.x;   // heavy (late) blocks first
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H, g = h / G;
  const int Hkv = H / G;
  const int t0 = kb * kBlockQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int32_t* cnt = counts + ((size_t)bh * n_blocks + kb) * 2;
  const int n_full = cnt[0], n_live = cnt[1];
  const int32_t* list = lists + ((size_t)bh * n_blocks + kb) * list_cap;
  const uint16_t* Kg = K + (size_t)(b * Hkv + g) * N * D;
  const uint16_t* Vg = V + (size_t)(b * Hkv + g) * N * D;
  const float* drow = delta + (size_t)bh * N;
  const int32_t* erow = evict + (size_t)bh * N;
  const uint16_t* Qb = Q + ((size_t)bh * N + t0) * D;

  // Q tile (rows past N zero-filled)
  {
    const uint32_t qbase = smem_u32(sm);
    for (int i = tid; i < kBlockQ * S::kRowChunks; i += kFwdThreads) {
      const int r = i / S::kRowChunks, c = i % S::kRowChunks;
      const bool ok = t0 + r < N;
      cp_async_16(qbase + swz(r, c, S::kRowChunks), Qb + (size_t)(ok ? r : 0) * D + c * 8, ok ? 16 : 0);
    }
    cp_async_commit();
  }
  const int n_tiles = (n_live + kBK - 1) / kBK;
  if (n_tiles > 0) fwd_load_tile<D>(sm, 0, 0, list, n_live, Kg, Vg, drow, erow);
  cp_async_commit();

  uint32_t qf[D / 16][4];
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int qr0 = warp * 16 + (lane >> 2);   // this thread's rows qr0 and qr0 + 8
  const int tq0 = t0 + qr0, tq1 = tq0 + 8;

  for (int it = 0; it < n_tiles; ++it) {
    const int stage = it & 1;
    if (it + 1 < n_tiles) {
      fwd_load_tile<D>(sm, stage ^ 1, it + 1, list, n_live, Kg, Vg, drow, erow);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (it == 0) {
      const uint32_t qbase = smem_u32(sm);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldmatrix_x4(qbase + swz(warp * 16 + (lane & 15), 2 * kk + (lane >> 4), S::kRowChunks), qf[kk][0],
                    qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    const uint32_t kbase = smem_u32(sm + S::kOffK + stage * S::kKVBytes);
    const uint32_t vbase = smem_u32(sm + S::kOffV + stage * S::kKVBytes);
    const int32_t* mj = reinterpret_cast<const int32_t*>(sm + S::kOffMeta) + stage * 3 * kBK;
    const float* md = reinterpret_cast<const float*>(mj + kBK);
    const int32_t* me = mj + 2 * kBK;

    // S = Q K^T (16 x 64 per warp)
    float s[kBK / 8][4];
#pragma unroll
    for (int i = 0; i < kBK / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < kBK / 16; ++np) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(kbase + swz(np * 16 + ((lane >> 4) << 3) + (lane & 7), 2 * kk + ((lane >> 3) & 1),
                                S::kRowChunks),
                    r0, r1, r2, r3);
        mma_bf16_16816(s[2 * np], qf[kk], r0, r1);
        mma_bf16_16816(s[2 * np + 1], qf[kk], r2, r3);
      }
    }
    // scale, bias, mask; row max
    const bool full_tile = (it + 1) * kBK <= n_full;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < kBK / 8; ++nt) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int col = nt * 8 + (lane & 3) * 2 + u;
        const float dl = md[col];
        float x0 = fmaf(s[nt][u], scale_log2, dl);
        float x1 = fmaf(s[nt][2 + u], scale_log2, dl);
        if (!full_tile) {
          const int jj = mj[col], ee = me[col];
          if (!(jj <= tq0 && tq0 < ee)) x0 = -INFINITY;
          if (!(jj <= tq1 && tq1 < ee)) x1 = -INFINITY;
        }
        s[nt][u] = x0;
        s[nt][2 + u] = x1;
        mx0 = fmaxf(mx0, x0);
        mx1 = fmaxf(mx1, x1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = fast_exp2(m0 - base0), a1 = fast_exp2(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kBK / 8; ++nt) {
      s[nt][0] = fast_exp2(s[nt][0] - base0);
      s[nt][1] = fast_exp2(s[nt][1] - base0);
      s[nt][2] = fast_exp2(s[nt][2] - base1);
      s[nt][3] = fast_exp2(s[nt][3] - base1);
      ps0 += s[nt][0] + s[nt][1];
      ps1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * a0 + ps0;
    l1 = l1 * a1 + ps1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= a0; o[i][1] *= a0;
      o[i][2] *= a1; o[i][3] *= a1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vbase + swz(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * dn + (lane >> 4),
                                      S::kRowChunks),
                          r0, r1, r2, r3);
        mma_bf16_16816(o[2 * dn], pa, r0, r1);
        mma_bf16_16816(o[2 * dn + 1], pa, r2, r3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // epilogue
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  OutT* Ob = O + ((size_t)bh * N) * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + (lane & 3) * 2;
    if (tq0 < N) {
      store_from_f32(Ob + (size_t)tq0 * D + col, o[i][0] * inv0);
      store_from_f32(Ob + (size_t)tq0 * D + col + 1, o[i][1] * inv0);
    }
    if (tq1 < N) {
      store_from_f32(Ob + (size_t)tq1 * D + col, o[i][2] * inv1);
      store_from_f32(Ob + (size_t)tq1 * D + col + 1, o[i][3] * inv1);
    }
  }
  if ((lane & 3) == 0) {
    if (tq0 < N) LSE[(size_t)bh * N + tq0] = (m0 + __log2f(l0)) * kLn2;
    if (tq1 < N) LSE[(size_t)bh * N + tq1] = (m1 + __log2f(l1)) * kLn2;
  }
}

// ---------------------------------------------------------------- decode

constexpr int kDecThreads = 128;

// One CTA per (split of kDecodeSplit selected keys, b*H + h).  Each warp works on four keys at a
// time, eight lanes per key row, each lane owning D/8 channels.  Writes an unnormalised partial
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
cudaError_t launch_fwd_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                         cudaStream_t s) {
  auto k = attn_fwd_kernel<D, OutT>;
  const int smem = FwdSmem<D>::kBytes;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  dim3 grid(P.n_blocks, P.B * P.H);
  k<<<grid, kFwdThreads, smem, s>>>(Q, K, V, delta, evict, ws_ptr<int32_t>(ws, P.off_counts),
                                    ws_ptr<int32_t>(ws, P.off_lists), (OutT*)O, LSE, P.H, P.G, P.N,
                                    P.n_blocks, P.list_cap, P.scale * kLog2e);
  return cudaGetLastError();
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

cudaError_t launch_attn_fwd_mma_sync(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                     const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                                     cudaStream_t s) {
  if (P.d == 128)
    return P.bf16 ? launch_fwd_t<128, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, s)
                  : launch_fwd_t<128, float>(P, Q, K, V, delta, evict, ws, O, LSE, s);
  return P.bf16 ? launch_fwd_t<64, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, s)
                : launch_fwd_t<64, float>(P, Q, K, V, delta, evict, ws, O, LSE, s);
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
