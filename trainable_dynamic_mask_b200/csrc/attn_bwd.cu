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
// Kernels here: rowdot (D), the key order, and dkv (key-major over 64-key tiles: key j only receives
// gradient from the queries t in [j, e_j), so each tile walks the query range [min j, max e_j) and
// masks per pair; the query heads of one KV group are summed in registers, so dK and dV need no
// atomics; mma.sync m16n8k16 bf16).  dQ is query-major over each block's live-key list, like the
// forward, so it needs no atomics either: the tcgen05 kernel of attn_bwd_tc.cu.
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

// ---------------------------------------------------------------- dK, dV, d delta
constexpr int kDkvThreads = 128;   // 4 warps x 16 keys = 64 keys
constexpr int kBQ2 = 64;           // queries per step

template <int D>
struct DkvSmem {
  static constexpr int kRowChunks = D / 8;
  static constexpr int kTile = 64 * D * 2;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;              // 2 stages
  static constexpr int kOffG = kOffQ + 2 * kTile;      // 2 stages
  static constexpr int kOffRow = kOffG + 2 * kTile;    // 2 stages x {lse2, D} x 64
  static constexpr int kBytes = kOffRow + 2 * 2 * kBQ2 * 4 + 16;
};

template <int D>
DMA_DEVINL void dkv_load_q(unsigned char* sm, int stage, int tq0, int N, const uint16_t* Qh,
                           const uint16_t* Gh, const float* lse, const float* Dr) {
  using S = DkvSmem<D>;
  const uint32_t qb = smem_u32(sm + S::kOffQ + stage * S::kTile);
  const uint32_t gb = smem_u32(sm + S::kOffG + stage * S::kTile);
  for (int i = threadIdx.x; i < kBQ2 * S::kRowChunks; i += kDkvThreads) {
    const int r = i / S::kRowChunks, c = i % S::kRowChunks;
    const int t = tq0 + r;
    const bool ok = t < N;
    cp_async_16(qb + swz(r, c, S::kRowChunks), Qh + (size_t)(ok ? t : 0) * D + c * 8, ok ? 16 : 0);
    cp_async_16(gb + swz(r, c, S::kRowChunks), Gh + (size_t)(ok ? t : 0) * D + c * 8, ok ? 16 : 0);
  }
  float* rl = reinterpret_cast<float*>(sm + S::kOffRow) + stage * 2 * kBQ2;
  for (int i = threadIdx.x; i < kBQ2; i += kDkvThreads) {
    const int t = tq0 + i;
    rl[i] = t < N ? lse[t] * kLog2e : 0.f;
    rl[kBQ2 + i] = t < N ? Dr[t] : 0.f;
  }
}

template <int D, typename OutT>
__global__ void __launch_bounds__(kDkvThreads, 1)
bwd_dkv_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
               const uint16_t* __restrict__ V, const uint16_t* __restrict__ dO,
               const float* __restrict__ delta, const int32_t* __restrict__ evict,
               const int32_t* __restrict__ perm, const float* __restrict__ LSE,
               const float* __restrict__ Drow, OutT* __restrict__ dK, OutT* __restrict__ dV,
               float* __restrict__ d_delta, int H, int G, int N, float scale_log2, float scale) {
  using S = DkvSmem<D>;
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ int qmax_sh, qmin_sh;
  __shared__ int tile_j[64];
  const int n_kt = (N + 63) / 64;
  const int kt = n_kt - 1 - (int)blockIdx.x;
  const int bg = blockIdx.y;   // b * Hkv + g
  const int Hkv = H / G;
  const int b = bg / Hkv, g = bg % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint16_t* Kg = K + (size_t)bg * N * D;
  const uint16_t* Vg = V + (size_t)bg * N * D;
  // this tile's keys: entries [64 kt, 64 kt + 64) of the group's key order (N past the end)
  if (tid < 64) tile_j[tid] = 64 * kt + tid < N ? perm[(size_t)bg * N + 64 * kt + tid] : N;
  __syncthreads();
  {
    const uint32_t kb = smem_u32(sm), vb = smem_u32(sm + S::kOffV);
    for (int i = tid; i < 64 * S::kRowChunks; i += kDkvThreads) {
      const int r = i / S::kRowChunks, c = i % S::kRowChunks;
      const int j = tile_j[r];
      const bool ok = j < N;
      cp_async_16(kb + swz(r, c, S::kRowChunks), Kg + (size_t)(ok ? j : 0) * D + c * 8, ok ? 16 : 0);
      cp_async_16(vb + swz(r, c, S::kRowChunks), Vg + (size_t)(ok ? j : 0) * D + c * 8, ok ? 16 : 0);
    }
    cp_async_commit();
  }
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  const int kr0 = warp * 16 + (lane >> 2);        // this thread's key rows kr0, kr0 + 8
  const int j_a = tile_j[kr0], j_b = tile_j[kr0 + 8];

  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    const size_t bh = (size_t)b * H + h;
    const float* drow = delta + bh * N;
    const int32_t* erow = evict + bh * N;
    const int e_a = j_a < N ? erow[j_a] : 0, e_b = j_b < N ? erow[j_b] : 0;
    const float dl_a = j_a < N ? drow[j_a] * kLog2e : 0.f, dl_b = j_b < N ? drow[j_b] * kLog2e : 0.f;
    if (tid == 0) { qmax_sh = 0; qmin_sh = N; }
    __syncthreads();
    {   // the query rows [qmin, qmax) that select some key of the tile in this head
      int mymax = 0, mymin = N;
      if (e_a > j_a) { mymax = max(mymax, e_a); mymin = min(mymin, j_a); }
      if (e_b > j_b) { mymax = max(mymax, e_b); mymin = min(mymin, j_b); }
      for (int o = 16; o > 0; o >>= 1) {
        mymax = max(mymax, __shfl_xor_sync(0xffffffffu, mymax, o));
        mymin = min(mymin, __shfl_xor_sync(0xffffffffu, mymin, o));
      }
      if (lane == 0) { atomicMax(&qmax_sh, mymax); atomicMin(&qmin_sh, mymin); }
    }
    __syncthreads();
    const int qmax = qmax_sh, j0 = qmin_sh;
    const uint16_t* Qh = Q + bh * N * D;
    const uint16_t* Gh = dO + bh * N * D;
    const float* lse = LSE + bh * N;
    const float* Dr = Drow + bh * N;
    const int nq = qmax > j0 ? (qmax - j0 + kBQ2 - 1) / kBQ2 : 0;
    float dd_a = 0.f, dd_b = 0.f;
    if (nq > 0) dkv_load_q<D>(sm, 0, j0, N, Qh, Gh, lse, Dr);
    cp_async_commit();
    for (int it = 0; it < nq; ++it) {
      const int stage = it & 1;
      const int tq0 = j0 + it * kBQ2;
      if (it + 1 < nq) {
        dkv_load_q<D>(sm, stage ^ 1, tq0 + kBQ2, N, Qh, Gh, lse, Dr);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint32_t kb = smem_u32(sm), vb = smem_u32(sm + S::kOffV);
      const uint32_t qb = smem_u32(sm + S::kOffQ + stage * S::kTile);
      const uint32_t gb = smem_u32(sm + S::kOffG + stage * S::kTile);
      const float* rl = reinterpret_cast<const float*>(sm + S::kOffRow) + stage * 2 * kBQ2;
      float s[kBQ2 / 8][4], dp[kBQ2 / 8][4];
#pragma unroll
      for (int i = 0; i < kBQ2 / 8; ++i) {
        s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
        dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t ka[4], va[4];
        ldmatrix_x4(kb + swz(warp * 16 + (lane & 15), 2 * kk + (lane >> 4), S::kRowChunks), ka[0], ka[1], ka[2],
                    ka[3]);
        ldmatrix_x4(vb + swz(warp * 16 + (lane & 15), 2 * kk + (lane >> 4), S::kRowChunks), va[0], va[1], va[2],
                    va[3]);
#pragma unroll
        for (int np = 0; np < kBQ2 / 16; ++np) {
          const int rr = np * 16 + ((lane >> 4) << 3) + (lane & 7), cc = 2 * kk + ((lane >> 3) & 1);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4(qb + swz(rr, cc, S::kRowChunks), r0, r1, r2, r3);
          mma_bf16_16816(s[2 * np], ka, r0, r1);
          mma_bf16_16816(s[2 * np + 1], ka, r2, r3);
          ldmatrix_x4(gb + swz(rr, cc, S::kRowChunks), r0, r1, r2, r3);
          mma_bf16_16816(dp[2 * np], va, r0, r1);
          mma_bf16_16816(dp[2 * np + 1], va, r2, r3);
        }
      }
      // P^T and dS^T (rows = keys, columns = queries)
#pragma unroll
      for (int nt = 0; nt < kBQ2 / 8; ++nt) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = nt * 8 + (lane & 3) * 2 + u;
          const int t = tq0 + col;
          const float l2 = rl[col], Dt = rl[kBQ2 + col];
          float pa = fast_exp2(fmaf(s[nt][u], scale_log2, dl_a) - l2);
          float pb = fast_exp2(fmaf(s[nt][2 + u], scale_log2, dl_b) - l2);
          if (!(j_a <= t && t < e_a)) pa = 0.f;
          if (!(j_b <= t && t < e_b)) pb = 0.f;
          const float dsa = pa * (dp[nt][u] - Dt), dsb = pb * (dp[nt][2 + u] - Dt);
          dd_a += dsa;
          dd_b += dsb;
          s[nt][u] = pa;
          s[nt][2 + u] = pb;
          dp[nt][u] = dsa;
          dp[nt][2 + u] = dsb;
        }
      }
      // dV += P^T dO, dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < kBQ2 / 16; ++kk) {
        uint32_t pa[4], sa[4];
        pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
        sa[0] = pack_bf16x2(dp[2 * kk][0], dp[2 * kk][1]);
        sa[1] = pack_bf16x2(dp[2 * kk][2], dp[2 * kk][3]);
        sa[2] = pack_bf16x2(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
        sa[3] = pack_bf16x2(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
#pragma unroll
        for (int dn = 0; dn < D / 16; ++dn) {
          const int rr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), cc = 2 * dn + (lane >> 4);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4_trans(gb + swz(rr, cc, S::kRowChunks), r0, r1, r2, r3);
          mma_bf16_16816(dv[2 * dn], pa, r0, r1);
          mma_bf16_16816(dv[2 * dn + 1], pa, r2, r3);
          ldmatrix_x4_trans(qb + swz(rr, cc, S::kRowChunks), r0, r1, r2, r3);
          mma_bf16_16816(dk[2 * dn], sa, r0, r1);
          mma_bf16_16816(dk[2 * dn + 1], sa, r2, r3);
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
    dd_a += __shfl_xor_sync(0xffffffffu, dd_a, 1);
    dd_a += __shfl_xor_sync(0xffffffffu, dd_a, 2);
    dd_b += __shfl_xor_sync(0xffffffffu, dd_b, 1);
    dd_b += __shfl_xor_sync(0xffffffffu, dd_b, 2);
    if ((lane & 3) == 0) {
      if (j_a < N) d_delta[bh * N + j_a] = dd_a;
      if (j_b < N) d_delta[bh * N + j_b] = dd_b;
    }
    __syncthreads();
  }
  OutT* dKo = dK + (size_t)bg * N * D;
  OutT* dVo = dV + (size_t)bg * N * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + (lane & 3) * 2;
    if (j_a < N) {
      store_from_f32(dKo + (size_t)j_a * D + col, dk[i][0] * scale);
      store_from_f32(dKo + (size_t)j_a * D + col + 1, dk[i][1] * scale);
      store_from_f32(dVo + (size_t)j_a * D + col, dv[i][0]);
      store_from_f32(dVo + (size_t)j_a * D + col + 1, dv[i][1]);
    }
    if (j_b < N) {
      store_from_f32(dKo + (size_t)j_b * D + col, dk[i][2] * scale);
      store_from_f32(dKo + (size_t)j_b * D + col + 1, dk[i][3] * scale);
      store_from_f32(dVo + (size_t)j_b * D + col, dv[i][2]);
      store_from_f32(dVo + (size_t)j_b * D + col + 1, dv[i][3]);
    }
  }
}

// Key order of the dK/dV pass.  A tile of 64 keys walks every query row that selects one of its keys
// in some head of the group, so tiles that mix long- and short-lived keys spend MMAs on masked pairs.
// Within each window of 256 positions the keys are therefore ordered by their group lifetime
// max_h e_j (longest first, then position); consecutive 64-entry runs of this order form the tiles.
constexpr int kOrderWin = 256;

__global__ void __launch_bounds__(kOrderWin)
bwd_key_order_kernel(const int32_t* __restrict__ evict, int32_t* __restrict__ perm, int H, int G, int N) {
  __shared__ uint32_t key[kOrderWin];
  const int w0 = blockIdx.x * kOrderWin, bg = blockIdx.y, tid = threadIdx.x;
  const int Hkv = H / G, b = bg / Hkv, g = bg % Hkv;
  const int j = w0 + tid;
  uint32_t k = 0xffffffffu;   // past N: last
  if (j < N) {
    int me = j;
    for (int hh = 0; hh < G; ++hh) me = max(me, evict[((size_t)b * H + g * G + hh) * N + j]);
    k = ((uint32_t)(N - me) << 16) | (uint32_t)j;   // ascending = lifetime end descending, then j
  }
  key[tid] = k;
  __syncthreads();
  for (int size = 2; size <= kOrderWin; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int partner = tid ^ stride;
      if (partner > tid) {
        const uint32_t a = key[tid], c = key[partner];
        const bool up = (tid & size) == 0;
        if ((a > c) == up) { key[tid] = c; key[partner] = a; }
      }
      __syncthreads();
    }
  if (j < N) perm[(size_t)bg * N + j] = (int32_t)(key[tid] & 0xffffu);
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
  {
    int32_t* perm = ws_ptr<int32_t>(ws, P.off_bwd_perm);
    bwd_key_order_kernel<<<dim3((P.N + kOrderWin - 1) / kOrderWin, P.B * P.Hkv), kOrderWin, 0, s>>>(
        evict, perm, P.H, P.G, P.N);
    auto k = bwd_dkv_kernel<D, OutT>;
    const int smem = DkvSmem<D>::kBytes;
    { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
    k<<<dim3((P.N + 63) / 64, P.B * P.Hkv), kDkvThreads, smem, s>>>(
        Q, K, V, dO, delta, evict, perm, LSE, Drow, (OutT*)dK, (OutT*)dV, d_delta, P.H, P.G, P.N,
        P.scale * kLog2e, P.scale);
  }
  return cudaGetLastError();
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
