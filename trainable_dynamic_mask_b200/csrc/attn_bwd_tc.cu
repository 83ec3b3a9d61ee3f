// Masked attention backward, dQ part, on the 5th-generation tensor cores.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Theoretical Guarantees for
// Safe Computation Skipping" (masked pairs have exactly zero gradient, so they are skipped) and
// section "Gradient Flow Integrity" (trainable end to end).
//
// With P the masked softmax (recomputed from the forward's LSE): dP = dO V^T, D_t = sum_c dO_tc O_tc,
// dS = P (dP - D), dQ = scale dS K.  Work item = (b, h, block of 128 query rows) over the block's
// live-key list (full keys first) in tiles of 128 keys; persistent CTAs, heaviest blocks first.
//
// Warp roles (384 threads):
//   warps 0-3  dS: thread r owns query row r (= TMEM lane r); per tile it reads S and dP in
//              32-column chunks, computes P = exp2(s scale log2(e) + delta_j log2(e) - LSE_t log2(e))
//              (mask j <= t < e_j on tiles that are not all full keys), dS = P (dP - D_t), and
//              writes dS (bf16) over the chunk's S columns; at the end of the item it writes dQ;
//   warp 4     allocates TMEM; one thread issues S = Q K^T and dP = dO V^T (operands in shared
//              memory) and dQ += dS K (dS from TMEM, K from shared memory read N-major);
//   warps 5-7  gather V rows; warps 8-11 gather Q, dO and K rows (TMA tile::gather4).
// TMEM: S buffers [0,128) and [384,512) (tile i uses buffer i % 2, so S of tile i + 1 is computed
// while dS of tile i feeds its dQ MMA), dP [128,256), dQ [256,256+D).
// Every wait is bounded (tc::mbar_wait); every TMEM access sits behind warp-uniform decisions.
#include <cuda.h>

#include "tc_ops.cuh"

namespace dma {
namespace {

constexpr int kBqThreads = 384;
constexpr int kBqMmaWarp = 4;
constexpr int kBqVWarp0 = 5;    // V producers: warps 5-7, row groups 11 + 11 + 10
constexpr int kBqKWarp0 = 8;    // Q, dO, K producers: warps 8-11, row groups 8 per warp
// setmaxnreg: launched with 168 per thread (384 x 168 = 64512); 128 x 232 + 256 x 56 = 44032.
constexpr int kBqRegsSoftmax = 232, kBqRegsOther = 56;
constexpr int kBqBK = 128;      // keys per tile
constexpr int kBqStages = 2;    // K and V stages
constexpr uint32_t kBqS0 = 0, kBqS1 = 384, kBqDP = 128, kBqDQ = 256;   // TMEM columns

enum : int { kErrBqQ = 0x100000, kErrBqK = 0x200000, kErrBqV = 0x400000, kErrBqS = 0x800000,
             kErrBqDS = 0x1000000, kErrBqDQ = 0x2000000, kErrBqEmpty = 0x4000000, kErrBqAlign = 0x8000000 };

template <int D>
struct BqSmem {
  static constexpr int kTile = (D / 64) * 128 * 128;   // 128 rows: [D/64][128][128 B]
  static constexpr int kQ = 0;
  static constexpr int kdO = kTile;
  static constexpr int kK = 2 * kTile;                  // [kBqStages]
  static constexpr int kV = kK + kBqStages * kTile;     // [kBqStages]
  static constexpr int kMeta = kV + kBqStages * kTile;  // [2 buffers][dl f32 | j | e - j][128]
  static constexpr int kBars = kMeta + 2 * 3 * kBqBK * 4;
  static constexpr int kBytes = kBars + 256;
};

struct BqBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kBqStages], k_empty[kBqStages], v_full[kBqStages], v_empty[kBqStages];
  uint64_t s_full, ds_full, dq_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};

DMA_DEVINL void bq_sync() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }

// 8 K steps of an M128 N128 product with both operands K-major SW128 (128-row tiles).
template <int KK, int NK>
struct BqSteps {
  DMA_DEVINL static void run(uint32_t d, uint64_t da, uint64_t db, uint32_t id) {
    mma_ss_at<(KK >> 2) * 16384 + (KK & 3) * 32>(d, da, db, id, KK > 0 ? 1u : 0u);
    BqSteps<KK + 1, NK>::run(d, da, db, id);
  }
};
template <int NK>
struct BqSteps<NK, NK> {
  DMA_DEVINL static void run(uint32_t, uint64_t, uint64_t, uint32_t) {}
};
// dQ (+)= dS K: 8 K steps of 16 keys, A = dS from TMEM, B = K tile read N-major.
template <int KK, int NK>
struct BqDqSteps {
  DMA_DEVINL static void run(uint32_t d, uint32_t a, uint64_t db, uint32_t id, uint32_t acc0) {
    mma_ts_at<KK>(d, a, db, id, KK > 0 ? 1u : acc0);
    BqDqSteps<KK + 1, NK>::run(d, a, db, id, acc0);
  }
};
template <int NK>
struct BqDqSteps<NK, NK> {
  DMA_DEVINL static void run(uint32_t, uint32_t, uint64_t, uint32_t, uint32_t) {}
};

DMA_DEVINL int bq_item_index(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

template <int D, typename OutT>
__global__ void __launch_bounds__(kBqThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                 const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const int32_t* __restrict__ counts, const int32_t* __restrict__ lists,
                 const float* __restrict__ delta, const int32_t* __restrict__ evict,
                 const float* __restrict__ LSE, const float* __restrict__ Drow, OutT* __restrict__ dQ,
                 int32_t* __restrict__ status, int BH, int H, int G, int N, int n_blocks, int list_cap,
                 float scale_log2, float scale) {
  using S = BqSmem<D>;
  extern __shared__ __align__(1024) unsigned char sm[];
  BqBars& bar = *reinterpret_cast<BqBars*>(sm + S::kBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = BH * n_blocks;
  const int cta = blockIdx.x, n_ctas = gridDim.x;
  volatile int* abort_flag = &bar.abort_flag;
  if (tid == 0) {
    bar.abort_flag = 0;
    if (smem_u32(sm) & 1023u) {
      atomicOr(status, kErrBqAlign);
      bar.abort_flag = 1;
    }
    tc::mbar_init(&bar.q_full, 32);
    tc::mbar_init(&bar.q_empty, 1);
    for (int i = 0; i < kBqStages; ++i) {
      tc::mbar_init(&bar.k_full[i], 32);
      tc::mbar_init(&bar.k_empty[i], 1);
      tc::mbar_init(&bar.v_full[i], 32);
      tc::mbar_init(&bar.v_empty[i], 1);
    }
    tc::mbar_init(&bar.s_full, 1);
    tc::mbar_init(&bar.ds_full, 128);
    tc::mbar_init(&bar.dq_done, 1);
    tc::mbar_init(&bar.drain, 1);
    tc::fence_mbar_init();
  }
  if (warp == kBqMmaWarp) {
    tc::tmem_alloc(&bar.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = bar.tmem_base;
  constexpr uint32_t kRowBytes = D * 2;

  if (warp >= kBqMmaWarp) {
    regs_dec<kBqRegsOther>();
    if (warp > kBqMmaWarp) {
      // ---------------------------------------------------------- producers (TMA gather4)
      const bool kside = warp >= kBqKWarp0;
      int grp, ngrp;
      if (kside) {
        grp = (warp - kBqKWarp0) * 8 + lane;
        ngrp = 8;
      } else {
        const int vw = warp - kBqVWarp0;
        grp = vw * 11 + lane;
        ngrp = vw < 2 ? 11 : 10;
      }
      const bool issuer = lane < ngrp;
      const uint32_t goff = (uint32_t)(4 * grp) * 128;
      uint64_t* full = kside ? bar.k_full : bar.v_full;
      uint64_t* empty = kside ? bar.k_empty : bar.v_empty;
      const CUtensorMap* map = kside ? &kmap : &vmap;
      const int tile_base = kside ? S::kK : S::kV;
      int tcount = 0, n_done = 0;
      bool ok = !*abort_flag;
      for (int r = 0; ok; ++r) {
        const int q = bq_item_index(r, cta, n_ctas);
        if (q >= n_items) break;
        const int bh = q % BH, kb = n_blocks - 1 - q / BH;
        const int n_live = counts[((size_t)bh * n_blocks + kb) * 2 + 1];
        const int n_tiles = (n_live + kBqBK - 1) / kBqBK;
        if (n_tiles == 0) continue;   // cannot happen: every query row selects at least one key
        const int t0 = kb * kBlockQ;
        const int b = bh / H, h = bh % H, g = h / G, Hkv = H / G;
        const int kvrow0 = (b * Hkv + g) * N;
        const int32_t* list = lists + ((size_t)bh * n_blocks + kb) * list_cap;
        if (kside) {
          if (n_done > 0 && !wait_all(&bar.q_empty, (n_done - 1) & 1, abort_flag, status, kErrBqEmpty)) {
            ok = false;
            break;
          }
          if (issuer) {   // Q and dO rows (rows past N repeat row N-1; their outputs are dropped)
            int rr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) rr[u] = bh * N + min(t0 + 4 * grp + u, N - 1);
            mbar_arrive_expect_tx(&bar.q_full, 8 * kRowBytes);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) {
              tma_gather4(smem_u32(sm + S::kQ) + hf * 16384 + goff, &qmap, hf * 64, rr[0], rr[1], rr[2], rr[3],
                          &bar.q_full);
              tma_gather4(smem_u32(sm + S::kdO) + hf * 16384 + goff, &domap, hf * 64, rr[0], rr[1], rr[2], rr[3],
                          &bar.q_full);
            }
          }
        }
        for (int i = 0; i < n_tiles; ++i, ++tcount) {
          const int st = tcount % kBqStages;
          if (tcount >= kBqStages &&
              !wait_all(&empty[st], ((tcount / kBqStages) - 1) & 1, abort_flag, status, kErrBqEmpty)) {
            ok = false;
            break;
          }
          if (issuer) {
            // entries past n_live are unspecified: fetch row 0 of the head there (dS is 0 for them)
            int rr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int li = i * kBqBK + 4 * grp + u;
              rr[u] = kvrow0 + (li < n_live ? max(list[li], 0) : 0);
            }
            mbar_arrive_expect_tx(&full[st], 4 * kRowBytes);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf)
              tma_gather4(smem_u32(sm + tile_base + st * S::kTile) + hf * 16384 + goff, map, hf * 64, rr[0], rr[1],
                          rr[2], rr[3], &full[st]);
          }
        }
        ++n_done;
      }
      if (!ok && issuer && tcount > 0) drain_wait(&full[(tcount - 1) % kBqStages], ((tcount - 1) / kBqStages) & 1);
    } else if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer (warp 4, one thread)
      constexpr uint32_t idss = tc::idesc_bf16(128, kBqBK, false, false);
      constexpr uint32_t iddq = tc::idesc_bf16(128, D, false, true);
      const uint64_t dq0 = tc::sdesc(smem_u32(sm + S::kQ), 16, 1024);
      const uint64_t ddo0 = tc::sdesc(smem_u32(sm + S::kdO), 16, 1024);
      const uint64_t dk0 = tc::sdesc(smem_u32(sm + S::kK), 16, 1024);
      const uint64_t dv0 = tc::sdesc(smem_u32(sm + S::kV), 16, 1024);
      const uint64_t dkn0 = tc::sdesc(smem_u32(sm + S::kK), 16384, 1024);   // K read N-major
      int tcount = 0, n_done = 0;
      bool ok = !*abort_flag;
      // S(T) = Q K^T into buffer T % 2 and dP(T) = dO V^T; K and V tiles are consumed in tile order,
      // so tile T sits in stage T % kBqStages of both
      // dq_wait: the dQ MMA to wait for before S(T) overwrites dS(T - 2).  A parity wait is only
      // sound on the barrier's newest or next phase, so it names the last dQ commit issued so far:
      // T - 2 inside an item (dQ(T - 1) follows this call), T - 1 at an item's first tile.
      auto issue_sdp = [&](int T, int dq_wait) -> bool {
        const int ks = T % kBqStages, vs = T % kBqStages;
        if (!tc::mbar_wait(&bar.k_full[ks], (T / kBqStages) & 1, abort_flag, status, kErrBqK)) return false;
        if (!tc::mbar_wait(&bar.v_full[vs], (T / kBqStages) & 1, abort_flag, status, kErrBqV)) return false;
        // the S buffer last held dS(T - 2); dP was last read by the dS pass of T - 1
        if (dq_wait >= 0 && !tc::mbar_wait(&bar.dq_done, dq_wait & 1, abort_flag, status, kErrBqDQ)) return false;
        if (T >= 1 && !tc::mbar_wait(&bar.ds_full, (T - 1) & 1, abort_flag, status, kErrBqDS)) return false;
        tc::fence_after();
        const uint32_t sbuf = tmem + ((T & 1) ? kBqS1 : kBqS0);
        BqSteps<0, D / 16>::run(sbuf, dq0, dk0 + (uint64_t)((ks * S::kTile) >> 4), idss);
        BqSteps<0, D / 16>::run(tmem + kBqDP, ddo0, dv0 + (uint64_t)((vs * S::kTile) >> 4), idss);
        tc::commit(&bar.s_full);
        tc::commit(&bar.v_empty[vs]);
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int q = bq_item_index(r, cta, n_ctas);
        if (q >= n_items) break;
        const int bh = q % BH, kb = n_blocks - 1 - q / BH;
        const int n_live = counts[((size_t)bh * n_blocks + kb) * 2 + 1];
        const int n_tiles = (n_live + kBqBK - 1) / kBqBK;
        if (n_tiles == 0) continue;
        if (!(ok = tc::mbar_wait(&bar.q_full, n_done & 1, abort_flag, status, kErrBqQ))) break;
        tc::fence_after();
        if (!(ok = issue_sdp(tcount, tcount - 1))) break;
        if (n_tiles == 1) tc::commit(&bar.q_empty);
        for (int i = 0; i < n_tiles && ok; ++i) {
          const int T = tcount + i;
          if (!(ok = tc::mbar_wait(&bar.ds_full, T & 1, abort_flag, status, kErrBqDS))) break;
          if (i + 1 < n_tiles) {
            if (!(ok = issue_sdp(T + 1, T - 1))) break;
            if (i + 2 == n_tiles) tc::commit(&bar.q_empty);   // Q and dO read for the last time
          }
          // dQ (+)= dS(T) K(T); then K(T)'s stage is free
          tc::fence_after();
          const int ks = T % kBqStages;
          const uint32_t sbuf = tmem + ((T & 1) ? kBqS1 : kBqS0);
          BqDqSteps<0, kBqBK / 16>::run(tmem + kBqDQ, sbuf, dkn0 + (uint64_t)((ks * S::kTile) >> 4), iddq,
                                        i == 0 ? 0u : 1u);
          tc::commit(&bar.dq_done);
          tc::commit(&bar.k_empty[ks]);
        }
        tcount += n_tiles;
        ++n_done;
      }
      tc::commit(&bar.drain);
      drain_wait(&bar.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS and dQ rows (warps 0-3)
    regs_inc<kBqRegsSoftmax>();
    const int r = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float* meta = reinterpret_cast<float*>(sm + S::kMeta);   // [2 buffers][dl | j | len][128]
    const uint64_t sc2 = f2(scale_log2, scale_log2);
    int tcount = 0;
    bool ok = !*abort_flag;
    for (int rr = 0; ok; ++rr) {
      const int q = bq_item_index(rr, cta, n_ctas);
      if (q >= n_items) break;
      const int bh = q % BH, kb = n_blocks - 1 - q / BH;
      const int32_t* cnt = counts + ((size_t)bh * n_blocks + kb) * 2;
      const int n_full = cnt[0], n_live = cnt[1];
      const int n_tiles = (n_live + kBqBK - 1) / kBqBK;
      if (n_tiles == 0) continue;
      const int t = kb * kBlockQ + r;
      const bool valid = t < N;
      // rows past N: P = 0 (their LSE is +inf), so their dS and dQ are 0 and dropped
      const float lse2 = valid ? LSE[(size_t)bh * N + t] * kLog2e : INFINITY;
      const float Dt = valid ? Drow[(size_t)bh * N + t] : 0.f;
      const uint64_t nl2 = f2(-lse2, -lse2), nD2 = f2(-Dt, -Dt);
      const int32_t* list = lists + ((size_t)bh * n_blocks + kb) * list_cap;
      const float* drow = delta + (size_t)bh * N;
      const int32_t* erow = evict + (size_t)bh * N;
      // this thread's entry of tile i: j (list), then delta_j and e_j - j; entries past n_live masked
      auto entry_j = [&](int i) { const int li = i * kBqBK + r; return li < n_live ? list[li] : -1; };
      int j_c = entry_j(0), j_n = n_tiles > 1 ? entry_j(1) : -1;
      float dl_c = j_c >= 0 ? drow[j_c] * kLog2e : 0.f;
      int ln_c = j_c >= 0 ? erow[j_c] - j_c : 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int T = tcount + i;
        // next tile's metadata loads (independent of this tile's work)
        const int j_nn = i + 2 < n_tiles ? entry_j(i + 2) : -1;
        const float dl_n = j_n >= 0 ? drow[j_n] * kLog2e : 0.f;
        const int ln_n = j_n >= 0 ? erow[j_n] - j_n : 0;
        float* buf = meta + (T & 1) * 3 * kBqBK;   // by the CTA's tile count: alternates across items too
        buf[r] = dl_c;
        reinterpret_cast<int32_t*>(buf)[kBqBK + r] = j_c;
        reinterpret_cast<int32_t*>(buf)[2 * kBqBK + r] = ln_c;
        if (!wait_all(&bar.s_full, T & 1, abort_flag, status, kErrBqS)) {
          ok = false;
          break;
        }
        tc::fence_after();
        bq_sync();
        const uint32_t sbuf = tmem + ((T & 1) ? kBqS1 : kBqS0) + lane_base;
        const uint32_t dpb = tmem + kBqDP + lane_base;
        const bool full_tile = (i + 1) * kBqBK <= n_full;
        const float2* dl2 = reinterpret_cast<const float2*>(buf);
        const int2* jj2 = reinterpret_cast<const int2*>(buf + kBqBK);
        const int2* ln2 = reinterpret_cast<const int2*>(buf + 2 * kBqBK);
#pragma unroll
        for (int c = 0; c < kBqBK / 32; ++c) {
          uint32_t sv[32], pv[32], pk[16];
          tc::tmem_ld32(sbuf + c * 32, sv);
          tc::tmem_ld32(dpb + c * 32, pv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int k = c * 32 + 2 * u;
            const float2 d = dl2[k / 2];
            // x = s scale log2(e) + delta_j log2(e) - LSE_t log2(e)
            const uint64_t x2 = f2_add(
                f2_fma(f2(__uint_as_float(sv[2 * u]), __uint_as_float(sv[2 * u + 1])), sc2, f2(d.x, d.y)), nl2);
            float x0, x1;
            f2_split(x2, x0, x1);
            float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            if (!full_tile) {
              const int2 jv = jj2[k / 2], lv = ln2[k / 2];
              p0 = (uint32_t)(t - jv.x) < (uint32_t)lv.x ? p0 : 0.f;
              p1 = (uint32_t)(t - jv.y) < (uint32_t)lv.y ? p1 : 0.f;
            }
            // dS = P (dP - D_t)
            const uint64_t ds2 =
                f2_mul(f2(p0, p1), f2_add(f2(__uint_as_float(pv[2 * u]), __uint_as_float(pv[2 * u + 1])), nD2));
            float ds0, ds1;
            f2_split(ds2, ds0, ds1);
            pk[u] = pack_bf16x2(ds0, ds1);
          }
          // dS of columns [32c, 32c + 32) goes to S columns [16c, 16c + 16), already read
          tc::tmem_st16(sbuf + c * 16, pk);
        }
        tc::tmem_wait_st();
        tc::fence_before();
        tc::mbar_arrive(&bar.ds_full);
        j_c = j_n;
        j_n = j_nn;
        dl_c = dl_n;
        ln_c = ln_n;
      }
      if (!ok) break;
      // ---- dQ row = scale * dQ_acc, after the item's last dQ MMA
      const int last = tcount + n_tiles - 1;
      if (!wait_all(&bar.dq_done, last & 1, abort_flag, status, kErrBqDQ)) {
        ok = false;
        break;
      }
      tc::fence_after();
      OutT* orow = dQ + ((size_t)bh * N + (valid ? t : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tc::tmem_ld32(tmem + kBqDQ + lane_base + c * 32, ov);
        tc::tmem_wait_ld();
        float of[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) of[u] = __uint_as_float(ov[u]) * scale;
        if (valid) store_row32(orow + c * 32, of);
      }
      tc::fence_before();
      tcount += n_tiles;
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == kBqMmaWarp) tc::tmem_dealloc(tmem, 512);
}

template <int D, typename OutT>
cudaError_t launch_dq_tc_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                           const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                           const float* LSE, const float* Drow, void* dQ, cudaStream_t s) {
  CUtensorMap qm, dom, km, vm;
  if (!make_row_map(&qm, Q, (uint64_t)P.B * P.H * P.N, D) || !make_row_map(&dom, dO, (uint64_t)P.B * P.H * P.N, D) ||
      !make_row_map(&km, K, (uint64_t)P.B * P.Hkv * P.N, D) || !make_row_map(&vm, V, (uint64_t)P.B * P.Hkv * P.N, D))
    return cudaErrorInvalidValue;
  auto k = bwd_dq_tc_kernel<D, OutT>;
  const int smem = BqSmem<D>::kBytes;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  const int n_items = P.B * P.H * P.n_blocks;
  const int grid = n_items < sm_count() ? n_items : sm_count();
  if (grid <= 0) return cudaSuccess;
  k<<<grid, kBqThreads, smem, s>>>(qm, dom, km, vm, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists),
                                   delta, evict, LSE, Drow, (OutT*)dQ, ws_ptr<int32_t>(ws, P.off_status), P.B * P.H,
                                   P.H, P.G, P.N, P.n_blocks, P.list_cap, P.scale * kLog2e, P.scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq_tc(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                             const float* LSE, const float* Drow, void* dQ, cudaStream_t s) {
  if (P.N > 32767) return cudaErrorInvalidValue;
  if (P.d == 128)
    return P.bf16 ? launch_dq_tc_t<128, uint16_t>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dQ, s)
                  : launch_dq_tc_t<128, float>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dQ, s);
  return P.bf16 ? launch_dq_tc_t<64, uint16_t>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dQ, s)
                : launch_dq_tc_t<64, float>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dQ, s);
}

}  // namespace dma
