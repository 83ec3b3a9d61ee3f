// Masked attention backward, dQ part, on the 5th-generation tensor cores.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Theoretical Guarantees for
// Safe Computation Skipping" (masked pairs have exactly zero gradient, so they are skipped) and
// section "Gradient Flow Integrity" (trainable end to end).
//
// With P the masked softmax (recomputed from the forward's LSE): dP = dO V^T, D_t = sum_c dO_tc O_tc,
// dS = P (dP - D), dQ = scale dS K.  Work item = (b, h, block of 128 query rows) over the block's
// live-key list (full keys first) in tiles of 96 keys; persistent CTAs, heaviest blocks first.
//
// Warp roles (512 threads):
//   warps 0-7  dS: warp w serves query rows 32 (w % 4) .. + 31 (= its TMEM lane quarter) and key
//              columns 48 (w / 4) .. + 47 of each tile: it reads S and dP, computes
//              P = exp2(s scale log2(e) + delta_j log2(e) - LSE_t log2(e)) (mask j <= t < e_j on tiles
//              that are not all full keys), dS = P (dP - D_t), and writes dS (bf16, two per column)
//              over the first 24 of its S columns; at the end of the item it writes half of dQ's row;
//   warp 8     allocates TMEM; its lane 0 issues S = Q K^T (operands in shared memory) and
//              dQ += dS K (dS from TMEM, K from shared memory read N-major);
//   warp 9     its lane 0 issues dP = dO V^T: one thread issues a tcgen05.mma about every 60-80
//              cycles, slower than the tensor pipe runs these 96-column products, so two threads on
//              different sub-partitions share the issue (each commit tracks its own thread's
//              products: barriers that wait for both count two arrivals);
//   warps 10-15 gather rows (TMA tile::gather4): Q and dO (warps 12-15), K (warps 12-14, which also
//              stage each K tile's key metadata delta_j log2(e), j, e_j - j in shared memory beside
//              it) and V (warps 10, 11, 15).
// TMEM: dQ [0, D); two tile buffers, each S (96 columns) then dP (96 columns), at 128 and 320, so
// that S and dP of tile T + 1 are computed while the dS pass of tile T runs.
// Every wait is bounded (tc::mbar_wait); every TMEM access sits behind warp-uniform decisions.
#include <cuda.h>

#include "tc_ops.cuh"

namespace dma {
namespace {

constexpr int kBqThreads = 512;
constexpr int kBqMmaWarp = 8;    // issues S and dQ
constexpr int kBqDpWarp = 9;     // issues dP
constexpr int kBqVWarp0 = 10;    // V: warps 10, 11 and 15, lanes 0-7 (row groups 0-23)
constexpr int kBqKWarp0 = 12;    // Q and dO: warps 12-15 (row groups 0-31); K: warps 12-14 (0-23)
// setmaxnreg: launched with 128 per thread (512 x 128 = 65536); 256 x 184 + 256 x 72 = 65536.
constexpr int kBqRegsDs = 184, kBqRegsOther = 72;
constexpr int kBqBK = 96;        // keys per tile
constexpr int kBqCols = 48;      // key columns per dS thread
// K and V stages (three each: four K stages and two V stages measured slower; seven do not fit).
constexpr int kBqKStages = 3, kBqVStages = 3;
constexpr uint32_t kBqDQ = 0, kBqBuf0 = 128, kBqBuf1 = 320, kBqDP = 96;   // TMEM columns (dP after S)

static_assert(kBqDpWarp == kBqMmaWarp + 1 && kBqVWarp0 == kBqDpWarp + 1, "warps 8 and 9 issue, the rest produce");

enum : int { kErrBqQ = 0x100000, kErrBqK = 0x200000, kErrBqV = 0x400000, kErrBqS = 0x800000,
             kErrBqDS = 0x1000000, kErrBqDQ = 0x2000000, kErrBqEmpty = 0x4000000, kErrBqAlign = 0x8000000 };

template <int D>
struct BqSmem {
  static constexpr int kHalves = D / 64;                 // 64-element column halves of a row
  static constexpr int kQTile = kHalves * 128 * 128;     // 128 rows: [halves][128][128 B]
  static constexpr int kKHalf = kBqBK * 128;             // bytes of one column half of a K or V tile
  static constexpr int kKTile = kHalves * kKHalf;        // 96 rows: [halves][96][128 B]
  static constexpr int kQ = 0;
  static constexpr int kdO = kQTile;
  static constexpr int kK = 2 * kQTile;                  // [kBqKStages]
  static constexpr int kV = kK + kBqKStages * kKTile;    // [kBqVStages]
  static constexpr int kMeta = kV + kBqVStages * kKTile; // [kBqKStages][dl f32 | j | e - j][kBqBK]
  static constexpr int kBars = kMeta + kBqKStages * 3 * kBqBK * 4;
  static constexpr int kBytes = kBars + 256;
};

struct BqBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kBqKStages], k_empty[kBqKStages], v_full[kBqVStages], v_empty[kBqVStages];
  uint64_t s_full[2], ds_full[2], dq_done, dq_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

// tcgen05.mma issued by the lane whose `leader` is non-zero (the whole warp runs the issue loop, so
// the descriptors stay warp-uniform), A and B from shared memory, descriptors advanced by OFFA / 16
// and OFFB / 16; ACC: accumulate into D (else overwrite it), or -1 to take `accumulate`.
template <uint32_t OFFA, uint32_t OFFB>
DMA_DEVINL void bq_mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate,
                          uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 a, b;\n\t"
      "add.s64 a, %1, %5;\n\t"
      "add.s64 b, %2, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %7, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(OFFA >> 4), "n"(OFFB >> 4), "r"(leader));
}
// The same with A from TMEM column a + ACOL and B from shared memory at descriptor + OFFB / 16.
template <uint32_t ACOL, uint32_t OFFB>
DMA_DEVINL void bq_mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t accumulate,
                          uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 b;\n\t.reg .b32 at;\n\t"
      "add.s64 b, %2, %5;\n\t"
      "add.u32 at, %1, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %7, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [at], b, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(OFFB >> 4), "n"(ACOL), "r"(leader));
}

// S = A B^T over D / 16 K steps, A a 128-row tile and B a 96-row tile, both K-major SW128.
template <int KK, int NK, int D>
struct BqSdp {
  DMA_DEVINL static void run(uint32_t d, uint64_t da, uint64_t db, uint32_t id, uint32_t leader) {
    bq_mma_ss<(KK >> 2) * BqSmem<D>::kQTile / (D / 64) + (KK & 3) * 32, (KK >> 2) * BqSmem<D>::kKHalf + (KK & 3) * 32>(
        d, da, db, id, KK > 0 ? 1u : 0u, leader);
    BqSdp<KK + 1, NK, D>::run(d, da, db, id, leader);
  }
};
template <int NK, int D>
struct BqSdp<NK, NK, D> {
  DMA_DEVINL static void run(uint32_t, uint64_t, uint64_t, uint32_t, uint32_t) {}
};
// dQ (+)= dS K over 6 K steps of 16 keys: keys 0-47 of dS sit in columns 0-23 of the S buffer and
// keys 48-95 in columns 48-71 (each dS thread writes over the S columns it has read); K is read
// N-major, 16 rows (2048 B) per step.
template <int KK>
struct BqDq {
  DMA_DEVINL static void run(uint32_t d, uint32_t a, uint64_t db, uint32_t id, uint32_t acc0, uint32_t leader) {
    bq_mma_ts<KK * 8 + (KK >= 3 ? 24 : 0), KK * 2048>(d, a, db, id, KK > 0 ? 1u : acc0, leader);
    BqDq<KK + 1>::run(d, a, db, id, acc0, leader);
  }
};
template <>
struct BqDq<kBqBK / 16> {
  DMA_DEVINL static void run(uint32_t, uint32_t, uint64_t, uint32_t, uint32_t, uint32_t) {}
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
    tc::mbar_init(&bar.q_empty, 2);
    for (int i = 0; i < kBqKStages; ++i) {
      tc::mbar_init(&bar.k_full[i], kBqBK / 4);
      tc::mbar_init(&bar.k_empty[i], 1);
    }
    for (int i = 0; i < kBqVStages; ++i) {
      tc::mbar_init(&bar.v_full[i], kBqBK / 4);
      tc::mbar_init(&bar.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar.s_full[i], 2);
      tc::mbar_init(&bar.ds_full[i], 8);
    }
    tc::mbar_init(&bar.dq_done, 1);
    tc::mbar_init(&bar.dq_free, 8);
    tc::mbar_init(&bar.drain, 2);
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
    if (warp >= kBqVWarp0) {
      // ---------------------------------------------------------- producers (TMA gather4)
      // A warp issues TMA requests one lane after another (about one per 64-72 cycles), so the
      // requests are spread over all six warps: Q and dO rows (32 groups of 4) over warps 12-15, K
      // rows (24 groups) over warps 12-14 and V rows (24 groups) over warps 10, 11 and 15, lanes 0-7.
      const bool q_role = warp >= kBqKWarp0;
      const bool kside = q_role && warp < kBqKWarp0 + 3;
      const int qgrp = (warp - kBqKWarp0) * 8 + lane;
      const int grp = kside ? qgrp : (q_role ? 16 : (warp - kBqVWarp0) * 8) + lane;
      const bool q_issuer = q_role && lane < 8;          // 32 groups of 4 query rows
      const bool t_issuer = lane < 8;                    // 24 groups of 4 key rows
      uint64_t* full = kside ? bar.k_full : bar.v_full;
      uint64_t* empty = kside ? bar.k_empty : bar.v_empty;
      const CUtensorMap* map = kside ? &kmap : &vmap;
      const int tile_base = kside ? S::kK : S::kV;
      const int n_st = kside ? kBqKStages : kBqVStages;
      float* meta0 = reinterpret_cast<float*>(sm + S::kMeta);
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
        const float* drow = delta + (size_t)bh * N;
        const int32_t* erow = evict + (size_t)bh * N;
        if (q_role) {
          if (n_done > 0 && !wait_all(&bar.q_empty, (n_done - 1) & 1, abort_flag, status, kErrBqEmpty)) {
            ok = false;
            break;
          }
          if (q_issuer) {   // Q and dO rows (rows past N repeat row N-1; their outputs are dropped)
            int rr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) rr[u] = bh * N + min(t0 + 4 * qgrp + u, N - 1);
            mbar_arrive_expect_tx(&bar.q_full, 8 * kRowBytes);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) {
              tma_gather4(smem_u32(sm + S::kQ) + hf * 128 * 128 + qgrp * 512, &qmap, hf * 64, rr[0], rr[1], rr[2],
                          rr[3], &bar.q_full);
              tma_gather4(smem_u32(sm + S::kdO) + hf * 128 * 128 + qgrp * 512, &domap, hf * 64, rr[0], rr[1], rr[2],
                          rr[3], &bar.q_full);
            }
          }
        }
        // Loads run ahead of their use so that no lane waits on one: the list entries two tiles
        // ahead, the delta and eviction values of the keys one tile ahead (K side).
        auto entries = [&](int i, int (&j)[4]) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int li = i * kBqBK + 4 * grp + u;
            j[u] = t_issuer && li < n_live ? list[li] : -1;
          }
        };
        auto key_values = [&](const int (&j)[4], float (&dv)[4], int (&lv)[4]) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            dv[u] = kside && j[u] >= 0 ? drow[j[u]] : 0.f;
            lv[u] = kside && j[u] >= 0 ? erow[j[u]] : 0;
          }
        };
        int jj[4], jn[4], jnn[4], lc[4], ln[4];
        float dc[4], dn[4];
        entries(0, jj);
        entries(1, jn);
        key_values(jj, dc, lc);
        for (int i = 0; i < n_tiles; ++i, ++tcount) {
          const int st = tcount % n_st;
          entries(i + 2, jnn);
          key_values(jn, dn, ln);
          if (tcount >= n_st && !wait_all(&empty[st], ((tcount / n_st) - 1) & 1, abort_flag, status, kErrBqEmpty)) {
            ok = false;
            break;
          }
          if (t_issuer) {
            // entries past n_live (j = -1) fetch row 0 of the head; their dS is 0
            const uint32_t dst = smem_u32(sm + tile_base + st * S::kKTile) + grp * 512;
            if (kside) {
              mbar_expect_tx(&full[st], 4 * kRowBytes);
            } else {
              mbar_arrive_expect_tx(&full[st], 4 * kRowBytes);
            }
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf)
              tma_gather4(dst + hf * S::kKHalf, map, hf * 64, kvrow0 + max(jj[0], 0), kvrow0 + max(jj[1], 0),
                          kvrow0 + max(jj[2], 0), kvrow0 + max(jj[3], 0), &full[st]);
            if (kside) {
              // the dS pass's per-key values, published by this lane's arrival on the K barrier
              float* meta = meta0 + st * 3 * kBqBK;
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int row = 4 * grp + u, j = jj[u];
                meta[row] = dc[u] * kLog2e;
                reinterpret_cast<int32_t*>(meta)[kBqBK + row] = j;
                reinterpret_cast<int32_t*>(meta)[2 * kBqBK + row] = j >= 0 ? lc[u] - j : 0;
              }
              tc::mbar_arrive(&full[st]);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            jj[u] = jn[u];
            jn[u] = jnn[u];
            dc[u] = dn[u];
            lc[u] = ln[u];
          }
        }
        ++n_done;
      }
      if (!ok && t_issuer && tcount > 0) drain_wait(&full[(tcount - 1) % n_st], ((tcount - 1) / n_st) & 1);
    } else {
      // ---------------------------------------------------------- MMA issue (warps 8 and 9, lane 0)
      constexpr uint32_t idss = tc::idesc_bf16(128, kBqBK, false, false);
      constexpr uint32_t iddq = tc::idesc_bf16(128, D, false, true);
      const bool sq = warp == kBqMmaWarp;   // S and dQ (else dP)
      const uint32_t leader = lane == 0 ? 1u : 0u;
      const uint64_t da0 = tc::sdesc(smem_u32(sm + (sq ? S::kQ : S::kdO)), 16, 1024);
      const uint64_t db0 = tc::sdesc(smem_u32(sm + (sq ? S::kK : S::kV)), 16, 1024);
      const uint64_t dkn0 = tc::sdesc(smem_u32(sm + S::kK), S::kKHalf, 1024);   // K read N-major
      auto commit = [&](uint64_t* b) {
        if (leader) tc::commit(b);
        __syncwarp();
      };
      int tcount = 0, n_done = 0;
      bool ok = !*abort_flag;
      // S(T) (warp 8) or dP(T) (warp 9) into buffer T % 2.  The buffer last held tile T - 2.  S: its
      // dS pass ended before warp 8 issued dQ(T - 2) (which waited for it), and dQ(T - 2) reads dS
      // there before S(T) writes it (one thread's tcgen05.mma run in issue order).  dP: warp 9 waits
      // for the dS pass of T - 2 itself.
      auto issue = [&](int T) -> bool {
        const int n_st = sq ? kBqKStages : kBqVStages, st = T % n_st;
        uint64_t* full = sq ? bar.k_full : bar.v_full;
        if (!wait_all(&full[st], (T / n_st) & 1, abort_flag, status, sq ? kErrBqK : kErrBqV)) return false;
        if (!sq && T >= 2 && !wait_all(&bar.ds_full[T & 1], ((T - 2) >> 1) & 1, abort_flag, status, kErrBqDS))
          return false;
        tc::fence_after();
        const uint32_t dst = tmem + ((T & 1) ? kBqBuf1 : kBqBuf0) + (sq ? 0u : kBqDP);
        BqSdp<0, D / 16, D>::run(dst, da0, db0 + (uint64_t)((st * S::kKTile) >> 4), idss, leader);
        commit(&bar.s_full[T & 1]);
        if (!sq) commit(&bar.v_empty[st]);
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int q = bq_item_index(r, cta, n_ctas);
        if (q >= n_items) break;
        const int bh = q % BH, kb = n_blocks - 1 - q / BH;
        const int n_live = counts[((size_t)bh * n_blocks + kb) * 2 + 1];
        const int n_tiles = (n_live + kBqBK - 1) / kBqBK;
        if (n_tiles == 0) continue;
        if (!(ok = wait_all(&bar.q_full, n_done & 1, abort_flag, status, kErrBqQ))) break;
        tc::fence_after();
        if (!sq) {
          for (int i = 0; i < n_tiles && ok; ++i) ok = issue(tcount + i);
          if (!ok) break;
          commit(&bar.q_empty);   // dO read for the last time
          tcount += n_tiles;
          ++n_done;
          continue;
        }
        if (!(ok = issue(tcount))) break;
        if (n_tiles == 1) commit(&bar.q_empty);
        for (int i = 0; i < n_tiles && ok; ++i) {
          const int T = tcount + i;
          if (i + 1 < n_tiles) {
            if (!(ok = issue(T + 1))) break;
            if (i + 2 == n_tiles) commit(&bar.q_empty);   // Q read for the last time
          }
          if (!(ok = wait_all(&bar.ds_full[T & 1], (T >> 1) & 1, abort_flag, status, kErrBqDS))) break;
          // the first dQ product of an item overwrites the accumulator the last item's rows were read from
          if (i == 0 && n_done > 0 &&
              !(ok = wait_all(&bar.dq_free, (n_done - 1) & 1, abort_flag, status, kErrBqDQ)))
            break;
          tc::fence_after();
          const int st = T % kBqKStages;
          BqDq<0>::run(tmem + kBqDQ, tmem + ((T & 1) ? kBqBuf1 : kBqBuf0), dkn0 + (uint64_t)((st * S::kKTile) >> 4),
                       iddq, i == 0 ? 0u : 1u, leader);
          commit(&bar.k_empty[st]);
          if (i + 1 == n_tiles) commit(&bar.dq_done);
        }
        tcount += n_tiles;
        ++n_done;
      }
      commit(&bar.drain);
      if (leader) drain_wait(&bar.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS and dQ rows (warps 0-7)
    regs_inc<kBqRegsDs>();
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;                       // query row of the block = TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int c0 = half * kBqCols;                           // this thread's key columns [c0, c0 + 48)
    const float* meta0 = reinterpret_cast<const float*>(sm + S::kMeta);
    const uint64_t sc2 = f2(scale_log2, scale_log2);
    int tcount = 0, n_done = 0;
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
      for (int i = 0; i < n_tiles; ++i) {
        const int T = tcount + i, st = T % kBqKStages;
        if (!wait_all(&bar.s_full[T & 1], (T >> 1) & 1, abort_flag, status, kErrBqS) ||
            !wait_all(&bar.k_full[st], (T / kBqKStages) & 1, abort_flag, status, kErrBqK)) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t sb = tmem + ((T & 1) ? kBqBuf1 : kBqBuf0) + lane_base + c0;
        uint32_t sa[32], sbv[16], pa[32], pb[16];
        tc::tmem_ld32(sb, sa);
        tc::tmem_ld16(sb + 32, sbv);
        tc::tmem_ld32(sb + kBqDP, pa);
        tc::tmem_ld16(sb + kBqDP + 32, pb);
        const float* meta = meta0 + st * 3 * kBqBK;
        const float2* dl2 = reinterpret_cast<const float2*>(meta) + c0 / 2;
        const int2* jj2 = reinterpret_cast<const int2*>(meta + kBqBK) + c0 / 2;
        const int2* ln2 = reinterpret_cast<const int2*>(meta + 2 * kBqBK) + c0 / 2;
        const bool full_tile = (i + 1) * kBqBK <= n_full;
        // dS of key columns c0 + 2u and c0 + 2u + 1, packed
        auto ds_pair = [&](int u, uint32_t s0, uint32_t s1, uint32_t d0, uint32_t d1) -> uint32_t {
          const float2 d = dl2[u];
          // x = s scale log2(e) + delta_j log2(e) - LSE_t log2(e)
          const uint64_t x2 = f2_add(f2_fma(f2(__uint_as_float(s0), __uint_as_float(s1)), sc2, f2(d.x, d.y)), nl2);
          float x0, x1;
          f2_split(x2, x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if (!full_tile) {
            const int2 jv = jj2[u], lv = ln2[u];
            p0 = (uint32_t)(t - jv.x) < (uint32_t)lv.x ? p0 : 0.f;
            p1 = (uint32_t)(t - jv.y) < (uint32_t)lv.y ? p1 : 0.f;
          }
          // dS = P (dP - D_t)
          const uint64_t ds2 = f2_mul(f2(p0, p1), f2_add(f2(__uint_as_float(d0), __uint_as_float(d1)), nD2));
          float ds0, ds1;
          f2_split(ds2, ds0, ds1);
          return pack_bf16x2(ds0, ds1);
        };
        uint32_t lo[16], hi[8];
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) lo[u] = ds_pair(u, sa[2 * u], sa[2 * u + 1], pa[2 * u], pa[2 * u + 1]);
#pragma unroll
        for (int u = 0; u < 8; ++u) hi[u] = ds_pair(16 + u, sbv[2 * u], sbv[2 * u + 1], pb[2 * u], pb[2 * u + 1]);
        // dS of columns [c0, c0 + 48) goes to S columns [c0, c0 + 24), already read by this thread
        tc::tmem_st16(sb, lo);
        tc::tmem_st8(sb + 16, hi);
        tc::tmem_wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bar.ds_full[T & 1]);
      }
      if (!ok) break;
      // ---- dQ row = scale * dQ_acc (this warp's half of the columns), after the item's last dQ MMA
      if (!wait_all(&bar.dq_done, n_done & 1, abort_flag, status, kErrBqDQ)) {
        ok = false;
        break;
      }
      tc::fence_after();
      OutT* orow = dQ + ((size_t)bh * N + (valid ? t : 0)) * D + half * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32];
        tc::tmem_ld32(tmem + kBqDQ + lane_base + half * (D / 2) + c * 32, ov);
        tc::tmem_wait_ld();
        float of[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) of[u] = __uint_as_float(ov[u]) * scale;
        if (valid) store_row32(orow + c * 32, of);
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar.dq_free);
      tcount += n_tiles;
      ++n_done;
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
