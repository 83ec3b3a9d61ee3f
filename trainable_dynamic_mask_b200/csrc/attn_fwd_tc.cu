// Masked attention forward on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient Sparse Attention
// Computation" (o_t equation), "Theoretical Guarantees for Safe Computation Skipping" (masked pairs
// have weight exactly 0 and are skipped) and "Hardware-Optimized Implementation" (block-wise,
// FlashAttention-style computation on tensor cores, O(n w d) work).
//
// Work item = (b, h, pair of query blocks: 256 rows), walking the pair's live-key list (the union
// of the two blocks' lists; full keys first) in tiles of 128 keys.  Each gathered K/V tile feeds
// both 128-row halves, so the gather traffic per tensor-core FLOP is half that of 128-row items.
// The kernel is persistent: one CTA per SM takes work units, heaviest first, from a global counter
// as it finishes earlier ones (greedy longest-first, balanced by the units' actual durations), and
// the next unit's Q and first tiles load while the current one finishes.  A unit is a
// pair, or one of S splits of a long pair's list: the split that finishes last merges the others'
// partial (O, m, l) with its own, so that few heavy pairs still spread evenly over the SMs.
//
// Warp roles (512 threads):
//   warps 0-3  softmax of query half 0, warps 4-7 softmax of half 1: thread r owns query row r of
//              its half = TMEM lane r.  It reads its S row from TMEM, applies scale, +delta_j and the
//              mask j <= t < e_j (tiles of full keys skip the test), keeps the running max and sum,
//              writes P (bf16) over S in TMEM, and rescales its O row whenever the running max
//              grows.  The reference of P is thus always the exact running max, so P <= 1 and the
//              key that holds the row's maximum enters with P = 1 exactly: a stale reference (P up
//              to 2^k) rounds the dominant weight to bf16 too, and in rows dominated by a few large
//              value rows (scaled keys of the long workload) that rounding alone moved outputs by
//              more than the parity tolerance.  An eighth of the exponentials run as a polynomial
//              on the FMA pipe to offload the MUFU pipe;
//   warp 8     allocates TMEM; one thread issues the MMAs: S_h = Q_h K^T (operands in shared
//              memory) and O_h += P_h V (P_h from TMEM, V from shared memory);
//   warps 9-11 gather V rows, warps 12-15 gather Q and K rows, with TMA tile::gather4 (128-byte
//              swizzled, the layout the MMA reads).  One warp's TMA issue rate caps its gather
//              throughput, so seven warps issue.
// TMEM: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [384,384+D); P_h aliases S_h.  The MMAs
// of one thread execute in issue order, so S_h of tile i + 1 is issued right behind the PV of tile i
// that reads P_h (no wait for that PV to complete): the tensor pipe holds both while the softmax of
// the other half runs.
// Stages: Q 1 (both halves), K 2, V 2.  Tile metadata (delta_j log2(e), j, e_j - j) is read by
// the softmax threads straight from the list, one entry per thread, through a shared buffer.
// Every wait is bounded (tc::mbar_wait) and reports a timeout through the workspace status word;
// every TMEM load/store (warp-collective) sits behind warp-uniform decisions.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <limits.h>

#include <mutex>

#include "tc_ops.cuh"

namespace dma {
namespace {

constexpr int kTcThreads = 512;
constexpr int kMmaWarp = 8;
constexpr int kVWarp0 = 9;                  // V producers: warps 9-11, row groups 11 + 11 + 10
constexpr int kKWarp0 = 12;                 // Q/K producers: warps 12-15, row groups 8 per warp
// Register split (setmaxnreg): launched with 128 per thread (512 x 128 = 65536), warpgroups 2 and 3
// give back to 48 and the softmax warpgroups take 208: 256 x 48 + 256 x 208 = 65536.
constexpr int kRegsSoftmax = 208, kRegsOther = 48;
constexpr int kTcBK = 128;                  // keys per tile
constexpr int kKStages = 2, kVStages = 2;
constexpr int kPolyEvery = 8;               // one pair in kPolyEvery takes the polynomial exp2
constexpr int kSchedRing = 4;               // units published ahead by the scheduling thread
constexpr int kSchedConsumers = 15;         // warps that read each published unit (all but the scheduler's)

enum : int { kErrTimeoutQ = 0x100, kErrTimeoutK = 0x200, kErrTimeoutS = 0x400, kErrTimeoutP = 0x800,
             kErrTimeoutPV = 0x1000, kErrTimeoutKEmpty = 0x2000, kErrTimeoutV = 0x4000,
             kErrTimeoutVEmpty = 0x8000, kErrTimeoutQEmpty = 0x10000, kErrTimeoutMerge = 0x20000, kErrSmemAlign = 0x40000,
             kErrTimeoutSched = 0x80000 };

template <int D>
struct TcSmem {
  static constexpr int kHalves = D / 64;              // 64-element column halves of a row
  static constexpr int kTile = kHalves * 128 * 128;   // [halves][128 rows][128 B]
  static constexpr int kQ = 0;                        // [2 query halves]
  static constexpr int kK = kQ + 2 * kTile;           // [kKStages]
  static constexpr int kV = kK + kKStages * kTile;    // [kVStages]
  static constexpr int kMeta = kV + kVStages * kTile; // [2 halves][2 buffers][dl f32 | j | e - j][128]
  static constexpr int kBars = kMeta + 2 * 2 * 3 * kTcBK * 4;
  static constexpr int kBytes = kBars + 512;
};

struct TcBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint64_t sched_full[kSchedRing], sched_empty[kSchedRing];
  int sched_slot[kSchedRing];   // the CTA's n-th unit in slot n % kSchedRing
  uint32_t tmem_base;
  int abort_flag;
  int merge_old[2];   // per softmax warpgroup: arrivals seen by its unit's merge counter
};

// Named barrier of one softmax warpgroup (ids 1 and 2; 0 is __syncthreads).
DMA_DEVINL void group_sync(int h) {
  if (h == 0) asm volatile("bar.sync 1, 128;\n" ::: "memory");
  else asm volatile("bar.sync 2, 128;\n" ::: "memory");
}

template <int KK, int NK>
struct QkSteps {
  DMA_DEVINL static void run(uint32_t d, uint64_t dq, uint64_t dk, uint32_t id) {
    mma_ss_at<(KK >> 2) * 16384 + (KK & 3) * 32>(d, dq, dk, id, KK > 0 ? 1u : 0u);
    QkSteps<KK + 1, NK>::run(d, dq, dk, id);
  }
};
template <int NK>
struct QkSteps<NK, NK> {
  DMA_DEVINL static void run(uint32_t, uint64_t, uint64_t, uint32_t) {}
};
template <int KK, int NK>
struct PvSteps {
  DMA_DEVINL static void run(uint32_t d, uint32_t a, uint64_t dv, uint32_t id, uint32_t acc0) {
    mma_ts_at<KK>(d, a, dv, id, KK > 0 ? 1u : acc0);
    PvSteps<KK + 1, NK>::run(d, a, dv, id, acc0);
  }
};
template <int NK>
struct PvSteps<NK, NK> {
  DMA_DEVINL static void run(uint32_t, uint32_t, uint64_t, uint32_t, uint32_t) {}
};

// S_h = Q_h K^T: Q half `half` (descriptor dq0 of half 0), K tile at descriptor dk; commits to `done`.
// (Shared addresses stay below 2^18, so adding offsets to the 14-bit address field never carries.)
template <int D>
DMA_DEVINL void issue_qk(uint32_t tmem, int half, uint64_t dq0, uint64_t dk, uint64_t* done) {
  constexpr uint32_t idq = tc::idesc_bf16(128, kTcBK, false, false);
  QkSteps<0, D / 16>::run(tmem + half * 128, dq0 + (uint64_t)((half * TcSmem<D>::kTile) >> 4), dk, idq);
  tc::commit(done);
}

// O_h (+)= P_h V: P_h from TMEM (aliasing S_h), V tile at descriptor dv; commits to `done`.
template <int D>
DMA_DEVINL void issue_pv(uint32_t tmem, int half, uint64_t dv, bool first, uint64_t* done) {
  constexpr uint32_t idv = tc::idesc_bf16(128, D, false, true);
  PvSteps<0, kTcBK / 16>::run(tmem + 256 + half * 128, tmem + half * 128, dv, idv, first ? 0u : 1u);
  tc::commit(done);
}

DMA_DEVINL int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Work unit u (see FwdSchedule): pair kp of row bh, split s of S (its list's tiles
// [s n / S, (s + 1) n / S)), partial-result slot (-1 when the pair is not split).
struct Unit { int bh, kp, s, S, slot; };
DMA_DEVINL Unit unit_of(const FwdSchedule& sc, int u) {
  int g = 0;
  while (g + 1 < sc.n_groups && u >= sc.g[g + 1].start) ++g;
  const int idx = u - sc.g[g].start, S = sc.g[g].S;
  return Unit{idx / S, sc.g[g].kp, idx % S, S, S > 1 ? sc.g[g].slot + idx : -1};
}
// Dynamic schedule: the CTAs take the units (ordered heaviest first) from a global counter as they
// finish earlier ones, the greedy longest-first assignment, which balances the SMs by the units'
// actual durations.  In each CTA one thread (lane 0 of the first Q/K producer warp, the role that
// runs ahead) takes the next unit and publishes it in a ring of kSchedRing slots; every other warp
// reads unit n from slot n % kSchedRing and releases the slot.  The counter ends above n_units;
// the last CTA to finish resets it (and the list kernel zeroes it with the mask).
DMA_DEVINL int sched_publish(TcBars& bar, int n, int32_t* ctr, int n_units, volatile int* abort_flag,
                             int32_t* status) {
  const int slot = n % kSchedRing;
  if (n >= kSchedRing &&
      !tc::mbar_wait(&bar.sched_empty[slot], ((n / kSchedRing) - 1) & 1, abort_flag, status, kErrTimeoutSched))
    return -1;
  int u = atomicAdd(ctr, 1);
  if (u > n_units) u = n_units;
  bar.sched_slot[slot] = u;
  tc::mbar_arrive(&bar.sched_full[slot]);
  return u;
}
DMA_DEVINL int sched_take(TcBars& bar, int n, volatile int* abort_flag, int32_t* status) {
  const int slot = n % kSchedRing;
  if (!tc::mbar_wait(&bar.sched_full[slot], (n / kSchedRing) & 1, abort_flag, status, kErrTimeoutSched)) return -1;
  const int u = *reinterpret_cast<volatile int*>(&bar.sched_slot[slot]);
  tc::mbar_arrive(&bar.sched_empty[slot]);
  return u;
}
// Warp-collective: lane 0 publishes (the scheduling warp) or takes unit n; every lane gets it.
DMA_DEVINL int sched_unit_warp(TcBars& bar, int n, bool scheduler, int32_t* ctr, int n_units,
                               volatile int* abort_flag, int32_t* status) {
  int u = -1;
  if ((threadIdx.x & 31) == 0)
    u = scheduler ? sched_publish(bar, n, ctr, n_units, abort_flag, status) : sched_take(bar, n, abort_flag, status);
  return __shfl_sync(0xffffffffu, u, 0);
}
// Tiles [tb, te) of the unit's pair list of n_live entries.
DMA_DEVINL void unit_tiles(const Unit& x, int n_live, int& tb, int& te) {
  const int n = (n_live + kTcBK - 1) / kTcBK;
  tb = x.s * n / x.S;
  te = (x.s + 1) * n / x.S;
}

template <int D, typename OutT>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ FwdSchedule sched,
                   const int32_t* __restrict__ pcounts, const int32_t* __restrict__ plists,
                   const int32_t* __restrict__ plen, const float* __restrict__ pdl, OutT* __restrict__ O,
                   float* __restrict__ LSE, uint16_t* __restrict__ Olo, float* __restrict__ fpart,
                   float* __restrict__ fml,
                   int32_t* __restrict__ fcnt, int32_t* __restrict__ sched_ctr, int32_t* __restrict__ status, int H,
                   int G, int N, int n_pairs,
                   int pair_cap, float scale_log2, int q0) {
  using S = TcSmem<D>;
  const int Nq = N - q0;   // the queries are positions [q0, N) (q0 > 0: a chunk of a longer sequence)
  extern __shared__ __align__(1024) unsigned char sm[];
  TcBars& bar = *reinterpret_cast<TcBars*>(sm + S::kBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_units = sched.n_units;
  volatile int* abort_flag = &bar.abort_flag;

  if (tid == 0) {
    bar.abort_flag = 0;
    if (smem_u32(sm) & 1023u) {   // the swizzled operand layout needs a 1024-byte aligned base
      atomicOr(status, kErrSmemAlign);
      bar.abort_flag = 1;
    }
    tc::mbar_init(&bar.q_full, 32);
    tc::mbar_init(&bar.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) { tc::mbar_init(&bar.k_full[i], 32); tc::mbar_init(&bar.k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { tc::mbar_init(&bar.v_full[i], 32); tc::mbar_init(&bar.v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar.s_full[i], 1);
      tc::mbar_init(&bar.p_full[i], 128);
      tc::mbar_init(&bar.pv_done[i], 1);
    }
    tc::mbar_init(&bar.drain, 1);
    for (int i = 0; i < kSchedRing; ++i) {
      tc::mbar_init(&bar.sched_full[i], 1);
      tc::mbar_init(&bar.sched_empty[i], kSchedConsumers);
    }
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&bar.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = bar.tmem_base;
  constexpr uint32_t kRowBytes = D * 2;

  if (warp >= kMmaWarp) {
    regs_dec<kRegsOther>();
    if (warp >= kVWarp0) {
      // ---------------------------------------------------------- producers (TMA gather4)
      const bool kside = warp >= kKWarp0;
      // row group (4 rows of a 128-row tile) of this lane, and whether the lane issues
      int grp, ngrp;
      if (kside) {
        grp = (warp - kKWarp0) * 8 + lane;
        ngrp = 8;
      } else {
        const int vw = warp - kVWarp0;
        grp = vw * 11 + lane;
        ngrp = vw < 2 ? 11 : 10;
      }
      const bool issuer = lane < ngrp;
      const uint32_t goff = (uint32_t)(4 * grp) * 128;
      uint64_t* full = kside ? bar.k_full : bar.v_full;
      uint64_t* empty = kside ? bar.k_empty : bar.v_empty;
      const CUtensorMap* map = kside ? &kmap : &vmap;
      const int tile_base = kside ? S::kK : S::kV;
      const int err_empty = kside ? kErrTimeoutKEmpty : kErrTimeoutVEmpty;
      int tc_count = 0;            // tiles issued by this role so far (stage = count % 2)
      int n_done = 0;              // items done (Q buffer phase)
      bool ok = !*abort_flag;
      for (int r = 0; ok; ++r) {
        const int u = sched_unit_warp(bar, r, warp == kKWarp0, sched_ctr, n_units, abort_flag, status);
        if (u < 0) {
          ok = false;
          break;
        }
        if (u >= n_units) break;
        const Unit it = unit_of(sched, u);
        const size_t lbase = ((size_t)it.bh * n_pairs + it.kp) * pair_cap;
        int tb, te;
        unit_tiles(it, pcounts[((size_t)it.bh * n_pairs + it.kp) * 2 + 1], tb, te);
        const int n_tiles = te - tb;
        const int t0 = it.kp * 256;
        const int b = it.bh / H, h = it.bh % H, g = h / G, Hkv = H / G;
        const int kvrow0 = (b * Hkv + g) * N;
        if (n_tiles == 0) continue;   // an empty split: nothing to load
        const int32_t* list = plists + lbase + (size_t)tb * kTcBK + 4 * grp;
        int4 jn = make_int4(0, 0, 0, 0);
        if (issuer) jn = *reinterpret_cast<const int4*>(list);
        if (kside) {
          // Q rows of both halves (rows past N repeat row N-1; their outputs are dropped)
          if (n_done > 0 && !wait_all(&bar.q_empty, (n_done - 1) & 1, abort_flag, status, kErrTimeoutQEmpty)) {
            ok = false;
            break;
          }
          if (issuer) {
            mbar_arrive_expect_tx(&bar.q_full, 8 * kRowBytes);
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
              int rr[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) rr[u] = it.bh * Nq + min(max(t0 + qh * 128 + 4 * grp + u - q0, 0), Nq - 1);
#pragma unroll
              for (int hf = 0; hf < D / 64; ++hf)
                tma_gather4(smem_u32(sm + S::kQ + qh * S::kTile) + hf * 16384 + goff, &qmap, hf * 64, rr[0], rr[1],
                            rr[2], rr[3], &bar.q_full);
            }
          }
        }
        for (int i = 0; i < n_tiles; ++i, ++tc_count) {
          const int4 jc = jn;
          if (issuer && i + 1 < n_tiles) jn = *reinterpret_cast<const int4*>(list + (i + 1) * kTcBK);
          const int st = tc_count % 2;
          if (tc_count >= 2 && !wait_all(&empty[st], ((tc_count / 2) - 1) & 1, abort_flag, status, err_empty)) {
            ok = false;
            break;
          }
          if (issuer) {
            // padding entries (-1) fetch row 0 of the head: they are masked for every query row
            const int r0 = kvrow0 + max(jc.x, 0), r1 = kvrow0 + max(jc.y, 0);
            const int r2 = kvrow0 + max(jc.z, 0), r3 = kvrow0 + max(jc.w, 0);
            mbar_arrive_expect_tx(&full[st], 4 * kRowBytes);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf)
              tma_gather4(smem_u32(sm + tile_base + st * S::kTile) + hf * 16384 + goff, map, hf * 64, r0, r1, r2, r3,
                          &full[st]);
          }
        }
        ++n_done;
      }
      // after an abort: let this lane's copies in flight land before the CTA exits
      if (!ok && issuer && tc_count > 0) drain_wait(&full[(tc_count - 1) % 2], ((tc_count - 1) / 2) & 1);
    } else {
      // ---------------------------------------------------------- MMA issuer (warp 8)
      if (lane == 0) {
        // descriptors of the operand bases
        const uint64_t dq0 = tc::sdesc(smem_u32(sm + S::kQ), 16, 1024);
        const uint64_t dk0 = tc::sdesc(smem_u32(sm + S::kK), 16, 1024);
        const uint64_t dv0 = tc::sdesc(smem_u32(sm + S::kV), 16384, 1024);
        int kc = 0, vc = 0;        // K / V tiles consumed
        int tcount = 0;            // tiles done per half (S, P and PV completions of each half)
        int n_done = 0;            // items done
        bool ok = !*abort_flag;
        for (int r = 0; ok; ++r) {
          const int u = sched_take(bar, r, abort_flag, status);
          if (u < 0) {
            ok = false;
            break;
          }
          if (u >= n_units) break;
          const Unit it = unit_of(sched, u);
          int tb, te;
          unit_tiles(it, pcounts[((size_t)it.bh * n_pairs + it.kp) * 2 + 1], tb, te);
          const int n_tiles = te - tb;
          if (n_tiles == 0) continue;
          if (!(ok = tc::mbar_wait(&bar.q_full, n_done & 1, abort_flag, status, kErrTimeoutQ))) break;
          // first K tile: both halves.  S_h overwrites P_h of the previous item's last tile, which that
          // item's last PV (issued earlier by this thread) reads: tcgen05.mma operations issued by one
          // thread execute in issue order, so the write cannot overtake the read and needs no wait.
          if (!(ok = tc::mbar_wait(&bar.k_full[kc % 2], (kc / 2) & 1, abort_flag, status, kErrTimeoutK))) break;
          tc::fence_after();
          for (int half = 0; half < 2; ++half)
            issue_qk<D>(tmem, half, dq0, dk0 + (uint64_t)(((kc % 2) * S::kTile) >> 4), &bar.s_full[half]);
          tc::commit(&bar.k_empty[kc % 2]);
          ++kc;
          if (n_tiles == 1) tc::commit(&bar.q_empty);
          for (int i = 0; i < n_tiles && ok; ++i) {
            const int t = tcount + i;
            const int vs = vc % 2;
            ok = tc::mbar_wait(&bar.v_full[vs], (vc / 2) & 1, abort_flag, status, kErrTimeoutV) &&
                 tc::mbar_wait(&bar.p_full[0], t & 1, abort_flag, status, kErrTimeoutP);
            if (!ok) break;
            tc::fence_after();
            issue_pv<D>(tmem, 0, dv0 + (uint64_t)((vs * S::kTile) >> 4), i == 0, &bar.pv_done[0]);
            const bool more = i + 1 < n_tiles;
            if (more) {
              // S_0 of the next tile goes over P_0, which the PV just issued reads: in-order execution
              // of this thread's MMAs orders the two (no wait for the PV to complete)
              if (!(ok = tc::mbar_wait(&bar.k_full[kc % 2], (kc / 2) & 1, abort_flag, status, kErrTimeoutK))) break;
              tc::fence_after();
              issue_qk<D>(tmem, 0, dq0, dk0 + (uint64_t)(((kc % 2) * S::kTile) >> 4), &bar.s_full[0]);
            }
            if (!(ok = tc::mbar_wait(&bar.p_full[1], t & 1, abort_flag, status, kErrTimeoutP))) break;
            tc::fence_after();
            issue_pv<D>(tmem, 1, dv0 + (uint64_t)((vs * S::kTile) >> 4), i == 0, &bar.pv_done[1]);
            tc::commit(&bar.v_empty[vs]);
            ++vc;
            if (more) {
              issue_qk<D>(tmem, 1, dq0, dk0 + (uint64_t)(((kc % 2) * S::kTile) >> 4), &bar.s_full[1]);
              tc::commit(&bar.k_empty[kc % 2]);
              ++kc;
              if (i + 2 == n_tiles) tc::commit(&bar.q_empty);
            }
          }
          tcount += n_tiles;
          ++n_done;
        }
        // let every MMA issued so far complete before TMEM is released
        tc::commit(&bar.drain);
        drain_wait(&bar.drain, 0);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax, query half h = warp / 4
    regs_inc<kRegsSoftmax>();
    const int h = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + h * 128 + lane_base, tO = tmem + 256 + h * 128 + lane_base;
    float* meta = reinterpret_cast<float*>(sm + S::kMeta) + h * 2 * 3 * kTcBK;   // [2 buffers][dl | j | len][128]
    const uint64_t sc2 = f2(scale_log2, scale_log2);
    int tcount = 0;
    bool ok = !*abort_flag;
    for (int rr = 0; ok; ++rr) {
      const int u = sched_unit_warp(bar, rr, false, sched_ctr, n_units, abort_flag, status);
      if (u < 0) {
        ok = false;
        break;
      }
      if (u >= n_units) break;
      const Unit it = unit_of(sched, u);
      const int32_t* cnt = pcounts + ((size_t)it.bh * n_pairs + it.kp) * 2;
      const int n_full = cnt[0];
      int tb, te;
      unit_tiles(it, cnt[1], tb, te);
      const int n_tiles = te - tb;
      const size_t lbase = ((size_t)it.bh * n_pairs + it.kp) * pair_cap + (size_t)tb * kTcBK;
      const int t = it.kp * 256 + h * 128 + r;   // this thread's query row
      float dl_n = n_tiles > 0 ? pdl[lbase + r] : 0.f;
      int jj_n = n_tiles > 0 ? plists[lbase + r] : -1;
      int ln_n = n_tiles > 0 ? plen[lbase + r] : 0;
      float m_used = -INFINITY, l = 0.f;
      for (int i = 0; i < n_tiles; ++i) {
        const int tt = tcount + i;
        if (!wait_all(&bar.s_full[h], tt & 1, abort_flag, status, kErrTimeoutS)) {
          ok = false;
          break;
        }
        tc::fence_after();
        uint32_t sr[kTcBK / 32][32];
#pragma unroll
        for (int c = 0; c < kTcBK / 32; ++c) tc::tmem_ld32(tS + c * 32, sr[c]);
        // this tile's metadata: entry r from this thread, the others through the shared buffer
        float* buf = meta + (tt & 1) * 3 * kTcBK;   // by the CTA's tile count: alternates across items too
        buf[r] = dl_n;
        reinterpret_cast<int32_t*>(buf)[kTcBK + r] = jj_n;
        reinterpret_cast<int32_t*>(buf)[2 * kTcBK + r] = ln_n;
        if (i + 1 < n_tiles) {
          dl_n = pdl[lbase + (i + 1) * kTcBK + r];
          jj_n = plists[lbase + (i + 1) * kTcBK + r];
          ln_n = plen[lbase + (i + 1) * kTcBK + r];
        }
        group_sync(h);
        tc::tmem_wait_ld();
        const float4* dl4 = reinterpret_cast<const float4*>(buf);
        const bool full_tile = (tb + i + 1) * kTcBK <= n_full;
        float mt = -INFINITY;
        if (full_tile) {
#pragma unroll
          for (int c4 = 0; c4 < kTcBK / 4; ++c4) {
            const float4 d = dl4[c4];
            const int c = 4 * c4;
            uint32_t* s4 = &sr[c / 32][c % 32];
            const uint64_t va = f2_fma(f2(__uint_as_float(s4[0]), __uint_as_float(s4[1])), sc2, f2(d.x, d.y));
            const uint64_t vb = f2_fma(f2(__uint_as_float(s4[2]), __uint_as_float(s4[3])), sc2, f2(d.z, d.w));
            float v0, v1, v2, v3;
            f2_split(va, v0, v1);
            f2_split(vb, v2, v3);
            mt = max3(mt, v0, v1);
            mt = max3(mt, v2, v3);
            s4[0] = __float_as_uint(v0);
            s4[1] = __float_as_uint(v1);
            s4[2] = __float_as_uint(v2);
            s4[3] = __float_as_uint(v3);
          }
        } else {
          // key j is selected by rows t in [j, j + len): (unsigned)(t - j) < len
          const int4* jj4 = reinterpret_cast<const int4*>(buf + kTcBK);
          const int4* ln4 = reinterpret_cast<const int4*>(buf + 2 * kTcBK);
#pragma unroll
          for (int c4 = 0; c4 < kTcBK / 4; ++c4) {
            const float4 d = dl4[c4];
            const int4 jv = jj4[c4], lv = ln4[c4];
            const int c = 4 * c4;
            uint32_t* s4 = &sr[c / 32][c % 32];
            const uint64_t va = f2_fma(f2(__uint_as_float(s4[0]), __uint_as_float(s4[1])), sc2, f2(d.x, d.y));
            const uint64_t vb = f2_fma(f2(__uint_as_float(s4[2]), __uint_as_float(s4[3])), sc2, f2(d.z, d.w));
            float v[4];
            f2_split(va, v[0], v[1]);
            f2_split(vb, v[2], v[3]);
            v[0] = (uint32_t)(t - jv.x) < (uint32_t)lv.x ? v[0] : -INFINITY;
            v[1] = (uint32_t)(t - jv.y) < (uint32_t)lv.y ? v[1] : -INFINITY;
            v[2] = (uint32_t)(t - jv.z) < (uint32_t)lv.z ? v[2] : -INFINITY;
            v[3] = (uint32_t)(t - jv.w) < (uint32_t)lv.w ? v[3] : -INFINITY;
#pragma unroll
            for (int u = 0; u < 4; ++u) s4[u] = __float_as_uint(v[u]);
            mt = max3(mt, v[0], v[1]);
            mt = max3(mt, v[2], v[3]);
          }
        }
        float alpha = 1.f;
        bool rescale = false;
        if (mt > m_used) {   // (also the first finite max: -inf < mt)
          alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
          m_used = mt;
          rescale = true;
        }
        const float base = m_used == -INFINITY ? 0.f : m_used;
        const uint64_t nb2 = f2(-base, -base);
        uint64_t psa = f2(0.f, 0.f), psb = f2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kTcBK / 64; ++c) {   // P (bf16 pairs) over columns [0, 64) of S_h
          uint32_t pk[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int k0 = c * 64 + 2 * u;
            const uint64_t x2 =
                f2_add(f2(__uint_as_float(sr[k0 / 32][k0 % 32]), __uint_as_float(sr[k0 / 32][k0 % 32 + 1])), nb2);
            float x0, x1, p0, p1;
            f2_split(x2, x0, x1);
            if (u % kPolyEvery == kPolyEvery - 1) {
              exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = fast_exp2(x0);
              p1 = fast_exp2(x1);
            }
            if (u & 1) psb = f2_add(psb, f2(p0, p1));
            else psa = f2_add(psa, f2(p0, p1));
            pk[u] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st32(tS + c * 32, pk);
        }
        // Rescale O_h now that the S row no longer occupies registers (PV of this tile waits for
        // p_full).  O_h holds this item's tiles < i: their PV completed before S_h of tile i was
        // computed.  The whole warp rescales when any of its rows needs it (alpha = 1 for the others).
        if (i > 0 && __any_sync(0xffffffffu, rescale)) {
          // the S row is dead: its registers take the whole O row, loaded with one wait
          uint32_t (&orow)[kTcBK / 32][32] = sr;
          static_assert(D <= kTcBK, "the O row reuses the S row's registers");
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tO + c * 32, orow[c]);
          tc::tmem_wait_ld();
          const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              float o0, o1;
              f2_split(f2_mul(f2(__uint_as_float(orow[c][u]), __uint_as_float(orow[c][u + 1])), a2), o0, o1);
              orow[c][u] = __float_as_uint(o0);
              orow[c][u + 1] = __float_as_uint(o1);
            }
            tc::tmem_st32(tO + c * 32, orow[c]);
          }
        }
        float s0, s1, s2, s3;
        f2_split(psa, s0, s1);
        f2_split(psb, s2, s3);
        l = l * alpha + ((s0 + s1) + (s2 + s3));
        tc::tmem_wait_st();
        tc::fence_before();
        tc::mbar_arrive(&bar.p_full[h]);
      }
      if (!ok) break;
      // ---- epilogue: O row = O_h / l, LSE = (m + log2 l) ln 2
      const bool own = n_tiles > 0;
      if (own) {
        const int last = tcount + n_tiles - 1;
        if (!wait_all(&bar.pv_done[h], last & 1, abort_flag, status, kErrTimeoutPV)) {
          ok = false;
          break;
        }
        tc::fence_after();
      }
      const bool valid = t >= q0 && t < N;   // a query row (rows of the first pair below q0 are not)
      OutT* orow = O + ((size_t)it.bh * Nq + (valid ? t - q0 : 0)) * D;
      // low-order bf16 part of the row (O - bf16(O)), kept for the backward's D = rowsum(dO * O), in
      // the blocked layout [b, h][128-row block][D / 8 column groups][128 rows][8]: this thread's row is
      // row r of block 2 kp + h (kept only when every position is a query, q0 = 0)
      uint16_t* lblk = Olo + ((size_t)it.bh * ((Nq + kBlockQ - 1) / kBlockQ) + it.kp * 2 + h) * kBlockQ * D;
      const bool keep_lo = valid && Olo != nullptr;
      if (it.S == 1) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tc::tmem_ld32(tO + c * 32, ov);
          tc::tmem_wait_ld();
          float of[32];
#pragma unroll
          for (int u2 = 0; u2 < 32; ++u2) of[u2] = __uint_as_float(ov[u2]) * inv;
          if (valid) store_row32(orow + c * 32, of);
          if (keep_lo) store_row32_lo(lblk + (size_t)c * 4 * kBlockQ * 8, r, of);
        }
        if (valid) LSE[(size_t)it.bh * Nq + t - q0] = ((m_used == -INFINITY ? 0.f : m_used) + __log2f(l)) * kLn2;
      } else {
        // Split pair: every split but the last to finish leaves (O unnormalised, m, l) in its slot;
        // the last one merges them with its own.  Counters per (pair, half): [arrivals, written].
        int32_t* mc = fcnt + ((size_t)it.bh * n_pairs + it.kp) * 4 + h * 2;
        if (r == 0) bar.merge_old[h] = atomicAdd(mc, 1);
        group_sync(h);
        const bool last = *reinterpret_cast<volatile int*>(&bar.merge_old[h]) == it.S - 1;
        const float mo = own ? m_used : -INFINITY, lo = own ? l : 0.f;
        if (!last) {
          float* po = fpart + ((size_t)it.slot * 2 + h) * D * kBlockQ;
          float* pml = fml + ((size_t)it.slot * 2 + h) * 2 * kBlockQ;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tc::tmem_ld32(tO + c * 32, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) po[(size_t)(c * 32 + u2) * kBlockQ + r] = own ? __uint_as_float(ov[u2]) : 0.f;
          }
          pml[r] = mo;
          pml[kBlockQ + r] = lo;
          __threadfence();
          group_sync(h);
          if (r == 0) atomicAdd(mc + 1, 1);
        } else {
          if (r == 0) {   // the others have arrived: wait (bounded) until their partials are written
            const long long c0 = clock64();
            while (ld_acquire(mc + 1) < it.S - 1) {
              if (clock64() - c0 > 4000000000LL) {
                *abort_flag = 1;
                atomicOr(status, kErrTimeoutMerge);
                break;
              }
              __nanosleep(100);
            }
          }
          group_sync(h);
          __threadfence();
          const size_t slot0 = (size_t)(it.slot - it.s);
          float mp[kMaxSplits], fp[kMaxSplits];
          float M = mo;
#pragma unroll
          for (int s2 = 0; s2 < kMaxSplits; ++s2) {
            mp[s2] = (s2 < it.S && s2 != it.s) ? __ldcg(fml + ((slot0 + s2) * 2 + h) * 2 * kBlockQ + r) : -INFINITY;
            M = fmaxf(M, mp[s2]);
          }
          const float Mb = M == -INFINITY ? 0.f : M;
          const float fo = mo == -INFINITY ? 0.f : fast_exp2(mo - Mb);
          float L = lo * fo;
#pragma unroll
          for (int s2 = 0; s2 < kMaxSplits; ++s2) {
            fp[s2] = mp[s2] == -INFINITY ? 0.f : fast_exp2(mp[s2] - Mb);
            if (fp[s2] != 0.f) L += __ldcg(fml + ((slot0 + s2) * 2 + h) * 2 * kBlockQ + kBlockQ + r) * fp[s2];
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tc::tmem_ld32(tO + c * 32, ov);
            tc::tmem_wait_ld();
            float of[32];
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) of[u2] = fo != 0.f ? __uint_as_float(ov[u2]) * fo : 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              if (fp[s2] == 0.f) continue;
              const float* po = fpart + ((slot0 + s2) * 2 + h) * D * kBlockQ + (size_t)(c * 32) * kBlockQ + r;
#pragma unroll
              for (int u2 = 0; u2 < 32; ++u2) of[u2] = fmaf(__ldcg(po + (size_t)u2 * kBlockQ), fp[s2], of[u2]);
            }
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) of[u2] *= inv;
            if (valid) store_row32(orow + c * 32, of);
            if (keep_lo) store_row32_lo(lblk + (size_t)c * 4 * kBlockQ * 8, r, of);
          }
          if (valid) LSE[(size_t)it.bh * Nq + t - q0] = (Mb + __log2f(L)) * kLn2;
          group_sync(h);
          if (r == 0) {   // leave the counters at zero for the next launch on the same mask
            mc[0] = 0;
            mc[1] = 0;
          }
        }
      }
      tc::fence_before();
      tcount += n_tiles;
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, 512);
  if (tid == 0) {   // the last CTA to finish leaves the schedule's counters at zero for the next launch
    __threadfence();
    if (atomicAdd(sched_ctr + 1, 1) == (int)gridDim.x - 1) {
      sched_ctr[0] = 0;
      sched_ctr[1] = 0;
    }
  }
}

template <int D, typename OutT>
cudaError_t launch_tc_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                        const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                        cudaStream_t s) {
  CUtensorMap qm, km, vm;
  if (!make_row_map(&qm, Q, (uint64_t)P.B * P.H * P.Nq, D) || !make_row_map(&km, K, (uint64_t)P.B * P.Hkv * P.N, D) ||
      !make_row_map(&vm, V, (uint64_t)P.B * P.Hkv * P.N, D))
    return cudaErrorInvalidValue;
  auto k = attn_fwd_tc_kernel<D, OutT>;
  const int smem = TcSmem<D>::kBytes;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  // persistent: one CTA per SM (the shared-memory footprint admits one), at most one per unit
  const int grid = P.sched.n_units < sm_count() ? P.sched.n_units : sm_count();
  if (grid <= 0) return cudaSuccess;
  // delta and e enter through the per-entry metadata that the list kernel wrote beside the lists
  (void)delta;
  (void)evict;
  k<<<grid, kTcThreads, smem, s>>>(qm, km, vm, P.sched, ws_ptr<int32_t>(ws, P.off_pcounts),
                                   ws_ptr<int32_t>(ws, P.off_plists), ws_ptr<int32_t>(ws, P.off_plen),
                                   ws_ptr<float>(ws, P.off_pdl), (OutT*)O, LSE,
                                   P.off_olo ? ws_ptr<uint16_t>(ws, P.off_olo) : nullptr,
                                   ws_ptr<float>(ws, P.off_fpart),
                                   ws_ptr<float>(ws, P.off_fml), ws_ptr<int32_t>(ws, P.off_fcnt),
                                   ws_ptr<int32_t>(ws, P.off_fcnt) + (size_t)P.B * P.H * P.n_pairs * 4,
                                   ws_ptr<int32_t>(ws, P.off_status), P.H, P.G, P.N, P.n_pairs, P.pair_cap,
                                   P.scale * kLog2e, P.q0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                               cudaStream_t s) {
  if (P.N > 32767) return cudaErrorInvalidValue;   // key indices are packed in 16 bits
  if (P.d == 128)
    return P.bf16 ? launch_tc_t<128, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, s)
                  : launch_tc_t<128, float>(P, Q, K, V, delta, evict, ws, O, LSE, s);
  return P.bf16 ? launch_tc_t<64, uint16_t>(P, Q, K, V, delta, evict, ws, O, LSE, s)
                : launch_tc_t<64, float>(P, Q, K, V, delta, evict, ws, O, LSE, s);
}

}  // namespace dma
