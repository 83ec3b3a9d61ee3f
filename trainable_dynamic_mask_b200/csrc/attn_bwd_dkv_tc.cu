// Masked attention backward, dK / dV / d delta part, on the 5th-generation tensor cores.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Theoretical Guarantees for
// Safe Computation Skipping" (masked pairs have exactly zero gradient, so they are skipped) and
// section "Gradient Flow Integrity" (trainable end to end).
//
// With P the masked softmax (recomputed from the forward's LSE), dP = dO V^T, D_t = sum_c dO_tc O_tc
// and dS = P (dP - D): dV_g = sum_{h in g} P_h^T dO_h, dK_g = scale sum_{h in g} dS_h^T Q_h and
// d delta_{h,j} = sum_t dS_{h,tj}.
//
// Key j receives gradient from the queries t in [j, e_j) only (the selection interval of the mask
// encoding).  The work is therefore organised per query head and key tile: within each window of
// 1024 positions, the head's live keys (e_j > j) are ordered by e_j, longest-lived first, and cut
// into tiles of 128; a tile walks the query steps of 64 rows covering [min j, max e_j) and masks per
// pair.  Keys of similar lifetime share a tile, so little of the walked range is masked.  Each
// (head, tile) item writes f32 partial dK_h, dV_h rows; a last kernel sums the G heads of each group.
//
// Kernels: order (per head and window: the key order and each tile's query range; d delta = 0),
// schedule (items by length, longest first), the tcgen05 kernel, reduce.
//
// tcgen05 kernel, per CTA (persistent, items dealt in snake order over the sorted list):
//   warps 0-7   elementwise: warp w owns key rows 32 (w % 4) .. + 31 (its TMEM lane quarter) and
//               query columns 32 (w / 4) .. + 31 of each step: P^T = exp2(s scale log2 e + delta_j
//               log2 e - LSE_t log2 e) with the mask j <= t < e_j, dS^T = P^T (dP^T - D_t); P^T and
//               dS^T (bf16) are written back over the columns of S^T and dP^T they were read from;
//               at the end of an item, warps 0-3 write dK (x scale) and warps 4-7 dV, and each
//               half adds its row sums of dS^T to d delta (two f32 adds onto 0: exact in any order);
//   warp 8      TMEM allocation; one thread issues S^T = K Q^T (operands in shared memory) and
//               dV += P^T dO (A from TMEM, B read N-major);
//   warp 10     one thread issues dP^T = V dO^T and dK += dS^T Q.  One thread issues a tcgen05.mma
//               about every 60-110 cycles, slower than the tensor pipe runs these M128 N64
//               products, so the products are split evenly over two threads on different SM
//               sub-partitions; each thread's commits track only its own MMAs, so the barriers
//               both feed count two arrivals;
//   warp 9      gathers the item's K and V rows (TMA tile::gather4), double-buffered across items;
//   warp 11     loads the Q and dO tiles of each step (TMA tiles of 64 rows), three stages.
// TMEM: S^T buffers at columns 0 and 128, dP^T at 64 and 192 (64 columns each; step T uses buffer
// T % 2, so the S^T/dP^T products of step T + 1 run while step T is elementwise), dK [256, 256 + D),
// dV [384, 384 + D).  Every wait is bounded (tc::mbar_wait).
#include <cuda.h>
#include <limits.h>

#include "tc_ops.cuh"

namespace dma {
namespace {

constexpr int kDkThreads = 384;
constexpr int kDkMmaWarp = 8;
constexpr int kDkKVWarp = 9, kDkGradWarp = 10, kDkQWarp = 11;
constexpr int kDkBK = 128;        // keys per item
constexpr int kDkBQ = 64;         // queries per step
constexpr int kDkQStages = 3;     // Q / dO stages
constexpr int kDkWin = 1024;      // positions per ordering window
constexpr int kDkTilesPerWin = kDkWin / kDkBK;
constexpr uint32_t kDkS = 0, kDkDP = 64, kDkBuf = 128, kDkDK = 256, kDkDV = 384;   // TMEM columns

// Device status codes: bit 0x10000000 marks this kernel, the other bits the wait that gave up
// (bits the other kernels use are avoided).
enum : int { kErrDkKV = 0x10000010, kErrDkQ = 0x10000020, kErrDkS = 0x10000040, kErrDkDS = 0x10000080,
             kErrDkAcc = 0x30000000, kErrDkEmpty = 0x50000000, kErrDkAlign = 0x10000008 };

DMA_DEVINL void store4_from_f32(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
DMA_DEVINL void store4_from_f32(uint16_t* p, float4 v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

template <int D>
struct DkSmem {
  static constexpr int kKV = (D / 64) * kDkBK * 128;   // 128 rows: [D/64][128][128 B]
  static constexpr int kQT = (D / 64) * kDkBQ * 128;   // 64 rows:  [D/64][64][128 B]
  static constexpr int kK = 0;                          // [2 item buffers]
  static constexpr int kV = 2 * kKV;                    // [2]
  static constexpr int kQ = 4 * kKV;                    // [kDkQStages]
  static constexpr int kdO = kQ + kDkQStages * kQT;     // [kDkQStages]
  static constexpr int kMeta = kdO + kDkQStages * kQT;  // [kDkQStages][64 columns] float2 (lse2, D)
  static constexpr int kBars = kMeta + kDkQStages * kDkBQ * 8;
  static constexpr int kBytes = kBars + 256;
};

struct DkBars {
  uint64_t kv_full[2], kv_empty[2];
  uint64_t qd_full[kDkQStages], qd_empty[kDkQStages];
  uint64_t s_full[2], ds_full[2];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};

// tcgen05.mma, A and B from shared memory, descriptors advanced by AOFF / 16 and BOFF / 16.
template <uint32_t AOFF, uint32_t BOFF>
DMA_DEVINL void mma_ss_off(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "add.s64 a, %1, %5;\n\t"
      "add.s64 b, %2, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(AOFF >> 4), "n"(BOFF >> 4));
}
// tcgen05.mma, A from TMEM column a_tmem + ACOL, B from shared memory at descriptor + BOFF / 16.
template <uint32_t ACOL, uint32_t BOFF>
DMA_DEVINL void mma_ts_off(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "add.s64 b, %2, %5;\n\t"
      "add.u32 a, %1, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(BOFF >> 4), "n"(ACOL));
}

// S^T or dP^T (M128 N64): A = a 128-row tile, B = a 64-row tile, both K-major SW128 with their
// 64-column halves 16384 and 8192 bytes apart; D / 16 K steps.
template <int KK, int NK>
struct DkSdpSteps {
  DMA_DEVINL static void run(uint32_t d, uint64_t da, uint64_t db, uint32_t id) {
    mma_ss_off<(KK >> 2) * 16384 + (KK & 3) * 32, (KK >> 2) * 8192 + (KK & 3) * 32>(d, da, db, id,
                                                                                    KK > 0 ? 1u : 0u);
    if constexpr (KK + 1 < NK) DkSdpSteps<KK + 1, NK>::run(d, da, db, id);
  }
};
// dV += P^T dO or dK += dS^T Q (M128 N=D, K = 64 queries in 4 steps of 16).  A: the bf16 pairs the
// elementwise warps stored, query columns [32 h, 32 h + 32) at TMEM columns [32 h, 32 h + 16) of
// the buffer; B: the 64-row tile read N-major (16 rows = 2048 bytes per K step).
template <int KK>
struct DkGradSteps {
  DMA_DEVINL static void run(uint32_t d, uint32_t a, uint64_t db, uint32_t id, uint32_t acc0) {
    mma_ts_off<32 * (KK >> 1) + 8 * (KK & 1), KK * 2048>(d, a, db, id, KK > 0 ? 1u : acc0);
    if constexpr (KK + 1 < kDkBQ / 16) DkGradSteps<KK + 1>::run(d, a, db, id, acc0);
  }
};

DMA_DEVINL int dk_item_index(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

// ---------------------------------------------------------------- order
// One CTA per (window of kDkWin positions, b * H + h).  Sorts the window's live keys by e_j
// descending (then position) and writes, per tile of kDkBK consecutive entries of that order, the
// item record {first query step row qlo (a multiple of kDkBQ), steps, keys, offset of its keys in
// perm}; steps = 0 marks an empty slot.  Sets d delta to 0 (it stays 0 for keys no query selects).
__global__ void __launch_bounds__(kDkWin)
bwd_dkv_order_kernel(const int32_t* __restrict__ evict, int32_t* __restrict__ perm, int4* __restrict__ slots,
                     float* __restrict__ d_delta, int N, int n_win) {
  __shared__ uint32_t key[kDkWin];
  __shared__ int tile_min[kDkWin / 32];
  const int win = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int w0 = win * kDkWin;
  const int j = w0 + tid;
  const int e = j < N ? evict[(size_t)bh * N + j] : 0;
  const bool live = j < N && e > j;
  if (j < N) d_delta[(size_t)bh * N + j] = 0.f;   // the tcgen05 kernel adds its two halves' sums
  // N - e < 2^15 (N <= 16384) above 10 bits of window position: ascending = e descending, then j
  key[tid] = live ? ((uint32_t)(N - e) << 10) | (uint32_t)tid : 0xffffffffu;
  const int n_live = __syncthreads_count(live);
  for (int size = 2; size <= kDkWin; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int partner = tid ^ stride;
      if (partner > tid) {
        const uint32_t a = key[tid], c = key[partner];
        const bool up = (tid & size) == 0;
        if ((a > c) == up) {
          key[tid] = c;
          key[partner] = a;
        }
      }
      __syncthreads();
    }
  const bool mine = tid < n_live;
  const int jj = mine ? w0 + (int)(key[tid] & 1023u) : INT_MAX;
  if (mine) perm[(size_t)bh * N + w0 + tid] = jj;
  int m = jj;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = min(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) tile_min[tid >> 5] = m;
  __syncthreads();
  if (tid < kDkTilesPerWin) {
    const int k = tid;
    int4 rec = make_int4(0, 0, 0, 0);
    if (k * kDkBK < n_live) {
      int mn = INT_MAX;
      for (int u = 0; u < kDkBK / 32; ++u) mn = min(mn, tile_min[k * (kDkBK / 32) + u]);
      const int emax = N - (int)(key[k * kDkBK] >> 10);   // the tile's first entry lives longest
      const int qlo = (mn / kDkBQ) * kDkBQ;
      rec.x = qlo;
      rec.y = (emax - qlo + kDkBQ - 1) / kDkBQ;
      rec.z = min(kDkBK, n_live - k * kDkBK);
      rec.w = bh * N + w0 + k * kDkBK;
    }
    slots[((size_t)bh * n_win + win) * kDkTilesPerWin + k] = rec;
  }
}

// ---------------------------------------------------------------- schedule
// One CTA: the non-empty slots ordered by steps, longest first (counting sort; the order among
// equal lengths is arbitrary and does not affect any result).  items[0 .. *n_items).
__global__ void __launch_bounds__(1024)
bwd_dkv_sched_kernel(const int4* __restrict__ slots, int n_slots, int max_steps, int32_t* __restrict__ items,
                     int32_t* __restrict__ n_items) {
  extern __shared__ int hist[];   // [max_steps + 1]: bin s holds length max_steps - s
  const int tid = threadIdx.x;
  for (int i = tid; i <= max_steps; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int s = tid; s < n_slots; s += blockDim.x) {
    const int st = slots[s].y;
    if (st > 0) atomicAdd(&hist[max_steps - min(st, max_steps)], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i <= max_steps; ++i) {
      const int c = hist[i];
      hist[i] = run;
      run += c;
    }
    *n_items = run;
  }
  __syncthreads();
  for (int s = tid; s < n_slots; s += blockDim.x) {
    const int st = slots[s].y;
    if (st > 0) items[atomicAdd(&hist[max_steps - min(st, max_steps)], 1)] = s;
  }
}

// ---------------------------------------------------------------- reduce
// dK_g = sum over the heads h of group g that select key j of the partial rows, likewise dV.
// One thread per 4 channels of a (b, g, j) row.
template <typename OutT>
__global__ void bwd_dkv_reduce_kernel(const float* __restrict__ part_k, const float* __restrict__ part_v,
                                      const int32_t* __restrict__ evict, OutT* __restrict__ dK,
                                      OutT* __restrict__ dV, int H, int G, int N, int D, size_t n_quads) {
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= n_quads) return;
  const int dq = D / 4;
  const size_t row = q / dq;   // (b * Hkv + g) * N + j
  const int c = (int)(q % dq) * 4;
  const int j = (int)(row % N);
  const size_t bg = row / N;
  const int Hkv = H / G;
  const int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
  float4 ak = make_float4(0.f, 0.f, 0.f, 0.f), av = ak;
  for (int hh = 0; hh < G; ++hh) {
    const size_t bh = (size_t)b * H + g * G + hh;
    if (evict[bh * N + j] > j) {
      const float4 k4 = *reinterpret_cast<const float4*>(part_k + (bh * N + j) * D + c);
      const float4 v4 = *reinterpret_cast<const float4*>(part_v + (bh * N + j) * D + c);
      ak.x += k4.x; ak.y += k4.y; ak.z += k4.z; ak.w += k4.w;
      av.x += v4.x; av.y += v4.y; av.z += v4.z; av.w += v4.w;
    }
  }
  store4_from_f32(dK + row * D + c, ak);
  store4_from_f32(dV + row * D + c, av);
}

// ---------------------------------------------------------------- tcgen05 kernel
template <int D>
__global__ void __launch_bounds__(kDkThreads, 1)
bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                  const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const int4* __restrict__ slots, const int32_t* __restrict__ items,
                  const int32_t* __restrict__ n_items_p, const int32_t* __restrict__ perm,
                  const float* __restrict__ delta, const int32_t* __restrict__ evict,
                  const float* __restrict__ LSE, const float* __restrict__ Drow, float* __restrict__ part_k,
                  float* __restrict__ part_v, float* __restrict__ d_delta, int32_t* __restrict__ status, int H,
                  int G, int N, int n_win, float scale_log2, float scale) {
  using S = DkSmem<D>;
  extern __shared__ __align__(1024) unsigned char sm[];
  DkBars& bar = *reinterpret_cast<DkBars*>(sm + S::kBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, n_ctas = gridDim.x;
  const int n_items = *n_items_p;
  volatile int* abort_flag = &bar.abort_flag;
  if (tid == 0) {
    bar.abort_flag = 0;
    if (smem_u32(sm) & 1023u) {
      atomicOr(status, kErrDkAlign);
      bar.abort_flag = 1;
    }
    for (int i = 0; i < 2; ++i) {   // barriers both issuers feed count two arrivals
      tc::mbar_init(&bar.kv_full[i], 32);
      tc::mbar_init(&bar.kv_empty[i], 2);
      tc::mbar_init(&bar.s_full[i], 2);
      tc::mbar_init(&bar.ds_full[i], 8);   // one arrival per elementwise warp
    }
    for (int i = 0; i < kDkQStages; ++i) {
      tc::mbar_init(&bar.qd_full[i], 32);   // the loader warp's lanes
      tc::mbar_init(&bar.qd_empty[i], 2);   // both MMA issuers read the stage
    }
    tc::mbar_init(&bar.acc_full, 2);
    tc::mbar_init(&bar.acc_empty, 8);
    tc::mbar_init(&bar.drain, 2);
    tc::fence_mbar_init();
  }
  if (warp == kDkMmaWarp) {
    tc::tmem_alloc(&bar.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = bar.tmem_base;
  constexpr uint32_t kRowBytes = D * 2;
  // The r-th item of this CTA: its record and b * H + h; false past the last item.  Every role walks
  // the same sequence.
  auto item_at = [&](int r, int4& rec, int& bh) -> bool {
    const int idx = dk_item_index(r, cta, n_ctas);
    if (idx >= n_items) return false;
    const int slot = items[idx];
    rec = slots[slot];
    bh = slot / (n_win * kDkTilesPerWin);
    return true;
  };
  int4 rec;
  int bh;

  if (warp == kDkKVWarp) {
    // ------------------------------------------------------------ K and V rows of each item (gather4)
    int n = 0;
    bool ok = !*abort_flag;
    for (int r = 0; ok && item_at(r, rec, bh); ++r, ++n) {
      const int buf = n & 1;
      if (n >= 2 && !wait_all(&bar.kv_empty[buf], ((n >> 1) - 1) & 1, abort_flag, status, kErrDkEmpty)) {
        ok = false;
        break;
      }
      const int b = bh / H, h = bh % H, Hkv = H / G;
      const int kvrow0 = (b * Hkv + h / G) * N;
      int rr[4];   // this lane's 4 rows; rows past the tile's keys fetch row 0 (their P and dS are 0)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int li = 4 * lane + u;
        rr[u] = kvrow0 + (li < rec.z ? perm[rec.w + li] : 0);
      }
      mbar_arrive_expect_tx(&bar.kv_full[buf], 8 * kRowBytes);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        tma_gather4(smem_u32(sm + S::kK + buf * S::kKV) + hf * (kDkBK * 128) + lane * 512, &kmap, hf * 64, rr[0],
                    rr[1], rr[2], rr[3], &bar.kv_full[buf]);
        tma_gather4(smem_u32(sm + S::kV + buf * S::kKV) + hf * (kDkBK * 128) + lane * 512, &vmap, hf * 64, rr[0],
                    rr[1], rr[2], rr[3], &bar.kv_full[buf]);
      }
    }
    if (!ok)
      for (int m = n >= 2 ? n - 2 : 0; m < n; ++m) drain_wait(&bar.kv_full[m & 1], (m >> 1) & 1);
  } else if (warp == kDkQWarp) {
    // ------------------------------------------------------------ Q and dO tiles of each step
    // Lane 0 loads the tiles; every lane also stages (LSE_t log2 e, D_t) of two of the step's 64
    // query columns in shared memory beside them (published by its arrival on the stage's barrier;
    // the values are loaded a step ahead, so no lane waits on a load).  Columns past N get
    // (+inf, 0): P = 0 there.
    int T = 0;
    bool ok = !*abort_flag;
    float2* metaq = reinterpret_cast<float2*>(sm + S::kMeta);
    for (int r = 0; ok && item_at(r, rec, bh); ++r) {
      const size_t hrow = (size_t)bh * N;
      auto load_meta = [&](int i, float4& m) {
        const int t = rec.x + i * kDkBQ + 2 * lane;
        m.x = t < N ? LSE[hrow + t] * kLog2e : INFINITY;
        m.y = t < N ? Drow[hrow + t] : 0.f;
        m.z = t + 1 < N ? LSE[hrow + t + 1] * kLog2e : INFINITY;
        m.w = t + 1 < N ? Drow[hrow + t + 1] : 0.f;
      };
      float4 mc, mn;
      load_meta(0, mc);
      for (int i = 0; i < rec.y; ++i, ++T) {
        const int st = T % kDkQStages;
        if (i + 1 < rec.y) load_meta(i + 1, mn);
        if (T >= kDkQStages &&
            !wait_all(&bar.qd_empty[st], ((T / kDkQStages) - 1) & 1, abort_flag, status, kErrDkEmpty)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          // rows past this head's N belong to the next head or lie past the tensor (zero fill): the
          // mask drops every pair with t >= N
          const int y = bh * N + rec.x + i * kDkBQ;
          mbar_expect_tx(&bar.qd_full[st], 2 * kDkBQ * kRowBytes);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            tma_tile_2d(smem_u32(sm + S::kQ + st * S::kQT) + hf * (kDkBQ * 128), &qmap, hf * 64, y, &bar.qd_full[st]);
            tma_tile_2d(smem_u32(sm + S::kdO + st * S::kQT) + hf * (kDkBQ * 128), &domap, hf * 64, y,
                        &bar.qd_full[st]);
          }
        }
        reinterpret_cast<float4*>(metaq + st * kDkBQ)[lane] = mc;
        tc::mbar_arrive(&bar.qd_full[st]);
        mc = mn;
      }
    }
    if (!ok && lane == 0)
      for (int m = T >= kDkQStages ? T - kDkQStages : 0; m < T; ++m)
        drain_wait(&bar.qd_full[m % kDkQStages], (m / kDkQStages) & 1);
  } else if (warp == kDkMmaWarp || warp == kDkGradWarp) {
    // ------------------------------------------------------------ MMA issue (lane 0 of warps 8 and 10)
    // Warp 8 issues S^T = K Q^T and dV += P^T dO, warp 10 dP^T = V dO^T and dK += dS^T Q.  Each
    // buffer reuse is ordered by one thread's issue order: S^T(U) (dP^T(U)) overwrites the P^T (dS^T)
    // that the same thread's dV (dK) product of step U - 2 reads, issued after the elementwise pass
    // of U - 2 ended (tcgen05.mma of one thread run in issue order).
    if (lane == 0) {
      const bool sv = warp == kDkMmaWarp;
      constexpr uint32_t id_sdp = tc::idesc_bf16(128, kDkBQ, false, false);
      constexpr uint32_t id_grad = tc::idesc_bf16(128, D, false, true);
      const uint32_t sdp_col = sv ? kDkS : kDkDP;   // S^T / P^T or dP^T / dS^T columns of a buffer
      const uint32_t acc_col = sv ? kDkDV : kDkDK;
      const int a_off = sv ? S::kK : S::kV;         // A of the S^T (dP^T) product: K (V) rows
      const int b_off = sv ? S::kQ : S::kdO;        // its B: the Q (dO) tile
      const int g_off = sv ? S::kdO : S::kQ;        // B of the gradient product, read N-major
      int T = 0, n = 0;
      bool ok = !*abort_flag;
      auto sdp = [&](int U, uint64_t ad) -> bool {
        const int b = U & 1, st = U % kDkQStages;
        if (!tc::mbar_wait(&bar.qd_full[st], (U / kDkQStages) & 1, abort_flag, status, kErrDkQ)) return false;
        tc::fence_after();
        const uint64_t bd = tc::sdesc(smem_u32(sm + b_off + st * S::kQT), 16, 1024);
        DkSdpSteps<0, D / 16>::run(tmem + b * kDkBuf + sdp_col, ad, bd, id_sdp);
        tc::commit(&bar.s_full[b]);
        return true;
      };
      for (int r = 0; ok && item_at(r, rec, bh); ++r, ++n) {
        const int kvb = n & 1;
        if (!(ok = tc::mbar_wait(&bar.kv_full[kvb], (n >> 1) & 1, abort_flag, status, kErrDkKV))) break;
        const uint64_t ad = tc::sdesc(smem_u32(sm + a_off + kvb * S::kKV), 16, 1024);
        const int steps = rec.y;
        if (!(ok = sdp(T, ad))) break;
        if (steps == 1) tc::commit(&bar.kv_empty[kvb]);
        for (int i = 0; i < steps; ++i) {
          const int U = T + i, b = U & 1, st = U % kDkQStages;
          if (i + 1 < steps) {
            if (!(ok = sdp(U + 1, ad))) break;
            if (i + 2 == steps) tc::commit(&bar.kv_empty[kvb]);   // K (V) of the item read for the last time
          }
          // dV (dK) += P^T (dS^T) of step U times its dO (Q) tile; the first step of an item starts
          // the accumulator, which the previous item's epilogue must have read
          if (!(ok = tc::mbar_wait(&bar.ds_full[b], (U >> 1) & 1, abort_flag, status, kErrDkDS))) break;
          if (i == 0 && n >= 1 && !(ok = tc::mbar_wait(&bar.acc_empty, (n - 1) & 1, abort_flag, status, kErrDkAcc)))
            break;
          tc::fence_after();
          const uint64_t gd = tc::sdesc(smem_u32(sm + g_off + st * S::kQT), kDkBQ * 128, 1024);
          DkGradSteps<0>::run(tmem + acc_col, tmem + b * kDkBuf + sdp_col, gd, id_grad, i == 0 ? 0u : 1u);
          tc::commit(&bar.qd_empty[st]);
        }
        if (!ok) break;
        tc::commit(&bar.acc_full);
        T += steps;
      }
      tc::commit(&bar.drain);
      drain_wait(&bar.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise (warps 0-7)
    const int hf = warp >> 2, qd = warp & 3;
    const int r = 32 * qd + lane;   // key row of the item = TMEM lane
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const float2* metaq = reinterpret_cast<const float2*>(sm + S::kMeta);   // [stage][64 columns]
    const uint64_t sc2 = f2(scale_log2, scale_log2);
    int T = 0, n = 0;
    bool ok = !*abort_flag;
    for (int rr = 0; ok && item_at(rr, rec, bh); ++rr, ++n) {
      const int steps = rec.y;
      const size_t hrow = (size_t)bh * N;
      const int jr = r < rec.z ? perm[rec.w + r] : -1;
      const int e = jr >= 0 ? evict[hrow + jr] : 0;
      const float dl = jr >= 0 ? delta[hrow + jr] * kLog2e : 0.f;
      const int len = jr >= 0 ? e - jr : 0;
      const uint64_t dl2 = f2(dl, dl);
      float dd = 0.f;
      for (int i = 0; i < steps; ++i) {
        const int U = T + i, b = U & 1, st = U % kDkQStages;
        // (LSE_t log2 e, D_t) of the step's columns, staged beside its Q / dO tiles
        if (!wait_all(&bar.s_full[b], (U >> 1) & 1, abort_flag, status, kErrDkS) ||
            !wait_all(&bar.qd_full[st], (U / kDkQStages) & 1, abort_flag, status, kErrDkQ)) {
          ok = false;
          break;
        }
        tc::fence_after();
        const float4* meta4 = reinterpret_cast<const float4*>(metaq + st * kDkBQ + 32 * hf);
        const uint32_t sb = tmem + b * kDkBuf + kDkS + lane_base + 32 * hf;
        const uint32_t pb = tmem + b * kDkBuf + kDkDP + lane_base + 32 * hf;
        uint32_t sv[32], pv[32], pk[16], dk[16];
        tc::tmem_ld32(sb, sv);
        tc::tmem_ld32(pb, pv);
        tc::tmem_wait_ld();
        const int t0 = rec.x + i * kDkBQ + 32 * hf;   // first column of this warp
        const bool full = __all_sync(0xffffffffu, jr >= 0 && jr <= t0 && e >= t0 + 32);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 m = meta4[u];   // (lse2, D) of columns 2u, 2u + 1
          const uint64_t x2 = f2_sub(
              f2_fma(f2(__uint_as_float(sv[2 * u]), __uint_as_float(sv[2 * u + 1])), sc2, dl2), f2(m.x, m.z));
          float x0, x1;
          f2_split(x2, x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if (!full) {
            const int t = t0 + 2 * u;
            p0 = (uint32_t)(t - jr) < (uint32_t)len ? p0 : 0.f;
            p1 = (uint32_t)(t + 1 - jr) < (uint32_t)len ? p1 : 0.f;
          }
          const uint64_t ds2 =
              f2_mul(f2(p0, p1), f2_sub(f2(__uint_as_float(pv[2 * u]), __uint_as_float(pv[2 * u + 1])), f2(m.y, m.w)));
          float ds0, ds1;
          f2_split(ds2, ds0, ds1);
          dd += ds0 + ds1;
          pk[u] = pack_bf16x2(p0, p1);
          dk[u] = pack_bf16x2(ds0, ds1);
        }
        // P^T over S^T and dS^T over dP^T, into the first 16 of the 32 columns just read
        tc::tmem_st16(sb, pk);
        tc::tmem_st16(pb, dk);
        tc::tmem_wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bar.ds_full[b]);
      }
      if (!ok) break;
      // ---- epilogue: dK (warps 0-3) or dV (warps 4-7) rows of the item's keys, f32 partials
      if (!wait_all(&bar.acc_full, n & 1, abort_flag, status, kErrDkAcc)) {
        ok = false;
        break;
      }
      tc::fence_after();
      {
        const uint32_t acc = tmem + (hf == 0 ? kDkDK : kDkDV) + lane_base;
        float* dst = (hf == 0 ? part_k : part_v) + (hrow + (jr >= 0 ? jr : 0)) * D;
        const float mul = hf == 0 ? scale : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tc::tmem_ld32(acc + 32 * c, v);
          tc::tmem_wait_ld();
          if (jr >= 0) {
#pragma unroll
            for (int u = 0; u < 32; u += 4)
              *reinterpret_cast<float4*>(dst + 32 * c + u) =
                  make_float4(__uint_as_float(v[u]) * mul, __uint_as_float(v[u + 1]) * mul,
                              __uint_as_float(v[u + 2]) * mul, __uint_as_float(v[u + 3]) * mul);
          }
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar.acc_empty);
      if (jr >= 0) atomicAdd(d_delta + hrow + jr, dd);
      T += steps;
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == kDkMmaWarp) tc::tmem_dealloc(tmem, 512);
}

template <int D, typename OutT>
cudaError_t launch_dkv_tc_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                            const float* LSE, const float* Drow, void* dK, void* dV, float* d_delta,
                            cudaStream_t s) {
  const int BH = P.B * P.H;
  const int n_win = (P.N + kDkWin - 1) / kDkWin;
  const int n_slots = BH * n_win * kDkTilesPerWin;
  int32_t* perm = ws_ptr<int32_t>(ws, P.off_dkv_perm);
  int4* slots = ws_ptr<int4>(ws, P.off_dkv_slots);
  int32_t* items = ws_ptr<int32_t>(ws, P.off_dkv_items);
  int32_t* n_items = items + n_slots;
  float* part_k = ws_ptr<float>(ws, P.off_dkv_part);
  float* part_v = part_k + (size_t)BH * P.N * D;
  bwd_dkv_order_kernel<<<dim3(n_win, BH), kDkWin, 0, s>>>(evict, perm, slots, d_delta, P.N, n_win);
  const int max_steps = (P.N + kDkBQ - 1) / kDkBQ + 1;
  bwd_dkv_sched_kernel<<<1, 1024, (max_steps + 1) * sizeof(int), s>>>(slots, n_slots, max_steps, items, n_items);
  CUtensorMap qm, dom, km, vm;
  if (!make_tile_map(&qm, Q, (uint64_t)BH * P.N, D, kDkBQ) || !make_tile_map(&dom, dO, (uint64_t)BH * P.N, D, kDkBQ) ||
      !make_row_map(&km, K, (uint64_t)P.B * P.Hkv * P.N, D) || !make_row_map(&vm, V, (uint64_t)P.B * P.Hkv * P.N, D))
    return cudaErrorInvalidValue;
  auto k = bwd_dkv_tc_kernel<D>;
  const int smem = DkSmem<D>::kBytes;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  const int grid = n_slots < sm_count() ? n_slots : sm_count();
  k<<<grid, kDkThreads, smem, s>>>(qm, dom, km, vm, slots, items, n_items, perm, delta, evict, LSE, Drow, part_k,
                                   part_v, d_delta, ws_ptr<int32_t>(ws, P.off_status), P.H, P.G, P.N, n_win,
                                   P.scale * kLog2e, P.scale);
  const size_t n_quads = (size_t)P.B * P.Hkv * P.N * (D / 4);
  bwd_dkv_reduce_kernel<OutT><<<(unsigned)((n_quads + 255) / 256), 256, 0, s>>>(
      part_k, part_v, evict, (OutT*)dK, (OutT*)dV, P.H, P.G, P.N, D, n_quads);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkv_tc(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              const uint16_t* dO, const float* delta, const int32_t* evict, void* ws,
                              const float* LSE, const float* Drow, void* dK, void* dV, float* d_delta,
                              cudaStream_t s) {
  if (P.N > kTopwMaxN) return cudaErrorInvalidValue;
  if (P.d == 128)
    return P.bf16 ? launch_dkv_tc_t<128, uint16_t>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dK, dV, d_delta, s)
                  : launch_dkv_tc_t<128, float>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dK, dV, d_delta, s);
  return P.bf16 ? launch_dkv_tc_t<64, uint16_t>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dK, dV, d_delta, s)
                : launch_dkv_tc_t<64, float>(P, Q, K, V, dO, delta, evict, ws, LSE, Drow, dK, dV, d_delta, s);
}

}  // namespace dma
