// Masked attention forward on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient Sparse Attention
// Computation" (o_t equation), "Theoretical Guarantees for Safe Computation Skipping" (masked pairs
// have weight exactly 0 and are skipped) and "Hardware-Optimized Implementation" (block-wise,
// FlashAttention-style computation on tensor cores, O(n w d) work).
//
// One CTA per (b, h, block of 128 query rows), walking the block's live-key list (full keys first)
// in tiles of 128 keys.  The tiles are split into two interleaved streams, A (even tiles) and B
// (odd tiles), each with its own S, P, O and softmax state, so that two softmax warps share every
// SM sub-partition and the tensor core always has the other stream's work while one stream runs
// its softmax.  The two partial results are merged at the end.
//
// Warp roles (512 threads; warps 9-11 only complete the third warpgroup):
//   warps 0-3  softmax of stream A, warps 4-7 softmax of stream B: thread r owns query row
//              r = TMEM lane r.  It reads its S row from TMEM, applies scale, +delta_j and the mask
//              j <= t < e_j (tiles of full keys skip the test), keeps the running max and sum in
//              registers, writes P (bf16) back over S in TMEM, and rescales its O row only when the
//              running max grows by more than 2^8 (the stale max otherwise stays the reference);
//   warp 8     allocates TMEM; one thread issues the MMAs: S = Q K^T (A and B from shared memory)
//              and O += P V (A = P from TMEM, B = V from shared memory);
//   warps 12-15 producers: thread p owns row p of every tile (its list entry, delta*log2(e) and
//              (j, e_j)); lanes 0-7 of each warp gather 4 rows each of K and V with TMA tile::gather4
//              (128-byte swizzled, the layout the MMA reads).  The TMA issue rate of one warp caps
//              gather throughput, so four warps issue.
// TMEM: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [384,384+D); P_X aliases S_X.
// Stages: K 3, V 2 (each stream owns one V stage), metadata 4 (released by the softmax).
// Every wait is bounded (tc::mbar_wait) and reports a timeout through the workspace status word;
// every TMEM load/store (warp-collective) sits behind warp-uniform decisions.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <limits.h>

#include <mutex>

#include "tc.cuh"

namespace dma {
namespace {

constexpr int kTcThreads = 512;       // 4 warpgroups: softmax A, softmax B, MMA (+3 idle), producers
constexpr int kProdWarp0 = 12, kProdWarps = 4, kProdThreads = kProdWarps * 32;
// Register split between the warpgroups (setmaxnreg): launched with 128 per thread (512 x 128 =
// 65536), the MMA and producer warpgroups give back to 48 and the softmax warpgroups take 208:
// 256 x 48 + 256 x 208 = 65536, so the increase can always be satisfied.
constexpr int kRegsSoftmax = 208, kRegsOther = 48;
constexpr int kTcBK = 128;            // keys per tile
constexpr int kKStages = 3, kVStages = 2, kMStages = 4;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

enum : int { kErrTimeoutQ = 0x100, kErrTimeoutK = 0x200, kErrTimeoutS = 0x400, kErrTimeoutP = 0x800,
             kErrTimeoutPV = 0x1000, kErrTimeoutKEmpty = 0x2000, kErrTimeoutV = 0x4000,
             kErrTimeoutVEmpty = 0x8000, kErrTimeoutM = 0x10000, kErrTimeoutMEmpty = 0x20000,
             kErrSmemAlign = 0x40000 };

template <int D>
struct TcSmem {
  static constexpr int kHalves = D / 64;              // 64-element column halves of a row
  static constexpr int kTile = kHalves * 128 * 128;   // [halves][128 rows][128 B]
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;               // [kKStages]
  static constexpr int kV = kK + kKStages * kTile;    // [kVStages]
  static constexpr int kMeta = kV + kVStages * kTile; // [kMStages][dl (f32), jj|ee (i32)][128]
  static constexpr int kMerge = kMeta + kMStages * 2 * kTcBK * 4;   // [2 streams][m, l][128]
  static constexpr int kBars = kMerge + 2 * 2 * 128 * 4;
  static constexpr int kBytes = kBars + 512;
};

struct TcBars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t m_full[kMStages], m_empty[kMStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
  int abort_flag;
};

DMA_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}\n" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Four rows (r0..r3) x 64 columns starting at column `col` of a 2-D tensor map, written as four
// consecutive 128-byte rows at `dst` (the map's 128-byte swizzle applies); completion is counted
// in bytes on `bar`.
DMA_DEVINL void tma_gather4(uint32_t dst, const CUtensorMap* map, int col, int r0, int r1, int r2, int r3,
                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

DMA_DEVINL void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Warp-uniform bounded wait (every lane of the warp calls it).
DMA_DEVINL bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status, int code) {
  return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, abort_flag, status, code));
}

DMA_DEVINL void softmax_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

template <int R> DMA_DEVINL void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R)); }
template <int R> DMA_DEVINL void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R)); }

template <int D, typename OutT>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const int32_t* __restrict__ counts, const int32_t* __restrict__ lists,
                   const int32_t* __restrict__ list_je, const float* __restrict__ list_dl,
                   OutT* __restrict__ O, float* __restrict__ LSE,
                   int32_t* __restrict__ status, int H, int G, int N, int n_blocks, int list_cap,
                   float scale_log2) {
  using S = TcSmem<D>;
  extern __shared__ __align__(1024) unsigned char sm[];
  TcBars& bar = *reinterpret_cast<TcBars*>(sm + S::kBars);
  float* m_dl = reinterpret_cast<float*>(sm + S::kMeta);                        // [kMStages][128]
  int32_t* m_je = reinterpret_cast<int32_t*>(sm + S::kMeta) + kMStages * kTcBK;  // [kMStages][128]
  float* merge = reinterpret_cast<float*>(sm + S::kMerge);                       // [2][2][128]

  const int kb = n_blocks - 1 - (int)blockIdx.x;   // heavy (late) blocks first
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H, g = h / G, Hkv = H / G;
  const int t0 = kb * kBlockQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t* cnt = counts + ((size_t)bh * n_blocks + kb) * 2;
  const int n_full = cnt[0], n_live = cnt[1];
  const int n_tiles = (n_live + kTcBK - 1) / kTcBK;
  volatile int* abort_flag = &bar.abort_flag;

  if (tid == 0) {
    bar.abort_flag = 0;
    if (smem_u32(sm) & 1023u) {   // the swizzled operand layout needs a 1024-byte aligned base
      atomicOr(status, kErrSmemAlign);
      bar.abort_flag = 1;
    }
    tc::mbar_init(&bar.q_full, 32);
    for (int i = 0; i < kKStages; ++i) { tc::mbar_init(&bar.k_full[i], 32); tc::mbar_init(&bar.k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { tc::mbar_init(&bar.v_full[i], 32); tc::mbar_init(&bar.v_empty[i], 1); }
    for (int i = 0; i < kMStages; ++i) {
      tc::mbar_init(&bar.m_full[i], kProdThreads);
      tc::mbar_init(&bar.m_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar.s_full[i], 1);
      tc::mbar_init(&bar.p_full[i], 128);
      tc::mbar_init(&bar.pv_done[i], 1);
    }
    tc::fence_mbar_init();
  }
  if (warp == 8) {
    tc::tmem_alloc(&bar.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = bar.tmem_base;
  const bool run = n_tiles > 0 && !*abort_flag;
  if (warp >= 8) {
    regs_dec<kRegsOther>();   // warpgroups 2 and 3 give registers back
  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers (TMA gather4)
    const int pw = warp - kProdWarp0;            // producer warp 0..3
    const int prow = pw * 32 + lane;             // the tile row this thread owns
    const int kvrow0 = (b * Hkv + g) * N;
    const size_t lbase = ((size_t)bh * n_blocks + kb) * list_cap;
    const int32_t* list = lists + lbase;
    const int32_t* lje = list_je + lbase;
    const float* ldl = list_dl + lbase;
    constexpr uint32_t kRowBytes = D * 2;
    const bool issuer = lane < 8;                // lanes 0-7 gather rows pw*32 + 4*lane .. +3
    const uint32_t goff = (uint32_t)(pw * 32 + 4 * (lane & 7)) * 128;
    if (run && issuer) {   // Q rows (rows past N repeat row N-1; their outputs are dropped)
      int r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) r[u] = bh * N + min(t0 + pw * 32 + 4 * lane + u, N - 1);
      mbar_arrive_expect_tx(&bar.q_full, 4 * kRowBytes);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf)
        tma_gather4(smem_u32(sm + S::kQ) + hf * 16384 + goff, &qmap, hf * 64, r[0], r[1], r[2], r[3], &bar.q_full);
    }
    // Software pipeline over tiles: this row's list entry and its metadata (written beside the list
    // by the list kernel, so no load depends on another) are loaded two tiles ahead.
    struct Entry { int j, je; float dl; };
    auto entry_at = [&](int i) {
      const int li = i * kTcBK + prow;
      Entry x{-1, 0xffff, 0.f};
      if (i < n_tiles && li < n_live) { x.j = list[li]; x.je = lje[li]; x.dl = ldl[li]; }
      return x;
    };
    Entry ec = entry_at(0), en = entry_at(1);
    int jv = -1;
    for (int i = 0; run && i <= n_tiles; ++i) {
      const Entry enn = entry_at(i + 2);
      const int jc = ec.j;
      if (i < n_tiles) {
        const int ks = i % kKStages, ms = i % kMStages;
        if (i >= kMStages &&
            !wait_all(&bar.m_empty[ms], ((i / kMStages) - 1) & 1, abort_flag, status, kErrTimeoutMEmpty))
          break;
        m_dl[ms * kTcBK + prow] = ec.dl;
        m_je[ms * kTcBK + prow] = ec.je;
        tc::mbar_arrive(&bar.m_full[ms]);
        if (i >= kKStages &&
            !wait_all(&bar.k_empty[ks], ((i / kKStages) - 1) & 1, abort_flag, status, kErrTimeoutKEmpty))
          break;
        int r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = __shfl_sync(0xffffffffu, jc, 4 * (lane & 7) + u);
          r[u] = kvrow0 + (j >= 0 ? j : 0);
        }
        if (issuer) {
          mbar_arrive_expect_tx(&bar.k_full[ks], 4 * kRowBytes);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_gather4(smem_u32(sm + S::kK + ks * S::kTile) + hf * 16384 + goff, &kmap, hf * 64, r[0], r[1], r[2],
                        r[3], &bar.k_full[ks]);
        }
      }
      if (i >= 1) {
        // V of tile i-1 (its stage belongs to the tile's stream)
        const int vi = i - 1, vs = vi % kVStages;
        if (vi >= kVStages &&
            !wait_all(&bar.v_empty[vs], ((vi / kVStages) - 1) & 1, abort_flag, status, kErrTimeoutVEmpty))
          break;
        int r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = __shfl_sync(0xffffffffu, jv, 4 * (lane & 7) + u);
          r[u] = kvrow0 + (j >= 0 ? j : 0);
        }
        if (issuer) {
          mbar_arrive_expect_tx(&bar.v_full[vs], 4 * kRowBytes);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_gather4(smem_u32(sm + S::kV + vs * S::kTile) + hf * 16384 + goff, &vmap, hf * 64, r[0], r[1], r[2],
                        r[3], &bar.v_full[vs]);
        }
      }
      jv = jc;
      ec = en;
      en = enn;
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && run) {
      constexpr uint32_t idq = tc::idesc_bf16(128, kTcBK, false, false);
      constexpr uint32_t idv = tc::idesc_bf16(128, D, false, true);
      const uint32_t qs = smem_u32(sm + S::kQ);
      bool ok = tc::mbar_wait(&bar.q_full, 0, abort_flag, status, kErrTimeoutQ);
      for (int i = 0; ok && i <= n_tiles; ++i) {
        if (i < n_tiles) {   // S_x = Q K_i^T
          const int x = i & 1, ks = i % kKStages;
          if (!tc::mbar_wait(&bar.k_full[ks], (i / kKStages) & 1, abort_flag, status, kErrTimeoutK)) break;
          if (i >= 2 && !tc::mbar_wait(&bar.pv_done[x], ((i >> 1) - 1) & 1, abort_flag, status, kErrTimeoutPV))
            break;
          tc::fence_after();
          const uint32_t kbase = smem_u32(sm + S::kK + ks * S::kTile);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_ss(tmem + x * 128, tc::sdesc(qs + off, 16, 1024), tc::sdesc(kbase + off, 16, 1024), idq,
                            kk > 0 ? 1u : 0u);
          }
          tc::commit(&bar.s_full[x]);
          tc::commit(&bar.k_empty[ks]);
        }
        if (i >= 1) {        // O_x += P_x V_{i-1}
          const int pi = i - 1, x = pi & 1, vs = pi % kVStages;
          if (!tc::mbar_wait(&bar.p_full[x], (pi >> 1) & 1, abort_flag, status, kErrTimeoutP)) break;
          if (!tc::mbar_wait(&bar.v_full[vs], (pi / kVStages) & 1, abort_flag, status, kErrTimeoutV)) break;
          tc::fence_after();
          const uint32_t vbase = smem_u32(sm + S::kV + vs * S::kTile);
#pragma unroll
          for (int kk = 0; kk < kTcBK / 16; ++kk)
            mma_bf16_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, tc::sdesc(vbase + kk * 2048, 16384, 1024),
                        idv, (pi >= 2 || kk > 0) ? 1u : 0u);
          tc::commit(&bar.pv_done[x]);
          tc::commit(&bar.v_empty[vs]);
        }
      }
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax, stream x = warp / 4
    regs_inc<kRegsSoftmax>();
    const int x = warp >> 2;
    const int r = tid & 127;
    const int t = t0 + r;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + x * 128 + lane_base, tO = tmem + 256 + x * 128 + lane_base;
    float m_used = -INFINITY, l = 0.f;
    int my_tiles = 0;
    bool ok = run;
    for (int i = x; ok && i < n_tiles; i += 2) {
      const int k = i >> 1, ms = i % kMStages;
      if (!wait_all(&bar.s_full[x], k & 1, abort_flag, status, kErrTimeoutS)) { ok = false; break; }
      tc::fence_after();
      uint32_t sr[kTcBK / 32][32];
#pragma unroll
      for (int c = 0; c < kTcBK / 32; ++c) tc::tmem_ld32(tS + c * 32, sr[c]);
      if (!wait_all(&bar.m_full[ms], (i / kMStages) & 1, abort_flag, status, kErrTimeoutM)) {
        tc::tmem_wait_ld();
        ok = false;
        break;
      }
      tc::tmem_wait_ld();
      const float4* dl4 = reinterpret_cast<const float4*>(m_dl + ms * kTcBK);
      const bool full_tile = (i + 1) * kTcBK <= n_full;
      float mt = -INFINITY;
      if (full_tile) {
#pragma unroll
        for (int c4 = 0; c4 < kTcBK / 4; ++c4) {
          const float4 d4 = dl4[c4];
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c4 * 4 + u;
            const float v = fmaf(__uint_as_float(sr[c / 32][c % 32]), scale_log2, dd[u]);
            sr[c / 32][c % 32] = __float_as_uint(v);
            mt = fmaxf(mt, v);
          }
        }
      } else {
        const int4* je4 = reinterpret_cast<const int4*>(m_je + ms * kTcBK);
#pragma unroll
        for (int c4 = 0; c4 < kTcBK / 4; ++c4) {
          const float4 d4 = dl4[c4];
          const int4 w4 = je4[c4];
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
          const int ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c4 * 4 + u;
            const int jj = (int)(int16_t)(ww[u] & 0xffff), ee = ww[u] >> 16;
            float v = fmaf(__uint_as_float(sr[c / 32][c % 32]), scale_log2, dd[u]);
            v = (jj >= 0 && jj <= t && t < ee) ? v : -INFINITY;
            sr[c / 32][c % 32] = __float_as_uint(v);
            mt = fmaxf(mt, v);
          }
        }
      }
      tc::mbar_arrive(&bar.m_empty[ms]);
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_used + kRescaleThreshold || (m_used == -INFINITY && mt != -INFINITY)) {
        alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
        m_used = mt;
        rescale = true;
      }
      // O_x is stable here: S_x of this tile was computed after the stream's previous PV finished.
      // The whole warp rescales when any of its rows needs it (alpha = 1 for the others).
      if (my_tiles > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orow[32];
          tc::tmem_ld32(tO + c * 32, orow);
          tc::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) orow[u] = __float_as_uint(__uint_as_float(orow[u]) * alpha);
          tc::tmem_st32(tO + c * 32, orow);
        }
      }
      const float base = m_used == -INFINITY ? 0.f : m_used;
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < kTcBK / 64; ++c) {   // P (bf16 pairs) over columns [0, 64) of S_x
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int k0 = c * 64 + 2 * u;
          const float p0 = fast_exp2(__uint_as_float(sr[k0 / 32][k0 % 32]) - base);
          const float p1 = fast_exp2(__uint_as_float(sr[(k0 + 1) / 32][(k0 + 1) % 32]) - base);
          ps += p0 + p1;
          pk[u] = pack_bf16x2(p0, p1);
        }
        tc::tmem_st32(tS + c * 32, pk);
      }
      l = l * alpha + ps;
      tc::tmem_wait_st();
      tc::fence_before();
      tc::mbar_arrive(&bar.p_full[x]);
      ++my_tiles;
    }
    // ---- merge the two streams
    // wait for this stream's last PV
    bool done = ok;
    if (ok && my_tiles > 0) {
      const int last = x + 2 * (my_tiles - 1);
      done = wait_all(&bar.pv_done[x], (last >> 1) & 1, abort_flag, status, kErrTimeoutPV);
    }
    merge[(x * 2 + 0) * 128 + r] = m_used;
    merge[(x * 2 + 1) * 128 + r] = l;
    softmax_sync();
    const float m0 = merge[0 * 128 + r], l0 = merge[1 * 128 + r];
    const float m1 = merge[2 * 128 + r], l1 = merge[3 * 128 + r];
    const float M = fmaxf(m0, m1);
    const float Mb = M == -INFINITY ? 0.f : M;
    const float s0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - Mb), s1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - Mb);
    const float L = l0 * s0 + l1 * s1;
    const bool have1 = n_tiles > 1;   // stream B has at least one tile
    // stream B scales its O rows in place; stream A then writes (O_A s0 + O_B') / L
    if (x == 1 && have1 && __all_sync(0xffffffffu, done)) {
      tc::fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tc::tmem_ld32(tO + c * 32, ov);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * s1);
        tc::tmem_st32(tO + c * 32, ov);
      }
      tc::tmem_wait_st();
    }
    tc::fence_before();
    softmax_sync();
    tc::fence_after();
    if (x == 0 && run && __all_sync(0xffffffffu, done && !*abort_flag)) {
      const uint32_t tO1 = tmem + 384 + lane_base;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      OutT* orow = O + ((size_t)bh * N + t) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t oa[32], ob[32];
        tc::tmem_ld32(tO + c * 32, oa);
        if (have1) tc::tmem_ld32(tO1 + c * 32, ob);
        tc::tmem_wait_ld();
        float of[32];
#pragma unroll
        for (int u = 0; u < 32; ++u)
          of[u] = (__uint_as_float(oa[u]) * s0 + (have1 ? __uint_as_float(ob[u]) : 0.f)) * inv;
        if (t < N) {
          if constexpr (sizeof(OutT) == 2) {
#pragma unroll
            for (int u = 0; u < 32; u += 8) {
              uint4 v;
              v.x = pack_bf16x2(of[u], of[u + 1]);
              v.y = pack_bf16x2(of[u + 2], of[u + 3]);
              v.z = pack_bf16x2(of[u + 4], of[u + 5]);
              v.w = pack_bf16x2(of[u + 6], of[u + 7]);
              *reinterpret_cast<uint4*>(orow + c * 32 + u) = v;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 4)
              *reinterpret_cast<float4*>(orow + c * 32 + u) = make_float4(of[u], of[u + 1], of[u + 2], of[u + 3]);
          }
        }
      }
      if (t < N) LSE[(size_t)bh * N + t] = (Mb + __log2f(L)) * kLn2;
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 8) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side: tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view [rows, d] of a row-major bf16 tensor; boxes of 64 columns x 1 row (the gather4 form),
// 128-byte swizzle.
bool make_row_map(CUtensorMap* map, const void* base, uint64_t rows, int d) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, typename OutT>
cudaError_t launch_tc_t(const Plan& P, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                        const float* delta, const int32_t* evict, void* ws, void* O, float* LSE,
                        cudaStream_t s) {
  CUtensorMap qm, km, vm;
  if (!make_row_map(&qm, Q, (uint64_t)P.B * P.H * P.N, D) || !make_row_map(&km, K, (uint64_t)P.B * P.Hkv * P.N, D) ||
      !make_row_map(&vm, V, (uint64_t)P.B * P.Hkv * P.N, D))
    return cudaErrorInvalidValue;
  auto k = attn_fwd_tc_kernel<D, OutT>;
  const int smem = TcSmem<D>::kBytes;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  dim3 grid(P.n_blocks, P.B * P.H);
  // delta and e enter through the per-entry metadata that the list kernel wrote beside the lists
  (void)delta;
  (void)evict;
  k<<<grid, kTcThreads, smem, s>>>(qm, km, vm, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists),
                                   ws_ptr<int32_t>(ws, P.off_list_je), ws_ptr<float>(ws, P.off_list_dl),
                                   (OutT*)O, LSE,
                                   ws_ptr<int32_t>(ws, P.off_status), P.H, P.G, P.N, P.n_blocks, P.list_cap,
                                   P.scale * kLog2e);
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
