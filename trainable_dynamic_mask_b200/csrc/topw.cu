// Causal top-w selection kernels.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Dynamic Sparse Mask
// Generation", m_t equation (top_w of delta plus the causal constraint, f sending the rest to
// -inf).  Order: delta descending, ties to the lower key index; a query with t+1 <= w keeps all of
// its causal keys.
//
// Encoding.  delta depends on the key only, so the rank of key j among keys 0..t can only grow
// with t: key j is selected exactly for t in [j, e_j).  The prefill kernels compute e for every key
// and, per block of DMA_BLOCK_Q queries, the list of keys live in the block.
//
// Algorithm:
//  1. ranks of the row in the order (delta desc, index asc): the row's composite keys are cut into
//     segments, each segment sorted by its own CTA, and a key's rank is the number of smaller keys
//     over all sorted segments: p[r] = position of rank r, rank[j] = rank of position j (rank 0 =
//     best);
//  2. T_k = rank of the w-th best key among positions [0, kC) for every chunk boundary k
//     (C = 128), from a [rank bucket][position chunk] count table with prefix sums over chunks
//     (T_k = N when kC <= w: nothing evicted yet);
//  3. chunk k (positions [kC, kC+C)) resolves exactly the keys evicted inside it: old keys with rank
//     in (T_{k+1}, T_k] and new keys with rank above T_{k+1}.  For such a key of rank r,
//     e = max(j, first t >= kC at which #{i <= t : rank_i < r} reaches w), where the count of old
//     keys better than r follows from T_k and the sorted candidate list.  New keys that survive to
//     the end (rank <= T at the last boundary) get e = N.  Every key's e is written exactly once.
//  4. one CTA per (row, pair of query blocks) compacts the live keys of the two blocks and of the
//     pair: full keys (selected by every existing row of the range: j <= t0 and e_j >= t1) first,
//     then the partial ones (keys evicted inside the range and the range's own keys), each in
//     ascending order.
#include <limits.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kC = kBlockQ;         // chunk = query block = 128

DMA_DEVINL uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// n-th (0-based) set bit of x; x must have more than n set bits.
DMA_DEVINL int nth_set_bit(uint32_t x, int n) {
  for (int i = 0; i < n; ++i) x &= x - 1;
  return __ffs(x) - 1;
}

// ---------------------------------------------------------------- ranks + thresholds (per row)
//
// The order (delta descending, index ascending) is that of the 64-bit composite key
// (~order_key(delta_j)) << 32 | j taken ascending; the keys of a row are distinct.  A row is cut
// into nseg segments of L keys (padding keys 2^64 - 1 sort last); each segment is sorted by one CTA
// (bitonic network in shared memory), then the rank of a key is the number of smaller keys summed
// over the sorted segments (its own index in its segment plus a lower bound in every other one).
// Many CTAs per row keep the SMs busy even for a few (b, h) rows.

DMA_DEVINL uint64_t topw_key(float delta, int j) {
  return ((uint64_t)(~order_key(delta)) << 32) | (uint32_t)j;
}

// One CTA (L/2 threads) sorts segment blockIdx.x of row blockIdx.y ascending into skeys.
template <int L>
__global__ void __launch_bounds__(L / 2)
topw_segsort_kernel(const float* __restrict__ delta, uint64_t* __restrict__ skeys, int N, int npad) {
  __shared__ uint64_t sk[L];
  const int seg = blockIdx.x, row = blockIdx.y, tid = threadIdx.x;
  const float* drow = delta + (size_t)row * N;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = tid + u * (L / 2);
    const int j = seg * L + i;
    sk[i] = j < N ? topw_key(drow[j], j) : ~0ull;
  }
  __syncthreads();
  for (int k = 2; k <= L; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const int i = 2 * jj * (tid / jj) + (tid % jj);   // lower element of this thread's pair
      const bool up = (i & k) == 0;
      const uint64_t x = sk[i], y = sk[i + jj];
      if ((x > y) == up) {
        sk[i] = y;
        sk[i + jj] = x;
      }
      __syncthreads();
    }
  }
  uint64_t* out = skeys + (size_t)row * npad + (size_t)seg * L;
#pragma unroll
  for (int u = 0; u < 2; ++u) out[tid + u * (L / 2)] = sk[tid + u * (L / 2)];
}

// Ranks of segment blockIdx.x of row blockIdx.y: rank[j] (position -> rank) and p[r] (rank ->
// position).  The row's sorted segments are staged in shared memory; one key per thread (two for
// L = 2048).
template <int L>
constexpr int rank_threads() { return L < 1024 ? L : 1024; }

template <int L>
__global__ void __launch_bounds__(rank_threads<L>())
topw_rank_kernel(const uint64_t* __restrict__ skeys, int32_t* __restrict__ p_out, int32_t* __restrict__ rank_out,
                 int N, int nseg) {
  constexpr int kT = rank_threads<L>();
  extern __shared__ __align__(16) uint64_t rk[];   // [nseg * L]
  const int seg = blockIdx.x, row = blockIdx.y, tid = threadIdx.x;
  const int npad = nseg * L;
  const uint64_t* src = skeys + (size_t)row * npad;
  for (int i = tid * 2; i < npad; i += 2 * kT) *reinterpret_cast<uint4*>(rk + i) = *reinterpret_cast<const uint4*>(src + i);
  __syncthreads();
  int32_t* prow = p_out + (size_t)row * N;
  int32_t* rrow = rank_out + (size_t)row * N;
#pragma unroll
  for (int u = 0; u < L / kT; ++u) {
    const int i = tid + u * kT;
    const uint64_t key = rk[seg * L + i];
    const uint32_t j = (uint32_t)key;
    if (j >= (uint32_t)N) continue;   // padding
    int r = i;
    for (int s2 = 0; s2 < nseg; ++s2) {
      if (s2 == seg) continue;
      const uint64_t* a = rk + s2 * L;
      int lo = 0;                       // lower bound: first index with a[] >= key (keys are distinct)
#pragma unroll
      for (int step = L / 2; step > 0; step >>= 1)
        if (a[lo + step - 1] < key) lo += step;
      lo += a[lo] < key ? 1 : 0;
      r += lo;
    }
    rrow[j] = r;
    prow[r] = (int32_t)j;
  }
}

constexpr int kThThreads = 1024;
constexpr int kThWarps = kThThreads / 32;

// T_k = rank of the w-th best key among positions [0, kC) for every chunk boundary k (N when
// kC <= w: nothing evicted yet), from a [rank bucket][position chunk] count table with prefix sums
// over chunks.  One CTA per row.
__global__ void __launch_bounds__(kThThreads)
topw_thresh_kernel(const int32_t* __restrict__ p_in, const int32_t* __restrict__ rank_in, int32_t* __restrict__ T_out,
                   int N, int w_max, const int32_t* __restrict__ w_heads, int H) {
  extern __shared__ __align__(16) uint32_t table[];   // [nch][nch + 1]
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w = row_window(w_heads, row, H, w_max);
  const int nch = (N + kC - 1) / kC, cw = nch + 1;
  const int32_t* prow = p_in + (size_t)row * N;
  const int32_t* rrow = rank_in + (size_t)row * N;
  for (int i = tid; i < nch * cw; i += kThThreads) table[i] = 0;
  __syncthreads();
  for (int j = tid; j < N; j += kThThreads) atomicAdd(&table[(rrow[j] >> 7) * cw + (j >> 7)], 1u);
  __syncthreads();
  for (int rb = tid; rb < nch; rb += kThThreads) {
    uint32_t prev = 0;
    for (int k = 0; k <= nch; ++k) {
      const uint32_t t = table[rb * cw + k];
      table[rb * cw + k] = prev;
      prev += t;
    }
  }
  __syncthreads();
  // boundaries with kC <= w evict nothing (T = N); warps take the others, from the first
  for (int k = tid; k <= nch; k += kThThreads)
    if (min(k * kC, N) <= w) T_out[(size_t)row * cw + k] = N;
  const int kfirst = N > w ? w / kC + 1 : nch + 1;   // first k with kC > w
  for (int k = kfirst + warp; k <= nch; k += kThWarps) {
    const int Pk = min(k * kC, N);
    int before = 0, rbs = -1;
    for (int rb0 = 0; rb0 < nch && rbs < 0; rb0 += 32) {
      const int rb = rb0 + lane;
      const int v = rb < nch ? (int)table[rb * cw + k] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, before + incl >= w);
      if (hit) {
        const int l = __ffs(hit) - 1;
        rbs = rb0 + l;
        before += __shfl_sync(0xffffffffu, incl - v, l);
      } else {
        before += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    // the w-th key with position < Pk lies in rank bucket rbs: its 128 positions, loaded together
    const int rend = min(rbs * 128 + 128, N);
    int pos[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = rbs * 128 + 32 * u + lane;
      pos[u] = r < rend ? prow[r] : INT_MAX;
    }
    int need = w - before, Tk = N;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t m = __ballot_sync(0xffffffffu, pos[u] < Pk);
      const int c = __popc(m);
      if (need > 0 && c >= need) {
        Tk = rbs * 128 + 32 * u + nth_set_bit(m, need - 1);
        need = 0;
      } else if (need > 0) {
        need -= c;
      }
    }
    if (lane == 0) T_out[(size_t)row * cw + k] = Tk;
  }
}

// ---------------------------------------------------------------- eviction index (per chunk)

constexpr int kEvThreads = 128;
constexpr int kEvOwnTMaxN = kEvThreads * 32;   // rows up to this length: thresholds inside the kernel

// Index of the w-th (1-based) set bit of a bitmap of nw <= kEvThreads words, one word per thread;
// every thread of the CTA calls it and gets the result.  The bitmap must hold at least w set bits.
DMA_DEVINL int nth_bit_of_block(const uint32_t* bm, int nw, int w, int* warp_sums, int* result) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t x = tid < nw ? bm[tid] : 0u;
  const int c = __popc(x);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < warp; ++i) before += warp_sums[i];
  const int excl = before + incl - c;
  if (c > 0 && excl < w && w <= excl + c) *result = 32 * tid + nth_set_bit(x, w - excl - 1);
  __syncthreads();
  const int r = *result;
  __syncthreads();   // warp_sums and result are reused by the next call
  return r;
}

// One CTA per (chunk k, row).  Chunk k = positions [t0, t1) resolves exactly the keys evicted
// inside it: old keys (position < t0) with rank in (T_{k+1}, T_k], and its own keys with rank above
// T_{k+1}.  For such a key of rank r, e = max(j, first t >= t0 with #{i <= t : rank_i < r} >= w);
// the count over old positions follows from T_k: Sk - #{old candidates with rank >= r}, Sk being
// min(t0, w).  Its own keys that survive the last boundary get e = N.
// T_in == nullptr (rows of at most kEvOwnTMaxN keys): the CTA finds its boundaries' thresholds
// itself, as the w-th smallest rank among positions [0, t0) and [0, t1), from a bitmap over ranks
// (the ranks of a row are a permutation of 0 .. N-1; over the whole row the w-th smallest is w - 1).
__global__ void __launch_bounds__(kEvThreads)
topw_evict_kernel(const int32_t* __restrict__ p_in, const int32_t* __restrict__ rank_in,
                  const int32_t* __restrict__ T_in, int32_t* __restrict__ evict, int32_t* __restrict__ status,
                  int N, int w_max, const int32_t* __restrict__ w_heads, int H) {
  constexpr int kEvU = 4;            // ranks scanned per thread per round
  __shared__ __align__(16) int32_t crank[kC];   // ranks of the chunk's own keys (INT_MAX past the end)
  __shared__ int32_t L[kC];          // old candidates, ascending rank
  __shared__ int32_t Lpos[kC];       // their positions
  __shared__ int32_t wcount[kEvU][kEvThreads / 32];
  const int k = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w = row_window(w_heads, row, H, w_max);
  const int nch = (N + kC - 1) / kC;
  const int t0 = k * kC, t1 = min(t0 + kC, N);
  const int32_t* prow = p_in + (size_t)row * N;
  const int32_t* rrow = rank_in + (size_t)row * N;
  int32_t* erow = evict + (size_t)row * N;
  const int Sk = min(t0, w);
  crank[tid] = tid < t1 - t0 ? rrow[t0 + tid] : INT_MAX;
  int Ta, Tb, Tf;
  if (T_in != nullptr) {
    const int32_t* T = T_in + (size_t)row * (nch + 1);
    Ta = T[k];
    Tb = T[k + 1];
    Tf = T[nch];
  } else {
    __shared__ uint32_t bm[kEvOwnTMaxN / 32];
    __shared__ int warp_sums[kEvThreads / 32];
    __shared__ int result;
    const int nw = (N + 31) / 32;
    for (int i = tid; i < nw; i += kEvThreads) bm[i] = 0u;
    __syncthreads();
    for (int j = tid; j < t0; j += kEvThreads) {
      const int r = rrow[j];
      atomicOr(&bm[r >> 5], 1u << (r & 31));
    }
    __syncthreads();
    Ta = t0 <= w ? N : nth_bit_of_block(bm, nw, w, warp_sums, &result);
    if (tid < t1 - t0) atomicOr(&bm[crank[tid] >> 5], 1u << (crank[tid] & 31));
    __syncthreads();
    Tb = t1 <= w ? N : nth_bit_of_block(bm, nw, w, warp_sums, &result);
    Tf = N <= w ? N : w - 1;
  }
  // old candidates in rank order: the ranks in (Tb, Ta] held by positions < t0; all loads of a round
  // are issued before its ballots
  int nL = 0;
  const int rhi = min(Ta, N - 1);
  for (int r0 = Tb + 1; r0 <= rhi; r0 += kEvThreads * kEvU) {
    int pos[kEvU];
#pragma unroll
    for (int u = 0; u < kEvU; ++u) {
      const int r = r0 + u * kEvThreads + tid;
      pos[u] = r <= rhi ? prow[r] : INT_MAX;
    }
    uint32_t m[kEvU];
#pragma unroll
    for (int u = 0; u < kEvU; ++u) {
      m[u] = __ballot_sync(0xffffffffu, pos[u] < t0);
      if (lane == 0) wcount[u][warp] = __popc(m[u]);
    }
    __syncthreads();
    int before = nL;   // candidates at ranks before this thread's first one (rank order = u, warp, lane)
    int total = 0;
#pragma unroll
    for (int u = 0; u < kEvU; ++u) {
      int bu = 0, tu = 0;
      for (int i = 0; i < kEvThreads / 32; ++i) {
        if (i < warp) bu += wcount[u][i];
        tu += wcount[u][i];
      }
      if (pos[u] < t0) {
        const int slot = before + total + bu + __popc(m[u] & lanemask_lt());
        if (slot < kC) {
          L[slot] = r0 + u * kEvThreads + tid;
          Lpos[slot] = pos[u];
        }
      }
      total += tu;
    }
    nL += total;
    __syncthreads();
  }
  if (nL > kC) {   // cannot happen: at most C keys are evicted per chunk
    if (tid == 0) atomicOr(status, 2);
    nL = kC;
  }
  __syncthreads();
  // The chunk's keys in rank order, and pmask[q] = offsets (t - t0) of the chunk's q best keys:
  // the chunk keys better than rank r are pmask[#{chunk ranks < r}].  pmask is the exclusive
  // prefix OR, over the chunk ranks q, of the one-bit mask of the offset holding rank q.
  __shared__ int32_t srank[kC];
  __shared__ int32_t soff[kC];
  __shared__ uint32_t pmask[kC + 1][kEvThreads / 32];
  __shared__ uint32_t wor[kEvThreads / 32][kEvThreads / 32];
  static_assert(kEvThreads == kC, "one thread per chunk offset");
  const int nc = t1 - t0;
  if (tid < nc) {   // q = rank of offset tid among the chunk's keys
    const int my = crank[tid];
    int q = 0;
    const int4* c4 = reinterpret_cast<const int4*>(crank);
#pragma unroll 8
    for (int i = 0; i < kC / 4; ++i) {
      const int4 v = c4[i];
      q += (v.x < my) + (v.y < my) + (v.z < my) + (v.w < my);
    }
    srank[q] = my;
    soff[q] = tid;
  }
  __syncthreads();
  {
    // thread q: one-bit mask of the offset of chunk rank q, then an inclusive OR scan over q
    uint32_t v[kEvThreads / 32];
    const int o = tid < nc ? soff[tid] : -1;
#pragma unroll
    for (int wd = 0; wd < kEvThreads / 32; ++wd) v[wd] = (o >> 5) == wd ? 1u << (o & 31) : 0u;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
#pragma unroll
      for (int wd = 0; wd < kEvThreads / 32; ++wd) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v[wd], sh);
        if (lane >= sh) v[wd] |= y;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int wd = 0; wd < kEvThreads / 32; ++wd) wor[warp][wd] = v[wd];
    }
    __syncthreads();
#pragma unroll
    for (int wd = 0; wd < kEvThreads / 32; ++wd) {
      uint32_t acc = v[wd];
      for (int i = 0; i < warp; ++i) acc |= wor[i][wd];
      pmask[tid + 1][wd] = acc;
      if (tid == 0) pmask[0][wd] = 0u;
    }
  }
  __syncthreads();
  const int ncand = nL + (t1 - t0);
  for (int c = tid; c < ncand; c += kEvThreads) {
    int r, j, base, e = -1;
    bool scan = false;
    if (c < nL) {
      r = L[c];
      j = Lpos[c];
      base = Sk - (nL - c);
      scan = true;
    } else {
      j = t0 + (c - nL);
      r = crank[c - nL];
      base = 0;
      if (r <= Tb) {
        if (r <= Tf) e = N;            // never evicted
      } else if (Ta < N && r > Ta) {
        e = j;                         // never selected
      } else {
        int lo = 0, n = nL;            // old members with rank in (r, Ta]: L is ascending
        while (n > 0) {
          const int half = n >> 1;
          if (L[lo + half] <= r) { lo += half + 1; n -= half + 1; }
          else n = half;
        }
        base = Sk - (nL - lo);
        if (base >= w) e = j;
        else scan = true;
      }
    }
    if (scan) {
      // e = the chunk position at which the count of keys better than r, starting from base,
      // reaches w: the (w - base)-th chunk key better than r in position order
      int lo = 0, n = nc;
      while (n > 0) {
        const int half = n >> 1;
        if (srank[lo + half] < r) { lo += half + 1; n -= half + 1; }
        else n = half;
      }
      int left = w - base;
      e = -2;
#pragma unroll
      for (int wd = 0; wd < kEvThreads / 32; ++wd) {
        const uint32_t m = pmask[lo][wd];
        const int cnt = __popc(m);
        if (cnt >= left) {
          e = max(j, t0 + 32 * wd + nth_set_bit(m, left - 1));
          break;
        }
        left -= cnt;
      }
      if (e == -2) {                   // cannot happen: such keys are evicted inside the chunk
        e = t1;
        atomicOr(status, 4);
      }
    }
    if (e >= 0) erow[j] = e;
  }
}

// Live keys of a range of query rows [t0, t1): j < t1 and e_j > max(j, t0).  The "full" ones
// (j <= t0 and e_j >= t1: selected by every row of the range) come first, then the others, each
// group in ascending key order.  One CTA per (row, pair of blocks) builds three lists: those of its
// two blocks (the mask encoding of the interface) and that of the pair (the attention forward's work
// item), whose entries also carry e_j - j (the number of queries selecting the key) and
// delta_j * log2(e), and which is padded to a multiple of 128 entries with key -1 and e - j = 0
// (masked for every row).
//
// The keys before the pair's first row t0 that are still live at t0 are among the w best keys of
// [0, t0): the ranks 0 .. T_k of the row (T_k, the rank of the w-th best key of [0, t0), from the
// thresholds kernel; k = t0 / 128).  So the CTA scans whichever is shorter, those ranks (through the
// rank -> position map) or the positions [0, t0) -- about w N / t0 against t0 entries -- and then the
// pair's own positions [t0, t1).  Each list is kept as two bitmaps over positions (full, partial),
// compacted at the end in ascending order.
constexpr int kListThreads = 256;
constexpr int kListWords = kTopwMaxN / 32;   // bitmap words of a whole row
constexpr int kListStreamMaxN = 4096;        // rows up to this length take the streaming kernel below

__global__ void __launch_bounds__(kListThreads)
topw_lists_kernel(const int32_t* __restrict__ evict, const float* __restrict__ delta,
                  const int32_t* __restrict__ p_in, const int32_t* __restrict__ T_in,
                  int32_t* __restrict__ counts, int32_t* __restrict__ lists,
                  int32_t* __restrict__ pcounts, int32_t* __restrict__ plists,
                  int32_t* __restrict__ plen, float* __restrict__ pdl, int32_t* __restrict__ fcnt, int N,
                  int list_cap, int pair_cap, int n_blocks, int n_pairs, int kp0) {
  __shared__ uint32_t bm[6][kListWords];   // list L: bm[2L] full keys, bm[2L + 1] partial keys
  __shared__ uint32_t wsum3[3][kListThreads / 32];
  const int kp = kp0 + (int)blockIdx.x, row = blockIdx.y;   // pairs from kp0: the ones holding a query
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = kp * kPairQ;
  const bool has_b = t0 + kC < N;
  // list 0: block 2kp, list 1: block 2kp + 1, list 2: the pair
  const int lo[3] = {t0, t0 + kC, t0};
  const int hi[3] = {min(t0 + kC, N), min(t0 + kPairQ, N), min(t0 + kPairQ, N)};
  const int cap[3] = {list_cap, list_cap, pair_cap};
  const int t1 = hi[2];
  const int nw = (t1 + 31) / 32;
  const int32_t* erow = evict + (size_t)row * N;
  const float* drow = delta + (size_t)row * N;
  const int32_t* prow = p_in + (size_t)row * N;
  // the attention forward's merge counters of this pair start at zero for every new mask
  if (tid < 4) fcnt[((size_t)row * n_pairs + kp) * 4 + tid] = 0;
  // and its dynamic schedule's counters (after the merge counters of every pair)
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid < 2) fcnt[(size_t)gridDim.y * n_pairs * 4 + tid] = 0;
  // bit 2L (full) or 2L + 1 (partial) of key j < t1 evicted at e, for each list it is live in
  auto classify = [&](int j, int e) -> uint32_t {
    uint32_t m = 0;
#pragma unroll
    for (int L = 0; L < 3; ++L) {
      const bool live = (L != 1 || has_b) && j < hi[L] && e > max(j, lo[L]);
      const bool full = live && j <= lo[L] && e >= hi[L];
      if (live) m |= 1u << (2 * L + (full ? 0 : 1));
    }
    return m;
  };
  for (int i = tid; i < 6 * kListWords; i += kListThreads)
    if ((i % kListWords) < nw) bm[i / kListWords][i % kListWords] = 0;
  __syncthreads();
  const int Tk = T_in[(size_t)row * (n_blocks + 1) + 2 * kp];
  constexpr int kBatch = 8;   // keys per thread whose loads are issued together
  if (Tk < N && Tk + 1 < t0) {
    // the ranks 0 .. T_k: their positions before t0 (bits set one key at a time)
    for (int r0 = 0; r0 <= Tk; r0 += kListThreads * kBatch) {
      int jb[kBatch], eb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int r = r0 + u * kListThreads + tid;
        jb[u] = r <= Tk ? prow[r] : INT_MAX;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) eb[u] = jb[u] < t0 ? erow[jb[u]] : 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = jb[u];
        if (j < t0) {
          const uint32_t m = classify(j, eb[u]);
#pragma unroll
          for (int b = 0; b < 6; ++b)
            if ((m >> b) & 1u) atomicOr(&bm[b][j >> 5], 1u << (j & 31));
        }
      }
    }
  } else {
    // the positions [0, t0) (t0 is a multiple of 256: every warp's 32 positions are a whole word)
    for (int base0 = 0; base0 < t0; base0 += kListThreads * kBatch) {
      int eb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = base0 + u * kListThreads + warp * 32 + lane;
        eb[u] = j < t0 ? erow[j] : 0;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int base = base0 + u * kListThreads + warp * 32;
        if (base >= t0) break;   // warp-uniform
        const uint32_t m = classify(base + lane, eb[u]);
#pragma unroll
        for (int b = 0; b < 6; ++b) {
          const uint32_t word = __ballot_sync(0xffffffffu, (m >> b) & 1u);
          if (lane == 0) bm[b][base >> 5] = word;
        }
      }
    }
  }
  {
    // the pair's own positions [t0, t1): one per thread, whole words per warp
    const int j = t0 + tid;
    const uint32_t m = j < t1 ? classify(j, erow[j]) : 0u;
#pragma unroll
    for (int b = 0; b < 6; ++b) {
      const uint32_t word = __ballot_sync(0xffffffffu, (m >> b) & 1u);
      if (lane == 0 && t0 + warp * 32 < t1) bm[b][(t0 >> 5) + warp] = word;
    }
  }
  __syncthreads();
  // compaction: the bitmaps' bytes are dealt in equal runs of upt consecutive bytes per thread (so
  // that every thread has about the same number of keys to write, however short the range).  One
  // block scan of the six counts (packed two per 32-bit word, 16 bits each: a list holds < 2^16 keys)
  // gives every key its index: full keys of a list first, then its partial keys.
  const int nbytes = 4 * nw;
  const int upt = (nbytes + kListThreads - 1) / kListThreads;   // <= 8
  const int u0 = tid * upt;
  auto byte_of = [&](int b, int u) -> uint32_t {
    return u < nbytes ? (bm[b][u >> 2] >> (8 * (u & 3))) & 0xffu : 0u;
  };
  uint32_t pk[3] = {0u, 0u, 0u};
#pragma unroll
  for (int b = 0; b < 6; ++b) {
    int c = 0;
    for (int u = 0; u < upt; ++u) c += __popc(byte_of(b, u0 + u));
    pk[b >> 1] += (uint32_t)c << (16 * (b & 1));
  }
  uint32_t inc[3] = {pk[0], pk[1], pk[2]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc[q], o);
      if (lane >= o) inc[q] += y;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int q = 0; q < 3; ++q) wsum3[q][warp] = inc[q];
  }
  __syncthreads();
  int start[6], total[6];
#pragma unroll
  for (int b = 0; b < 6; ++b) {
    const int q = b >> 1, sh = 16 * (b & 1);
    int before = 0, tot = 0;
#pragma unroll
    for (int v = 0; v < kListThreads / 32; ++v) {
      const int x = (int)((wsum3[q][v] >> sh) & 0xffffu);
      before += v < warp ? x : 0;
      tot += x;
    }
    start[b] = before + (int)(((inc[q] - pk[q]) >> sh) & 0xffffu);
    total[b] = tot;
  }
  int n_out[3][2];
#pragma unroll
  for (int L = 0; L < 3; ++L) {
    n_out[L][0] = min(total[2 * L], cap[L]);
    n_out[L][1] = min(total[2 * L + 1], cap[L] - n_out[L][0]);
  }
#pragma unroll
  for (int L = 0; L < 3; ++L) {
    if (L == 1 && !has_b) continue;
    int32_t* dst = L == 0 ? lists + ((size_t)row * n_blocks + 2 * kp) * list_cap
                 : L == 1 ? lists + ((size_t)row * n_blocks + 2 * kp + 1) * list_cap
                          : plists + ((size_t)row * n_pairs + kp) * pair_cap;
#pragma unroll
    for (int kind = 0; kind < 2; ++kind) {
      const int b = 2 * L + kind;
      int o = start[b] + (kind == 1 ? n_out[L][0] : 0);
      const int lim = kind == 0 ? n_out[L][0] : n_out[L][0] + n_out[L][1];
      for (int u = 0; u < upt; ++u) {
        uint32_t x = byte_of(b, u0 + u);
        while (x) {
          const int jj = 8 * (u0 + u) + __ffs(x) - 1;
          x &= x - 1;
          if (o < lim) dst[o] = jj;
          ++o;
        }
      }
    }
  }
  __syncthreads();   // the pair list is complete for the pass below
  {
    // the pair list's e_j - j and delta_j log2(e), entry by entry (global writes of this CTA made
    // before the barrier above are visible to it)
    const size_t pb = ((size_t)row * n_pairs + kp) * pair_cap;
    const int n2 = n_out[2][0] + n_out[2][1];
    for (int i0 = 0; i0 < n2; i0 += kListThreads * kBatch) {
      int jb[kBatch], eb[kBatch];
      float db[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kListThreads + tid;
        jb[u] = i < n2 ? plists[pb + i] : -1;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        eb[u] = jb[u] >= 0 ? erow[jb[u]] : 0;
        db[u] = jb[u] >= 0 ? drow[jb[u]] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kListThreads + tid;
        if (i < n2) {
          plen[pb + i] = eb[u] - jb[u];
          pdl[pb + i] = db[u] * kLog2e;
        }
      }
    }
  }
  const int nlive = n_out[2][0] + n_out[2][1];
  const int nround = min(pair_cap, (nlive + kC - 1) / kC * kC);
  {
    const size_t pb = ((size_t)row * n_pairs + kp) * pair_cap;
    for (int i = nlive + tid; i < nround; i += kListThreads) {
      plists[pb + i] = -1;
      plen[pb + i] = 0;
      pdl[pb + i] = 0.f;
    }
  }
  if (tid == 0) {
    int32_t* ca = counts + ((size_t)row * n_blocks + 2 * kp) * 2;
    ca[0] = n_out[0][0];
    ca[1] = n_out[0][0] + n_out[0][1];
    if (has_b) {
      ca[2] = n_out[1][0];
      ca[3] = n_out[1][0] + n_out[1][1];
    }
    int32_t* cp = pcounts + ((size_t)row * n_pairs + kp) * 2;
    cp[0] = n_out[2][0];
    cp[1] = nlive;
  }
}

// The same lists by one streaming pass over all keys j < t1 in ascending order (four keys per
// thread per round, e_j and delta_j loaded a round ahead, packed per-warp counters): no bitmaps and
// no rank map, cheaper than the kernel above while t1 is short (rows of up to 4096 keys), dearer on
// long rows, where the ranks up to T_k are far fewer than the positions before t0.
constexpr int kListWarps = kListThreads / 32;
constexpr int kListBits = 10;                    // packed per-warp counters (a warp counts <= 128)
constexpr int kListMask = (1 << kListBits) - 1;

__global__ void __launch_bounds__(kListThreads)
topw_lists_stream_kernel(const int32_t* __restrict__ evict, const float* __restrict__ delta,
                  int32_t* __restrict__ counts, int32_t* __restrict__ lists,
                  int32_t* __restrict__ pcounts, int32_t* __restrict__ plists,
                  int32_t* __restrict__ plen, float* __restrict__ pdl, int32_t* __restrict__ fcnt, int N,
                  int list_cap, int pair_cap, int n_blocks, int n_pairs, int kp0) {
  // partial keys: block a (<= 2C), block b (<= 2C), pair (<= 4C)
  __shared__ int32_t part[8 * kC];
  __shared__ int32_t wsum[6][kListWarps];   // per warp: full count of list 0..2, partial count of 0..2
  const int kp = kp0 + (int)blockIdx.x, row = blockIdx.y;   // pairs from kp0: the ones holding a query
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = kp * kPairQ;
  const bool has_b = t0 + kC < N;
  // list 0: block 2kp, list 1: block 2kp + 1, list 2: the pair
  const int lo[3] = {t0, t0 + kC, t0};
  const int hi[3] = {min(t0 + kC, N), min(t0 + kPairQ, N), min(t0 + kPairQ, N)};
  const int pcap[3] = {2 * kC, 2 * kC, 4 * kC};
  const int poff[3] = {0, 2 * kC, 4 * kC};
  const int cap[3] = {list_cap, list_cap, pair_cap};
  const int t1 = hi[2];
  const int32_t* erow = evict + (size_t)row * N;
  const float* drow = delta + (size_t)row * N;
  int32_t* out[3];
  out[0] = lists + ((size_t)row * n_blocks + 2 * kp) * list_cap;
  out[1] = has_b ? out[0] + list_cap : out[0];
  const size_t pbase = ((size_t)row * n_pairs + kp) * pair_cap;
  out[2] = plists + pbase;
  int32_t* olen = plen + pbase;
  float* odl = pdl + pbase;
  int nfull[3] = {0, 0, 0}, npart[3] = {0, 0, 0};
  // the attention forward's merge counters of this pair start at zero for every new mask
  if (tid < 4) fcnt[((size_t)row * n_pairs + kp) * 4 + tid] = 0;
  // and its dynamic schedule's counters (after the merge counters of every pair)
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid < 2) fcnt[(size_t)gridDim.y * n_pairs * 4 + tid] = 0;
  // e_j and delta_j of this thread's 4 keys, loaded one round ahead
  int enext[4];
  float dnext[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = tid * 4 + u;
    enext[u] = j < t1 ? erow[j] : 0;
    dnext[u] = j < t1 ? drow[j] : 0.f;
  }
  for (int base = 0; base < t1; base += kListThreads * 4) {
    int ecur[4];
    float dcur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ecur[u] = enext[u];
      dcur[u] = dnext[u];
      const int jn = base + kListThreads * 4 + tid * 4 + u;
      enext[u] = jn < t1 ? erow[jn] : 0;
      dnext[u] = jn < t1 ? drow[jn] : 0.f;
    }
    int cf = 0, cq = 0;              // packed counts of this thread's full / partial keys
    uint32_t fbits = 0, qbits = 0;   // bit 3u + L: key u is full / partial in list L
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + tid * 4 + u;
      const int e = ecur[u];
#pragma unroll
      for (int L = 0; L < 3; ++L) {
        const bool valid = L != 1 || has_b;
        bool full, part;
        if (j <= t0) {   // j <= every range's first row: live iff e > lo, full iff e >= hi
          full = valid && e >= hi[L];
          part = valid && e > lo[L] && e < hi[L];
        } else {
          const bool live = valid && j < hi[L] && e > max(j, lo[L]);
          full = live && j <= lo[L] && e >= hi[L];
          part = live && !full;
        }
        fbits |= (uint32_t)full << (3 * u + L);
        qbits |= (uint32_t)part << (3 * u + L);
        cf += (int)full << (kListBits * L);
        cq += (int)part << (kListBits * L);
      }
    }
    int incf = cf, incq = cq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yf = __shfl_up_sync(0xffffffffu, incf, o);
      const int yq = __shfl_up_sync(0xffffffffu, incq, o);
      if (lane >= o) { incf += yf; incq += yq; }
    }
    if (lane == 31) {
#pragma unroll
      for (int L = 0; L < 3; ++L) {
        wsum[L][warp] = (incf >> (kListBits * L)) & kListMask;
        wsum[3 + L][warp] = (incq >> (kListBits * L)) & kListMask;
      }
    }
    __syncthreads();
    int of[3], oq[3], tf[3], tq[3];
#pragma unroll
    for (int L = 0; L < 3; ++L) {
      int bf = 0, bq = 0, sf = 0, sq = 0;
      for (int i = 0; i < kListWarps; ++i) {
        const int vf = wsum[L][i], vq = wsum[3 + L][i];
        if (i < warp) { bf += vf; bq += vq; }
        sf += vf;
        sq += vq;
      }
      of[L] = nfull[L] + bf + (((incf - cf) >> (kListBits * L)) & kListMask);
      oq[L] = npart[L] + bq + (((incq - cq) >> (kListBits * L)) & kListMask);
      tf[L] = sf;
      tq[L] = sq;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + tid * 4 + u;
#pragma unroll
      for (int L = 0; L < 3; ++L) {
        if ((fbits >> (3 * u + L)) & 1u) {
          if (of[L] < cap[L]) {
            out[L][of[L]] = j;
            if (L == 2) {
              olen[of[L]] = ecur[u] - j;
              odl[of[L]] = dcur[u] * kLog2e;
            }
          }
          ++of[L];
        }
        if ((qbits >> (3 * u + L)) & 1u) {
          if (oq[L] < pcap[L]) part[poff[L] + oq[L]] = j;
          ++oq[L];
        }
      }
    }
#pragma unroll
    for (int L = 0; L < 3; ++L) {
      nfull[L] += tf[L];
      npart[L] += tq[L];
    }
    __syncthreads();   // wsum is rewritten next round
  }
  // Caps: a block list holds at most w live keys at its first row plus C new ones (<= list_cap);
  // its partial keys are at most C evicted plus C new ones.  A pair: w + 2C and 2C + 2C.
#pragma unroll
  for (int L = 0; L < 3; ++L) {
    nfull[L] = min(nfull[L], cap[L]);
    npart[L] = min(min(npart[L], pcap[L]), cap[L] - nfull[L]);
  }
#pragma unroll
  for (int L = 0; L < 3; ++L) {
    if (L == 1 && !has_b) continue;
    for (int i = tid; i < npart[L]; i += kListThreads) {
      const int j = part[poff[L] + i];
      out[L][nfull[L] + i] = j;
      if (L == 2) {
        olen[nfull[L] + i] = erow[j] - j;
        odl[nfull[L] + i] = drow[j] * kLog2e;
      }
    }
  }
  const int nlive = nfull[2] + npart[2];
  const int nround = min(pair_cap, (nlive + kC - 1) / kC * kC);
  for (int i = nlive + tid; i < nround; i += kListThreads) {
    out[2][i] = -1;
    olen[i] = 0;
    odl[i] = 0.f;
  }
  if (tid == 0) {
    int32_t* ca = counts + ((size_t)row * n_blocks + 2 * kp) * 2;
    ca[0] = nfull[0];
    ca[1] = nfull[0] + npart[0];
    if (has_b) {
      ca[2] = nfull[1];
      ca[3] = nfull[1] + npart[1];
    }
    int32_t* cp = pcounts + ((size_t)row * n_pairs + kp) * 2;
    cp[0] = nfull[2];
    cp[1] = nlive;
  }
}

// ---------------------------------------------------------------- decode selection

constexpr int kSelThreads = 512;                // two CTAs per SM: a row per CTA, all rows in one wave
constexpr int kSelBatch = 8;                   // rounds of loads issued together
constexpr int kSelBits = 12;                   // histogram window
constexpr int kSelBins = 1 << kSelBits;
constexpr int kSelCand = 6144;                 // candidates kept in shared memory
constexpr int kSelWarps = kSelThreads / 32;

struct SelShared {
  uint32_t hist[kSelBins];
  uint32_t cand_key[kSelCand];
  uint32_t red[2][kSelWarps];
  int32_t scan[2][kSelBatch * kSelWarps];   // exclusive prefix of (greater, equal) counts per (round, warp)
  uint32_t bin, above, ncand;
};

// The bin (from the highest) in which the count accumulated from the highest bin reaches `need`,
// and the count of the bins above it, into S.bin / S.above.  hist must be complete.
DMA_DEVINL void sel_find_bin(SelShared& S, uint32_t need, int nbins, int tid) {
  if (tid < 32) {
    const int lane = tid;
    const int per = (nbins + 31) / 32;   // bins per lane, lane 0 takes the highest
    uint32_t sum = 0;
    for (int u = 0; u < per; ++u) {
      const int q = lane * per + u;
      if (q < nbins) sum += S.hist[nbins - 1 - q];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need);
    const int l = __ffs(hit) - 1;
    if (lane == l) {
      uint32_t above = incl - sum;
      for (int u = 0; u < per; ++u) {
        const int q = lane * per + u;
        if (q >= nbins) break;
        const uint32_t bin = (uint32_t)(nbins - 1 - q);
        if (above + S.hist[bin] >= need) {
          S.bin = bin;
          S.above = above;
          break;
        }
        above += S.hist[bin];
      }
    }
  }
  __syncthreads();
}

// Top-w of the whole row (the query at position N-1), in the order (delta desc, index asc).
// Selection by histograms over a 12-bit window of the order key, starting at the highest bit in
// which the row's keys differ (delta values crowd into a few exponents, so a fixed top-byte pass
// would separate almost nothing).  Passes over the row narrow the window until the bin holding the
// w-th best key has at most kSelCand keys; those are then resolved in shared memory.  A last pass
// writes the selected positions in ascending order.
__global__ void __launch_bounds__(kSelThreads, 2)
topw_decode_kernel(const float* __restrict__ delta, int32_t* __restrict__ sel, float* __restrict__ seld, int N,
                   int w_max, const int32_t* __restrict__ w_heads, int H, int sel_stride) {
  extern __shared__ __align__(16) unsigned char sel_raw[];
  SelShared& S = *reinterpret_cast<SelShared*>(sel_raw);
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* drow = delta + (size_t)row * N;
  const int k = min(row_window(w_heads, row, H, w_max), N);
  int32_t* out = sel + (size_t)row * sel_stride;
  float* outd = seld != nullptr ? seld + (size_t)row * sel_stride : nullptr;   // delta of each selected key
  if (k == N) {
    for (int i = tid; i < N; i += kSelThreads) {
      out[i] = i;
      if (outd) outd[i] = drow[i];
    }
    return;
  }
  // ---- key range of the row
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int i0 = 0; i0 < N; i0 += kSelThreads * kSelBatch) {
    uint32_t kb[kSelBatch];
#pragma unroll
    for (int u = 0; u < kSelBatch; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      kb[u] = i < N ? order_key(drow[i]) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kSelBatch; ++u) {
      if (i0 + u * kSelThreads + tid < N) {
        kmin = min(kmin, kb[u]);
        kmax = max(kmax, kb[u]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) { S.red[0][warp] = kmin; S.red[1][warp] = kmax; }
  __syncthreads();
  kmin = 0xffffffffu;
  kmax = 0u;
  for (int i = 0; i < kSelWarps; ++i) { kmin = min(kmin, S.red[0][i]); kmax = max(kmax, S.red[1][i]); }
  __syncthreads();
  // ---- narrowing.  Keys in play: (key >> (shift + width)) == pre, where [shift, shift + width) is
  // the current window; when every key is equal the threshold is that key.
  uint32_t need = (uint32_t)k;
  uint32_t thr = kmin;
  if (kmin != kmax) {
    const int top = 31 - __clz(kmin ^ kmax);   // highest bit in which the keys differ
    int width = top + 1 < kSelBits ? top + 1 : kSelBits;
    int shift = top + 1 - width;
    uint32_t pre = top == 31 ? 0u : kmin >> (top + 1);
    bool in_smem = false;   // candidates collected in shared memory
    int ncand = 0;
    while (true) {
      // histogram of the window over the keys in play
      for (int i = tid; i < kSelBins; i += kSelThreads) S.hist[i] = 0;
      __syncthreads();
      const uint32_t wmask = (1u << width) - 1u;
      const int hs = shift + width;   // bits above the window
      if (!in_smem) {
        for (int i0 = 0; i0 < N; i0 += kSelThreads * kSelBatch) {
          uint32_t kb[kSelBatch];
#pragma unroll
          for (int u = 0; u < kSelBatch; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            kb[u] = i < N ? order_key(drow[i]) : 0u;
          }
#pragma unroll
          for (int u = 0; u < kSelBatch; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            const uint32_t hi = hs >= 32 ? 0u : kb[u] >> hs;
            if (i < N && hi == pre) atomicAdd(&S.hist[(kb[u] >> shift) & wmask], 1u);
          }
        }
      } else {
        for (int c = tid; c < ncand; c += kSelThreads) {
          const uint32_t key = S.cand_key[c];
          const uint32_t hi = hs >= 32 ? 0u : key >> hs;
          if (hi == pre) atomicAdd(&S.hist[(key >> shift) & wmask], 1u);
        }
      }
      __syncthreads();
      sel_find_bin(S, need, 1 << width, tid);
      const uint32_t bin = S.bin, cnt = S.hist[S.bin];
      need -= S.above;
      pre = (hs >= 32 ? 0u : pre << width) | bin;
      __syncthreads();
      if (shift == 0) {   // the bin is a single key value
        thr = pre;
        break;
      }
      if (!in_smem && cnt <= (uint32_t)kSelCand) {
        // collect the bin's keys (their order does not matter: only the threshold is sought)
        if (tid == 0) S.ncand = 0;
        __syncthreads();
        for (int i0 = 0; i0 < N; i0 += kSelThreads * kSelBatch) {
          uint32_t kb[kSelBatch];
#pragma unroll
          for (int u = 0; u < kSelBatch; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            kb[u] = i < N ? order_key(drow[i]) : 0u;
          }
#pragma unroll
          for (int u = 0; u < kSelBatch; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            if (i < N && (kb[u] >> shift) == pre) {
              const uint32_t slot = atomicAdd(&S.ncand, 1u);
              if (slot < (uint32_t)kSelCand) S.cand_key[slot] = kb[u];
            }
          }
        }
        __syncthreads();
        ncand = (int)min(S.ncand, (uint32_t)kSelCand);
        in_smem = true;
      }
      width = shift < kSelBits ? shift : kSelBits;
      shift -= width;
      __syncthreads();
    }
  }
  // ---- thr = key of the k-th best: take keys above it and the first `need` equal ones, in index
  // order.  out position of a taken key = #greater before it + min(#equal before it, need).
  int gt_run = 0, eq_run = 0;
  for (int i0 = 0; i0 < N; i0 += kSelThreads * kSelBatch) {
    uint32_t kb[kSelBatch];
    float dv[kSelBatch];
#pragma unroll
    for (int u = 0; u < kSelBatch; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      dv[u] = i < N ? drow[i] : 0.f;
      kb[u] = order_key(dv[u]);
    }
    uint32_t mg[kSelBatch], me[kSelBatch];
#pragma unroll
    for (int u = 0; u < kSelBatch; ++u) {
      const bool in = i0 + u * kSelThreads + tid < N;
      mg[u] = __ballot_sync(0xffffffffu, in && kb[u] > thr);
      me[u] = __ballot_sync(0xffffffffu, in && kb[u] == thr);
      if (lane == 0) {
        S.scan[0][u * kSelWarps + warp] = __popc(mg[u]);
        S.scan[1][u * kSelWarps + warp] = __popc(me[u]);
      }
    }
    __syncthreads();
    if (warp < 2) {   // exclusive scans in (round, warp) order: warp 0 the greater, warp 1 the equal
      constexpr int kPer = kSelBatch * kSelWarps / 32;
      int v[kPer], sum = 0;
#pragma unroll
      for (int u = 0; u < kPer; ++u) { v[u] = S.scan[warp][lane * kPer + u]; sum += v[u]; }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
#pragma unroll
      for (int u = 0; u < kPer; ++u) { S.scan[warp][lane * kPer + u] = run; run += v[u]; }
      if (lane == 31) S.red[warp][0] = (uint32_t)run;   // batch totals
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kSelBatch; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      const uint32_t lt = (1u << lane) - 1u;
      const int gb = gt_run + S.scan[0][u * kSelWarps + warp] + __popc(mg[u] & lt);
      const int eb = eq_run + S.scan[1][u * kSelWarps + warp] + __popc(me[u] & lt);
      const bool g = (mg[u] >> lane) & 1u, e = (me[u] >> lane) & 1u;
      if (g || (e && eb < (int)need)) {
        const int o = gb + min(eb, (int)need);
        if (o < k) {
          out[o] = i;
          if (outd) outd[o] = dv[u];
        }
      }
    }
    gt_run += (int)S.red[0][0];
    eq_run += (int)S.red[1][0];
    __syncthreads();
  }
}

}  // namespace

template <int L>
cudaError_t launch_topw_rank(const Plan& P, const float* delta, uint64_t* skeys, int32_t* pbuf, int32_t* rbuf,
                             cudaStream_t s) {
  const int rows = P.B * P.H;
  const int nseg = (P.N + L - 1) / L;
  topw_segsort_kernel<L><<<dim3(nseg, rows), L / 2, 0, s>>>(delta, skeys, P.N, nseg * L);
  const int smem = nseg * L * (int)sizeof(uint64_t);
  { cudaError_t ea = ensure_smem_limit(topw_rank_kernel<L>, smem); if (ea != cudaSuccess) return ea; }
  topw_rank_kernel<L><<<dim3(nseg, rows), rank_threads<L>(), smem, s>>>(skeys, pbuf, rbuf, P.N, nseg);
  return cudaGetLastError();
}

cudaError_t launch_topw_prefill(const Plan& P, const float* delta, int32_t* evict, void* ws,
                                cudaStream_t s) {
  const int rows = P.B * P.H;
  const int nch = P.n_blocks;
  int32_t* pbuf = ws_ptr<int32_t>(ws, P.off_tw_p);
  int32_t* rbuf = ws_ptr<int32_t>(ws, P.off_tw_rank);
  int32_t* Tbuf = ws_ptr<int32_t>(ws, P.off_tw_T);
  uint64_t* skeys = ws_ptr<uint64_t>(ws, P.off_tw_keys);
  cudaError_t e;
  switch (topw_seg_len(P.N)) {
    case 512: e = launch_topw_rank<512>(P, delta, skeys, pbuf, rbuf, s); break;
    case 1024: e = launch_topw_rank<1024>(P, delta, skeys, pbuf, rbuf, s); break;
    default: e = launch_topw_rank<2048>(P, delta, skeys, pbuf, rbuf, s); break;
  }
  if (e != cudaSuccess) return e;
  // rows the streaming list kernel takes need the thresholds only here, inside the eviction kernel
  const bool own_T = P.N <= kListStreamMaxN;
  static_assert(kListStreamMaxN <= kEvOwnTMaxN, "the eviction kernel's rank bitmap covers those rows");
  if (!own_T) {
    const int tsmem = nch * (nch + 1) * (int)sizeof(uint32_t);
    { cudaError_t ea = ensure_smem_limit(topw_thresh_kernel, tsmem); if (ea != cudaSuccess) return ea; }
    topw_thresh_kernel<<<rows, kThThreads, tsmem, s>>>(pbuf, rbuf, Tbuf, P.N, P.w, P.w_heads, P.H);
  }
  topw_evict_kernel<<<dim3(nch, rows), kEvThreads, 0, s>>>(pbuf, rbuf, own_T ? nullptr : Tbuf, evict,
                                                            ws_ptr<int32_t>(ws, P.off_status), P.N, P.w,
                                                            P.w_heads, P.H);
  const int kp0 = P.q0 / kPairQ;
  if (P.N > kListStreamMaxN)
    topw_lists_kernel<<<dim3(P.n_pairs - kp0, rows), kListThreads, 0, s>>>(
        evict, delta, pbuf, Tbuf, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists),
        ws_ptr<int32_t>(ws, P.off_pcounts), ws_ptr<int32_t>(ws, P.off_plists), ws_ptr<int32_t>(ws, P.off_plen),
        ws_ptr<float>(ws, P.off_pdl), ws_ptr<int32_t>(ws, P.off_fcnt), P.N, P.list_cap, P.pair_cap, P.n_blocks,
        P.n_pairs, kp0);
  else
    topw_lists_stream_kernel<<<dim3(P.n_pairs - kp0, rows), kListThreads, 0, s>>>(
        evict, delta, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists),
        ws_ptr<int32_t>(ws, P.off_pcounts), ws_ptr<int32_t>(ws, P.off_plists), ws_ptr<int32_t>(ws, P.off_plen),
        ws_ptr<float>(ws, P.off_pdl), ws_ptr<int32_t>(ws, P.off_fcnt), P.N, P.list_cap, P.pair_cap, P.n_blocks,
        P.n_pairs, kp0);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- decode: one key appended
constexpr int kAppThreads = 256;

// One CTA per (b, h) row: the selection over [0, L) from the one over [0, L-1) (rows of sel_stride
// entries; the row's window w holds its w keys when L - 1 > w, every key 0 .. L-2 when L - 1 <= w,
// then not read).  The worst selected key is the smallest
// (order key, ~index) composite: the smallest delta, the larger index among equal ones.  The new
// key L - 1 enters iff its order key is strictly larger; it then has the largest index, so the
// ascending list loses the worst key's entry and gains L - 1 at its end.
__global__ void __launch_bounds__(kAppThreads)
topw_append_kernel(const float* __restrict__ delta, int32_t* __restrict__ sel, float* __restrict__ seld, int L,
                   int w_max, const int32_t* __restrict__ w_heads, int H, int sel_stride) {
  __shared__ uint64_t wmin[kAppThreads / 32];
  __shared__ int pos;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* drow = delta + (size_t)row * L;
  const int w = row_window(w_heads, row, H, w_max);
  const int kp = min(L - 1, w);
  int32_t* out = sel + (size_t)row * sel_stride;
  float* outd = seld + (size_t)row * sel_stride;   // delta of each selected key, kept beside it
  if (kp < w) {   // every key is selected
    for (int i = tid; i < L; i += kAppThreads) {
      out[i] = i;
      outd[i] = drow[i];
    }
    return;
  }
  const bool implicit = L - 1 == w;   // the previous selection is every key 0 .. L-2
  uint64_t c = ~0ull;
  for (int i = tid; i < w; i += kAppThreads) {
    const int j = implicit ? i : out[i];
    c = min(c, ((uint64_t)order_key(drow[j]) << 32) | (uint64_t)(~(uint32_t)j));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c = min(c, __shfl_xor_sync(0xffffffffu, c, o));
  if (lane == 0) wmin[warp] = c;
  if (tid == 0) pos = w;
  __syncthreads();
  c = wmin[0];
#pragma unroll
  for (int i = 1; i < kAppThreads / 32; ++i) c = min(c, wmin[i]);
  const uint32_t okw = (uint32_t)(c >> 32);
  const int jw = (int)~(uint32_t)c;
  const bool enter = order_key(drow[L - 1]) > okw;
  if (implicit) {
    for (int i = tid; i < w; i += kAppThreads) {
      const int j = (!enter || i < jw) ? i : i + 1;
      out[i] = j;
      outd[i] = drow[j];
    }
    return;
  }
  if (!enter) return;
  for (int i = tid; i < w; i += kAppThreads)
    if (out[i] == jw) pos = i;   // the keys are distinct: one writer
  __syncthreads();
  const int p0 = pos;
  // entries [p0, w - 1) move down by one, then L - 1 at the end; rounds in ascending order read
  // every entry before it is overwritten
  for (int base = (p0 / kAppThreads) * kAppThreads; base < w; base += kAppThreads) {
    const int i = base + tid;
    int v = 0;
    float dv = 0.f;
    if (i >= p0 && i < w) {
      v = i + 1 < w ? out[i + 1] : L - 1;
      dv = i + 1 < w ? outd[i + 1] : drow[L - 1];
    }
    __syncthreads();
    if (i >= p0 && i < w) {
      out[i] = v;
      outd[i] = dv;
    }
    __syncthreads();
  }
}

cudaError_t launch_topw_append(const Plan& P, const float* delta, void* ws, cudaStream_t s) {
  topw_append_kernel<<<P.B * P.H, kAppThreads, 0, s>>>(delta, ws_ptr<int32_t>(ws, P.off_sel),
                                                       ws_ptr<float>(ws, P.off_seld), P.N, P.w, P.w_heads, P.H,
                                                       P.sel_len);
  return cudaGetLastError();
}

cudaError_t launch_topw_select_rows(const float* delta, int rows, int N, int w, const int32_t* w_heads, int H,
                                    int32_t* sel, float* seld, int sel_stride, cudaStream_t s) {
  const int smem = (int)sizeof(SelShared);
  { cudaError_t ea = ensure_smem_limit(topw_decode_kernel, smem); if (ea != cudaSuccess) return ea; }
  topw_decode_kernel<<<rows, kSelThreads, smem, s>>>(delta, sel, seld, N, w, w_heads, H, sel_stride);
  return cudaGetLastError();
}

cudaError_t launch_topw_decode(const Plan& P, const float* delta, void* ws, cudaStream_t s) {
  return launch_topw_select_rows(delta, P.B * P.H, P.N, P.w, P.w_heads, P.H, ws_ptr<int32_t>(ws, P.off_sel),
                                 ws_ptr<float>(ws, P.off_seld), P.sel_len, s);
}

}  // namespace dma
