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
// Algorithm (one CTA per (b, h) row, the row resident in shared memory):
//  1. stable LSD radix sort of the row by (delta desc, index asc): p[r] = position of rank r,
//     rank[j] = rank of position j (rank 0 = best);
//  2. T_k = rank of the w-th best key among positions [0, kC) for every chunk boundary k
//     (C = 128), from a [rank bucket][position chunk] count table with prefix sums over chunks
//     (T_k = N when kC <= w: nothing evicted yet);
//  3. chunk k (positions [kC, kC+C)) resolves exactly the keys evicted inside it: old keys with rank
//     in (T_{k+1}, T_k] and new keys with rank above T_{k+1}.  For such a key of rank r,
//     e = max(j, first t >= kC at which #{i <= t : rank_i < r} reaches w), where the count of old
//     keys better than r follows from T_k and the sorted candidate list.  New keys that survive to
//     the end (rank <= T at the last boundary) get e = N.  Every key's e is written exactly once.
// A second kernel (one CTA per (row, query block)) compacts the live keys of each block:
// full keys (selected by every existing row: j <= t0 and e_j >= min(t0 + C, N)) first, then the
// partial ones (at most 2C: keys evicted inside the block and the block's own keys), each in
// ascending order.
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

// ---------------------------------------------------------------- sort + thresholds (per row)

constexpr int kSortThreads2 = 1024;
constexpr int kSortWarps2 = kSortThreads2 / 32;
constexpr int kMaxItems = kTopwMaxN / kSortThreads2;   // 16 keys per thread at most

// Shared-memory index with one pad word every 32: thread t's run [IT*t, IT*t + IT) starts in a
// different bank for every lane of a warp when IT is a power of two.
DMA_DEVINL int pad32(int i) { return i + (i >> 5); }

// One CTA per (b, h) row: stable LSD radix sort of the row by (delta descending, index ascending)
// with 4-bit digits, thread-private digit counters and a block-wide scan per pass (digit positions
// where every key agrees are skipped); then the threshold ranks T_k for every chunk boundary.
// Writes p (rank -> position), rank (position -> rank) and T to global scratch.
__global__ void __launch_bounds__(kSortThreads2, 1)
topw_sort_kernel(const float* __restrict__ delta, int32_t* __restrict__ p_out, int32_t* __restrict__ rank_out,
                 int32_t* __restrict__ T_out, int N, int w) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = (N + kC - 1) / kC;
  const int Np = pad32(N) + 32;
  const int Npi = (Np + 7) & ~7;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smraw);                         // [Np]   (later: table)
  uint16_t* idx = reinterpret_cast<uint16_t*>(keys + Np);                      // [Npi]  ping
  uint16_t* idx2 = idx + Npi;                                                  // [Npi]  pong
  uint16_t* cnt = idx2 + Npi;                                                  // [16][1024] (later: rank)
  int32_t* wsum = reinterpret_cast<int32_t*>(cnt + 16 * kSortThreads2);        // [32]
  __shared__ uint32_t red_and[kSortWarps2], red_or[kSortWarps2];

  const float* drow = delta + (size_t)row * N;
  const int IT = (N + kSortThreads2 - 1) / kSortThreads2;
  uint32_t kand = 0xffffffffu, kor = 0u;
  {
    float dv[kMaxItems];   // all loads first, then the stores
#pragma unroll
    for (int u = 0; u < kMaxItems; ++u) {
      const int i = tid + u * kSortThreads2;
      dv[u] = i < N ? drow[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kMaxItems; ++u) {
      const int i = tid + u * kSortThreads2;
      if (i < N) {
        const uint32_t k = ~order_key(dv[u]);   // ascending k = delta descending
        keys[pad32(i)] = k;
        idx[pad32(i)] = (uint16_t)i;
        kand &= k;
        kor |= k;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    kor |= __shfl_xor_sync(0xffffffffu, kor, o);
  }
  if (lane == 0) { red_and[warp] = kand; red_or[warp] = kor; }
  __syncthreads();
  uint32_t varying = 0;
  {
    uint32_t a = 0xffffffffu, o = 0u;
    for (int i = 0; i < kSortWarps2; ++i) { a &= red_and[i]; o |= red_or[i]; }
    varying = a ^ o;
  }

  for (int shift = 0; shift < 32; shift += 4) {
    if (((varying >> shift) & 0xFu) == 0) continue;   // every key has the same digit here
    uint32_t kk[kMaxItems];
#pragma unroll
    for (int c = 0; c < 16; ++c) cnt[c * kSortThreads2 + tid] = 0;
#pragma unroll
    for (int i = 0; i < kMaxItems; ++i) {
      const int pos = tid * IT + i;
      if (i < IT && pos < N) {
        kk[i] = keys[pad32(pos)];
        const uint32_t dg = (kk[i] >> shift) & 0xFu;
        cnt[dg * kSortThreads2 + tid] += 1;
      }
    }
    __syncthreads();
    {  // exclusive scan of cnt in (digit, thread) order: 16 entries per thread
      uint32_t v[16], sum = 0;
#pragma unroll
      for (int c = 0; c < 16; ++c) { v[c] = cnt[tid * 16 + c]; sum += v[c]; }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wsum[warp] = (int32_t)incl;
      __syncthreads();
      if (warp == 0) {
        const uint32_t x = (uint32_t)wsum[lane];
        uint32_t xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, xi, o);
          if (lane >= o) xi += y;
        }
        wsum[lane] = (int32_t)(xi - x);
      }
      __syncthreads();
      uint32_t run = (uint32_t)wsum[warp] + incl - sum;
#pragma unroll
      for (int c = 0; c < 16; ++c) { cnt[tid * 16 + c] = (uint16_t)run; run += v[c]; }
    }
    __syncthreads();
    // every read of `keys` in this pass happened before the barriers above, so items can be
    // written as soon as their destinations are known; indices go to the other buffer
#pragma unroll
    for (int i = 0; i < kMaxItems; ++i) {
      const int pos = tid * IT + i;
      if (i < IT && pos < N) {
        const uint32_t dg = (kk[i] >> shift) & 0xFu;
        const int dst = cnt[dg * kSortThreads2 + tid];
        cnt[dg * kSortThreads2 + tid] = (uint16_t)(dst + 1);
        keys[pad32(dst)] = kk[i];
        idx2[pad32(dst)] = idx[pad32(pos)];
      }
    }
    __syncthreads();
    uint16_t* t = idx; idx = idx2; idx2 = t;
  }
  // p[r] = idx[pad32(r)];  rank[j] in the counter area
  uint16_t* rank = cnt;
  int32_t* prow = p_out + (size_t)row * N;
  int32_t* rrow = rank_out + (size_t)row * N;
  for (int r = tid; r < N; r += kSortThreads2) {
    const int j = idx[pad32(r)];
    rank[j] = (uint16_t)r;
    prow[r] = j;
    rrow[j] = r;
  }
  // thresholds: table[rb][k] = #positions < k*C whose rank is in bucket rb (u32, reuses keys)
  uint32_t* table = keys;
  const int cw = nch + 1;
  for (int i = tid; i < nch * cw; i += kSortThreads2) table[i] = 0;
  __syncthreads();
  for (int j = tid; j < N; j += kSortThreads2) atomicAdd(&table[(rank[j] >> 7) * cw + (j >> 7)], 1u);
  __syncthreads();
  for (int rb = tid; rb < nch; rb += kSortThreads2) {
    uint32_t prev = 0;
    for (int k = 0; k <= nch; ++k) {
      const uint32_t t = table[rb * cw + k];
      table[rb * cw + k] = prev;
      prev += t;
    }
  }
  __syncthreads();
  for (int k = warp; k <= nch; k += kSortWarps2) {
    const int Pk = min(k * kC, N);
    int Tk = N;
    if (Pk > w) {
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
      int need = w - before;
      for (int r0 = rbs * 128; r0 < min(rbs * 128 + 128, N); r0 += 32) {
        const int r = r0 + lane;
        const uint32_t m = __ballot_sync(0xffffffffu, r < N && (int)idx[pad32(min(r, N - 1))] < Pk);
        const int c = __popc(m);
        if (c >= need) { Tk = r0 + nth_set_bit(m, need - 1); break; }
        need -= c;
      }
    }
    if (lane == 0) T_out[(size_t)row * cw + k] = Tk;
  }
}

// ---------------------------------------------------------------- eviction index (per chunk)

constexpr int kEvThreads = 128;

// One CTA per (chunk k, row).  Chunk k = positions [t0, t1) resolves exactly the keys evicted
// inside it: old keys (position < t0) with rank in (T_{k+1}, T_k], and its own keys with rank above
// T_{k+1}.  For such a key of rank r, e = max(j, first t >= t0 with #{i <= t : rank_i < r} >= w);
// the count over old positions follows from T_k: Sk - #{old candidates with rank >= r}, Sk being
// min(t0, w).  Its own keys that survive the last boundary get e = N.
__global__ void __launch_bounds__(kEvThreads)
topw_evict_kernel(const int32_t* __restrict__ p_in, const int32_t* __restrict__ rank_in,
                  const int32_t* __restrict__ T_in, int32_t* __restrict__ evict, int32_t* __restrict__ status,
                  int N, int w) {
  __shared__ int32_t crank[kC];      // ranks of the chunk's own keys
  __shared__ int32_t L[kC];          // old candidates, ascending rank
  __shared__ int32_t wcount[kEvThreads / 32];
  const int k = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = (N + kC - 1) / kC;
  const int t0 = k * kC, t1 = min(t0 + kC, N);
  const int32_t* prow = p_in + (size_t)row * N;
  const int32_t* rrow = rank_in + (size_t)row * N;
  const int32_t* T = T_in + (size_t)row * (nch + 1);
  int32_t* erow = evict + (size_t)row * N;
  const int Ta = T[k], Tb = T[k + 1], Tf = T[nch];
  const int Sk = min(t0, w);
  if (tid < t1 - t0) crank[tid] = rrow[t0 + tid];
  // old candidates in rank order
  int nL = 0;
  const int rhi = min(Ta, N - 1);
  for (int r0 = Tb + 1; r0 <= rhi; r0 += kEvThreads) {
    const int r = r0 + tid;
    const bool in = r <= rhi && prow[r] < t0;
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    if (lane == 0) wcount[warp] = __popc(m);
    __syncthreads();
    int before = nL, total = 0;
    for (int i = 0; i < kEvThreads / 32; ++i) {
      if (i < warp) before += wcount[i];
      total += wcount[i];
    }
    if (in) {
      const int slot = before + __popc(m & lanemask_lt());
      if (slot < kC) L[slot] = r;
    }
    nL += total;
    __syncthreads();
  }
  if (nL > kC) {   // cannot happen: at most C keys are evicted per chunk
    if (tid == 0) atomicOr(status, 2);
    nL = kC;
  }
  __syncthreads();
  const int ncand = nL + (t1 - t0);
  for (int c = tid; c < ncand; c += kEvThreads) {
    int r, j, base, e = -1;
    bool scan = false;
    if (c < nL) {
      r = L[c];
      j = prow[r];
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
        int above = 0;                 // old members with rank in (r, Ta]
        for (int i = 0; i < nL; ++i) above += L[i] > r;
        base = Sk - above;
        if (base >= w) e = j;
        else scan = true;
      }
    }
    if (scan) {
      int count = base;
      e = -2;
      for (int t = t0; t < t1; ++t) {
        if (crank[t - t0] < r && ++count >= w) { e = max(j, t); break; }
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
// group in ascending key order.  One CTA scans the keys of a pair of blocks (kPairQ rows) once and
// builds three lists from them: those of its two blocks (the mask encoding of the interface) and
// that of the pair (the attention forward's work item), whose entries also carry j | e_j << 16
// and delta_j * log2(e) and which is padded to a multiple of 128 entries with key -1 (masked for
// every row: e = 0).
constexpr int kListThreads = 256;
constexpr int kListWarps = kListThreads / 32;
constexpr int kListBits = 10;                    // packed per-warp counters (a warp counts <= 128)
constexpr int kListMask = (1 << kListBits) - 1;

__global__ void __launch_bounds__(kListThreads)
topw_lists_kernel(const int32_t* __restrict__ evict, const float* __restrict__ delta,
                  int32_t* __restrict__ counts, int32_t* __restrict__ lists,
                  int32_t* __restrict__ pcounts, int32_t* __restrict__ plists,
                  int32_t* __restrict__ pje, float* __restrict__ pdl, int N, int list_cap, int pair_cap,
                  int n_blocks, int n_pairs) {
  // partial keys: block a (<= 2C), block b (<= 2C), pair (<= 4C)
  __shared__ int32_t part[8 * kC];
  __shared__ int32_t wsum[6][kListWarps];   // per warp: full count of list 0..2, partial count of 0..2
  const int kp = blockIdx.x, row = blockIdx.y;
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
  int32_t* oje = pje + pbase;
  float* odl = pdl + pbase;
  int nfull[3] = {0, 0, 0}, npart[3] = {0, 0, 0};
  int enext[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = tid * 4 + u;
    enext[u] = j < t1 ? erow[j] : 0;
  }
  for (int base = 0; base < t1; base += kListThreads * 4) {
    int ecur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ecur[u] = enext[u];
      const int jn = base + kListThreads * 4 + tid * 4 + u;   // prefetch the next round
      enext[u] = jn < t1 ? erow[jn] : 0;
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
        const bool live = valid && j < hi[L] && e > max(j, lo[L]);
        const bool full = live && j <= lo[L] && e >= hi[L];
        fbits |= (uint32_t)full << (3 * u + L);
        qbits |= (uint32_t)(live && !full) << (3 * u + L);
        cf += (int)full << (kListBits * L);
        cq += (int)(live && !full) << (kListBits * L);
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
              oje[of[L]] = (j & 0xffff) | (ecur[u] << 16);
              odl[of[L]] = drow[j] * kLog2e;
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
        oje[nfull[L] + i] = (j & 0xffff) | (erow[j] << 16);
        odl[nfull[L] + i] = drow[j] * kLog2e;
      }
    }
  }
  const int nlive = nfull[2] + npart[2];
  const int nround = min(pair_cap, (nlive + kC - 1) / kC * kC);
  for (int i = nlive + tid; i < nround; i += kListThreads) {
    out[2][i] = -1;
    oje[i] = 0xffff;
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

constexpr int kSelThreads = 1024;

// Top-w of the whole row (query at position N-1): 4-pass MSB-first radix select on the order key,
// then an order-preserving compaction of the selected positions.
__global__ void __launch_bounds__(kSelThreads)
topw_decode_kernel(const float* __restrict__ delta, int32_t* __restrict__ sel, int N, int w) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_prefix, sh_need;
  __shared__ int32_t wcnt[2][kSelThreads / 32];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* drow = delta + (size_t)row * N;
  const int k = min(w, N);
  int32_t* out = sel + (size_t)row * k;
  if (k == N) {
    for (int i = tid; i < N; i += kSelThreads) out[i] = i;
    return;
  }
  uint32_t prefix = 0, mask = 0, need = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < N; i0 += kSelThreads) {
      const int i = i0 + tid;
      const bool valid = i < N;
      uint32_t key = valid ? order_key(drow[i]) : 0u;
      const bool in = valid && ((key & mask) == prefix);
      const uint32_t imask = __ballot_sync(0xffffffffu, in);
      if (in) {
        const uint32_t dig = (key >> shift) & 255u;
        const uint32_t peers = __match_any_sync(imask, dig);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[dig], __popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // digits from high to low: lane l owns digits 255-8l .. 248-8l
      uint32_t v[8], s = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { v[u] = hist[255 - (lane * 8 + u)]; s += v[u]; }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need);
      const int l = __ffs(hit) - 1;
      if (lane == l) {
        uint32_t above = incl - s;
        for (int u = 0; u < 8; ++u) {
          if (above + v[u] >= need) {
            sh_prefix = prefix | ((uint32_t)(255 - (lane * 8 + u)) << shift);
            sh_need = need - above;
            break;
          }
          above += v[u];
        }
      }
    }
    __syncthreads();
    prefix = sh_prefix;
    need = sh_need;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix = order key of the k-th best; take keys above it and the first `need` equal ones
  int taken = 0, eqseen = 0;
  for (int i0 = 0; i0 < N; i0 += kSelThreads) {
    const int i = i0 + tid;
    const uint32_t key = i < N ? order_key(drow[i]) : 0u;
    const bool gt = i < N && key > prefix;
    const bool eq = i < N && key == prefix;
    const uint32_t meq = __ballot_sync(0xffffffffu, eq);
    int eq_before_in_warp = __popc(meq & lanemask_lt());
    if (lane == 0) wcnt[1][warp] = __popc(meq);
    __syncthreads();
    int eq_before = eqseen + eq_before_in_warp, eq_tot = 0;
    for (int u = 0; u < kSelThreads / 32; ++u) {
      if (u < warp) eq_before += wcnt[1][u];
      eq_tot += wcnt[1][u];
    }
    const bool take = gt || (eq && eq_before < (int)need);
    const uint32_t mt = __ballot_sync(0xffffffffu, take);
    if (lane == 0) wcnt[0][warp] = __popc(mt);
    __syncthreads();
    int t_before = taken + __popc(mt & lanemask_lt()), t_tot = 0;
    for (int u = 0; u < kSelThreads / 32; ++u) {
      if (u < warp) t_before += wcnt[0][u];
      t_tot += wcnt[0][u];
    }
    if (take && t_before < k) out[t_before] = i;
    taken += t_tot;
    eqseen += eq_tot;
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_topw_prefill(const Plan& P, const float* delta, int32_t* evict, void* ws,
                                cudaStream_t s) {
  const int rows = P.B * P.H;
  const int nch = P.n_blocks;
  const int Np = P.N + (P.N >> 5) + 32;
  const size_t smem = (size_t)Np * 4 + (size_t)((Np + 7) & ~7) * 2 * 2 + 16 * kSortThreads2 * 2 + 32 * 4 +
                      (size_t)(nch + 1) * 4;
  if ((size_t)nch * (nch + 1) * 4 > (size_t)Np * 4) return cudaErrorInvalidValue;   // table must fit
  { cudaError_t ea = ensure_smem_limit(topw_sort_kernel, (int)smem); if (ea != cudaSuccess) return ea; }
  int32_t* pbuf = ws_ptr<int32_t>(ws, P.off_tw_p);
  int32_t* rbuf = ws_ptr<int32_t>(ws, P.off_tw_rank);
  int32_t* Tbuf = ws_ptr<int32_t>(ws, P.off_tw_T);
  topw_sort_kernel<<<rows, kSortThreads2, smem, s>>>(delta, pbuf, rbuf, Tbuf, P.N, P.w);
  topw_evict_kernel<<<dim3(nch, rows), kEvThreads, 0, s>>>(pbuf, rbuf, Tbuf, evict,
                                                            ws_ptr<int32_t>(ws, P.off_status), P.N, P.w);
  topw_lists_kernel<<<dim3(P.n_pairs, rows), kListThreads, 0, s>>>(
      evict, delta, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists),
      ws_ptr<int32_t>(ws, P.off_pcounts), ws_ptr<int32_t>(ws, P.off_plists), ws_ptr<int32_t>(ws, P.off_pje),
      ws_ptr<float>(ws, P.off_pdl), P.N, P.list_cap, P.pair_cap, P.n_blocks, P.n_pairs);
  return cudaGetLastError();
}

cudaError_t launch_topw_decode(const Plan& P, const float* delta, void* ws, cudaStream_t s) {
  topw_decode_kernel<<<P.B * P.H, kSelThreads, 0, s>>>(delta, ws_ptr<int32_t>(ws, P.off_sel), P.N,
                                                       P.w);
  return cudaGetLastError();
}

}  // namespace dma
