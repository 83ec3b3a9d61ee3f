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
constexpr int kSortWarps = 16;
constexpr int kSortThreads = kSortWarps * 32;

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

struct TopwSmem {
  uint32_t* keyA;   // [N]   (later: count table, shared with keyB)
  uint32_t* keyB;   // [N]
  uint16_t* idxA;   // [N]   after sorting: p[r]
  uint16_t* idxB;   // [N]   after sorting: rank[j]
  uint32_t* hist;   // [256 * kSortWarps]
  int32_t* T;       // [nch + 1]
  uint16_t* cand;   // [kSortWarps][kC]
  int32_t* scan;    // [kSortThreads]
};

__global__ void __launch_bounds__(kSortThreads, 1)
topw_rows_kernel(const float* __restrict__ delta, int32_t* __restrict__ evict,
                 int32_t* __restrict__ status, int N, int w) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = (N + kC - 1) / kC;
  const int Nal = (N + 7) & ~7;
  TopwSmem S;
  S.keyA = reinterpret_cast<uint32_t*>(smraw);
  S.keyB = S.keyA + Nal;
  S.idxA = reinterpret_cast<uint16_t*>(S.keyB + Nal);
  S.idxB = S.idxA + Nal;
  S.hist = reinterpret_cast<uint32_t*>(S.idxB + Nal);
  S.T = reinterpret_cast<int32_t*>(S.hist + 256 * kSortWarps);
  S.cand = reinterpret_cast<uint16_t*>(S.T + ((nch + 1 + 3) & ~3));
  S.scan = reinterpret_cast<int32_t*>(S.cand + kSortWarps * kC);

  const float* drow = delta + (size_t)row * N;
  int32_t* erow = evict + (size_t)row * N;

  // ---- 1. stable radix sort, ascending on ~order_key (= delta descending, index ascending)
  for (int i = tid; i < N; i += kSortThreads) {
    S.keyA[i] = ~order_key(drow[i]);
    S.idxA[i] = (uint16_t)i;
  }
  const int seg = ((N + kSortWarps - 1) / kSortWarps + 31) & ~31;
  const int wbeg = warp * seg, wend = min(N, wbeg + seg);
  uint32_t* kin = S.keyA;
  uint32_t* kout = S.keyB;
  uint16_t* iin = S.idxA;
  uint16_t* iout = S.idxB;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = pass * 8;
    for (int i = tid; i < 256 * kSortWarps; i += kSortThreads) S.hist[i] = 0;
    __syncthreads();
    for (int base = wbeg; base < wend; base += 32) {
      const int i = base + lane;
      const bool valid = i < wend;
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const uint32_t dig = (kin[i] >> shift) & 255u;
        const uint32_t peers = __match_any_sync(vmask, dig);
        if (lane == __ffs(peers) - 1) S.hist[dig * kSortWarps + warp] += __popc(peers);
      }
      __syncwarp();
    }
    __syncthreads();
    {  // exclusive scan of hist in (digit, warp) order: 4096 entries, 8 per thread
      uint32_t v[8], sum = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) { v[k] = S.hist[tid * 8 + k]; sum += v[k]; }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) S.scan[warp] = (int32_t)incl;
      __syncthreads();
      if (warp == 0) {
        uint32_t ws = lane < kSortWarps ? (uint32_t)S.scan[lane] : 0u;
        uint32_t wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
          if (lane >= o) wi += y;
        }
        if (lane < kSortWarps) S.scan[lane] = (int32_t)(wi - ws);
      }
      __syncthreads();
      uint32_t run = (uint32_t)S.scan[warp] + incl - sum;
#pragma unroll
      for (int k = 0; k < 8; ++k) { S.hist[tid * 8 + k] = run; run += v[k]; }
    }
    __syncthreads();
    for (int base = wbeg; base < wend; base += 32) {
      const int i = base + lane;
      const bool valid = i < wend;
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      uint32_t key = 0, dig = 0, peers = 0, dst = 0;
      uint16_t idx = 0;
      if (valid) {
        key = kin[i];
        idx = iin[i];
        dig = (key >> shift) & 255u;
        peers = __match_any_sync(vmask, dig);
        dst = S.hist[dig * kSortWarps + warp] + __popc(peers & lanemask_lt());
      }
      __syncwarp();
      if (valid) {
        kout[dst] = key;
        iout[dst] = idx;
        if (lane == __ffs(peers) - 1) S.hist[dig * kSortWarps + warp] += __popc(peers);
      }
      __syncwarp();
    }
    __syncthreads();
    uint32_t* tk = kin; kin = kout; kout = tk;
    uint16_t* ti = iin; iin = iout; iout = ti;
  }
  // after 4 passes the sorted order is back in (keyA, idxA)
  const uint16_t* p = S.idxA;   // p[r]
  uint16_t* rank = S.idxB;      // rank[j]
  for (int r = tid; r < N; r += kSortThreads) rank[p[r]] = (uint16_t)r;

  // ---- 2. thresholds T_k, k = 0..nch
  uint32_t* cnt = S.keyA;   // [nch][nch + 1] (spans keyA and keyB)
  const int cw = nch + 1;
  for (int i = tid; i < nch * cw; i += kSortThreads) cnt[i] = 0;
  __syncthreads();
  for (int j = tid; j < N; j += kSortThreads) atomicAdd(&cnt[(rank[j] >> 7) * cw + (j >> 7)], 1u);
  __syncthreads();
  for (int rb = tid; rb < nch; rb += kSortThreads) {
    uint32_t prev = 0;
    for (int k = 0; k <= nch; ++k) {
      const uint32_t t = cnt[rb * cw + k];
      cnt[rb * cw + k] = prev;   // positions < k*C with rank in bucket rb
      prev += t;
    }
  }
  __syncthreads();
  for (int k = warp; k <= nch; k += kSortWarps) {
    const int Pk = min(k * kC, N);
    int Tk = N;
    if (Pk > w) {
      int before = 0, rbs = -1;
      for (int rb0 = 0; rb0 < nch && rbs < 0; rb0 += 32) {
        const int rb = rb0 + lane;
        const int v = rb < nch ? (int)cnt[rb * cw + k] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          int y = __shfl_up_sync(0xffffffffu, incl, o);
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
      int need = w - before;   // >= 1: the need-th present rank in bucket rbs
      for (int r0 = rbs * 128; r0 < min(rbs * 128 + 128, N); r0 += 32) {
        const int r = r0 + lane;
        const uint32_t m = __ballot_sync(0xffffffffu, r < N && p[r] < Pk);
        const int c = __popc(m);
        if (c >= need) { Tk = r0 + nth_set_bit(m, need - 1); break; }
        need -= c;
      }
    }
    if (lane == 0) S.T[k] = Tk;
  }
  __syncthreads();

  // ---- 3. eviction index, chunk by chunk
  const int Tf = S.T[nch];
  uint16_t* L = S.cand + warp * kC;
  for (int k = warp; k < nch; k += kSortWarps) {
    const int t0 = k * kC, t1 = min(t0 + kC, N);
    const int Ta = S.T[k], Tb = S.T[k + 1];
    const int Sk = min(t0, w);
    // old candidates: rank in (Tb, min(Ta, N-1)] and position < t0, ascending rank
    int nL = 0;
    const int rhi = min(Ta, N - 1);
    for (int r0 = Tb + 1; r0 <= rhi; r0 += 32) {
      const int r = r0 + lane;
      const bool in = r <= rhi && p[r] < t0;
      const uint32_t m = __ballot_sync(0xffffffffu, in);
      if (in) {
        const int slot = nL + __popc(m & lanemask_lt());
        if (slot < kC) L[slot] = (uint16_t)r;
      }
      nL += __popc(m);
    }
    if (nL > kC) {   // cannot happen: at most C keys are evicted per chunk
      if (lane == 0) atomicOr(status, 2);
      nL = kC;
    }
    __syncwarp();
    // candidates: old (index < nL) then new (positions t0..t1-1)
    const int ncand = nL + (t1 - t0);
    for (int c0 = 0; c0 < ncand; c0 += 32) {
      const int c = c0 + lane;
      int r = 0, j = 0, base = 0, e = -1;
      bool scan = false;
      if (c < nL) {
        r = L[c];
        j = p[r];
        base = Sk - (nL - c);
        scan = true;
      } else if (c < ncand) {
        j = t0 + (c - nL);
        r = rank[j];
        if (r <= Tb) {
          if (r <= Tf) e = N;          // never evicted
        } else if (Ta < N && r > Ta) {
          e = j;                       // never selected
        } else {
          int above = 0;               // old members with rank in (r, Ta]
          for (int i = 0; i < nL; ++i) above += (int)L[i] > r;
          base = Sk - above;
          if (base >= w) e = j;
          else scan = true;
        }
      }
      bool active = scan;
      int count = base;
      for (int t = t0; t < t1 && __any_sync(0xffffffffu, active); ++t) {
        const int rt = rank[t];
        if (active && rt < r) {
          if (++count >= w) { e = max(j, t); active = false; }
        }
      }
      if (active) {   // cannot happen: such keys are evicted inside the chunk
        e = t1;
        atomicOr(status, 4);
      }
      if (c < ncand && e >= 0) erow[j] = e;
    }
    __syncwarp();
  }
}

// Live keys of query block k: j < t1 and e_j > max(j, t0).  Full keys (j <= t0, e_j >= t1) first.
constexpr int kListThreads = 256;

__global__ void __launch_bounds__(kListThreads)
topw_lists_kernel(const int32_t* __restrict__ evict, int32_t* __restrict__ counts,
                  int32_t* __restrict__ lists, int N, int list_cap, int n_blocks) {
  __shared__ int32_t partial[2 * kC];
  __shared__ int32_t wsum[2][kListThreads / 32];
  const int k = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = k * kC, t1 = min(t0 + kC, N);
  const int32_t* erow = evict + (size_t)row * N;
  int32_t* out = lists + ((size_t)row * n_blocks + k) * list_cap;
  int nfull = 0, npart = 0;
  for (int base = 0; base < t1; base += kListThreads * 4) {
    int f[4], q[4];
    int cf = 0, cq = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + tid * 4 + u;
      int e = j < t1 ? erow[j] : 0;
      const bool live = j < t1 && e > max(j, t0);
      const bool full = live && j <= t0 && e >= t1;
      f[u] = full;
      q[u] = live && !full;
      cf += f[u];
      cq += q[u];
    }
    int incf = cf, incq = cq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int yf = __shfl_up_sync(0xffffffffu, incf, o);
      int yq = __shfl_up_sync(0xffffffffu, incq, o);
      if (lane >= o) { incf += yf; incq += yq; }
    }
    if (lane == 31) { wsum[0][warp] = incf; wsum[1][warp] = incq; }
    __syncthreads();
    int wf = 0, wq = 0, tf = 0, tq = 0;
    for (int i = 0; i < kListThreads / 32; ++i) {
      if (i < warp) { wf += wsum[0][i]; wq += wsum[1][i]; }
      tf += wsum[0][i];
      tq += wsum[1][i];
    }
    int of = nfull + wf + incf - cf, oq = npart + wq + incq - cq;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + tid * 4 + u;
      if (f[u]) { if (of < list_cap) out[of] = j; ++of; }
      if (q[u]) { if (oq < 2 * kC) partial[oq] = j; ++oq; }
    }
    nfull += tf;
    npart += tq;
    __syncthreads();
  }
  // at most C evicted old keys plus C new keys; a live set never exceeds list_cap
  nfull = min(nfull, list_cap);
  npart = min(min(npart, 2 * kC), list_cap - nfull);
  for (int i = tid; i < npart; i += kListThreads) out[nfull + i] = partial[i];
  if (tid == 0) {
    counts[((size_t)row * n_blocks + k) * 2 + 0] = nfull;
    counts[((size_t)row * n_blocks + k) * 2 + 1] = nfull + npart;
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

size_t topw_rows_smem_bytes(int N) {
  const int nch = (N + kC - 1) / kC;
  const size_t Nal = (size_t)((N + 7) & ~7);
  size_t b = Nal * 4 * 2 + Nal * 2 * 2 + 256 * kSortWarps * 4 + (size_t)((nch + 1 + 3) & ~3) * 4 +
             kSortWarps * kC * 2 + kSortThreads * 4;
  // the count table [nch][nch+1] u32 reuses keyA+keyB
  const size_t table = (size_t)nch * (nch + 1) * 4;
  if (table > Nal * 8) b += table - Nal * 8;   // only for tiny N
  return b;
}

cudaError_t launch_topw_prefill(const Plan& P, const float* delta, int32_t* evict, void* ws,
                                cudaStream_t s) {
  const int rows = P.B * P.H;
  size_t smem = topw_rows_smem_bytes(P.N);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  { cudaError_t ea = ensure_smem_limit(topw_rows_kernel, (int)smem); if (ea != cudaSuccess) return ea; }
  topw_rows_kernel<<<rows, kSortThreads, smem, s>>>(delta, evict, ws_ptr<int32_t>(ws, P.off_status),
                                                   P.N, P.w);
  topw_lists_kernel<<<dim3(P.n_blocks, rows), kListThreads, 0, s>>>(
      evict, ws_ptr<int32_t>(ws, P.off_counts), ws_ptr<int32_t>(ws, P.off_lists), P.N, P.list_cap,
      P.n_blocks);
  return cudaGetLastError();
}

cudaError_t launch_topw_decode(const Plan& P, const float* delta, void* ws, cudaStream_t s) {
  topw_decode_kernel<<<P.B * P.H, kSelThreads, 0, s>>>(delta, ws_ptr<int32_t>(ws, P.off_sel), P.N,
                                                       P.w);
  return cudaGetLastError();
}

}  // namespace dma
