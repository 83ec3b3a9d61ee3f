// Context-parallel prefill: the sequence is split into contiguous shards, one per rank, and one
// exchange of each shard's best keys lets every rank rebuild an exact stand-in for the prefix in
// front of its shard.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Dynamic Sparse Mask
// Generation", m_t equation: a query at position t keeps the best min(t+1, w) keys of [0, t] by
// delta (ties to the lower position).  The best keys of a union are among the best keys of its
// parts, so for every query of shard r the selection lies in (the best keys of the prefix) + (the
// shard's own keys), and the best keys of the prefix lie among the best keys of every earlier shard.
//
//   dma_cp_candidates  per (b, h): the best min(W_h, len) keys of the shard (the decode selection
//                      kernel over the shard's delta row), packed with their global position, delta
//                      and K, V rows into a fixed-size candidate buffer (the unit of the exchange);
//   dma_cp_compact     from the candidates of every earlier shard: per (b, h) the best keys of the
//                      whole prefix (the same selection kernel over the merged candidates), per
//                      (b, g) the union of its heads' sets in position order behind padding rows,
//                      then the shard's own keys: a sequence of P + len rows whose selection and
//                      attention for the shard's queries equal those of the whole sequence (delta of
//                      a union key is -inf for a head that did not select it, and of padding rows
//                      -inf for every head: neither is ever among a query's best keys once the
//                      prefix holds w keys; a shorter prefix is kept whole).
#include "common.cuh"
#include "internal.h"

namespace dma {
namespace {

constexpr int kCpThreads = 256;
constexpr int kCpUnionThreads = 1024;
constexpr int kCpMaxUnion = 16384;   // G * w: union entries a (b, g) sorts in shared memory
constexpr int kCpErrUnion = 0x20000000;   // workspace status bit: a union larger than its rows

struct CpLayout {
  size_t cand_bytes, off_pos, off_delta, off_k, off_v;
  size_t ws_bytes, off_status, off_sel, off_dm, off_sel2, off_src;
  int prefix_rows, elt, cap;
};

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

CpLayout cp_layout_of(const Plan& P, int prefix_len, int n_prev) {
  CpLayout L;
  const size_t BH = (size_t)P.B * P.H, w = (size_t)P.w;
  L.elt = P.bf16 ? 2 : 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.off_pos = take(BH * w * 4);
  L.off_delta = take(BH * w * 4);
  L.off_k = take(BH * w * P.d * L.elt);
  L.off_v = take(BH * w * P.d * L.elt);
  L.cand_bytes = off;
  off = 0;
  L.off_status = take(256);
  L.off_sel = take(BH * w * 4);
  L.off_dm = take(BH * (size_t)(n_prev > 0 ? n_prev : 1) * w * 4);
  L.off_sel2 = take(BH * w * 4);
  L.off_src = take(BH * w * 8);   // >= B Hkv P source entries (P <= G w)
  L.ws_bytes = off;
  L.prefix_rows = (int)((size_t)P.G * w < (size_t)prefix_len ? (size_t)P.G * w : (size_t)prefix_len);
  L.cap = next_pow2(P.G * P.w);
  return L;
}

// 16-byte chunks of one row of `nch` chunks, copied by the lanes `lane0 + 32 k` of a warp.
DMA_DEVINL void copy_row(uint4* dst, const uint4* src, int nch, int lane) {
  for (int c = lane; c < nch; c += 32) dst[c] = src != nullptr ? src[c] : make_uint4(0, 0, 0, 0);
}

// One CTA per (b, h, kCpThreads entries): the shard's selection (ascending shard positions, stride w)
// packed into the candidate buffer; entries past the row's count get position -1, delta -inf and zero
// rows.
__global__ void __launch_bounds__(kCpThreads)
cp_pack_kernel(const int32_t* __restrict__ sel, const float* __restrict__ delta, const unsigned char* __restrict__ K,
               const unsigned char* __restrict__ V, int32_t* __restrict__ cpos, float* __restrict__ cdl,
               unsigned char* __restrict__ cK, unsigned char* __restrict__ cV, int H, int G, int len, int w,
               const int32_t* __restrict__ w_heads, int shard_start, int row_bytes) {
  const int row = blockIdx.x, b = row / H, h = row % H, Hkv = H / G, g = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = blockIdx.y * kCpThreads, i1 = min(i0 + kCpThreads, w);
  const int k = min(row_window(w_heads, row, H, w), len);
  const size_t base = (size_t)row * w;
  if (i0 + tid < i1) {
    const int i = i0 + tid;
    const int j = i < k ? sel[base + i] : -1;
    cpos[base + i] = j >= 0 ? shard_start + j : -1;
    cdl[base + i] = j >= 0 ? delta[(size_t)row * len + j] : -INFINITY;
  }
  const int nch = row_bytes / 16;
  const size_t kvrow0 = (size_t)(b * Hkv + g) * len;
  for (int i = i0 + warp; i < i1; i += kCpThreads / 32) {
    const int j = i < k ? sel[base + i] : -1;
    const uint4* sk = j >= 0 ? reinterpret_cast<const uint4*>(K + (kvrow0 + j) * row_bytes) : nullptr;
    const uint4* sv = j >= 0 ? reinterpret_cast<const uint4*>(V + (kvrow0 + j) * row_bytes) : nullptr;
    copy_row(reinterpret_cast<uint4*>(cK + (base + i) * row_bytes), sk, nch, lane);
    copy_row(reinterpret_cast<uint4*>(cV + (base + i) * row_bytes), sv, nch, lane);
  }
}

// dm[row][q w + i] = delta of entry i of shard q's candidates of row: the merged candidates of the
// prefix, in shard order (= ascending position for the real entries).
__global__ void cp_gather_delta_kernel(const unsigned char* __restrict__ cands, size_t cand_bytes, size_t off_delta,
                                       float* __restrict__ dm, int rows, int n_prev, int w) {
  const size_t n = (size_t)rows * n_prev * w;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % w);
    const size_t rq = e / w;
    const int q = (int)(rq % n_prev);
    const size_t row = rq / n_prev;
    dm[e] = reinterpret_cast<const float*>(cands + q * cand_bytes + off_delta)[row * w + i];
  }
}

// One CTA per (b, g): the union, over the heads of group g, of each head's best keys of the prefix
// (sel2: ascending indices q w + i into the merged candidates, stride w), in position order behind
// P - |union| padding rows; then delta per head (-inf where the head did not select the key).
__global__ void __launch_bounds__(kCpUnionThreads)
cp_union_kernel(const unsigned char* __restrict__ cands, size_t cand_bytes, size_t off_pos, size_t off_delta,
                size_t off_k, size_t off_v, const int32_t* __restrict__ sel2, float* __restrict__ delta_c,
                int32_t* __restrict__ pos_c, int64_t* __restrict__ src, int32_t* __restrict__ status, int H, int G,
                int n_prev, int w, const int32_t* __restrict__ w_heads, int P, int Nc, int cap, int64_t n_rows_w) {
  extern __shared__ __align__(16) unsigned char cp_sm[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(cp_sm);                   // [cap]
  int32_t* first = reinterpret_cast<int32_t*>(keys + cap);              // [cap]: 1 for the first of a position
  __shared__ int count, wsum[kCpUnionThreads / 32];
  const int bg = blockIdx.x, Hkv = H / G, b = bg / Hkv, g = bg % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) count = 0;
  (void)off_k;
  (void)off_v;
  // prefix rows start at delta -inf for every head of the group
  for (int hh = 0; hh < G; ++hh) {
    float* dc = delta_c + (size_t)(b * H + g * G + hh) * Nc;
    for (int i = tid; i < P; i += kCpUnionThreads) dc[i] = -INFINITY;
  }
  __syncthreads();
  // the selected real entries of every head: key = position << 32 | head << 24 | merged index
  for (int hh = 0; hh < G; ++hh) {
    const int row = b * H + g * G + hh;
    const int kh = min(row_window(w_heads, row, H, w), n_prev * w);
    for (int i = tid; i < kh; i += kCpUnionThreads) {
      const int idx = sel2[(size_t)row * w + i];
      const int q = idx / w, ii = idx % w;
      const int pos = reinterpret_cast<const int32_t*>(cands + q * cand_bytes + off_pos)[(size_t)row * w + ii];
      if (pos < 0) continue;
      const int slot = atomicAdd(&count, 1);
      if (slot < cap) keys[slot] = ((uint64_t)(uint32_t)pos << 32) | ((uint64_t)hh << 24) | (uint64_t)idx;
    }
  }
  __syncthreads();
  const int n = count;
  if (n > cap) {   // cannot happen (each head selects at most w keys, cap >= G w): reported, nothing written
    if (tid == 0) atomicOr(status, kCpErrUnion);
    return;
  }
  for (int s = n + tid; s < cap; s += kCpUnionThreads) keys[s] = ~0ull;
  __syncthreads();
  // bitonic sort ascending
  for (int size = 2; size <= cap; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < cap; i += kCpUnionThreads) {
        const int partner = i ^ stride;
        if (partner > i) {
          const uint64_t a = keys[i], c = keys[partner];
          const bool up = (i & size) == 0;
          if ((a > c) == up) {
            keys[i] = c;
            keys[partner] = a;
          }
        }
      }
      __syncthreads();
    }
  // rank of each distinct position: exclusive scan of the first-of-a-position flags, in contiguous
  // segments of per = cap / threads entries per thread
  const int per = (cap + kCpUnionThreads - 1) / kCpUnionThreads;
  int local = 0;
  for (int u = 0; u < per; ++u) {
    const int s = tid * per + u;
    int f = 0;
    if (s < n) f = (s == 0 || (keys[s] >> 32) != (keys[s - 1] >> 32)) ? 1 : 0;
    if (s < cap) first[s] = f;
    local += f;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int i = 0; i < warp; ++i) wbase += wsum[i];
  int total = 0;
  for (int i = 0; i < kCpUnionThreads / 32; ++i) total += wsum[i];
  int run = wbase + incl - local;   // distinct positions before this thread's segment
  for (int u = 0; u < per; ++u) {
    const int s = tid * per + u;
    if (s < cap) {
      const int f = first[s];
      first[s] = run + f - 1;       // rank of the position of entry s
      run += f;
    }
  }
  __syncthreads();
  const int base = P - total;   // total <= P: union of G sets of <= w keys within the prefix
  if (base < 0) {                // cannot happen either: reported, nothing more written
    if (tid == 0) atomicOr(status, kCpErrUnion);
    return;
  }
  // delta of every (position, head) entry
  for (int s = tid; s < n; s += kCpUnionThreads) {
    const uint64_t key = keys[s];
    const int hh = (int)((key >> 24) & 0xff), idx = (int)(key & 0xffffff);
    const int q = idx / w, ii = idx % w, row = b * H + g * G + hh;
    delta_c[(size_t)row * Nc + base + first[s]] =
        reinterpret_cast<const float*>(cands + q * cand_bytes + off_delta)[(size_t)row * w + ii];
  }
  // position and source entry of each prefix row (the entry that comes first for a position: every
  // head of the group holds the same K and V rows for it); padding rows -1.  cp_rows_kernel copies.
  for (int s = tid; s < n; s += kCpUnionThreads) {
    const uint64_t key = keys[s];
    if (s > 0 && (keys[s - 1] >> 32) == (key >> 32)) continue;
    const int hh = (int)((key >> 24) & 0xff), idx = (int)(key & 0xffffff);
    const int q = idx / w, ii = idx % w, row = b * H + g * G + hh;
    const int out = base + first[s];
    pos_c[(size_t)bg * Nc + out] = (int32_t)(key >> 32);
    src[(size_t)bg * P + out] = (int64_t)q * n_rows_w + (int64_t)row * w + ii;
  }
  for (int i = tid; i < base; i += kCpUnionThreads) {
    pos_c[(size_t)bg * Nc + i] = -1;
    src[(size_t)bg * P + i] = -1;
  }
}

// K and V rows [0, P) of every (b, g) of the compacted sequence, from their source entries (16-byte
// chunks over the whole grid; padding rows zero).
__global__ void cp_rows_kernel(const unsigned char* __restrict__ cands, size_t cand_bytes, size_t off_k, size_t off_v,
                               const int64_t* __restrict__ src, unsigned char* __restrict__ Kc,
                               unsigned char* __restrict__ Vc, int BHkv, int P, int Nc, int64_t n_rows_w,
                               int row_bytes) {
  const int nch = row_bytes / 16;
  const size_t n = (size_t)BHkv * P * nch;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t r = e / nch;
    const int c = (int)(e % nch);
    const size_t bg = r / P, i = r % P, out = bg * Nc + i;
    const int64_t sidx = src[r];
    uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
    if (sidx >= 0) {
      const unsigned char* cb = cands + (size_t)(sidx / n_rows_w) * cand_bytes;
      const size_t ent = (size_t)(sidx % n_rows_w);
      kv = reinterpret_cast<const uint4*>(cb + off_k + ent * row_bytes)[c];
      vv = reinterpret_cast<const uint4*>(cb + off_v + ent * row_bytes)[c];
    }
    reinterpret_cast<uint4*>(Kc + out * row_bytes)[c] = kv;
    reinterpret_cast<uint4*>(Vc + out * row_bytes)[c] = vv;
  }
}

// The shard's own keys behind the prefix stand-in: rows P .. P + len - 1 of Kc, Vc, pos_c and delta_c.
__global__ void cp_own_kernel(const float* __restrict__ delta, const unsigned char* __restrict__ K,
                              const unsigned char* __restrict__ V, float* __restrict__ delta_c,
                              unsigned char* __restrict__ Kc, unsigned char* __restrict__ Vc,
                              int32_t* __restrict__ pos_c, int BH, int BHkv, int len, int P, int Nc, int prefix_len,
                              int row_bytes) {
  const int nch = row_bytes / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t t0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t nrow = (size_t)BHkv * len;
  for (size_t e = t0; e < nrow * nch; e += stride) {
    const size_t r = e / nch;
    const int c = (int)(e % nch);
    const size_t bg = r / len, i = r % len, out = bg * Nc + P + i;
    reinterpret_cast<uint4*>(Kc + out * row_bytes)[c] = reinterpret_cast<const uint4*>(K + r * row_bytes)[c];
    reinterpret_cast<uint4*>(Vc + out * row_bytes)[c] = reinterpret_cast<const uint4*>(V + r * row_bytes)[c];
    if (c == 0) pos_c[out] = prefix_len + (int)i;
  }
  for (size_t e = t0; e < (size_t)BH * len; e += stride) {
    const size_t bh = e / len, i = e % len;
    delta_c[bh * Nc + P + i] = delta[e];
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

// The shard problem: p as given with every position a query (the selection kernels are row-wise).
dma_status_t shard_plan(const dma_params_t* p, Plan* P) {
  if (p == nullptr) return DMA_ERR_INVALID_ARG;
  dma_params_t q = *p;
  q.Nq = q.N;
  dma_status_t st = make_plan(&q, P);
  if (st != DMA_OK) return st;
  if ((size_t)P->G * P->w > (size_t)kCpMaxUnion || P->G > 255) return DMA_ERR_UNSUPPORTED;
  return DMA_OK;
}

}  // namespace
}  // namespace dma

using namespace dma;

extern "C" {

dma_status_t dma_cp_layout(const dma_params_t* p, int32_t prefix_len, int32_t n_prev, dma_cp_layout_t* out) {
  Plan P;
  dma_status_t st = shard_plan(p, &P);
  if (st != DMA_OK) return st;
  if (out == nullptr || prefix_len < 0 || n_prev < 0 || (prefix_len > 0) != (n_prev > 0)) return DMA_ERR_INVALID_ARG;
  if ((int64_t)n_prev * P.w >= (1 << 24)) return DMA_ERR_UNSUPPORTED;
  const CpLayout L = cp_layout_of(P, prefix_len, n_prev);
  out->cand_bytes = L.cand_bytes;
  out->off_pos = L.off_pos;
  out->off_delta = L.off_delta;
  out->off_k = L.off_k;
  out->off_v = L.off_v;
  out->ws_bytes = L.ws_bytes;
  out->off_status = L.off_status;
  out->prefix_rows = L.prefix_rows;
  out->reserved = 0;
  return DMA_OK;
}

dma_status_t dma_cp_candidates(const dma_params_t* p, int32_t shard_start, const float* delta, const void* K,
                               const void* V, void* cand, size_t cand_bytes, void* workspace, size_t workspace_bytes,
                               void* stream) {
  Plan P;
  dma_status_t st = shard_plan(p, &P);
  if (st != DMA_OK) return st;
  if (shard_start < 0 || !ok_ptr(delta) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(cand)) return DMA_ERR_INVALID_ARG;
  const CpLayout L = cp_layout_of(P, 0, 0);
  if (cand_bytes < L.cand_bytes) return DMA_ERR_INVALID_ARG;
  if (!ok_ptr(workspace) || workspace_bytes < L.ws_bytes) return DMA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* sel = ws_ptr<int32_t>(workspace, L.off_sel);
  cudaError_t e = launch_topw_select_rows(delta, P.B * P.H, P.N, P.w, P.w_heads, P.H, sel, nullptr, P.w, s);
  if (e != cudaSuccess) return DMA_ERR_CUDA;
  unsigned char* c = static_cast<unsigned char*>(cand);
  cp_pack_kernel<<<dim3(P.B * P.H, (P.w + kCpThreads - 1) / kCpThreads), kCpThreads, 0, s>>>(sel, delta, (const unsigned char*)K, (const unsigned char*)V,
                                                  reinterpret_cast<int32_t*>(c + L.off_pos),
                                                  reinterpret_cast<float*>(c + L.off_delta), c + L.off_k, c + L.off_v,
                                                  P.H, P.G, P.N, P.w, P.w_heads, shard_start, P.d * L.elt);
  return cudaGetLastError() == cudaSuccess ? DMA_OK : DMA_ERR_CUDA;
}

dma_status_t dma_cp_compact(const dma_params_t* p, int32_t prefix_len, int32_t n_prev, const void* cands,
                            size_t cands_bytes, const float* delta, const void* K, const void* V, float* delta_c,
                            void* Kc, void* Vc, int32_t* pos_c, void* workspace, size_t workspace_bytes,
                            void* stream) {
  Plan P;
  dma_status_t st = shard_plan(p, &P);
  if (st != DMA_OK) return st;
  if (prefix_len < 0 || n_prev < 0 || (prefix_len > 0) != (n_prev > 0)) return DMA_ERR_INVALID_ARG;
  if ((int64_t)n_prev * P.w >= (1 << 24)) return DMA_ERR_UNSUPPORTED;
  const CpLayout L = cp_layout_of(P, prefix_len, n_prev);
  if (!ok_ptr(delta) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(delta_c) || !ok_ptr(Kc) || !ok_ptr(Vc) || !ok_ptr(pos_c))
    return DMA_ERR_INVALID_ARG;
  if (n_prev > 0 && (!ok_ptr(cands) || cands_bytes < (size_t)n_prev * L.cand_bytes)) return DMA_ERR_INVALID_ARG;
  if (!ok_ptr(workspace) || workspace_bytes < L.ws_bytes) return DMA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int Pr = L.prefix_rows, Nc = Pr + P.N, rb = P.d * L.elt;
  const unsigned char* cb = static_cast<const unsigned char*>(cands);
  if (n_prev > 0) {
    float* dm = ws_ptr<float>(workspace, L.off_dm);
    int32_t* sel2 = ws_ptr<int32_t>(workspace, L.off_sel2);
    const size_t n = (size_t)P.B * P.H * n_prev * P.w;
    cp_gather_delta_kernel<<<(unsigned)((n + 255) / 256 < 148 * 8 ? (n + 255) / 256 : 148 * 8), 256, 0, s>>>(
        cb, L.cand_bytes, L.off_delta, dm, P.B * P.H, n_prev, P.w);
    cudaError_t e = launch_topw_select_rows(dm, P.B * P.H, n_prev * P.w, P.w, P.w_heads, P.H, sel2, nullptr, P.w, s);
    if (e != cudaSuccess) return DMA_ERR_CUDA;
    const size_t smem = (size_t)L.cap * (sizeof(uint64_t) + sizeof(int32_t));
    if (ensure_smem_limit(cp_union_kernel, (int)smem) != cudaSuccess) return DMA_ERR_CUDA;
    int64_t* src = ws_ptr<int64_t>(workspace, L.off_src);
    const int64_t n_rows_w = (int64_t)P.B * P.H * P.w;   // entries of one candidate buffer
    cp_union_kernel<<<P.B * P.Hkv, kCpUnionThreads, smem, s>>>(
        cb, L.cand_bytes, L.off_pos, L.off_delta, L.off_k, L.off_v, sel2, delta_c, pos_c, src,
        ws_ptr<int32_t>(workspace, L.off_status), P.H, P.G, n_prev, P.w, P.w_heads, Pr, Nc, L.cap, n_rows_w);
    const size_t work = (size_t)P.B * P.Hkv * Pr * (rb / 16);
    if (work > 0)
      cp_rows_kernel<<<(unsigned)((work + 255) / 256 < 148 * 8 ? (work + 255) / 256 : 148 * 8), 256, 0, s>>>(
          cb, L.cand_bytes, L.off_k, L.off_v, src, (unsigned char*)Kc, (unsigned char*)Vc, P.B * P.Hkv, Pr, Nc,
          n_rows_w, rb);
  }
  const size_t work = (size_t)P.B * P.Hkv * P.N * (rb / 16);
  const unsigned grid = (unsigned)((work + 255) / 256 < 148 * 8 ? (work + 255) / 256 : 148 * 8);
  cp_own_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(delta, (const unsigned char*)K, (const unsigned char*)V, delta_c,
                                                    (unsigned char*)Kc, (unsigned char*)Vc, pos_c, P.B * P.H,
                                                    P.B * P.Hkv, P.N, Pr, Nc, prefix_len, rb);
  return cudaGetLastError() == cudaSuccess ? DMA_OK : DMA_ERR_CUDA;
}

}  // extern "C"
