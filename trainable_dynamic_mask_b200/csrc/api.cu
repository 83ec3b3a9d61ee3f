// C-ABI entry points of libdma: argument validation, workspace plan, dispatch to launchers.
// Nothing is launched before every argument has been checked.
#include <math.h>
#include <string.h>

#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"
#include "internal.h"

using namespace dma;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

dma_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? DMA_OK : DMA_ERR_CUDA; }

// Validates the workspace for plan P.
dma_status_t check_ws(const Plan& P, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned16(ws)) return DMA_ERR_WORKSPACE;
  if (ws_bytes < P.bytes) return DMA_ERR_WORKSPACE;
  return DMA_OK;
}

}  // namespace

namespace dma {

cudaError_t ensure_smem_limit_impl(const void* kernel, int bytes) {
  // The limit is raised to the device's opt-in maximum (minus the kernel's static shared memory)
  // the first time a kernel is launched on a device, whatever this launch needs.
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  int optin = 0;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
  const int limit = optin - (int)fa.sharedSizeBytes;
  if (bytes > limit) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

// Work units of the attention forward (see FwdSchedule).  The split counts depend only on the
// problem's shape and a fixed reference of 148 SMs, so that the workspace plan and the launch agree.
// A pair's list length is estimated as min(t1, min(w, N) + 128) keys.  The persistent CTAs take the
// units heaviest first as they finish earlier ones, so the kernel ends when the CTA with the most
// tiles does.
// A unit of more than half the average tiles per SM ("big") cannot share a CTA with another big
// one without pushing that CTA past the average: when there are more big units than SMs (e.g. 208
// of ~9 tiles on 148 SMs for 16 heads x 16 pairs), whole groups of big pairs, heaviest first, are
// split in two until the big units fit one per SM.  Each split costs a second pipeline start and a
// merge of partial (O, m, l) by the split that finishes last (a few us), which is why pairs are not
// split further.  When there are fewer pairs than SMs, each pair gets
// min(kMaxSplits, ceil(SMs / pairs), tiles) units.
void fwd_schedule(const Plan& P, FwdSchedule* S) {
  constexpr int kRefSMs = 148;
  const int BH = P.B * P.H;
  const int minwn = P.w < P.N ? P.w : P.N;
  const int kp0 = P.q0 / kPairQ;        // pairs below the first query row have no query (chunked prefill)
  const int np = P.n_pairs - kp0;
  const long items = (long)BH * np;
  const long want = items >= kRefSMs ? 1 : (kRefSMs + items - 1) / items;
  int est[kMaxPairs], split[kMaxPairs], order[kMaxPairs];
  long total = 0;
  for (int kp = kp0; kp < P.n_pairs; ++kp) {
    const int t1 = (kp + 1) * kPairQ < P.N ? (kp + 1) * kPairQ : P.N;
    const int live = t1 < minwn + kBlockQ ? t1 : minwn + kBlockQ;
    est[kp] = (live + kBlockQ - 1) / kBlockQ;
    total += est[kp];
    long sp = want < kMaxSplits ? want : kMaxSplits;
    if (sp > est[kp]) sp = est[kp];
    split[kp] = (int)(sp < 1 ? 1 : sp);
    order[kp - kp0] = kp;
  }
  total *= BH;
  if (want == 1) {
    // big: 2 * est * SMs > total (more than half the average per SM)
    auto is_big = [&](long tiles, long parts) { return 2 * tiles * kRefSMs > total * parts; };
    long big = 0;
    for (int kp = kp0; kp < P.n_pairs; ++kp)
      if (is_big(est[kp], 1)) big += BH;
    while (big > kRefSMs) {
      int pick = -1;
      for (int kp = kp0; kp < P.n_pairs; ++kp)
        if (split[kp] == 1 && est[kp] >= 2 && is_big(est[kp], 1) && (pick < 0 || est[kp] >= est[pick])) pick = kp;
      if (pick < 0) break;
      split[pick] = 2;
      big -= BH;
      if (is_big(est[pick], 2)) big += 2L * BH;
    }
  }
  // heaviest units first: cost est / S, ties to the later pair
  for (int a = 1; a < np; ++a)
    for (int b = a; b > 0; --b) {
      const int x = order[b - 1], y = order[b];
      if ((long)est[y] * split[x] > (long)est[x] * split[y] ||
          ((long)est[y] * split[x] == (long)est[x] * split[y] && y > x)) {
        order[b - 1] = y;
        order[b] = x;
      } else {
        break;
      }
    }
  memset(S, 0, sizeof(*S));
  int start = 0, slot = 0;
  for (int i = 0; i < np; ++i) {
    const int kp = order[i];
    S->g[i].kp = kp;
    S->g[i].S = split[kp];
    S->g[i].start = start;
    S->g[i].slot = split[kp] > 1 ? slot : -1;
    start += BH * split[kp];
    if (split[kp] > 1) slot += BH * split[kp];
  }
  S->n_groups = np;
  S->n_units = start;
  S->n_slots = slot;
}

dma_status_t make_plan(const dma_params_t* p, Plan* P) {
  if (p == nullptr || P == nullptr) return DMA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->Hkv < 1 || p->N < 1 || p->Nq < 1 || p->d < 1 || p->w < 1)
    return DMA_ERR_INVALID_ARG;
  if (p->H % p->Hkv != 0) return DMA_ERR_INVALID_ARG;
  if (p->dtype != DMA_BF16 && p->dtype != DMA_F32) return DMA_ERR_INVALID_ARG;
  if (p->Nq > p->N) return DMA_ERR_INVALID_ARG;
  if (!(p->scale == p->scale) || isinf(p->scale)) return DMA_ERR_INVALID_ARG;
  if (p->w_heads != nullptr && (reinterpret_cast<uintptr_t>(p->w_heads) & 15u) != 0) return DMA_ERR_INVALID_ARG;
  if ((p->flags & ~DMA_FLAG_FORWARD_ONLY) != 0) return DMA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return DMA_ERR_UNSUPPORTED;
  if ((int64_t)p->B * p->H > 65535) return DMA_ERR_UNSUPPORTED;
  Plan& R = *P;
  memset(&R, 0, sizeof(R));
  R.B = p->B; R.H = p->H; R.Hkv = p->Hkv; R.N = p->N; R.Nq = p->Nq; R.d = p->d; R.w = p->w;
  R.w_heads = p->w_heads;
  R.fwd_only = (p->flags & DMA_FLAG_FORWARD_ONLY) != 0;
  R.G = p->H / p->Hkv;
  R.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
  R.bf16 = p->dtype == DMA_BF16;
  R.decode = (p->Nq == 1 && p->N > 1);
  R.q0 = p->N - p->Nq;
  if (!R.decode && p->N > kTopwMaxN) return DMA_ERR_UNSUPPORTED;
  if (R.decode && p->N > (1 << 24)) return DMA_ERR_UNSUPPORTED;

  const size_t BH = (size_t)R.B * R.H;
  const int minwn = R.w < R.N ? R.w : R.N;
  R.n_blocks = (R.N + kBlockQ - 1) / kBlockQ;
  {
    size_t cap = align_up((size_t)minwn + kBlockQ, kBlockQ);
    size_t ncap = align_up((size_t)R.N, kBlockQ);
    R.list_cap = (int)(cap < ncap ? cap : ncap);
    // a pair's live set: the <= w keys live at its first row plus at most kPairQ new keys
    size_t pcap = align_up((size_t)minwn + kPairQ, kBlockQ);
    R.pair_cap = (int)(pcap < ncap ? pcap : ncap);
  }
  R.n_pairs = (R.N + kPairQ - 1) / kPairQ;
  // with per-head windows the selection rows keep the stride w whatever N is, so that an appended
  // key never moves a row (each row holds min(w_h, N) keys)
  R.sel_len = R.w_heads != nullptr ? R.w : minwn;
  R.n_split = (R.sel_len + kDecodeSplit - 1) / kDecodeSplit;
  // decode combines its splits' (m, l) in shared memory, within kDecodeSplit * d * 2 bytes
  if (R.decode && (size_t)R.n_split * 2 * sizeof(float) > (size_t)kDecodeSplit * R.d * 2) return DMA_ERR_UNSUPPORTED;
  R.n_slices = (R.N + kGateSlice - 1) / kGateSlice;

  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  R.off_status = take(256);
  if (!R.decode) {
    R.off_counts = take(BH * R.n_blocks * 2 * sizeof(int32_t));
    R.off_lists = take(BH * R.n_blocks * (size_t)R.list_cap * sizeof(int32_t));
    R.off_pcounts = take(BH * R.n_pairs * 2 * sizeof(int32_t));
    R.off_plists = take(BH * R.n_pairs * (size_t)R.pair_cap * sizeof(int32_t));
    R.off_plen = take(BH * R.n_pairs * (size_t)R.pair_cap * sizeof(int32_t));
    R.off_pdl = take(BH * R.n_pairs * (size_t)R.pair_cap * sizeof(float));
    fwd_schedule(R, &R.sched);
    R.off_fpart = take((size_t)R.sched.n_slots * 2 * R.d * kBlockQ * sizeof(float));
    R.off_fml = take((size_t)R.sched.n_slots * 2 * 2 * kBlockQ * sizeof(float));
    R.off_fcnt = take((BH * R.n_pairs * 4 + 2) * sizeof(int32_t));   // + the forward's unit counters
    R.off_rowD = take(BH * R.Nq * sizeof(float));
    // the forward keeps the low-order bf16 part of O for the backward (training: every position a query)
    if (R.bf16 && R.q0 == 0 && !R.fwd_only) R.off_olo = take(BH * R.n_blocks * (size_t)kBlockQ * R.d * 2);
    {
      const size_t n_slots = BH * ((R.N + 1023) / 1024) * 8;   // windows of 1024 keys, tiles of 128
      R.off_dkv_perm = take(BH * R.N * sizeof(int32_t));
      R.off_dkv_slots = take(n_slots * 4 * sizeof(int32_t));
      R.off_dkv_items = take((n_slots + 1) * sizeof(int32_t));
      R.off_dkv_part = take(2 * BH * R.N * (size_t)R.d * sizeof(float));
    }
    R.off_tw_p = take(BH * R.N * sizeof(int32_t));
    R.off_tw_rank = take(BH * R.N * sizeof(int32_t));
    R.off_tw_T = take(BH * (R.n_blocks + 1) * sizeof(int32_t));
    {
      const size_t L = (size_t)topw_seg_len(R.N);
      R.off_tw_keys = take(BH * ((R.N + L - 1) / L) * L * sizeof(uint64_t));
    }
  } else {
    R.off_sel = take(BH * R.sel_len * sizeof(int32_t));
    R.off_seld = take(BH * R.sel_len * sizeof(float));
    R.off_dec_part = take(BH * R.n_split * (size_t)(R.d + 2) * sizeof(float));
  }
  if (!R.bf16) {
    R.off_q16 = take(BH * R.Nq * R.d * 2);
    R.off_k16 = take((size_t)R.B * R.Hkv * R.N * R.d * 2);
    R.off_v16 = take((size_t)R.B * R.Hkv * R.N * R.d * 2);
    R.off_do16 = take(BH * R.Nq * R.d * 2);
  }
  R.off_gx = take(BH * R.N * sizeof(float));
  R.off_dA_part = take(BH * ((R.N + 1023) / 1024) * sizeof(float));
  R.off_dDelta_part = take((size_t)R.n_slices * R.B * R.Hkv * R.d * R.H * sizeof(float));
  R.bytes = off;
  return DMA_OK;
}

}  // namespace dma

extern "C" {

const char* dma_status_string(dma_status_t s) {
  switch (s) {
    case DMA_OK: return "DMA_OK";
    case DMA_ERR_INVALID_ARG: return "DMA_ERR_INVALID_ARG: invalid argument";
    case DMA_ERR_UNSUPPORTED: return "DMA_ERR_UNSUPPORTED: valid request outside implemented limits";
    case DMA_ERR_WORKSPACE: return "DMA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case DMA_ERR_CUDA: return "DMA_ERR_CUDA: a CUDA launch failed";
    case DMA_ERR_TIMEOUT: return "DMA_ERR_TIMEOUT: a device-side bounded wait gave up";
  }
  return "DMA_ERR_UNKNOWN";
}

int32_t dma_abi_version(void) { return DMA_ABI_VERSION; }

dma_status_t dma_workspace_size(const dma_params_t* p, size_t* bytes) {
  if (bytes == nullptr) return DMA_ERR_INVALID_ARG;
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  *bytes = P.bytes;
  return DMA_OK;
}

dma_status_t dma_workspace_layout(const dma_params_t* p, dma_ws_layout_t* L) {
  if (L == nullptr) return DMA_ERR_INVALID_ARG;
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  memset(L, 0, sizeof(*L));
  L->bytes = P.bytes;
  L->off_status = P.off_status;
  L->off_counts = P.off_counts;
  L->off_lists = P.off_lists;
  L->off_sel = P.off_sel;
  L->n_blocks = P.decode ? 0 : P.n_blocks;
  L->list_cap = P.decode ? 0 : P.list_cap;
  L->sel_len = P.decode ? P.sel_len : 0;
  return DMA_OK;
}

dma_status_t dma_gate(const dma_params_t* p, const void* V, const void* Delta, const float* A,
                      float* delta, float* x_save, void* workspace, size_t workspace_bytes,
                      void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(V) || !ok_ptr(Delta) || !ok_ptr(A) || !ok_ptr(delta)) return DMA_ERR_INVALID_ARG;
  if (x_save != nullptr && !aligned16(x_save)) return DMA_ERR_INVALID_ARG;
  if (P.H > kGateMaxH) return DMA_ERR_UNSUPPORTED;
  return cuda_status(launch_gate_fwd(P, V, Delta, A, delta, x_save, (cudaStream_t)stream));
}

dma_status_t dma_topk_mask(const dma_params_t* p, const float* delta, int32_t* evict,
                           void* workspace, size_t workspace_bytes, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(delta)) return DMA_ERR_INVALID_ARG;
  if (P.decode ? (evict != nullptr) : !ok_ptr(evict)) return DMA_ERR_INVALID_ARG;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (P.decode) return cuda_status(launch_topw_decode(P, delta, workspace, s));
  return cuda_status(launch_topw_prefill(P, delta, evict, workspace, s));
}

dma_status_t dma_topk_append(const dma_params_t* p, const float* delta, void* workspace,
                             size_t workspace_bytes, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!P.decode || !ok_ptr(delta)) return DMA_ERR_INVALID_ARG;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  return cuda_status(launch_topw_append(P, delta, workspace, (cudaStream_t)stream));
}

dma_status_t dma_gate_append(const dma_params_t* p, const void* V, const void* Delta, const float* A,
                             float* delta, float* x_save, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(V) || !ok_ptr(Delta) || !ok_ptr(A) || !ok_ptr(delta) || (x_save != nullptr && !ok_ptr(x_save)))
    return DMA_ERR_INVALID_ARG;
  return cuda_status(launch_gate_append(P, V, Delta, A, delta, x_save, (cudaStream_t)stream));
}

dma_status_t dma_attn_fwd(const dma_params_t* p, const void* Q, const void* K, const void* V,
                          const float* delta, const int32_t* evict, void* workspace,
                          size_t workspace_bytes, void* O, float* LSE, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(delta) || !ok_ptr(O) || !ok_ptr(LSE))
    return DMA_ERR_INVALID_ARG;
  if (P.decode ? (evict != nullptr) : !ok_ptr(evict)) return DMA_ERR_INVALID_ARG;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const uint16_t *q16 = (const uint16_t*)Q, *k16 = (const uint16_t*)K, *v16 = (const uint16_t*)V;
  cudaError_t e = cudaSuccess;
  if (!P.bf16) {
    const size_t nq = (size_t)P.B * P.H * P.Nq * P.d, nk = (size_t)P.B * P.Hkv * P.N * P.d;
    uint16_t* q = ws_ptr<uint16_t>(workspace, P.off_q16);
    uint16_t* k = ws_ptr<uint16_t>(workspace, P.off_k16);
    uint16_t* v = ws_ptr<uint16_t>(workspace, P.off_v16);
    if ((e = launch_convert_f32_to_bf16((const float*)Q, q, nq, s)) != cudaSuccess) return DMA_ERR_CUDA;
    if ((e = launch_convert_f32_to_bf16((const float*)K, k, nk, s)) != cudaSuccess) return DMA_ERR_CUDA;
    if ((e = launch_convert_f32_to_bf16((const float*)V, v, nk, s)) != cudaSuccess) return DMA_ERR_CUDA;
    q16 = q; k16 = k; v16 = v;
  }
  if (P.decode) e = launch_decode_attn(P, q16, k16, v16, delta, workspace, O, LSE, s);
  else e = launch_attn_fwd(P, q16, k16, v16, delta, evict, workspace, O, LSE, s);
  return cuda_status(e);
}

dma_status_t dma_attn_bwd(const dma_params_t* p, const void* Q, const void* K, const void* V,
                          const float* delta, const int32_t* evict, void* workspace,
                          size_t workspace_bytes, const void* O, const float* LSE,
                          const void* dO, void* dQ, void* dK, void* dV, float* d_delta,
                          void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (P.decode || P.q0 != 0 || P.fwd_only) return DMA_ERR_UNSUPPORTED;   // training: every position a query
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(delta) || !ok_ptr(evict) || !ok_ptr(O) ||
      !ok_ptr(LSE) || !ok_ptr(dO) || !ok_ptr(dQ) || !ok_ptr(dK) || !ok_ptr(dV) || !ok_ptr(d_delta))
    return DMA_ERR_INVALID_ARG;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const uint16_t *q16 = (const uint16_t*)Q, *k16 = (const uint16_t*)K, *v16 = (const uint16_t*)V,
                 *do16 = (const uint16_t*)dO;
  if (!P.bf16) {
    const size_t nq = (size_t)P.B * P.H * P.Nq * P.d, nk = (size_t)P.B * P.Hkv * P.N * P.d;
    uint16_t* q = ws_ptr<uint16_t>(workspace, P.off_q16);
    uint16_t* k = ws_ptr<uint16_t>(workspace, P.off_k16);
    uint16_t* v = ws_ptr<uint16_t>(workspace, P.off_v16);
    uint16_t* g = ws_ptr<uint16_t>(workspace, P.off_do16);
    if (launch_convert_f32_to_bf16((const float*)Q, q, nq, s) != cudaSuccess) return DMA_ERR_CUDA;
    if (launch_convert_f32_to_bf16((const float*)K, k, nk, s) != cudaSuccess) return DMA_ERR_CUDA;
    if (launch_convert_f32_to_bf16((const float*)V, v, nk, s) != cudaSuccess) return DMA_ERR_CUDA;
    if (launch_convert_f32_to_bf16((const float*)dO, g, nq, s) != cudaSuccess) return DMA_ERR_CUDA;
    q16 = q; k16 = k; v16 = v; do16 = g;
  }
  return cuda_status(launch_attn_bwd(P, q16, k16, v16, delta, evict, workspace, O, LSE, do16, dQ,
                                     dK, dV, d_delta, s));
}

dma_status_t dma_gate_bwd(const dma_params_t* p, const void* V, const void* Delta,
                          const float* A, const float* x_save, const float* delta,
                          const float* d_delta, float* dDelta, float* dA, float* dV_gate,
                          void* workspace, size_t workspace_bytes, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(V) || !ok_ptr(Delta) || !ok_ptr(A) || !ok_ptr(x_save) || !ok_ptr(delta) ||
      !ok_ptr(d_delta) || !ok_ptr(dDelta) || !ok_ptr(dA) || !ok_ptr(dV_gate))
    return DMA_ERR_INVALID_ARG;
  if (P.H > kGateMaxH) return DMA_ERR_UNSUPPORTED;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  return cuda_status(launch_gate_bwd(P, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate,
                                     workspace, (cudaStream_t)stream));
}

dma_status_t dma_check_device_status(const dma_params_t* p, void* workspace, void* stream,
                                     int32_t* code) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (workspace == nullptr || code == nullptr) return DMA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws_ptr<int32_t>(workspace, P.off_status), sizeof(v),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DMA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DMA_ERR_CUDA;
  *code = v;
  return v == 0 ? DMA_OK : DMA_ERR_TIMEOUT;
}

dma_status_t dma_selftest_bounded_wait(const dma_params_t* p, void* workspace, size_t workspace_bytes,
                                       int64_t limit_cycles, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (limit_cycles < 1 || limit_cycles > ((int64_t)1 << 34)) return DMA_ERR_INVALID_ARG;
  if ((st = check_ws(P, workspace, workspace_bytes)) != DMA_OK) return st;
  return cuda_status(launch_selftest_wait(P, workspace, (long long)limit_cycles, (cudaStream_t)stream));
}

dma_status_t dma_clear_device_status(const dma_params_t* p, void* workspace, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (workspace == nullptr) return DMA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws_ptr<int32_t>(workspace, P.off_status), 0, sizeof(int32_t),
                                     (cudaStream_t)stream));
}

}  // extern "C"
