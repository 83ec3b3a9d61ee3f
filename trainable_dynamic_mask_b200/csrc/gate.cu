// Gate kernels: delta = exp(A * softplus(v Delta)) and its backward.
//
// Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Dynamic Sparse Mask
// Generation", delta equation ("Dynamic Weight Computation"); Delta and A are learnable, and the
// method is trainable end to end (section "Gradient Flow Integrity").
//
// x[b,h,j] = sum_r v_j[r] Delta[r,h] with v_j the concatenation of the Hkv value heads at key
// position j (r = g*d + c).  The contraction is narrow (H = 2..32 columns), so it runs on the FMA
// pipe with float32 accumulation: bf16 products are exact in float32, and float32 inputs keep
// their full precision.  Each CTA stages a 64-position tile of one value head, transposed to
// [channel][position], plus the matching Delta rows, and each thread accumulates a 4x4
// (position x head) register tile.
#include "common.cuh"

namespace dma {
namespace {

constexpr int kGatePT = 64;  // positions per CTA (backward kernels)

// 8 consecutive elements (16-byte aligned) widened to float.
DMA_DEVINL void load8_as_f32(const uint16_t* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
DMA_DEVINL void load8_as_f32(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

DMA_DEVINL float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }
DMA_DEVINL float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// CTA = 32 key positions of one batch row, 256 threads = 8 reduction groups x 32 threads.  The
// reduction dimension r = g*d + c is processed in chunks of kGateR; inside a chunk group k takes
// r = k, k+8, ...  Each thread holds a 4-position x HPT-head register tile (thread = 8 position
// groups x 4 head groups); the 8 partial tiles are summed through shared memory at the end.
constexpr int kGateP = 32;      // positions per CTA
constexpr int kGateR = 256;     // reduction rows staged per chunk
constexpr int kGateThreads = 256;

template <typename T, int HPT>
__global__ void __launch_bounds__(kGateThreads)
gate_fwd_kernel(const T* __restrict__ V, const T* __restrict__ Delta, const float* __restrict__ A,
                float* __restrict__ delta, float* __restrict__ x_save, int H, int Hkv, int N, int d) {
  constexpr int HP = 4 * HPT;                       // padded head count
  extern __shared__ __align__(16) float sm[];
  float* Vt = sm;                                   // [kGateR][kGateP]   V transposed
  float* Ds = Vt + kGateR * kGateP;                 // [kGateR][HP]
  float* red = Ds + kGateR * HP;                    // [8][kGateP][HP]
  const int b = blockIdx.y, p0 = blockIdx.x * kGateP;
  const int tid = threadIdx.x, kg = tid >> 5, lane = tid & 31;
  const int pg = lane & 7, hg = lane >> 3;
  const int R = Hkv * d;
  float acc[4][HPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < HPT; ++j) acc[i][j] = 0.f;

  for (int r0 = 0; r0 < R; r0 += kGateR) {
    const int rn = min(kGateR, R - r0);
    __syncthreads();
    // stage V rows r = g*d + c in [r0, r0 + rn), positions p0..p0+31: lanes run over positions,
    // each loading 8 consecutive channels, so the transposed stores are conflict-free.  All loads
    // of a thread are issued before any store so that their latencies overlap.
    constexpr int kVLoads = kGateP * (kGateR / 8) / kGateThreads;   // 4
    float v8[kVLoads][8];
#pragma unroll
    for (int u = 0; u < kVLoads; ++u) {
      const int e = tid + u * kGateThreads;
      const int p = e % kGateP, o = e / kGateP;
      const int r = r0 + o * 8, g = r / d, c = r % d;
      const int pos = p0 + p;
      if (o * 8 < rn && pos < N) load8_as_f32(V + ((size_t)(b * Hkv + g) * N + pos) * d + c, v8[u]);
      else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[u][i] = 0.f;
      }
    }
    constexpr int kDLoads = kGateR * HP / kGateThreads;   // HP
    float dl[kDLoads];
#pragma unroll
    for (int u = 0; u < kDLoads; ++u) {
      const int e = tid + u * kGateThreads;
      const int rr = e / HP, h = e % HP;
      dl[u] = (rr < rn && h < H) ? load_as_f32(Delta + (size_t)(r0 + rr) * H + h) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kVLoads; ++u) {
      const int e = tid + u * kGateThreads;
      const int p = e % kGateP, o = e / kGateP;
#pragma unroll
      for (int i = 0; i < 8; ++i) Vt[(o * 8 + i) * kGateP + p] = v8[u][i];
    }
#pragma unroll
    for (int u = 0; u < kDLoads; ++u) Ds[tid + u * kGateThreads] = dl[u];
    __syncthreads();
    for (int rr = kg; rr < rn; rr += 8) {
      const float4 v4 = *reinterpret_cast<const float4*>(Vt + rr * kGateP + pg * 4);
      const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
      float dd[HPT];
      if constexpr (HPT % 4 == 0) {
#pragma unroll
        for (int j = 0; j < HPT; j += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(Ds + rr * HP + hg * HPT + j);
          dd[j] = d4.x; dd[j + 1] = d4.y; dd[j + 2] = d4.z; dd[j + 3] = d4.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < HPT; ++j) dd[j] = Ds[rr * HP + hg * HPT + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < HPT; ++j) acc[i][j] = fmaf(vv[i], dd[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < HPT; ++j) red[(kg * kGateP + pg * 4 + i) * HP + hg * HPT + j] = acc[i][j];
  __syncthreads();
  for (int o = tid; o < kGateP * HP; o += kGateThreads) {
    const int p = o / HP, h = o % HP;
    const int pos = p0 + p;
    if (h >= H || pos >= N) continue;
    float x = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) x += red[(k * kGateP + p) * HP + h];
    const size_t off = (size_t)(b * H + h) * N + pos;
    delta[off] = expf(A[h] * softplus_f(x));
    if (x_save) x_save[off] = x;
  }
}

__global__ void convert_f32_bf16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst,
                                        size_t n) {
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t n4 = n / 4;
  for (size_t k = i; k < n4; k += stride) {
    float4 v = reinterpret_cast<const float4*>(src)[k];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(dst)[k] = o;
  }
  for (size_t k = n4 * 4 + i; k < n; k += stride) dst[k] = f32_to_bf16(src[k]);
}

// ---------------------------------------------------------------- backward

// gx = d_delta * delta * A * sigmoid(x); partial sums of d_delta * delta * softplus(x) for dA.
__global__ void gate_bwd_pointwise_kernel(const float* __restrict__ x, const float* __restrict__ delta,
                                          const float* __restrict__ dd, const float* __restrict__ A,
                                          float* __restrict__ gx, float* __restrict__ dA_part,
                                          int H, int N) {
  __shared__ float red[32];
  const int row = blockIdx.y;   // b*H + h
  const int h = row % H;
  const float a = A[h];
  const size_t base = (size_t)row * N;
  float part = 0.f;
  for (int k = 0; k < 4; ++k) {
    const int j = blockIdx.x * 1024 + k * 256 + threadIdx.x;
    if (j < N) {
      const float xv = x[base + j], dv = delta[base + j], g = dd[base + j];
      gx[base + j] = g * dv * a * sigmoid_f(xv);
      part += g * dv * softplus_f(xv);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) dA_part[(size_t)row * gridDim.x + blockIdx.x] = v;
  }
}

// dV_gate[b,g,j,c] = sum_h gx[b,h,j] * Delta[g*d+c, h]
// dV_gate[b, g, j, c] = sum_h gx[b, h, j] Delta[g d + c, h]: per (64 positions, g, b) a
// [64 x H] x [H x d] product in float32.  Thread = PP = d / 32 positions x 8 channels (register
// tile), reading gx as [h][64 positions] and Delta as [h][d] from shared memory with 16-byte loads;
// a warp stores 512 contiguous bytes per position.
template <typename T, int D>
__global__ void __launch_bounds__(256)
gate_bwd_dv_kernel(const float* __restrict__ gx, const T* __restrict__ Delta, float* __restrict__ dVg, int H,
                   int Hkv, int N) {
  constexpr int CG = D / 8, PP = kGatePT * CG / 256;   // channel groups; positions per thread
  extern __shared__ __align__(16) float sm[];
  float* Gs = sm;                    // [H][kGatePT]
  float* Ds = sm + H * kGatePT;      // [H][D]
  const int j0 = blockIdx.x * kGatePT, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, cg = tid % CG, pg = tid / CG;
  for (int e = tid; e < H * kGatePT; e += 256) {
    const int h = e / kGatePT, p = e % kGatePT;
    Gs[e] = (j0 + p < N) ? gx[(size_t)(b * H + h) * N + j0 + p] : 0.f;
  }
  for (int e = tid; e < D * H; e += 256) {
    const int c = e / H, h = e % H;   // coalesced over the row-major Delta
    Ds[h * D + c] = load_as_f32(Delta + (size_t)(g * D + c) * H + h);
  }
  __syncthreads();
  float acc[PP][8];
#pragma unroll
  for (int p = 0; p < PP; ++p)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[p][c] = 0.f;
  for (int h = 0; h < H; ++h) {
    const float4 d0 = *reinterpret_cast<const float4*>(Ds + h * D + cg * 8);
    const float4 d1 = *reinterpret_cast<const float4*>(Ds + h * D + cg * 8 + 4);
    const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    float gg[PP];
#pragma unroll
    for (int p = 0; p < PP; ++p) gg[p] = Gs[h * kGatePT + pg * PP + p];
#pragma unroll
    for (int p = 0; p < PP; ++p)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[p][c] = fmaf(gg[p], dd[c], acc[p][c]);
  }
#pragma unroll
  for (int p = 0; p < PP; ++p) {
    const int j = j0 + pg * PP + p;
    if (j >= N) continue;
    float* o = dVg + ((size_t)(b * Hkv + g) * N + j) * D + cg * 8;
    *reinterpret_cast<float4*>(o) = make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
    *reinterpret_cast<float4*>(o + 4) = make_float4(acc[p][4], acc[p][5], acc[p][6], acc[p][7]);
  }
}

// partial[(s*B + b)][g*d + c][h] = sum_{j in slice s} V[b,g,j,c] * gx[b,h,j].  Thread = 8 channels x
// 4 heads (register tile); the NT = (d / 8) x ceil(H / 4) tiles are repeated 256 / NT times over
// disjoint positions of each 64-position chunk and summed through shared memory at the end.
template <typename T, int D>
__global__ void __launch_bounds__(256)
gate_bwd_ddelta_partial_kernel(const T* __restrict__ V, const float* __restrict__ gx, float* __restrict__ part,
                               int B, int H, int Hkv, int N) {
  constexpr int CG = D / 8;
  extern __shared__ __align__(16) float sm[];
  const int HG = (H + 3) / 4, HP = HG * 4, NT = CG * HG, NQ = 256 / NT;
  float* Vs = sm;                    // [64][D]
  float* Gs = sm + 64 * D;           // [64][HP]
  float* red = Gs + 64 * HP;         // [NQ][NT][32]
  const int s = blockIdx.x, b = blockIdx.y, g = blockIdx.z;
  const int tid = threadIdx.x;
  const int q = tid / NT, t = tid % NT, cg = t % CG, hg = t / CG;
  float acc[8][4];
#pragma unroll
  for (int c = 0; c < 8; ++c)
#pragma unroll
    for (int h = 0; h < 4; ++h) acc[c][h] = 0.f;
  const T* Vg = V + (size_t)(b * Hkv + g) * N * D;
  const int jend = min(N, (s + 1) * kGateSlice);
  for (int j0 = s * kGateSlice; j0 < jend; j0 += 64) {
    __syncthreads();
    for (int e = tid; e < 64 * D; e += 256) {
      const int p = e / D, c = e % D;
      Vs[e] = (j0 + p < N) ? load_as_f32(Vg + (size_t)(j0 + p) * D + c) : 0.f;
    }
    for (int e = tid; e < HP * 64; e += 256) {
      const int h = e / 64, p = e % 64;
      Gs[p * HP + h] = (h < H && j0 + p < N) ? gx[(size_t)(b * H + h) * N + j0 + p] : 0.f;
    }
    __syncthreads();
    if (q < NQ) {
      for (int p = q; p < 64; p += NQ) {
        const float4 v0 = *reinterpret_cast<const float4*>(Vs + p * D + cg * 8);
        const float4 v1 = *reinterpret_cast<const float4*>(Vs + p * D + cg * 8 + 4);
        const float4 g4 = *reinterpret_cast<const float4*>(Gs + p * HP + hg * 4);
        const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int h = 0; h < 4; ++h) acc[c][h] = fmaf(vv[c], gg[h], acc[c][h]);
      }
    }
  }
  __syncthreads();
  if (q < NQ) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
      for (int h = 0; h < 4; ++h) red[((size_t)q * NT + t) * 32 + c * 4 + h] = acc[c][h];
  }
  __syncthreads();
  for (int e = tid; e < NT * 32; e += 256) {
    const int tt = e / 32, ch = e % 32, c = ch / 4, h = ch % 4;
    float v = 0.f;
    for (int qq = 0; qq < NQ; ++qq) v += red[((size_t)qq * NT + tt) * 32 + ch];
    const int cc = (tt % CG) * 8 + c, hh = (tt / CG) * 4 + h;
    if (hh < H) part[((size_t)(s * B + b) * Hkv * D + (size_t)g * D + cc) * H + hh] = v;
  }
}

__global__ void gate_bwd_reduce_kernel(const float* __restrict__ part, const float* __restrict__ dA_part,
                                       float* __restrict__ dDelta, float* __restrict__ dA, int nparts,
                                       int RH, int H, int B, int nchunk) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < RH) {
    float acc = 0.f;
    for (int k = 0; k < nparts; ++k) acc += part[(size_t)k * RH + i];
    dDelta[i] = acc;
  }
  if (i < H) {
    float acc = 0.f;
    for (int b = 0; b < B; ++b)
      for (int k = 0; k < nchunk; ++k) acc += dA_part[((size_t)b * H + i) * nchunk + k];
    dA[i] = acc;
  }
}

// bf16 values: x = v_cat Delta as a [positions x Hkv*d] x [Hkv*d x H] product on the tensor cores
// (mma.sync m16n8k16, float32 accumulation; bf16 products are exact in float32).  CTA = 16 key
// positions of one batch row, 8 warps splitting the reduction in 16-wide steps (step s to warp
// s % 8); the 8 partial [16 x H] tiles are summed through shared memory.  The V rows of the 16
// positions (all Hkv heads: 16 rows of Hkv*d) and Delta (zero-padded to HT*8 columns) are staged
// with coalesced 16-byte async copies, all issued before one wait; A fragments come from a
// 16-byte-chunk XOR swizzle (conflict-free ldmatrix), B fragments from ldmatrix.trans of the
// row-major Delta.
constexpr int kGmP = 16;
constexpr int kGmThreads = 256;

template <int HT>   // Delta column tiles of 8 (H <= 8 * HT), HT even
__global__ void __launch_bounds__(kGmThreads)
gate_fwd_mma_kernel(const uint16_t* __restrict__ V, const uint16_t* __restrict__ Delta, const float* __restrict__ A,
                    float* __restrict__ delta, float* __restrict__ x_save, int H, int Hkv, int N, int d) {
  extern __shared__ __align__(128) unsigned char gsm[];
  const int K = Hkv * d, KC = K / 8;                        // reduction length, its 16-byte chunks
  uint16_t* Vs = reinterpret_cast<uint16_t*>(gsm);          // [16][K], chunk c of row p at c ^ (p & 7)
  uint16_t* Ds = Vs + kGmP * K;                             // [K][8 HT]
  float* red = reinterpret_cast<float*>(Ds + (size_t)K * 8 * HT);   // [8 warps][16][8 HT]
  const int b = blockIdx.y, p0 = blockIdx.x * kGmP;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dch = d / 8;
  // ---- stage V (16 positions x K) and Delta (K x H, padded to 8 HT columns): every 16-byte
  // copy of both is issued before the first wait (one memory round trip)
  for (int q = tid; q < kGmP * KC; q += kGmThreads) {
    const int p = q / KC, kc = q % KC;
    const int g = kc / dch, c = kc % dch;
    const int pos = p0 + p;
    const bool in = pos < N;
    const uint16_t* src = in ? V + ((size_t)(b * Hkv + g) * N + pos) * d + c * 8 : V;
    cp_async_16(smem_u32(Vs + (size_t)p * K + ((kc ^ (p & 7)) * 8)), src, in ? 16 : 0);
  }
  if ((H & 7) == 0) {
    const int hc = H / 8;
    for (int q = tid; q < K * HT; q += kGmThreads) {
      const int r = q / HT, c = q % HT;
      const bool in = c < hc;
      cp_async_16(smem_u32(Ds + (size_t)r * 8 * HT + c * 8), in ? Delta + (size_t)r * H + c * 8 : Delta, in ? 16 : 0);
    }
  } else {
    for (int q = tid; q < K * 8 * HT; q += kGmThreads) {
      const int r = q / (8 * HT), h = q % (8 * HT);
      Ds[q] = h < H ? Delta[(size_t)r * H + h] : (uint16_t)0;
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  // ---- partial products over this warp's reduction steps
  float acc[HT][4];
#pragma unroll
  for (int n = 0; n < HT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
  const uint32_t vs_base = smem_u32(Vs), ds_base = smem_u32(Ds);
  const int arow = lane & 15, achunk = lane >> 4;               // ldmatrix.x4 address of this lane
  const int brow = (lane & 7) + ((lane >> 3) & 1) * 8, btile = lane >> 4;
  for (int ks = warp; ks < K / 16; ks += 8) {
    uint32_t a[4];
    const int kc = ks * 2 + achunk;
    ldmatrix_x4(vs_base + (uint32_t)(arow * K + ((kc ^ (arow & 7)) * 8)) * 2, a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n = 0; n < HT; n += 2) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(ds_base + (uint32_t)((ks * 16 + brow) * 8 * HT + (n + btile) * 8) * 2, b0, b1, b2, b3);
      mma_bf16_16816(acc[n], a, b0, b1);
      mma_bf16_16816(acc[n + 1], a, b2, b3);
    }
  }
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < HT; ++n) {
    float* rw = red + (size_t)warp * kGmP * 8 * HT;
    rw[g * 8 * HT + n * 8 + 2 * t] = acc[n][0];
    rw[g * 8 * HT + n * 8 + 2 * t + 1] = acc[n][1];
    rw[(g + 8) * 8 * HT + n * 8 + 2 * t] = acc[n][2];
    rw[(g + 8) * 8 * HT + n * 8 + 2 * t + 1] = acc[n][3];
  }
  __syncthreads();
  for (int o = tid; o < kGmP * H; o += kGmThreads) {
    const int p = o / H, h = o % H;
    const int pos = p0 + p;
    if (pos >= N) continue;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) x += red[((size_t)w * kGmP + p) * 8 * HT + h];
    const size_t off = (size_t)(b * H + h) * N + pos;
    delta[off] = expf(A[h] * softplus_f(x));
    if (x_save) x_save[off] = x;
  }
}

template <int HT>
cudaError_t launch_gate_fwd_mma(const Plan& P, const void* V, const void* Delta, const float* A, float* delta,
                                float* x_save, cudaStream_t s) {
  const int K = P.Hkv * P.d;
  const size_t smem = (size_t)kGmP * K * 2 + (size_t)K * 8 * HT * 2 + (size_t)8 * kGmP * 8 * HT * 4;
  auto k = gate_fwd_mma_kernel<HT>;
  { cudaError_t ea = ensure_smem_limit(k, (int)smem); if (ea != cudaSuccess) return ea; }
  dim3 grid((P.N + kGmP - 1) / kGmP, P.B);
  k<<<grid, kGmThreads, smem, s>>>((const uint16_t*)V, (const uint16_t*)Delta, A, delta, x_save, P.H, P.Hkv, P.N,
                                   P.d);
  return cudaGetLastError();
}

// Shared memory of the tensor-core gate for problem P (0 when it does not apply).
size_t gate_mma_smem(const Plan& P) {
  if (!P.bf16 || P.H > 64) return 0;
  const int HT = P.H <= 16 ? 2 : P.H <= 32 ? 4 : 8;
  const size_t K = (size_t)P.Hkv * P.d;
  const size_t smem = kGmP * K * 2 + K * 8 * HT * 2 + (size_t)8 * kGmP * 8 * HT * 4;
  return smem <= 200 * 1024 ? smem : 0;
}

template <typename T, int HPT>
cudaError_t launch_gate_fwd_t(const Plan& P, const void* V, const void* Delta, const float* A, float* delta,
                              float* x_save, cudaStream_t s) {
  constexpr int HP = 4 * HPT;
  const int smem = (kGateR * kGateP + kGateR * HP + 8 * kGateP * HP) * (int)sizeof(float);
  auto k = gate_fwd_kernel<T, HPT>;
  { cudaError_t ea = ensure_smem_limit(k, smem); if (ea != cudaSuccess) return ea; }
  dim3 grid((P.N + kGateP - 1) / kGateP, P.B);
  k<<<grid, kGateThreads, smem, s>>>((const T*)V, (const T*)Delta, A, delta, x_save, P.H, P.Hkv, P.N, P.d);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gate_fwd_h(const Plan& P, const void* V, const void* Delta, const float* A, float* delta,
                              float* x_save, cudaStream_t s) {
  if (P.H <= 4) return launch_gate_fwd_t<T, 1>(P, V, Delta, A, delta, x_save, s);
  if (P.H <= 8) return launch_gate_fwd_t<T, 2>(P, V, Delta, A, delta, x_save, s);
  if (P.H <= 16) return launch_gate_fwd_t<T, 4>(P, V, Delta, A, delta, x_save, s);
  if (P.H <= 32) return launch_gate_fwd_t<T, 8>(P, V, Delta, A, delta, x_save, s);
  if (P.H <= 64) return launch_gate_fwd_t<T, 16>(P, V, Delta, A, delta, x_save, s);
  return cudaErrorInvalidValue;
}

}  // namespace

// ---------------------------------------------------------------- gate of the last position
// One warp per (b, h): x = sum_{g,c} V[b, g, N-1, c] Delta[g*d + c, h] in float32, then
// delta = exp(A_h softplus(x)), at position N - 1 only.
template <typename T>
__global__ void gate_append_kernel(const T* __restrict__ V, const T* __restrict__ Delta, const float* __restrict__ A,
                                   float* __restrict__ delta, float* __restrict__ x_save, int BH, int H, int Hkv,
                                   int N, int d) {
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (gw >= BH) return;
  const int b = gw / H, h = gw % H;
  float acc = 0.f;
  for (int r = lane; r < Hkv * d; r += 32) {
    const int g = r / d, c = r % d;
    acc = fmaf(load_as_f32(V + ((size_t)(b * Hkv + g) * N + (N - 1)) * d + c), load_as_f32(Delta + (size_t)r * H + h),
               acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const size_t off = (size_t)gw * N + (N - 1);
    delta[off] = expf(A[h] * softplus_f(acc));
    if (x_save) x_save[off] = acc;
  }
}

cudaError_t launch_gate_append(const Plan& P, const void* V, const void* Delta, const float* A, float* delta,
                               float* x_save, cudaStream_t s) {
  const int BH = P.B * P.H;
  const unsigned blocks = (unsigned)((BH * 32 + 255) / 256);
  if (P.bf16)
    gate_append_kernel<uint16_t><<<blocks, 256, 0, s>>>((const uint16_t*)V, (const uint16_t*)Delta, A, delta, x_save,
                                                        BH, P.H, P.Hkv, P.N, P.d);
  else
    gate_append_kernel<float><<<blocks, 256, 0, s>>>((const float*)V, (const float*)Delta, A, delta, x_save, BH, P.H,
                                                     P.Hkv, P.N, P.d);
  return cudaGetLastError();
}

cudaError_t launch_gate_fwd(const Plan& P, const void* V, const void* Delta, const float* A,
                            float* delta, float* x_save, cudaStream_t s) {
  if (gate_mma_smem(P) > 0) {
    if (P.H <= 16) return launch_gate_fwd_mma<2>(P, V, Delta, A, delta, x_save, s);
    if (P.H <= 32) return launch_gate_fwd_mma<4>(P, V, Delta, A, delta, x_save, s);
    return launch_gate_fwd_mma<8>(P, V, Delta, A, delta, x_save, s);
  }
  return P.bf16 ? launch_gate_fwd_h<uint16_t>(P, V, Delta, A, delta, x_save, s)
                : launch_gate_fwd_h<float>(P, V, Delta, A, delta, x_save, s);
}

cudaError_t launch_convert_f32_to_bf16(const float* src, uint16_t* dst, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n / 4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks == 0) blocks = 1;
  convert_f32_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, dst, n);
  return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const Plan& P, const void* V, const void* Delta, const float* A,
                            const float* x_save, const float* delta, const float* d_delta,
                            float* dDelta, float* dA, float* dV_gate, void* ws, cudaStream_t s) {
  if ((P.d / 8) * ((P.H + 3) / 4) > 256) return cudaErrorInvalidValue;   // one register tile per thread
  float* gx = ws_ptr<float>(ws, P.off_gx);
  float* dA_part = ws_ptr<float>(ws, P.off_dA_part);
  float* part = ws_ptr<float>(ws, P.off_dDelta_part);
  const int nchunk = (P.N + 1023) / 1024;
  gate_bwd_pointwise_kernel<<<dim3(nchunk, P.B * P.H), 256, 0, s>>>(x_save, delta, d_delta, A, gx,
                                                                     dA_part, P.H, P.N);
  const size_t smem_dv = (size_t)(P.H * kGatePT + P.d * P.H) * sizeof(float);
  const int HP = (P.H + 3) / 4 * 4, NT = (P.d / 8) * (HP / 4);
  const size_t smem_dd = (size_t)(64 * P.d + 64 * HP + (256 / NT) * NT * 32) * sizeof(float);
  dim3 gdv((P.N + kGatePT - 1) / kGatePT, P.Hkv, P.B);
  dim3 gdd(P.n_slices, P.B, P.Hkv);
  auto launch = [&](auto kdv, auto kdd, const auto* Vp, const auto* Dp) -> cudaError_t {
    { cudaError_t ea = ensure_smem_limit(kdv, (int)smem_dv); if (ea != cudaSuccess) return ea; }
    kdv<<<gdv, 256, smem_dv, s>>>(gx, Dp, dV_gate, P.H, P.Hkv, P.N);
    { cudaError_t ea = ensure_smem_limit(kdd, (int)smem_dd); if (ea != cudaSuccess) return ea; }
    kdd<<<gdd, 256, smem_dd, s>>>(Vp, gx, part, P.B, P.H, P.Hkv, P.N);
    return cudaSuccess;
  };
  cudaError_t e;
  if (P.bf16) {
    const uint16_t* Vp = (const uint16_t*)V;
    const uint16_t* Dp = (const uint16_t*)Delta;
    e = P.d == 128 ? launch(gate_bwd_dv_kernel<uint16_t, 128>, gate_bwd_ddelta_partial_kernel<uint16_t, 128>, Vp, Dp)
                   : launch(gate_bwd_dv_kernel<uint16_t, 64>, gate_bwd_ddelta_partial_kernel<uint16_t, 64>, Vp, Dp);
  } else {
    const float* Vp = (const float*)V;
    const float* Dp = (const float*)Delta;
    e = P.d == 128 ? launch(gate_bwd_dv_kernel<float, 128>, gate_bwd_ddelta_partial_kernel<float, 128>, Vp, Dp)
                   : launch(gate_bwd_dv_kernel<float, 64>, gate_bwd_ddelta_partial_kernel<float, 64>, Vp, Dp);
  }
  if (e != cudaSuccess) return e;
  const int RH = P.Hkv * P.d * P.H;
  gate_bwd_reduce_kernel<<<(RH + 255) / 256, 256, 0, s>>>(part, dA_part, dDelta, dA,
                                                          P.n_slices * P.B, RH, P.H, P.B, nchunk);
  return cudaGetLastError();
}

}  // namespace dma
