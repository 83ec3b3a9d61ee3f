// Device helpers shared by the DMA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

#define DMA_DEVINL __device__ __forceinline__

namespace dma {

// ---------------------------------------------------------------- conversions

DMA_DEVINL float bf16_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// round-to-nearest-even float -> bf16 (inputs are finite)
DMA_DEVINL uint16_t f32_to_bf16(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// two floats -> packed bf16x2 (lo in the low half)
DMA_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T> DMA_DEVINL float load_as_f32(const T* p);
template <> DMA_DEVINL float load_as_f32<float>(const float* p) { return *p; }
template <> DMA_DEVINL float load_as_f32<uint16_t>(const uint16_t* p) { return bf16_to_f32(*p); }

template <typename T> DMA_DEVINL void store_from_f32(T* p, float v);
template <> DMA_DEVINL void store_from_f32<float>(float* p, float v) { *p = v; }
template <> DMA_DEVINL void store_from_f32<uint16_t>(uint16_t* p, float v) { *p = f32_to_bf16(v); }

// Order-preserving map of a float to uint32 for the selection order (larger = better).
// -0.0 is mapped like +0.0 so that it ties with it.
DMA_DEVINL uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Window of selection row `row` (= b * H + h): w_heads[h] clamped to [1, w], or w when there are no
// per-head windows.
DMA_DEVINL int row_window(const int32_t* w_heads, int row, int H, int w) {
  if (w_heads == nullptr) return w;
  const int v = __ldg(w_heads + row % H);
  return v < 1 ? 1 : (v > w ? w : v);
}

// ---------------------------------------------------------------- shared-memory access

DMA_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes == 0 zero-fills the destination.
DMA_DEVINL void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
DMA_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> DMA_DEVINL void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

DMA_DEVINL void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
DMA_DEVINL void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
DMA_DEVINL void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

DMA_DEVINL float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk `c` of row `r` in a tile whose rows are `row_chunks` chunks long,
// XOR-swizzled on the low three chunk bits so that eight consecutive rows of one chunk column
// fall in eight different bank groups (conflict-free ldmatrix).
DMA_DEVINL uint32_t swz(int r, int c, int row_chunks) {
  return (uint32_t)((r * row_chunks + (c ^ (r & 7))) * 16);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device) -- the attribute lives
// in the device context -- so that no such call happens while a caller captures a stream into a
// CUDA graph.
cudaError_t ensure_smem_limit_impl(const void* kernel, int bytes);
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel k, int bytes) {
  return ensure_smem_limit_impl(reinterpret_cast<const void*>(k), bytes);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace dma
