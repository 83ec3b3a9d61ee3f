// Shared building blocks of the tcgen05 attention kernels: TMA gathers, tcgen05.mma with
// in-asm descriptor offsets, bounded warp-uniform waits, setmaxnreg, packed f32x2 arithmetic and a
// polynomial exp2.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace dma {

DMA_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}\n" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Raises the barrier's expected transaction bytes without arriving (the arrival comes later).
DMA_DEVINL void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
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

// The box of a 2-D tensor map whose first element is (x = column, y = row), written to `dst` (the
// map's swizzle applies); completion is counted in bytes on `bar`.  Rows past the tensor read 0.
DMA_DEVINL void tma_tile_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Warp-uniform bounded wait (every lane of the warp calls it).
DMA_DEVINL bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status, int code) {
  return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, abort_flag, status, code));
}

// Wait that ignores the abort flag, for draining copies in flight after an abort (bounded).
DMA_DEVINL void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!tc::mbar_try_wait_sleep(bar, parity, 20000u) && clock64() - t0 < 200000000LL) {
  }
}

template <int R> DMA_DEVINL void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R)); }
template <int R> DMA_DEVINL void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R)); }

// ---- packed f32x2 arithmetic (two lanes of FP32 work per instruction on sm_100)
DMA_DEVINL uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
DMA_DEVINL void f2_split(uint64_t v, float& lo, float& hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v)); }
DMA_DEVINL uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
DMA_DEVINL uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
DMA_DEVINL uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
DMA_DEVINL uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
DMA_DEVINL float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of x <= ~8 on the FMA pipe: x = i + f with i = round(x), f in [-1/2, 1/2];
// 2^f ~ 1 + f (c1 + f (c2 + f c3)), a cubic fitted here for minimum relative error on [-1/2, 1/2]
// (max 1.02e-4, far below bf16's half ulp 2^-9, the precision P is stored in); i is added to the
// exponent field.  x is clamped at -127, where f = 0, p = 1 exactly and the exponent sum wraps to
// +0: masked entries (x = -inf) give exactly 0, as the MUFU path does.  Round-to-nearest uses the
// 1.5 * 2^23 shift: the integer lands in the low mantissa bits of x + 1.5 * 2^23.
DMA_DEVINL void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  constexpr float kShift = 12582912.0f;   // 1.5 * 2^23
  constexpr float c1 = 0.6932829022407532f, c2 = 0.24221068620681763f, c3 = 0.05500871315598488f;
  x0 = fmaxf(x0, -127.f);
  x1 = fmaxf(x1, -127.f);
  const uint64_t x = f2(x0, x1);
  const uint64_t r = f2_add(x, f2(kShift, kShift));
  const uint64_t f = f2_sub(x, f2_sub(r, f2(kShift, kShift)));
  uint64_t p = f2_fma(f, f2(c3, c3), f2(c2, c2));
  p = f2_fma(f, p, f2(c1, c1));
  p = f2_fma(f, p, f2(1.f, 1.f));
  float r0, r1, q0, q1;
  f2_split(r, r0, r1);
  f2_split(p, q0, q1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(r0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(r1) << 23));
}

// tcgen05.mma (kind::f16, A and B from shared memory) with both descriptors advanced by OFF / 16
// inside the asm block: the 8 K steps then need no live descriptor registers each.
template <uint32_t OFF>
DMA_DEVINL void mma_ss_at(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "add.s64 a, %1, %5;\n\t"
      "add.s64 b, %2, %5;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(OFF >> 4));
}
// tcgen05.mma with A = P from TMEM column a_tmem + 8 KK and B = V at descriptor + KK * 2048 / 16.
template <int KK>
DMA_DEVINL void mma_ts_at(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "add.s64 b, %2, %5;\n\t"
      "add.u32 a, %1, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(KK * 2048 / 16), "n"(KK * 8));
}


// 32 consecutive outputs of a row (16-byte stores).
DMA_DEVINL void store_row32(uint16_t* dst, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 32; u += 8) {
    uint4 w;
    w.x = pack_bf16x2(v[u], v[u + 1]);
    w.y = pack_bf16x2(v[u + 2], v[u + 3]);
    w.z = pack_bf16x2(v[u + 4], v[u + 5]);
    w.w = pack_bf16x2(v[u + 6], v[u + 7]);
    *reinterpret_cast<uint4*>(dst + u) = w;
  }
}
// The low-order parts v - bf16(v) of 32 outputs, as bf16: with the row stored by store_row32,
// hi + lo carries v to about 16 significant bits.  Blocked layout: the 8-column group k of row r of
// a 128-row block sits at dst_k + r * 8 (dst_k = the group's [128][8] slice), so that the 32 lanes
// of a warp, 32 consecutive rows, store 512 contiguous bytes per instruction.
DMA_DEVINL void store_row32_lo(uint16_t* group0, int r, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 32; u += 8) {
    float q[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) q[k] = v[u + k] - bf16_to_f32(f32_to_bf16(v[u + k]));
    uint4 w;
    w.x = pack_bf16x2(q[0], q[1]);
    w.y = pack_bf16x2(q[2], q[3]);
    w.z = pack_bf16x2(q[4], q[5]);
    w.w = pack_bf16x2(q[6], q[7]);
    *reinterpret_cast<uint4*>(group0 + (size_t)(u / 8) * 128 * 8 + (size_t)r * 8) = w;
  }
}
DMA_DEVINL void store_row32(float* dst, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 32; u += 4) *reinterpret_cast<float4*>(dst + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
}
}  // namespace dma
