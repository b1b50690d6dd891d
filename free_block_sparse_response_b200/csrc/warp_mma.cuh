// Warp-level bf16 tensor-core primitives (mma.sync m16n8k16), ldmatrix and cp.async.
//
// Fragment layouts (lane = 4*g + t, g = lane/4, t = lane%4):
//   A 16x16 row-major : a0 (row g,   k 2t..2t+1)  a1 (row g+8, k 2t..2t+1)
//                       a2 (row g,   k 2t+8..+9)  a3 (row g+8, k 2t+8..+9)
//   B 16x8  (k x n)   : b0 (k 2t..2t+1, col g)    b1 (k 2t+8..+9, col g)
//   C 16x8  fp32      : c0,c1 (row g, cols 2t,2t+1)  c2,c3 (row g+8, cols 2t,2t+1)
//
// Shared-memory tiles hold rows of D bf16 values (D/8 chunks of 16 bytes); chunk c of
// row r lives at chunk slot c ^ (r & 7), so the 8 rows an ldmatrix phase touches hit 8
// different bank groups.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace spr {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// 16-byte async copy global->shared; src_bytes < 16 zero-fills the rest (0 = all zero).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Split x into bf16 hi + bf16 lo (x ~= hi + lo to ~16 significant bits) for a pair.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  float2 hf = __bfloat1622float2(h);
  __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a swizzled tile of D bf16 columns.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

}  // namespace spr
