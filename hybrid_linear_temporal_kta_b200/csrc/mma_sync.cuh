// mma_sync.cuh -- warp-level bf16 tensor-core tiles (m16n8k16, fp32 accumulate), ldmatrix and
// cp.async wrappers for the chunked linear-attention kernels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace kta {

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p)))
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p)))
               : "memory");
}

// Two 8x8 matrices (one n8 B tile, both k halves), transposed; lanes 0-15 give row addresses.
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p)))
               : "memory");
}

// c += a * b for one m16n8k16 bf16 tile.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte async global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Lane address helpers for 16x16 bf16 fragments of a row-major smem matrix with row stride ld
// (elements). "rows" is the fragment's first row, "cols" its first column.
//  A operand, stored [m][k]:                     ldsm_x4   at a_rowmajor
//  B operand pair (two n8 tiles), stored [n][k]: ldsm_x4   at b_nmajor   -> {b0,b1} n0, {b2,b3} n1
//  B operand pair, stored [k][n]:                ldsm_x4_t at b_kmajor   -> {b0,b1} n0, {b2,b3} n1
//  A operand, stored [k][m]:                     ldsm_x4_t at a_kmajor
__device__ __forceinline__ int frag_a_rowmajor(int lane, int row0, int col0, int ld) {
  return (row0 + (lane & 15)) * ld + col0 + (lane >> 4) * 8;
}
__device__ __forceinline__ int frag_b_nmajor(int lane, int n0, int k0, int ld) {
  return (n0 + (lane & 7) + (lane >> 4) * 8) * ld + k0 + ((lane >> 3) & 1) * 8;
}
__device__ __forceinline__ int frag_b_kmajor(int lane, int k0, int n0, int ld) {
  return (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0 + (lane >> 4) * 8;
}
__device__ __forceinline__ int frag_a_kmajor(int lane, int m0, int k0, int ld) {
  const int mat = lane >> 3;
  return (k0 + (lane & 7) + (mat >> 1) * 8) * ld + m0 + (mat & 1) * 8;
}

}  // namespace kta
