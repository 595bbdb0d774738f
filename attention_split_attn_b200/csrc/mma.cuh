// mma.cuh -- warp-level tensor-core tiles for the GQA kernels (decode and
// selected-key): mma.sync m16n8k16 with f32 accumulation, ldmatrix from
// 128-byte-swizzled shared-memory tiles written by TMA (SWIZZLE_128B).
//
// Tile layout in shared memory: a [32 cells][D] tile of 16-bit values is
// stored as D/64 sub-tiles of [32 rows][128 bytes]; within a row the 16-byte
// chunk c sits at position c ^ (row & 7) (the TMA 128-byte swizzle, with each
// sub-tile 1024-byte aligned), so eight rows read at one chunk index hit
// eight different bank groups.
#pragma once

#include "common.cuh"

namespace attn {

template <typename KT> struct MmaType;
template <> struct MmaType<__nv_bfloat16> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  // two floats -> packed pair, round to nearest even (lo in the low half)
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  }
};
template <> struct MmaType<__half> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                        uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                              uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// Byte offset of 16-byte chunk `chunk` (0 .. D/8-1) of row `row` in a
// swizzled [ROWS][D] tile of 16-bit values (D/64 sub-tiles of ROWS x 128 B).
template <int ROWS = 32>
__device__ __forceinline__ uint32_t swz_offset(int row, int chunk) {
  const int sub = chunk >> 3, c = chunk & 7;
  return (uint32_t)(sub * (ROWS * 128) + row * 128 + ((c ^ (row & 7)) << 4));
}

// Transpose an 8x8 matrix of 16-bit values held one row-pair per lane (the
// m16n8k16 accumulator/operand fragment layout) across the warp.
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

}  // namespace attn
