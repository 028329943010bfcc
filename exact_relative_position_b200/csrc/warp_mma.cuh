// warp_mma.cuh -- warp-level tensor-core helpers (mma.sync m16n8k16 for
// 16-bit inputs), ldmatrix and cp.async staging with a
// 128-byte XOR swizzle for [rows x 64] 16-bit tiles.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace relpos {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-byte chunk c (0..7) of row r in a [rows x 64] 16-bit tile
// whose 128-byte rows are XOR-swizzled by (r & 7), so that ldmatrix of 8
// consecutive rows at one chunk touches 8 distinct bank groups.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
// 4-byte copy (any 4-byte aligned address); src_bytes = 0 writes zeros
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Stage rows [r0, r0 + ROWS) of a [*, 64] 16-bit matrix (row pitch `pitch`
// elements) into a swizzled tile; rows >= nrows are zero-filled.
template <int ROWS, int NTHREADS, typename T>
__device__ __forceinline__ void load_tile_async(uint32_t sbase, const T* g, int r0, int nrows, int tid,
                                                int pitch = 64) {
#pragma unroll
  for (int it = 0; it < ROWS * 8 / NTHREADS; ++it) {
    const int idx = it * NTHREADS + tid;
    const int r = idx >> 3, c = idx & 7;
    const int gr = r0 + r;
    const bool ok = gr < nrows;
    const T* src = g + (size_t)(ok ? gr : 0) * pitch + c * 8;
    cp_async16(sbase + swz(r, c), src, ok ? 16 : 0);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <typename T> struct MmaOp;
template <> struct MmaOp<__half> {
  static __device__ __forceinline__ void run(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};
template <> struct MmaOp<__nv_bfloat16> {
  static __device__ __forceinline__ void run(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};

// A fragments (16 rows x 64 cols, 4 k16 steps) of a swizzled [rows x 64] tile.
__device__ __forceinline__ void load_a_frags(uint32_t sbase, int row0, int lane, uint32_t (&a)[4][4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = row0 + (lane & 15);
    const int c = kk * 2 + (lane >> 4);
    ldsm_x4(sbase + swz(r, c), a[kk][0], a[kk][1], a[kk][2], a[kk][3]);
  }
}

// C[16 x 8*NT] += A[16 x 64] * B^T where B is a swizzled [8*NT rows x 64]
// tile (rows = output columns, contiguous along the contraction).
template <typename T, int NT>
__device__ __forceinline__ void mma_abt(float (&c)[NT][4], const uint32_t (&a)[4][4], uint32_t sb, int n0, int lane) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t b0, b1, b2, b3;
      const int r = n0 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int ch = kk * 2 + ((lane >> 3) & 1);
      ldsm_x4(sb + swz(r, ch), b0, b1, b2, b3);
      MmaOp<T>::run(c[2 * np], a[kk], b0, b1);
      MmaOp<T>::run(c[2 * np + 1], a[kk], b2, b3);
    }
  }
}

// C[16 x 64] += P[16 x 16*KS] * B where B is a swizzled [16*KS rows x 64]
// tile (rows = contraction index, contiguous along the output columns);
// p holds the A fragments of P per k16 step.
template <typename T, int KS>
__device__ __forceinline__ void mma_ab(float (&c)[8][4], const uint32_t (&p)[KS][4], uint32_t sb, int k0, int lane) {
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
    for (int dp = 0; dp < 4; ++dp) {
      uint32_t b0, b1, b2, b3;
      const int r = k0 + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int ch = dp * 2 + (lane >> 4);
      ldsm_x4_t(sb + swz(r, ch), b0, b1, b2, b3);
      MmaOp<T>::run(c[2 * dp], p[kk], b0, b1);
      MmaOp<T>::run(c[2 * dp + 1], p[kk], b2, b3);
    }
  }
}

}  // namespace relpos
