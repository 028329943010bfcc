// band.cuh -- per-score relation terms of BAND tiles and the by-offset
// relation-gradient stores of the backward passes (digest of "Fast and Exact
// Relative-Position Attention via Structure-Aware Kernels": Eq. (2) and
// Eq. (4); "constant tiles and the saturated region").
//
// A BAND tile straddles the diagonal band of interior offsets, so its scores
// need one scalar per cell: Z^Q[i, e], Z^K[j, e] and b[e] with
// e = clamp(j - i, E_lo, E_hi) - E_lo.
//
// The gathers are branch-free: every index is clamped into the stored
// columns (and rows) of its projection group, so a masked cell reads a
// harmless in-bounds value that the caller's mask overwrites, and the code
// stays small enough for the instruction cache.
#pragma once

#include "common.cuh"

namespace relpos {

// Bytes of one warp's staging area: the 16-bit dS rows of the by-offset
// store (32 rows x 64 columns, kDsPitch elements per row).
constexpr int kDsPitch = 72;
constexpr uint32_t kStageWarpBytes = 32u * kDsPitch * 2u;

// Row = query i (forward, Q-parallel backward).  x[c] (c < NC) holds the raw
// score of key j0 + coff + c and becomes (score + relation terms) * sc.
//   zq_row: Z^Q row of i, indexable by expanded column in [eq0, eq1]
//   zk_tile: Z^K of the key tile's key t at zk_tile[t * zS + e], e in [ek0, ek1], t <= kmax
template <bool AQ, bool AK, bool BIAS, int NC>
__device__ __forceinline__ void band_terms_q(float* x, int E_lo, int E_hi, int i, int j0, int coff,
                                             const float* zq_row, int eq0, int eq1, const float* zk_tile, int zS,
                                             int kmax, int ek0, int ek1, const float* bexp, float sc) {
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 32) {
#pragma unroll
    for (int c = c0; c < c0 + 32; ++c) {
      const int e = iclamp(j0 + coff + c - i, E_lo, E_hi) - E_lo;
      float rel = 0.f;
      if (AQ) rel += __ldg(zq_row + iclamp(e, eq0, eq1));
      if (AK) rel += __ldg(zk_tile + (long long)imin(coff + c, kmax) * zS + iclamp(e, ek0, ek1));
      if (BIAS) rel += __ldg(bexp + e);
      x[c] = (x[c] + rel) * sc;
    }
    asm volatile("" ::: "memory");
  }
}

// Row = key j (K-parallel backward).  x[c] holds the raw score of query qb + coff + c.
template <bool AQ, bool AK, bool BIAS, int NC>
__device__ __forceinline__ void band_terms_k(float* x, int E_lo, int E_hi, int j, int qb, int coff,
                                             const float* zk_row, int ek0, int ek1, const float* zq_tile, int zS,
                                             int qmax, int eq0, int eq1, const float* bexp, float sc) {
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 32) {
#pragma unroll
    for (int c = c0; c < c0 + 32; ++c) {
      const int e = iclamp(j - qb - coff - c, E_lo, E_hi) - E_lo;
      float rel = 0.f;
      if (AQ) rel += __ldg(zq_tile + (long long)imin(coff + c, qmax) * zS + iclamp(e, eq0, eq1));
      if (AK) rel += __ldg(zk_row + iclamp(e, ek0, ek1));
      if (BIAS) rel += __ldg(bexp + e);
      x[c] = (x[c] + rel) * sc;
    }
    asm volatile("" ::: "memory");
  }
}

// Interior relation-gradient entries of one BAND tile, stored by offset from
// the warp's 16-bit dS rows (rows = this side's positions, 64 columns = the
// other side's) as those 16-bit values (the consumers apply tau).  Warp-cooperative and coalesced: the warp walks its 32 rows
// and its lanes cover the columns, whose offsets are consecutive.  Interior
// offsets E_lo < d < E_hi have exactly one cell per (row, offset), so every
// entry has one writer; the two saturated offsets are summed by the caller.
//   key_rows = false: row = query i = row0 + rbase + rr, column = key j = col0 + cbeg + c, d = j - i
//   key_rows = true:  row = key j = row0 + rbase + rr, column = query i = col0 + cbeg + c, d = j - i
//   dz_base + (rbase + rr) * S + (d - E_lo - e0) is the entry of (row, d)
template <typename T>
__device__ __forceinline__ void dz_band_store(const T* stage16, int rbase, int lane, bool key_rows, int row0, int col0,
                                              int cbeg, int nrows, int nkv, int N, int causal, int E_lo, int E_hi,
                                              T* dz_base, long long S, int e0) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int c = lane + 32 * q;
    const int col = col0 + cbeg + c;
    // the warp's 32 rows x this 32-column chunk: when every cell is kept and
    // interior (warp-uniform), the entries of a lane form a line of slope
    // S -+ 1 through dZ, walked with one pointer step per row
    const int r0 = row0 + rbase, c0 = col0 + cbeg + 32 * q;
    const int dmin = key_rows ? r0 - (c0 + 31) : c0 - (r0 + 31);
    const int dmax = key_rows ? r0 + 31 - c0 : c0 + 31 - r0;
    const int imx = key_rows ? c0 + 31 : r0 + 31, jmx = key_rows ? r0 + 31 : c0 + 31;
    if (rbase + 31 < nrows && dmin > E_lo && dmax < E_hi && imx < N && jmx < nkv && !(causal && dmax > 0)) {
      T* ptr = dz_base + (long long)rbase * S + (key_rows ? r0 - col : col - r0) - E_lo - e0;
      const long long step = key_rows ? S + 1 : S - 1;
#pragma unroll 8
      for (int rr = 0; rr < 32; ++rr) {
        *ptr = stage16[rr * kDsPitch + c];
        ptr += step;
      }
      continue;
    }
#pragma unroll 4
    for (int rr = 0; rr < 32; ++rr) {
      const int row = rbase + rr;
      if (row >= nrows) break;
      T* dz_row = dz_base + (long long)row * S - e0 - E_lo;
      const int i = key_rows ? col : row0 + row;
      const int j = key_rows ? row0 + row : col;
      const int d = j - i;
      const bool kept = i < N && j < nkv && !(causal && j > i) && d > E_lo && d < E_hi;
      if (kept) dz_row[d] = stage16[rr * kDsPitch + c];
    }
  }
}

}  // namespace relpos
