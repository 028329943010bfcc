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

// band_terms_q for the Q-parallel pass with the q.aQ term read as aligned
// float4 vectors where it can: a 32-column chunk whose offsets, for every row
// of the warp, lie inside the row's stored columns (warp-uniform test) needs
// Z^Q[i, A + c] for 32 consecutive c, so the lane loads the aligned 16-byte
// pieces covering them (eight columns at a time: three pieces) and picks its
// values with the row's alignment shift s = (A + c) mod 4 (three selects), a
// third of the load requests of one gather per score.  Other chunks gather one
// by one (clamped).  zq_row as band_terms_q; its row storage starts on 16
// bytes (group stride and base are multiples of 8 floats) and extends to
// eq1 rounded up to 4 floats.
template <bool AK, bool BIAS, int NC>
__device__ __forceinline__ void band_terms_q_vec(float* x, int E_lo, int E_hi, int i, int lane, int j0, int coff,
                                                 const float* zq_row, int eq0, int eq1, const float* zk_tile, int zS,
                                                 int kmax, int ek0, int ek1, const float* bexp, float sc) {
  const int A = j0 + coff - i - E_lo;   // offset column of key j0 + coff for this row (before clamping)
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 32) {
    // warp-uniform: every lane's 32 offsets inside [E_lo, E_hi] and the stored columns
    const bool lane_in = A + c0 >= 0 && A + c0 + 31 <= E_hi - E_lo && A + c0 >= eq0 && A + c0 + 31 <= eq1;
    if (__all_sync(0xffffffffu, lane_in)) {
      const float* base = zq_row + (A + c0);
      const float4* vb = reinterpret_cast<const float4*>(reinterpret_cast<uintptr_t>(base) & ~uintptr_t(15));
      const int s = (int)((reinterpret_cast<uintptr_t>(base) >> 2) & 3);
      const bool s1 = (s & 1) != 0, s2 = (s & 2) != 0;
#pragma unroll
      for (int c8 = 0; c8 < 32; c8 += 8) {
        // the third piece of the last eight columns holds needed values only when
        // s > 0 (else it would start past them, possibly past the row's storage)
        const float4 a = __ldg(vb + c8 / 4), b = __ldg(vb + c8 / 4 + 1);
        const float4 d = (c8 < 24 || s != 0) ? __ldg(vb + c8 / 4 + 2) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float w[12] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w, d.x, d.y, d.z, d.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float zq = s2 ? (s1 ? w[u + 3] : w[u + 2]) : (s1 ? w[u + 1] : w[u]);
          const int c = c0 + c8 + u;
          const int e = A + c;   // inside [E_lo, E_hi] - E_lo here
          float rel = zq;
          if (AK) rel += __ldg(zk_tile + (long long)imin(coff + c, kmax) * zS + iclamp(e, ek0, ek1));
          if (BIAS) rel += __ldg(bexp + e);
          x[c] = (x[c] + rel) * sc;
        }
      }
    } else {
#pragma unroll
      for (int c = c0; c < c0 + 32; ++c) {
        const int e = iclamp(j0 + coff + c - i, E_lo, E_hi) - E_lo;
        float rel = __ldg(zq_row + iclamp(e, eq0, eq1));
        if (AK) rel += __ldg(zk_tile + (long long)imin(coff + c, kmax) * zS + iclamp(e, ek0, ek1));
        if (BIAS) rel += __ldg(bexp + e);
        x[c] = (x[c] + rel) * sc;
      }
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

// band_terms_k for the K-parallel pass with the k.aK term read as aligned
// float4 vectors where it can, as band_terms_q_vec: here the offsets fall with
// the column (e = A - c), so an interior chunk needs Z^K[j, A - c0 - 31 ..
// A - c0], and column c0 + c8 + u of an eight-column group is entry s + 7 - u of
// its three pieces.
template <bool AQ, bool BIAS, int NC>
__device__ __forceinline__ void band_terms_k_vec(float* x, int E_lo, int E_hi, int j, int qb, int coff,
                                                 const float* zk_row, int ek0, int ek1, const float* zq_tile, int zS,
                                                 int qmax, int eq0, int eq1, const float* bexp, float sc) {
  const int A = j - qb - coff - E_lo;   // offset column of query qb + coff for this key (before clamping)
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 32) {
    const bool lane_in = A - c0 - 31 >= 0 && A - c0 <= E_hi - E_lo && A - c0 - 31 >= ek0 && A - c0 <= ek1;
    if (__all_sync(0xffffffffu, lane_in)) {
      const float* base = zk_row + (A - c0 - 31);
      const float4* vb = reinterpret_cast<const float4*>(reinterpret_cast<uintptr_t>(base) & ~uintptr_t(15));
      const int s = (int)((reinterpret_cast<uintptr_t>(base) >> 2) & 3);
      const bool s1 = (s & 1) != 0, s2 = (s & 2) != 0;
#pragma unroll
      for (int c8 = 0; c8 < 32; c8 += 8) {
        // pieces 6 - c8/4 .. 8 - c8/4; the top one of the first group holds needed
        // values only when s > 0 (else it would start past them)
        const float4* pv = vb + (6 - c8 / 4);
        const float4 a = __ldg(pv), b = __ldg(pv + 1);
        const float4 d = (c8 > 0 || s != 0) ? __ldg(pv + 2) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float w[12] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w, d.x, d.y, d.z, d.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float zk = s2 ? (s1 ? w[10 - u] : w[9 - u]) : (s1 ? w[8 - u] : w[7 - u]);
          const int c = c0 + c8 + u;
          const int e = A - c;   // inside [E_lo, E_hi] - E_lo here
          float rel = zk;
          if (AQ) rel += __ldg(zq_tile + (long long)imin(coff + c, qmax) * zS + iclamp(e, eq0, eq1));
          if (BIAS) rel += __ldg(bexp + e);
          x[c] = (x[c] + rel) * sc;
        }
      }
    } else {
#pragma unroll
      for (int c = c0; c < c0 + 32; ++c) {
        const int e = iclamp(j - qb - coff - c, E_lo, E_hi) - E_lo;
        float rel = __ldg(zk_row + iclamp(e, ek0, ek1));
        if (AQ) rel += __ldg(zq_tile + (long long)imin(coff + c, qmax) * zS + iclamp(e, eq0, eq1));
        if (BIAS) rel += __ldg(bexp + e);
        x[c] = (x[c] + rel) * sc;
      }
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
