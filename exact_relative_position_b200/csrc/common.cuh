// common.cuh -- shared definitions of the relative-position attention library:
// offset maps, the expanded (bucket -> truncated) form, projection group
// geometry and the tile plan.  Host and device use the same functions, so the
// planner and the kernels agree by construction.
//
// Source: digest page of "Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels" -- Eq. (1)-(3), sections "grouped reachable range"
// and "constant tiles and the saturated region".
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "../../include/relpos_attn.h"

#define RP_HD __host__ __device__ __forceinline__

namespace relpos {

constexpr int kTile = RELPOS_TILE;   // tile edge and projection group size (128)
constexpr int kHeadDim = 64;
constexpr double kGuard = 1e-9;      // exact integer crossings of the log formulas round as in exact arithmetic

RP_HD int imin(int a, int b) { return a < b ? a : b; }
RP_HD int imax(int a, int b) { return a > b ? a : b; }
RP_HD int iclamp(int x, int lo, int hi) { return imin(imax(x, lo), hi); }
// Row stride of a projection group: a multiple of 8 elements, so that rows of
// the fp32 projection and of the 16-bit relation gradient both start on 16 bytes.
RP_HD int round_up8(int x) { return (x + 7) & ~7; }

// ---------------------------------------------------------------------------
// Offset maps phi(delta), delta = j - i.
// ---------------------------------------------------------------------------

// T5 buckets: half of the buckets per direction when bidirectional; within a
// half of size h, magnitudes below h/2 are exact and larger ones fall into
// h/2 + floor(ln(n/(h/2)) / ln(max_distance/(h/2)) * (h/2)) capped at h-1.
RP_HD int phi_t5(int delta, int num_buckets, int max_distance, int bidirectional) {
  int h = num_buckets, base = 0, n;
  if (bidirectional) {
    h = num_buckets / 2;
    base = delta > 0 ? h : 0;
    n = delta < 0 ? -delta : delta;
  } else {
    n = delta < 0 ? -delta : 0;
  }
  const int exact = h / 2;
  if (n < exact) return base + n;
  const double x = log((double)n / (double)exact) / log((double)max_distance / (double)exact) *
                   (double)(h - exact);
  const int large = exact + (int)floor(x + kGuard);
  return base + imin(large, h - 1);
}

// DeBERTa log buckets: |delta| <= mid = num_buckets/2 keeps the offset, beyond
// it sign * (mid + ceil(ln(n/mid) / ln((max_distance-1)/mid) * (mid-1)));
// the row is that position + num_buckets clamped to [0, 2 num_buckets).
RP_HD int phi_log(int delta, int num_buckets, int max_distance) {
  const int mid = num_buckets / 2;
  const int n = delta < 0 ? -delta : delta;
  int pos = delta;
  if (n > mid) {
    const double x = log((double)n / (double)mid) / log((double)(max_distance - 1) / (double)mid) *
                     (double)(mid - 1);
    const int lp = mid + (int)ceil(x - kGuard);
    pos = delta < 0 ? -lp : lp;
  }
  return iclamp(pos + num_buckets, 0, 2 * num_buckets - 1);
}

RP_HD int phi_of(const relpos_map_desc& m, int N, int delta) {
  switch (m.kind) {
    case RELPOS_MAP_TRUNCATED: return iclamp(delta, -m.clip, m.clip) + m.clip;
    case RELPOS_MAP_IDENTITY: return delta + N - 1;
    case RELPOS_MAP_BUCKET_T5: return phi_t5(delta, m.num_buckets, m.max_distance, m.bidirectional);
    case RELPOS_MAP_BUCKET_LOG_REVERSED: return phi_log(-delta, m.num_buckets, m.max_distance);
    default: return phi_log(delta, m.num_buckets, m.max_distance);
  }
}

// ---------------------------------------------------------------------------
// Plan passed by value to every kernel.
// ---------------------------------------------------------------------------

// Projection geometry of one 128-row group: its rows store the expanded
// columns [e0, e0 + W) with a row stride of S floats, starting `base` floats
// into the (batch, head) slice.
struct GroupInfo {
  int e0, W, S, pad;
  long long base;
};

struct Plan {
  int B, H, N;
  int E_lo, E_hi, Rexp;     // expanded offset range [E_lo, E_hi]; expanded row e = clamp(delta) - E_lo
  int nT;                   // number of 128-row tiles / groups
  int grouped;              // 1: per-group reachable columns; 0: every row stores all Rexp columns
  int causal, padding;
  float tau;
  long long zq_head, zk_head;   // floats per (batch, head) of Z^Q / Z^K (0 when absent)
  const GroupInfo* gq;          // device [nT]
  const GroupInfo* gk;          // device [nT]
  const int* key_len;           // device [B] or null
  // attention dropout (0 = off): keep a cell when its 8-bit Philox uniform is >= drop_thresh
  int dropout;
  uint32_t drop_thresh, seed_lo, seed_hi, drop_offset;
  float drop_scale;             // 1 / (1 - drop_thresh / 256)
  // limit of every bounded mbarrier wait in the fused kernels (ns); the host
  // lowers it only to exercise the timeout path
  unsigned long long wait_ns;
  // packed variable-length batch (0: the dense [B, H, N, 64] layout): sequence
  // b owns token rows cu[b] .. cu[b + 1] - 1 of token-major [T, H, 64] tensors
  // and of the LSE [H, T]; N is the longest sequence.  The workspace keeps
  // its dense per-(batch, head) layout of N rows.
  int packed, T;
  const int* cu;
  // query-tile order of the forward and Q-parallel grids: tile |qrev - blockIdx.x|
  // (0 in ascending order; under a causal mask the last tile index, so that the
  // longest rows go first)
  int qrev, qrev_pair;
};

// First token row and length of sequence b.  Packed offsets are clamped so
// that every row a kernel stores stays inside [0, T) and every length inside
// [0, N], whatever the offsets hold; the dense layout has length N.
struct SeqRows {
  int row0, len;
};
RP_HD SeqRows seq_rows(const Plan& p, int b) {
  SeqRows s;
  if (!p.packed) {
    s.row0 = 0;
    s.len = p.N;
    return s;
  }
  s.row0 = iclamp(p.cu[b], 0, p.T);
  s.len = iclamp(p.cu[b + 1] - s.row0, 0, imin(p.N, p.T - s.row0));
  return s;
}
// Row i of (b, h) of q / k / v / o / dout / dq / dk / dv, in units of 64-element rows.
RP_HD long long act_row(const Plan& p, const SeqRows& s, int b, int h, int i) {
  return p.packed ? (long long)(s.row0 + i) * p.H + h : ((long long)b * p.H + h) * p.N + i;
}
// Entry of row i of (b, h) in the LSE ([B, H, N] dense, [H, T] packed).
RP_HD long long lse_index(const Plan& p, const SeqRows& s, int b, int h, int i) {
  return p.packed ? (long long)h * p.T + s.row0 + i : ((long long)b * p.H + h) * p.N + i;
}
// Elements between consecutive rows of one (b, h).
RP_HD int act_pitch(const Plan& p) { return p.packed ? p.H * 64 : 64; }
// Coordinates (c1, c2) of row `row` of (b, h) for a TMA map made by
// make_rows_map: dense maps are {64, N, B H}, packed maps {64, H, T}.
RP_HD void tma_rows(const Plan& p, const SeqRows& s, int bh, int h, int row, int& c1, int& c2) {
  if (p.packed) { c1 = h; c2 = s.row0 + row; }
  else { c1 = row; c2 = bh; }
}

// Reachable expanded columns of query group g (key_side = 0) or key group g
// (key_side = 1): a query i reaches delta in [-i, N-1-i], a key j reaches
// [j-(N-1), j]; causal keeps delta <= 0.
RP_HD void group_columns(const Plan& p, int key_side, int g, int* e0, int* W) {
  if (!p.grouped) { *e0 = 0; *W = p.Rexp; return; }
  const int r0 = g * kTile, n = imin(kTile, p.N - r0);
  int lo, hi;
  if (!key_side) { lo = -(r0 + n - 1); hi = p.N - 1 - r0; }
  else { lo = r0 - (p.N - 1); hi = r0 + n - 1; }
  if (p.causal) hi = imin(hi, 0);
  lo = imax(lo, p.E_lo);
  hi = imin(hi, p.E_hi);
  if (hi < lo) hi = lo;
  *e0 = lo - p.E_lo;
  *W = hi - lo + 1;
}

// Fills GroupInfo for group g (prefix sum over the preceding groups).
RP_HD GroupInfo group_info(const Plan& p, int key_side, int g) {
  GroupInfo gi;
  long long base = 0;
  for (int t = 0; t < g; ++t) {
    int e0, W;
    group_columns(p, key_side, t, &e0, &W);
    base += (long long)imin(kTile, p.N - t * kTile) * round_up8(W);
  }
  group_columns(p, key_side, g, &gi.e0, &gi.W);
  gi.S = round_up8(gi.W);
  gi.pad = 0;
  gi.base = base;
  return gi;
}

RP_HD long long head_elems(const Plan& p, int key_side) {
  if (p.nT == 0) return 0;
  GroupInfo last = group_info(p, key_side, p.nT - 1);
  return last.base + (long long)imin(kTile, p.N - (p.nT - 1) * kTile) * last.S;
}

// ---------------------------------------------------------------------------
// Tile plan: the two comparisons of a tile's offset range with (E_lo, E_hi).
// ---------------------------------------------------------------------------
// Class of the cells with queries [i0, i1] and keys [j0, j1] (both ranges
// inside [0, N)): the same two comparisons as for a whole tile.
RP_HD int block_class(int i0, int i1, int j0, int j1, int nkv, int causal, int E_lo, int E_hi) {
  if (j0 >= nkv || (causal && j0 > i1)) return RELPOS_TILE_MASKED;
  const int j1v = imin(j1, nkv - 1);
  if (j1v - i0 <= E_lo) return RELPOS_TILE_CONST_LO;
  if (j0 - i1 >= E_hi) return RELPOS_TILE_CONST_HI;
  return RELPOS_TILE_BAND;
}

RP_HD int tile_class(int qi, int kj, int N, int nkv, int causal, int E_lo, int E_hi) {
  const int i0 = qi * kTile, i1 = imin(i0 + kTile, N) - 1;
  const int j0 = kj * kTile, j1 = imin(j0 + kTile, N) - 1;
  return block_class(i0, i1, j0, j1, nkv, causal, E_lo, E_hi);
}

// Class of the 64-column half h of tile (qi, kj) as the backward's compute
// warps see it: the half's columns are keys (key_cols) or queries; a half
// whose cells are all masked counts as CONST_LO (its values are masked to 0).
RP_HD int half_class(int qi, int kj, int h, bool key_cols, int N, int nkv, int causal, int E_lo, int E_hi) {
  int i0 = qi * kTile, i1 = imin(i0 + kTile, N) - 1;
  int j0 = kj * kTile, j1 = imin(j0 + kTile, N) - 1;
  if (key_cols) {
    j0 += 64 * h;
    j1 = imin(j1, j0 + 63);
    if (j0 > j1) return RELPOS_TILE_CONST_LO;
  } else {
    i0 += 64 * h;
    i1 = imin(i1, i0 + 63);
    if (i0 > i1) return RELPOS_TILE_CONST_LO;
  }
  const int c = block_class(i0, i1, j0, j1, nkv, causal, E_lo, E_hi);
  return c == RELPOS_TILE_MASKED ? RELPOS_TILE_CONST_LO : c;
}

// Segments of query tile qi: key tiles [0, lo_end) are CONST_LO, [lo_end,
// band_end) BAND, [band_end, live_end) CONST_HI, [live_end, nT) MASKED.
// Classes are monotone in kj (the offset range grows with kj and the
// masked tiles are the tail), so the bounds come from counting.
RP_HD void tile_segments(int qi, int nT, int N, int nkv, int causal, int E_lo, int E_hi, int seg[4]) {
  int nlo = 0, nband = 0, nhi = 0;
  for (int kj = 0; kj < nT; ++kj) {
    const int c = tile_class(qi, kj, N, nkv, causal, E_lo, E_hi);
    nlo += c == RELPOS_TILE_CONST_LO;
    nband += c == RELPOS_TILE_BAND;
    nhi += c == RELPOS_TILE_CONST_HI;
  }
  seg[0] = nlo;
  seg[1] = nlo + nband;
  seg[2] = nlo + nband + nhi;
  seg[3] = nT;
}

template <typename T> struct DT;
template <> struct DT<__half> {
  static constexpr bool kCoarse = false;
  static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
  static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  // sum of the two packed values, as fp32
  static __device__ __forceinline__ float pair_sum(uint32_t u) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    return f.x + f.y;
  }
};
template <> struct DT<__nv_bfloat16> {
  static constexpr bool kCoarse = true;
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float pair_sum(uint32_t u) {
    return __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
  }
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Attention dropout mask.  Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011), restated from its
// definition: ten rounds of (hi0, lo0) = M0 x0, (hi1, lo1) = M1 x2 (32 x 32 ->
// 64-bit), x = (hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0), the key bumped by
// (W0, W1) before every round after the first.  One call serves a block of
// 4 query rows x 4 keys: counter (j >> 2, i >> 2, bh, offset), key (seed_lo,
// seed_hi); query row i & 3 reads output word i & 3, key j & 3 its byte j & 3
// (least significant first), and the cell is kept when that byte is
// >= drop_thresh (= ceil(256 p)).
// ---------------------------------------------------------------------------
#ifdef __CUDACC__
__device__ __forceinline__ uint4 philox4x32_10(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, uint32_t k0,
                                               uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, x0), lo0 = 0xD2511F53u * x0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, x2), lo1 = 0xCD9E8D57u * x2;
    x0 = hi1 ^ x1 ^ k0;
    x1 = lo1;
    x2 = hi0 ^ x3 ^ k1;
    x3 = lo0;
  }
  return make_uint4(x0, x1, x2, x3);
}

// Keep bits of the four 8-bit uniforms of word w (bit b: byte b >= thresh).
// Bytes 0 / 2 and 1 / 3 are added, as 16-bit lanes, to 256 - thresh: the carry
// into bit 8 of a lane is the comparison (thresh <= 256, so no lane overflows).
__device__ __forceinline__ uint32_t keep4(uint32_t w, uint32_t thresh) {
  const uint32_t c = (256u - thresh) * 0x00010001u;
  const uint32_t e = ((w & 0x00FF00FFu) + c) & 0x01000100u;          // bytes 0, 2 -> bits 8, 24
  const uint32_t o = (((w >> 8) & 0x00FF00FFu) + c) & 0x01000100u;   // bytes 1, 3 -> bits 8, 24
  const uint32_t m = e | (o << 1);                                   // bits 8, 9, 24, 25
  return ((m >> 8) & 3u) | ((m >> 22) & 12u);
}

// Keep bits of 64 consecutive columns c0 .. c0 + 63 (c0 a multiple of 4) of
// this lane's row; bit c of km[c >> 5] keeps column c0 + c.  The whole warp
// calls this, with rows = 32 consecutive indices, lane = row & 31.
//  row_is_query: rows are queries i, columns keys; a block is the 4 rows of a
//    lane quad (i & 3) x 4 keys and gives row i & 3 the 4 bits of word i & 3.
//  otherwise: rows are keys j, columns queries; a block is 4 queries x the 4
//    keys of a lane quad (j & 3) and gives key j & 3 byte j & 3 of each word.
// Either way the quad's 16 blocks over the 64 columns are split so that each
// lane draws every fourth one (4 generator calls per lane for its 64 cells)
// and hands each of the other three lanes its 4 bits of each (three shuffles).
__device__ __forceinline__ void keep_mask64(const Plan& p, int bh, int row, int c0, bool row_is_query,
                                            uint32_t (&km)[2]) {
  km[0] = km[1] = 0u;
  const uint32_t th = p.drop_thresh;
  const int q4 = row & 3;                       // this lane's place in its quad
  uint32_t give[4] = {0u, 0u, 0u, 0u};          // 4 bits per drawn block for each lane of the quad
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int blk = 4 * t + q4;                 // block: columns c0 + 4 blk .. + 3
    const uint32_t cb = (uint32_t)(c0 + 4 * blk) >> 2, rb = (uint32_t)row >> 2;
    const uint4 r = row_is_query ? philox4x32_10(cb, rb, (uint32_t)bh, p.drop_offset, p.seed_lo, p.seed_hi)
                                 : philox4x32_10(rb, cb, (uint32_t)bh, p.drop_offset, p.seed_lo, p.seed_hi);
    const uint32_t k0 = keep4(r.x, th), k1 = keep4(r.y, th), k2 = keep4(r.z, th), k3 = keep4(r.w, th);
    if (row_is_query) {
      // lane q of the quad is query row q: word q, its 4 bits are the block's 4 keys
      give[0] |= k0 << (4 * t);
      give[1] |= k1 << (4 * t);
      give[2] |= k2 << (4 * t);
      give[3] |= k3 << (4 * t);
    } else {
      // lane q of the quad is key q: bit q of every word, one per query of the block
#pragma unroll
      for (int q = 0; q < 4; ++q)
        give[q] |= (((k0 >> q) & 1u) | (((k1 >> q) & 1u) << 1) | (((k2 >> q) & 1u) << 2) | (((k3 >> q) & 1u) << 3))
                   << (4 * t);
    }
  }
  // own bits first, then each partner's bits for this lane
  uint32_t mine = give[0];
  if (q4 == 1) mine = give[1];
  if (q4 == 2) mine = give[2];
  if (q4 == 3) mine = give[3];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int blk = 4 * t + q4;
    km[blk >> 3] |= ((mine >> (4 * t)) & 0xFu) << (4 * (blk & 7));
  }
#pragma unroll
  for (int d = 1; d < 4; ++d) {
    const int src = q4 ^ d;                     // the partner lane; it drew blocks 4 t + src
    uint32_t send = give[0];
    if (src == 1) send = give[1];
    if (src == 2) send = give[2];
    if (src == 3) send = give[3];
    const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, d);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int blk = 4 * t + src;
      km[blk >> 3] |= ((got >> (4 * t)) & 0xFu) << (4 * (blk & 7));
    }
  }
}
#endif

}  // namespace relpos
