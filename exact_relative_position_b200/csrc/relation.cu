// relation.cu -- relation-table side of exact relative-position attention
// (digest of "Fast and Exact Relative-Position Attention via Structure-Aware
// Kernels": Eq. (3), "grouped reachable range", "constant tiles and the
// saturated region" and the table-gradient GEMMs of the backward section).
//
//  * tables:      group geometry, expanded row -> table row map, expanded
//                 bias and (for bucketed maps) the expanded aQ/aK tables in
//                 which every bucket row is copied once per offset it covers.
//  * projection:  Z = X A_exp^T for every 128-row group over its reachable
//                 columns only (dense tensor-core GEMM, K = head dim).
//  * relgrad:     dQ += dZ^Q A_exp and dK += dZ^K A_exp (row epilogue),
//                 dA_exp = sum dZ^T X per fixed split of (batch, head, group),
//                 db_exp = column sums of dZ^Q, then a deterministic final
//                 pass that sums the splits in order and folds the copy
//                 columns of a bucket back into that bucket in ascending
//                 offset order.  No atomics.
#include <algorithm>

#include "kernels.cuh"
#include "warp_mma.cuh"

namespace relpos {

namespace {

// ------------------------------------------------------------------ tables
__global__ void groups_kernel(const Plan p, GroupInfo* gq, GroupInfo* gk) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= p.nT) return;
  gq[g] = group_info(p, 0, g);
  gk[g] = group_info(p, 1, g);
}

__global__ void phi_exp_kernel(const relpos_map_desc map, const int N, const int E_lo, const int Rexp, int* phi_exp) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < Rexp) phi_exp[e] = phi_of(map, N, E_lo + e);
}

__global__ void bias_exp_kernel(const relpos_map_desc map, const int N, const int E_lo, const int Rexp, const int R,
                                const int H, const float* __restrict__ b, float* __restrict__ b_exp) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)H * Rexp) return;
  const int h = (int)(idx / Rexp), e = (int)(idx - (long long)h * Rexp);
  b_exp[idx] = b[(size_t)h * R + phi_of(map, N, E_lo + e)];
}

// Copy of table row phi(E_lo + e) into expanded row e (16-byte chunks).
__global__ void table_exp_kernel(const relpos_map_desc map, const int N, const int E_lo, const int Rexp, const int R,
                                 const int Hq, const uint4* __restrict__ src, uint4* __restrict__ dst) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)Hq * Rexp * 8;
  if (idx >= total) return;
  const int c = (int)(idx & 7);
  const long long row = idx >> 3;
  const int h = (int)(row / Rexp), e = (int)(row - (long long)h * Rexp);
  const int r = phi_of(map, N, E_lo + e);
  dst[idx] = src[((size_t)h * R + r) * 8 + c];
}

__global__ void fold_mark_kernel(const int* __restrict__ phi_exp, const int Rexp, int* fold_lo, int* fold_hi) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= Rexp) return;
  const int r = phi_exp[e];
  if (e == 0 || phi_exp[e - 1] != r) fold_lo[r] = e;
  if (e == Rexp - 1 || phi_exp[e + 1] != r) fold_hi[r] = e + 1;
}

// ------------------------------------------------------------------ projection
// Z[b,h, group g rows, columns e0 + [c0, c0 + 64)] = X_rows A_exp[e0 + c0 ..]^T for
// kProjChunks consecutive 64-column chunks per CTA: the group's X rows are loaded
// once, and the next chunk's A rows arrive while the current chunk is stored.
constexpr int kProjChunks = 4;
constexpr int kProjSmem = 128 * 128 + 2 * 64 * 128;

template <typename T>
__global__ void __launch_bounds__(256) projection_kernel(const Plan p, const int key_side, const T* __restrict__ X,
                                                         const T* __restrict__ A, const long long a_hs,
                                                         float* __restrict__ Z, const long long z_head) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, bh = blockIdx.z;
  const int h = bh % p.H;
  const GroupInfo gi = key_side ? p.gk[g] : p.gq[g];
  const int cfirst = blockIdx.x * kProjChunks * 64;
  if (cfirst >= gi.W) return;
  const int nch = imin(kProjChunks, (gi.W - cfirst + 63) / 64);
  const int r0 = g * kTile;
  const uint32_t sX = smem_u32(smem), sA0 = sX + 128 * 128;
  // this sequence's rows of X (dense [B, H, N, 64] or packed [T, H, 64]); rows
  // past the sequence are zero-filled, so their projections are zero
  const int b = bh / p.H;
  const SeqRows sr = seq_rows(p, b);
  const T* Xh = X + (size_t)act_row(p, sr, b, h, 0) * 64;
  const T* Ah = A + (size_t)h * a_hs + (size_t)gi.e0 * 64;
  load_tile_async<128, 256>(sX, Xh, r0, sr.len, tid, act_pitch(p));
  load_tile_async<64, 256>(sA0, Ah + (size_t)cfirst * 64, 0, gi.W - cfirst, tid);
  cp_async_commit();
  const int g8 = lane >> 2, tq = lane & 3;
  float* Zg = Z + (size_t)bh * z_head + gi.base;
  uint32_t xa[4][4];
#pragma unroll 1
  for (int k = 0; k < nch; ++k) {
    const int c0 = cfirst + 64 * k;
    if (k + 1 < nch) {
      // buffer (k + 1) & 1 was last read in iteration k - 1, which ended with a barrier
      load_tile_async<64, 256>(sA0 + (uint32_t)((k + 1) & 1) * 64 * 128, Ah + (size_t)(c0 + 64) * 64, 0,
                               gi.W - c0 - 64, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (k == 0) load_a_frags(sX, warp * 16, lane, xa);
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    mma_abt<T, 8>(acc, xa, sA0 + (uint32_t)(k & 1) * 64 * 128, 0, lane);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int rr = warp * 16 + g8 + 8 * hf;
      if (r0 + rr >= p.N) continue;
      float* zrow = Zg + (long long)rr * gi.S;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int col = c0 + nt * 8 + 2 * tq;
        if (col < gi.W) *reinterpret_cast<float2*>(zrow + col) = make_float2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
      }
    }
    __syncthreads();   // every warp has read buffer k & 1 before iteration k + 1 refills it
  }
}

// ------------------------------------------------------------------ saturated key columns
// out[bh][0][j] = tau log2e Z^K[j, 0], out[bh][1][j] = tau log2e Z^K[j, R_exp - 1]
// (zero where the key's group does not store the column or j >= N), laid out
// contiguously so the fused forward can bulk-copy one key tile's worth.
__global__ void saturated_columns_kernel(const Plan p, const float* __restrict__ zk, float* __restrict__ out,
                                         const float scale) {
  const int npad = p.nT * kTile;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.B * p.H * npad) return;
  const int j = (int)(idx % npad);
  const long long bh = idx / npad;
  float lo = 0.f, hi = 0.f;
  if (j < p.N) {
    const GroupInfo gi = p.gk[j / kTile];
    const float* row = zk + bh * p.zk_head + gi.base + (long long)(j % kTile) * gi.S - gi.e0;
    if (gi.e0 == 0) lo = row[0] * scale;
    if (gi.e0 + gi.W >= p.Rexp) hi = row[p.Rexp - 1] * scale;
  }
  out[(bh * 2 + 0) * npad + j] = lo;
  out[(bh * 2 + 1) * npad + j] = hi;
}

// out[bh][0][i] = tau log2e (Z^Q[i, 0] + b_exp[0]) - LSE_i log2e, out[bh][1][i] =
// the same at R_exp - 1 (each term only when present; -inf where lse2 is +inf,
// i.e. past the sequence or for a row without a kept key): the row constants of
// saturated tiles for the backward passes, with the LSE folded in.
__global__ void saturated_rows_kernel(const Plan p, const float* __restrict__ zq, const float* __restrict__ b_exp,
                                      const float* __restrict__ lse2, float* __restrict__ out, const float scale) {
  const int npad = p.nT * kTile;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.B * p.H * npad) return;
  const int i = (int)(idx % npad);
  const long long bh = idx / npad;
  const int h = (int)(bh % p.H);
  float lo = 0.f, hi = 0.f;
  if (i < p.N) {
    if (zq) {
      const GroupInfo gi = p.gq[i / kTile];
      const float* row = zq + bh * p.zq_head + gi.base + (long long)(i % kTile) * gi.S - gi.e0;
      if (gi.e0 == 0) lo += row[0];
      if (gi.e0 + gi.W >= p.Rexp) hi += row[p.Rexp - 1];
    }
    if (b_exp) {
      lo += b_exp[(size_t)h * p.Rexp];
      hi += b_exp[(size_t)h * p.Rexp + p.Rexp - 1];
    }
  }
  const float l2 = lse2[bh * npad + i];
  out[(bh * 2 + 0) * npad + i] = lo * scale - l2;
  out[(bh * 2 + 1) * npad + i] = hi * scale - l2;
}

// ------------------------------------------------------------------ relgrad rows
// out[rows of group g] = acc_in[rows] + tau (dS_g[rows, :W] A_exp[e0 .. e0 + W)
//                        + s_lo A_exp[0] + s_hi A_exp[R_exp - 1])     (16-bit tensor cores)
// dS_g: the group's stored 16-bit relation gradient (interior offsets; zero at
// the saturated ones), (s_lo, s_hi): the row's fp32 saturated-offset sums.
// One CTA per (group, batch x head).  The reduction runs over the group's W
// stored columns, streamed in chunks of 32 columns through a 3-stage cp.async
// ring; warp w owns rows 16w .. 16w + 15 and all 64 output columns
// (mma m16n8k16, operands by ldmatrix).
namespace rg {
constexpr int kKC = 32;        // columns of dS (rows of the table) per chunk
constexpr int kStages = 3;
constexpr int kZP = 40;        // elements per row of a dS chunk [128][32] (80 bytes: conflict-free ldmatrix)
constexpr int kAP = 72;        // elements per row of a table chunk [32][64] (144 bytes)
template <typename T>
constexpr uint32_t stage_bytes() { return (uint32_t)(128 * kZP + kKC * kAP) * (uint32_t)sizeof(T); }
}  // namespace rg

template <typename T>
__global__ void __launch_bounds__(256) relgrad_rows_kernel(const Plan p, const int key_side, const T* __restrict__ dZ,
                                                           const long long z_head, const float* __restrict__ dz_sat,
                                                           const T* __restrict__ A, const long long a_hs,
                                                           const float* __restrict__ acc_in, T* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t rg_smem[];
  constexpr uint32_t kSB = rg::stage_bytes<T>();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (batch x heads, groups), the groups launched from the last one down:
  // under a causal mask a later group's rows reach more offsets, so the launch
  // ends on the shortest groups
  const int bh = blockIdx.x, g = (int)(gridDim.y - 1 - blockIdx.y), h = bh % p.H, b = bh / p.H;
  const GroupInfo gi = key_side ? p.gk[g] : p.gq[g];
  const int r0 = g * kTile;
  const SeqRows sr = seq_rows(p, b);
  const int nrows = imin(kTile, sr.len - r0);   // rows of this sequence in the group (may be <= 0)
  const T* Zg = dZ + (size_t)bh * z_head + gi.base;
  const T* Ah0 = A + (size_t)h * a_hs;
  const T* Ah = Ah0 + (size_t)gi.e0 * 64;
  const int nk = (gi.W + rg::kKC - 1) / rg::kKC;
  const uint32_t sbase = smem_u32(rg_smem);
  auto load = [&](int kc) {
    const uint32_t zs = sbase + (uint32_t)(kc % rg::kStages) * kSB;
    const uint32_t as = zs + 128u * rg::kZP * (uint32_t)sizeof(T);
    const int c0 = kc * rg::kKC;
    // dS: 128 rows x 4 pieces of 8 columns (rows start on 16 bytes: S and the
    // group base are multiples of 8); a piece at or past the row stride S or
    // a row past the group is zero-filled.  Columns in [W, S) are stored zeros.
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = u * 256 + tid;
      const int r = idx >> 2, pc = idx & 3;
      const int col = c0 + 8 * pc;
      const bool ok = r < nrows && col < gi.S;
      cp_async16(zs + (uint32_t)(r * rg::kZP + 8 * pc) * (uint32_t)sizeof(T), ok ? Zg + (long long)r * gi.S + col : Zg,
                 ok ? 16 : 0);
    }
    // table rows e0 + c0 .. + 31 (8 pieces of 8 elements each); rows past W are zero-filled
    const int r = tid >> 3, pc = tid & 7;
    const bool ok = c0 + r < gi.W;
    cp_async16(as + (uint32_t)(r * rg::kAP + 8 * pc) * (uint32_t)sizeof(T), ok ? Ah + (size_t)(c0 + r) * 64 + 8 * pc : Ah,
               ok ? 16 : 0);
  };
  const int g8 = lane >> 2, tq = lane & 3, rb = warp * 16;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
  for (int s = 0; s < rg::kStages - 1; ++s) {
    if (s < nk) load(s);
    cp_async_commit();
  }
  // ldmatrix lane addresses: A (dS rows) and B (table, transposed)
  const int mi = lane >> 3;
  const uint32_t a_off = (uint32_t)((rb + (lane & 15)) * rg::kZP + (lane >> 4) * 8) * (uint32_t)sizeof(T);
  const uint32_t b_off = (uint32_t)(((mi & 1) * 8 + (lane & 7)) * rg::kAP + (mi >> 1) * 8) * (uint32_t)sizeof(T);
  for (int kc = 0; kc < nk; ++kc) {
    cp_async_wait<rg::kStages - 2>();
    __syncthreads();   // chunk kc visible to all; the stage of chunk kc - 1 is free again
    if (kc + rg::kStages - 1 < nk) load(kc + rg::kStages - 1);
    cp_async_commit();
    const uint32_t zs = sbase + (uint32_t)(kc % rg::kStages) * kSB;
    const uint32_t as = zs + 128u * rg::kZP * (uint32_t)sizeof(T);
#pragma unroll
    for (int ks = 0; ks < rg::kKC / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(zs + a_off + (uint32_t)(ks * 16) * (uint32_t)sizeof(T), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(as + b_off + (uint32_t)(ks * 16 * rg::kAP + np * 16) * (uint32_t)sizeof(T), b0, b1, b2, b3);
        MmaOp<T>::run(acc[2 * np], a, b0, b1);
        MmaOp<T>::run(acc[2 * np + 1], a, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  const size_t npad = (size_t)p.nT * kTile;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int rr = rb + g8 + 8 * hf;
    if (rr >= nrows) continue;
    const float2 sat = *reinterpret_cast<const float2*>(dz_sat + 2 * ((size_t)bh * npad + r0 + rr));
    // the fp32 accumulator keeps the workspace's dense layout; the output is the caller's
    const size_t ai = ((size_t)bh * p.N + r0 + rr) * 64;
    const size_t ro = (size_t)act_row(p, sr, b, h, r0 + rr) * 64;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = nt * 8 + 2 * tq;
      const float2 base = *reinterpret_cast<const float2*>(acc_in + ai + c);
      const float lo0 = DT<T>::to_f(Ah0[c]), lo1 = DT<T>::to_f(Ah0[c + 1]);
      const float hi0 = DT<T>::to_f(Ah0[(size_t)(p.Rexp - 1) * 64 + c]), hi1 = DT<T>::to_f(Ah0[(size_t)(p.Rexp - 1) * 64 + c + 1]);
      const float v0 = acc[nt][2 * hf] + sat.x * lo0 + sat.y * hi0;
      const float v1 = acc[nt][2 * hf + 1] + sat.x * lo1 + sat.y * hi1;
      *reinterpret_cast<uint32_t*>(out + ro + c) = DT<T>::pack(fmaf(p.tau, v0, base.x), fmaf(p.tau, v1, base.y));
    }
  }
}

// ------------------------------------------------------------------ table partials
// part[s][hq][c0 + m][:] = tau x the sum over the split's (batch, head, group)
// items, in order, of dS_g[rows, c0 + m - e0] X[rows, :]   (16-bit tensor cores)
// plus, at the saturated offsets m = 0 and R_exp - 1, tau x the sum of the
// rows' fp32 saturated-offset sums times X[rows, :].
// Block (e-block of 256 expanded rows, table, split).  The split's positions
// are streamed in chunks of 32 rows of (dS, X, saturated sums) through a
// 3-stage cp.async ring that runs across item boundaries; items whose group
// stores none of the block's columns are skipped.  Warp w owns expanded rows
// 32w .. 32w + 31 (two m16 tiles), so every X fragment feeds two MMAs.  dS is
// copied in 16-byte pieces when the item's first column lines up with the
// block to 8 elements (every group of a map whose groups reach all offsets),
// else element by element.  With db_part (per-head tables on the query side,
// with a bias) the block also sums its dS columns in fp32 from the same staged
// chunks: db_part[s][h][c0 + m] = tau x (column sums + saturated sums), so the
// bias gradient needs no pass of its own over dS^Q.
namespace tp {
constexpr int kEB = 256;       // expanded rows per block
constexpr int kRC = 32;        // positions per chunk
constexpr int kStages = 3;
constexpr int kZP = 264;       // elements per row of a dS chunk [32][256] (528 bytes: conflict-free ldmatrix)
constexpr int kXP = 72;        // elements per row of an X chunk [32][64]
template <typename T>
constexpr uint32_t stage_bytes() { return (uint32_t)(kRC * kZP + kRC * kXP) * (uint32_t)sizeof(T) + kRC * 8u; }
}  // namespace tp

struct ItemCursor {
  long long it;   // current item
  int rc;         // first row of the next chunk inside it
};

template <typename T>
__global__ void __launch_bounds__(256) table_part_kernel(const Plan p, const int key_side, const T* __restrict__ dZ,
                                                         const long long z_head, const float* __restrict__ dz_sat,
                                                         const T* __restrict__ X, const int per_head, const int nsplit,
                                                         float* __restrict__ part, float* __restrict__ db_part) {
  extern __shared__ __align__(16) uint8_t tp_smem[];
  constexpr uint32_t kSB = tp::stage_bytes<T>();
  constexpr uint32_t kXOff = (uint32_t)tp::kRC * tp::kZP * (uint32_t)sizeof(T);
  constexpr uint32_t kSOff = kXOff + (uint32_t)tp::kRC * tp::kXP * (uint32_t)sizeof(T);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (splits, heads, expanded-row blocks), the blocks launched from the last
  // one down: under a causal identity map the blocks next to the diagonal carry
  // the most rows, and the launch then ends on the lightest ones
  const int s = blockIdx.x, hq = blockIdx.y, c0 = (int)(gridDim.z - 1 - blockIdx.z) * tp::kEB;
  const int Hq = per_head ? p.H : 1;
  const long long nitems = per_head ? (long long)p.B * p.nT : (long long)p.B * p.H * p.nT;
  const long long it0 = nitems * s / nsplit, it1 = nitems * (s + 1) / nsplit;
  const size_t npad = (size_t)p.nT * kTile;
  auto item = [&](long long it, int& bh, int& g) {
    if (per_head) {
      const int b = (int)(it / p.nT);
      g = (int)(it - (long long)b * p.nT);
      bh = b * p.H + hq;
    } else {
      bh = (int)(it / p.nT);
      g = (int)(it - (long long)bh * p.nT);
    }
  };
  // rows of group g that belong to the sequence of (b, h) (all of them in the dense layout)
  auto item_rows = [&](int bh, int g) { return iclamp(seq_rows(p, bh / p.H).len - g * kTile, 0, kTile); };
  auto useful = [&](int bh, int g) {
    const GroupInfo gi = key_side ? p.gk[g] : p.gq[g];
    return !(c0 + tp::kEB <= gi.e0 || c0 >= gi.e0 + gi.W) && item_rows(bh, g) > 0;
  };
  // number of chunks of this split (block-uniform)
  int nchunks = 0;
  for (long long it = it0; it < it1; ++it) {
    int bh, g;
    item(it, bh, g);
    if (useful(bh, g)) nchunks += (item_rows(bh, g) + tp::kRC - 1) / tp::kRC;
  }
  // load cursor: skips items that store none of the block's columns or no rows
  ItemCursor cur{it0, 0};
  auto skip = [&]() {
    while (cur.it < it1) {
      int bh, g;
      item(cur.it, bh, g);
      if (useful(bh, g)) break;
      ++cur.it;
    }
  };
  skip();
  const uint32_t sbase = smem_u32(tp_smem);
  auto load = [&](int q) {
    int bh, g;
    item(cur.it, bh, g);
    const GroupInfo gi = key_side ? p.gk[g] : p.gq[g];
    const int r0 = g * kTile, nrows = item_rows(bh, g);
    const T* Zg = dZ + (size_t)bh * z_head + gi.base;
    const int b = bh / p.H;
    const T* Xg = X + (size_t)act_row(p, seq_rows(p, b), b, bh - b * p.H, r0) * 64;
    const int xpitch = act_pitch(p);
    const uint32_t zs = sbase + (uint32_t)(q % tp::kStages) * kSB;
    // dS rows rc .. rc + 31, expanded columns c0 .. c0 + 255 (local column lc = c - e0)
    if (((c0 - gi.e0) & 7) == 0) {
      // 16-byte pieces: lc is a multiple of 8 and the row stride S too; the
      // columns [W, S) are stored zeros
#pragma unroll
      for (int u = 0; u < tp::kRC * tp::kEB / 8 / 256; ++u) {
        const int idx = u * 256 + tid;
        const int r = idx >> 5, c = (idx & 31) * 8;
        const int lc = c0 + c - gi.e0;
        const bool ok = cur.rc + r < nrows && lc >= 0 && lc < gi.S;
        cp_async16(zs + (uint32_t)(r * tp::kZP + c) * (uint32_t)sizeof(T),
                   ok ? Zg + (long long)(cur.rc + r) * gi.S + lc : Zg, ok ? 16 : 0);
      }
    } else {
      // a window not aligned to 8 elements (ragged N): plain 16-bit copies,
      // visible to the block after the barrier that makes the stage current
      T* zp = reinterpret_cast<T*>(tp_smem + (uint32_t)(q % tp::kStages) * kSB);
#pragma unroll 4
      for (int u = 0; u < tp::kRC * tp::kEB / 256; ++u) {
        const int idx = u * 256 + tid;
        const int r = idx >> 8, c = idx & 255;
        const int lc = c0 + c - gi.e0;
        const bool ok = cur.rc + r < nrows && lc >= 0 && lc < gi.W;
        zp[r * tp::kZP + c] = ok ? Zg[(long long)(cur.rc + r) * gi.S + lc] : DT<T>::from_f(0.f);
      }
    }
    {
      const int r = tid >> 3, pc = tid & 7;
      const bool ok = cur.rc + r < nrows;
      cp_async16(zs + kXOff + (uint32_t)(r * tp::kXP + 8 * pc) * (uint32_t)sizeof(T),
                 ok ? Xg + (size_t)(cur.rc + r) * xpitch + 8 * pc : Xg, ok ? 16 : 0);
    }
    if (tid < tp::kRC / 2) {
      // the rows' saturated-offset sums (s_lo, s_hi), two rows per piece
      const int r = 2 * tid;
      const bool ok = cur.rc + r < nrows;
      const float* src = dz_sat + 2 * ((size_t)bh * npad + r0 + cur.rc + r);
      cp_async16(zs + kSOff + (uint32_t)r * 8u, ok ? src : dz_sat, ok ? (cur.rc + r + 1 < nrows ? 16 : 8) : 0);
    }
    cur.rc += tp::kRC;
    if (cur.rc >= nrows) {
      cur.rc = 0;
      ++cur.it;
      skip();
    }
  };
  const int g8 = lane >> 2, tq = lane & 3, eb = warp * 32;
  float acc[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[mt][i][0] = acc[mt][i][1] = acc[mt][i][2] = acc[mt][i][3] = 0.f;
  // column sums of dS for db_part: rows g8 and g8 + 8 of each m16 tile
  const bool with_db = db_part != nullptr;   // block-uniform
  float dbs[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  // the saturated offsets 0 / R_exp - 1 in this block: sums over the rows of
  // s x X (thread: column sc, rows sr, sr + 4, ...) and, for db, of s
  const bool sat_lo_here = c0 == 0, sat_hi_here = c0 <= p.Rexp - 1 && p.Rexp - 1 < c0 + tp::kEB;
  const int sc = tid & 63, srg = tid >> 6;
  float sx_lo = 0.f, sx_hi = 0.f, ss_lo = 0.f, ss_hi = 0.f;
#pragma unroll
  for (int q = 0; q < tp::kStages - 1; ++q) {
    if (q < nchunks) load(q);
    cp_async_commit();
  }
  // ldmatrix lane addresses (both operands transposed from [position][.] rows)
  const int mi = lane >> 3;
  const uint32_t a_off = (uint32_t)(((mi >> 1) * 8 + (lane & 7)) * tp::kZP + eb + (mi & 1) * 8) * (uint32_t)sizeof(T);
  const uint32_t b_off = (uint32_t)(((mi & 1) * 8 + (lane & 7)) * tp::kXP + (mi >> 1) * 8) * (uint32_t)sizeof(T);
  for (int q = 0; q < nchunks; ++q) {
    cp_async_wait<tp::kStages - 2>();
    __syncthreads();   // chunk q visible to all; the stage of chunk q - 1 is free again
    if (q + tp::kStages - 1 < nchunks) load(q + tp::kStages - 1);
    cp_async_commit();
    const uint32_t zs = sbase + (uint32_t)(q % tp::kStages) * kSB;
#pragma unroll
    for (int ks = 0; ks < tp::kRC / 16; ++ks) {
      // A = dS^T: rows = expanded offsets, columns = positions
      uint32_t a[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        ldsm_x4_t(zs + a_off + (uint32_t)(ks * 16 * tp::kZP + 16 * mt) * (uint32_t)sizeof(T), a[mt][0], a[mt][1],
                  a[mt][2], a[mt][3]);
        if (with_db) {
          dbs[mt][0] += DT<T>::pair_sum(a[mt][0]) + DT<T>::pair_sum(a[mt][2]);
          dbs[mt][1] += DT<T>::pair_sum(a[mt][1]) + DT<T>::pair_sum(a[mt][3]);
        }
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(zs + kXOff + b_off + (uint32_t)(ks * 16 * tp::kXP + np * 16) * (uint32_t)sizeof(T), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          MmaOp<T>::run(acc[mt][2 * np], a[mt], b0, b1);
          MmaOp<T>::run(acc[mt][2 * np + 1], a[mt], b2, b3);
        }
      }
    }
    if (sat_lo_here || sat_hi_here) {   // block-uniform
      const T* Xs = reinterpret_cast<const T*>(tp_smem + (uint32_t)(q % tp::kStages) * kSB + kXOff);
      const float2* Ss = reinterpret_cast<const float2*>(tp_smem + (uint32_t)(q % tp::kStages) * kSB + kSOff);
#pragma unroll
      for (int rr = srg; rr < tp::kRC; rr += 4) {
        const float2 sv = Ss[rr];
        const float xv = DT<T>::to_f(Xs[rr * tp::kXP + sc]);
        sx_lo = fmaf(sv.x, xv, sx_lo);
        sx_hi = fmaf(sv.y, xv, sx_hi);
        ss_lo += sv.x;
        ss_hi += sv.y;
      }
    }
  }
  cp_async_wait<0>();
  float* P = part + ((size_t)s * Hq + hq) * (size_t)p.Rexp * 64;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int e = c0 + eb + 16 * mt + g8 + 8 * hf;
      if (e >= p.Rexp) continue;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int d = nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(P + (size_t)e * 64 + d) =
            make_float2(p.tau * acc[mt][nt][2 * hf], p.tau * acc[mt][nt][2 * hf + 1]);
      }
    }
  }
  float* DB = with_db ? db_part + ((size_t)s * p.H + hq) * p.Rexp : nullptr;
  if (with_db) {
    // the quad's four lanes hold the four position classes of the same rows
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v = dbs[mt][hf];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        const int e = c0 + eb + 16 * mt + g8 + 8 * hf;
        if (tq == 0 && e < p.Rexp) DB[e] = p.tau * v;
      }
  }
  if (sat_lo_here || sat_hi_here) {
    // saturated offsets: the four row classes added in order on top of the
    // (zero) stored columns 0 / R_exp - 1 written above
    __shared__ float sred[4][64][2];
    __shared__ float sdb[4][2];
    __syncthreads();
    sred[srg][sc][0] = sx_lo;
    sred[srg][sc][1] = sx_hi;
    if (sc == 0) { sdb[srg][0] = ss_lo; sdb[srg][1] = ss_hi; }
    __syncthreads();
    if (srg == 0) {
      const float lo = ((sred[0][sc][0] + sred[1][sc][0]) + sred[2][sc][0]) + sred[3][sc][0];
      const float hi = ((sred[0][sc][1] + sred[1][sc][1]) + sred[2][sc][1]) + sred[3][sc][1];
      if (sat_lo_here) P[sc] += p.tau * lo;
      if (sat_hi_here) P[(size_t)(p.Rexp - 1) * 64 + sc] += p.tau * hi;
      if (with_db && sc == 0) {
        if (sat_lo_here) DB[0] += p.tau * (((sdb[0][0] + sdb[1][0]) + sdb[2][0]) + sdb[3][0]);
        if (sat_hi_here) DB[p.Rexp - 1] += p.tau * (((sdb[0][1] + sdb[1][1]) + sdb[2][1]) + sdb[3][1]);
      }
    }
  }
}

// db_part[s][h][e] = tau x the sum over the split's (batch, group) items of
// column e of dS^Q (plus, at e = 0 and R_exp - 1, of the rows' fp32
// saturated-offset sums), for the block's 256 expanded columns.  Warp w takes
// the rows r = w (mod 8) of every item, lane l the columns l + 32 k; the eight
// warp sums are added in warp order at the end.
template <typename T>
__global__ void __launch_bounds__(256) bias_part_kernel(const Plan p, const T* __restrict__ dZ, const long long z_head,
                                                        const float* __restrict__ dz_sat, const int nsplit,
                                                        float* __restrict__ part) {
  __shared__ float red[8][256];
  __shared__ float sred[8][2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * 256, h = blockIdx.y, s = blockIdx.z;
  const long long nitems = (long long)p.B * p.nT;
  const long long it0 = nitems * s / nsplit, it1 = nitems * (s + 1) / nsplit;
  const size_t npad = (size_t)p.nT * kTile;
  const bool sat_lo_here = c0 == 0, sat_hi_here = c0 <= p.Rexp - 1 && p.Rexp - 1 < c0 + 256;
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  float ss_lo = 0.f, ss_hi = 0.f;
  for (long long it = it0; it < it1; ++it) {
    const int b = (int)(it / p.nT), g = (int)(it - (long long)b * p.nT);
    const GroupInfo gi = p.gq[g];
    if (c0 + 256 <= gi.e0 || c0 >= gi.e0 + gi.W) continue;   // block-uniform
    const int bh = b * p.H + h;
    const int nrows = iclamp(seq_rows(p, b).len - g * kTile, 0, kTile);
    const T* Zg = dZ + (size_t)bh * z_head + gi.base;
    int lc[8];
    bool okc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      lc[k] = c0 + lane + 32 * k - gi.e0;
      okc[k] = lc[k] >= 0 && lc[k] < gi.W;
      if (!okc[k]) lc[k] = 0;
    }
#pragma unroll 4
    for (int r = warp; r < nrows; r += 8) {
      const T* zr = Zg + (long long)r * gi.S;
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = okc[k] ? DT<T>::to_f(zr[lc[k]]) : 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += v[k];
      if ((sat_lo_here || sat_hi_here) && lane == 0) {
        const float2 sv = *reinterpret_cast<const float2*>(dz_sat + 2 * ((size_t)bh * npad + g * kTile + r));
        ss_lo += sv.x;
        ss_hi += sv.y;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[warp][lane + 32 * k] = acc[k];
  if (lane == 0) { sred[warp][0] = ss_lo; sred[warp][1] = ss_hi; }
  __syncthreads();
  const int e = c0 + tid;
  if (e < p.Rexp) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += red[w][tid];
    if (sat_lo_here && e == 0)
      for (int w = 0; w < 8; ++w) sum += sred[w][0];
    if (sat_hi_here && e == p.Rexp - 1)
      for (int w = 0; w < 8; ++w) sum += sred[w][1];
    part[((size_t)s * p.H + h) * p.Rexp + e] = p.tau * sum;
  }
}

// The fold below for maps whose every table row is one expanded row (R = R_exp:
// the identity and truncated maps) and with many rows: out[hq][r][c] = the sum
// over splits s, in order, of part[s][hq][fold_lo[r]][c], as a grid-stride
// pass over the output (one block per row would mostly schedule blocks).
__global__ void __launch_bounds__(256) fold_rows_kernel(const float* __restrict__ part, const int nsplit, const int Hq,
                                                        const int Rexp, const int R, const int C,
                                                        const int* __restrict__ fold_lo, float* __restrict__ out) {
  if (C == 64 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    // a table row as 16 float4: the row, its head and its fold source are found once
    // per four columns; the splits are added in the same order as below
    const float4* src4 = reinterpret_cast<const float4*>(part);
    const size_t split_stride = (size_t)Hq * Rexp * 16;
    const long long n4 = (long long)Hq * R * 16;
    for (long long idx = blockIdx.x * 256LL + threadIdx.x; idx < n4; idx += (long long)gridDim.x * 256) {
      const long long hr = idx >> 4;
      const int hq = (int)(hr / R), r = (int)(hr - (long long)hq * R);
      const float4* src = src4 + ((size_t)hq * Rexp + fold_lo[r]) * 16 + (idx & 15);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int sp = 0; sp < nsplit; ++sp) {
        const float4 v = __ldg(src + sp * split_stride);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      reinterpret_cast<float4*>(out)[idx] = acc;
    }
    return;
  }
  const long long n = (long long)Hq * R * C;
  for (long long idx = blockIdx.x * 256LL + threadIdx.x; idx < n; idx += (long long)gridDim.x * 256) {
    const int c = (int)(idx % C);
    const long long hr = idx / C;
    const int r = (int)(hr % R), hq = (int)(hr / R);
    const int e = fold_lo[r];
    float acc = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) acc += part[(((size_t)sp * Hq + hq) * Rexp + e) * C + c];
    out[idx] = acc;
  }
}

// out[hq][r][c] = sum over the pairs (e in the fold range of r, split s) of
// part[s][hq][e][c].  One block per (r, hq); C is 64 (tables) or 1 (bias).
// The 256 threads form 256 / C groups per column c; group k sums the pairs
// k, k + 256 / C, ... (pairs ordered by e, then s) and the group sums are
// added in group order, so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) fold_kernel(const float* __restrict__ part, const int nsplit, const int Hq,
                                                   const int Rexp, const int R, const int C,
                                                   const int* __restrict__ fold_lo, const int* __restrict__ fold_hi,
                                                   float* __restrict__ out) {
  __shared__ float red[256];
  const int r = blockIdx.x, hq = blockIdx.y, tid = threadIdx.x;
  const int G = 256 / C, c = tid % C, grp = tid / C;
  const int lo = fold_lo[r];
  const long long npairs = (long long)(fold_hi[r] - lo) * nsplit;
  float acc = 0.f;
#pragma unroll 4
  for (long long q = grp; q < npairs; q += G) {
    const int e = lo + (int)(q / nsplit), sp = (int)(q % nsplit);
    acc += part[(((size_t)sp * Hq + hq) * Rexp + e) * C + c];
  }
  red[tid] = acc;
  __syncthreads();
  if (tid < C) {
    float sum = 0.f;
    for (int k = 0; k < G; ++k) sum += red[k * C + tid];
    out[((size_t)hq * R + r) * C + tid] = sum;
  }
}

// ------------------------------------------------------------------ debug
__global__ void debug_phi_kernel(const relpos_map_desc map, const int N, int* out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < 2 * N - 1) out[t] = phi_of(map, N, t - (N - 1));
}

__global__ void debug_plan_kernel(const int B, const int N, const int causal, const int* key_len, const int E_lo,
                                  const int E_hi, int* classes, int* segs) {
  const int nT = (N + kTile - 1) / kTile;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * nT * nT) return;
  const int kj = (int)(idx % nT);
  const int qi = (int)((idx / nT) % nT);
  const int b = (int)(idx / ((long long)nT * nT));
  const int nkv = key_len ? iclamp(key_len[b], 0, N) : N;
  classes[idx] = tile_class(qi, kj, N, nkv, causal, E_lo, E_hi);
  if (kj == 0) {
    int sg[4];
    tile_segments(qi, nT, N, nkv, causal, E_lo, E_hi, sg);
    for (int c = 0; c < 4; ++c) segs[((size_t)b * nT + qi) * 4 + c] = sg[c];
  }
}

inline unsigned nblk(long long n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t launch_build_tables(const Plan& p, const relpos_map_desc& map, GroupInfo* gq, GroupInfo* gk, int* phi_exp,
                                int R, const void* aq, const void* ak, int table_per_head, void* aq_exp, void* ak_exp,
                                const float* b, float* b_exp, int is_bf16, int expand_tables, cudaStream_t s) {
  (void)is_bf16;
  { groups_kernel<<<nblk(p.nT, 128), 128, 0, s>>>(p, gq, gk); note_launch(1); }
  { phi_exp_kernel<<<nblk(p.Rexp, 256), 256, 0, s>>>(map, p.N, p.E_lo, p.Rexp, phi_exp); note_launch(1); }
  if (b) { bias_exp_kernel<<<nblk((long long)p.H * p.Rexp, 256), 256, 0, s>>>(map, p.N, p.E_lo, p.Rexp, R, p.H, b, b_exp); note_launch(1); }
  if (expand_tables) {
    const int Hq = table_per_head ? p.H : 1;
    const long long n = (long long)Hq * p.Rexp * 8;
    if (aq) { table_exp_kernel<<<nblk(n, 256), 256, 0, s>>>(map, p.N, p.E_lo, p.Rexp, R, Hq, (const uint4*)aq, (uint4*)aq_exp); note_launch(1); }
    if (ak) { table_exp_kernel<<<nblk(n, 256), 256, 0, s>>>(map, p.N, p.E_lo, p.Rexp, R, Hq, (const uint4*)ak, (uint4*)ak_exp); note_launch(1); }
  }
  return cudaGetLastError();
}

cudaError_t launch_fold_ranges(const Plan& p, const int* phi_exp, int R, int* fold_lo, int* fold_hi, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(fold_lo, 0, sizeof(int) * R, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(fold_hi, 0, sizeof(int) * R, s);
  if (e != cudaSuccess) return e;
  { fold_mark_kernel<<<nblk(p.Rexp, 256), 256, 0, s>>>(phi_exp, p.Rexp, fold_lo, fold_hi); note_launch(1); }
  return cudaGetLastError();
}

template <typename T>
static cudaError_t projection_typed(const Plan& p, const Tensors& t, cudaStream_t s, cudaStream_t sk) {
  cudaError_t e = cudaFuncSetAttribute(projection_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kProjSmem);
  if (e != cudaSuccess) return e;
  // widest group decides the chunk count; narrower groups exit early
  int wq = 0, wk = 0;
  if (!p.grouped) { wq = wk = p.Rexp; }
  else { wq = wk = p.N + kTile - 1; }
  if (t.zq && t.aq_exp) {
    dim3 grid((wq + 64 * kProjChunks - 1) / (64 * kProjChunks), p.nT, p.B * p.H);
    { projection_kernel<T><<<grid, 256, kProjSmem, s>>>(p, 0, (const T*)t.q, (const T*)t.aq_exp,
                                                      t.table_per_head ? t.aq_hs : 0, t.zq, p.zq_head); note_launch(1); }
  }
  if (t.zk && t.ak_exp) {
    dim3 grid((wk + 64 * kProjChunks - 1) / (64 * kProjChunks), p.nT, p.B * p.H);
    { projection_kernel<T><<<grid, 256, kProjSmem, sk>>>(p, 1, (const T*)t.k, (const T*)t.ak_exp,
                                                      t.table_per_head ? t.ak_hs : 0, t.zk, p.zk_head); note_launch(1); }
  }
  return cudaGetLastError();
}

cudaError_t launch_saturated_columns(const Plan& p, const Tensors& t, cudaStream_t s) {
  const long long n = (long long)p.B * p.H * p.nT * kTile;
  { saturated_columns_kernel<<<nblk(n, 256), 256, 0, s>>>(p, t.zk, t.zk_sat, p.tau * kLog2e); note_launch(1); }
  return cudaGetLastError();
}

cudaError_t launch_saturated_rows(const Plan& p, const Tensors& t, cudaStream_t s) {
  const long long n = (long long)p.B * p.H * p.nT * kTile;
  {
    saturated_rows_kernel<<<nblk(n, 256), 256, 0, s>>>(p, t.aq_exp ? t.zq : nullptr, t.b_exp, t.lse2, t.zq_sat,
                                                       p.tau * kLog2e);
    note_launch(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_projection(const Plan& p, const Tensors& t, cudaStream_t s, cudaStream_t key_stream) {
  return t.is_bf16 ? projection_typed<__nv_bfloat16>(p, t, s, key_stream) : projection_typed<__half>(p, t, s, key_stream);
}

// Table-gradient fold: the grid-stride pass when every row folds one expanded
// row and there are many rows, else one block per (row, head).
static void launch_fold(const float* part, int nsplit, int Hq, int Rexp, int R, int C, const int* fold_lo,
                        const int* fold_hi, float* out, cudaStream_t s) {
  if (R == Rexp && (long long)R * Hq >= 4096) {
    const long long n = (long long)Hq * R * C;
    const int blocks = (int)std::min<long long>((n + 255) / 256, 148LL * 8);
    { fold_rows_kernel<<<blocks, 256, 0, s>>>(part, nsplit, Hq, Rexp, R, C, fold_lo, out); note_launch(1); }
  } else {
    { fold_kernel<<<dim3(R, Hq), 256, 0, s>>>(part, nsplit, Hq, Rexp, R, C, fold_lo, fold_hi, out); note_launch(1); }
  }
}

// side 0: the query side (aQ rows, aQ table, bias); side 1: the key side (aK).
template <typename T>
static cudaError_t relgrad_typed(const Plan& p, const Tensors& t, int side, cudaStream_t s, cudaStream_t sr) {
  const int Hq = t.table_per_head ? p.H : 1;
  const int nE = (p.Rexp + tp::kEB - 1) / tp::kEB;
  constexpr uint32_t kRowsSmem = rg::kStages * rg::stage_bytes<T>();
  constexpr uint32_t kPartSmem = tp::kStages * tp::stage_bytes<T>();
  cudaError_t e = cudaFuncSetAttribute(relgrad_rows_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowsSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(table_part_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPartSmem);
  if (e != cudaSuccess) return e;
  // per-head aQ tables with a bias: the aQ table-gradient pass also sums the
  // bias gradient's columns (its splits are the workspace's bias splits)
  const bool fuse_db = t.aq_exp && t.b_exp && t.table_per_head && t.nsplit_b == t.nsplit_q;
  if (side == 0 && t.aq_exp) {
    { relgrad_rows_kernel<T><<<dim3(p.B * p.H, p.nT), 256, kRowsSmem, sr>>>(p, 0, (const T*)t.dzq, p.zq_head, t.dzq_sat,
                                                                        (const T*)t.aq_exp,
                                                                        t.table_per_head ? t.aq_hs : 0, t.dq_acc, (T*)t.dq); note_launch(1); }
    { table_part_kernel<T><<<dim3(t.nsplit_q, Hq, nE), 256, kPartSmem, s>>>(p, 0, (const T*)t.dzq, p.zq_head,
                                                                           t.dzq_sat, (const T*)t.q,
                                                                           t.table_per_head, t.nsplit_q, t.daq_part,
                                                                           fuse_db ? t.db_part : nullptr); note_launch(1); }
    launch_fold(t.daq_part, t.nsplit_q, Hq, p.Rexp, t.R, 64, t.fold_lo, t.fold_hi, t.daq, s);
  }
  if (side == 1 && t.ak_exp) {
    { relgrad_rows_kernel<T><<<dim3(p.B * p.H, p.nT), 256, kRowsSmem, sr>>>(p, 1, (const T*)t.dzk, p.zk_head, t.dzk_sat,
                                                                        (const T*)t.ak_exp,
                                                                        t.table_per_head ? t.ak_hs : 0, t.dk_acc, (T*)t.dk); note_launch(1); }
    { table_part_kernel<T><<<dim3(t.nsplit_k, Hq, nE), 256, kPartSmem, s>>>(p, 1, (const T*)t.dzk, p.zk_head,
                                                                           t.dzk_sat, (const T*)t.k,
                                                                           t.table_per_head, t.nsplit_k, t.dak_part,
                                                                           nullptr); note_launch(1); }
    launch_fold(t.dak_part, t.nsplit_k, Hq, p.Rexp, t.R, 64, t.fold_lo, t.fold_hi, t.dak, s);
  }
  if (side == 0 && t.b_exp) {
    if (!fuse_db)
    { bias_part_kernel<T><<<dim3((p.Rexp + 255) / 256, p.H, t.nsplit_b), 256, 0, s>>>(p, (const T*)t.dzq, p.zq_head,
                                                                                     t.dzq_sat, t.nsplit_b, t.db_part); note_launch(1); }
    launch_fold(t.db_part, t.nsplit_b, p.H, p.Rexp, t.R, 1, t.fold_lo, t.fold_hi, t.db, s);
  }
  return cudaGetLastError();
}

cudaError_t launch_relgrad(const Plan& p, const Tensors& t, int side, cudaStream_t s, cudaStream_t rows_stream) {
  return t.is_bf16 ? relgrad_typed<__nv_bfloat16>(p, t, side, s, rows_stream)
                   : relgrad_typed<__half>(p, t, side, s, rows_stream);
}

cudaError_t launch_debug_phi(const relpos_map_desc& map, int N, int* out, cudaStream_t s) {
  { debug_phi_kernel<<<nblk(2LL * N - 1, 256), 256, 0, s>>>(map, N, out); note_launch(1); }
  return cudaGetLastError();
}

cudaError_t launch_debug_tile_plan(int B, int N, int causal, const int* key_len, int E_lo, int E_hi, int* classes,
                                   int* segs, cudaStream_t s) {
  const int nT = (N + kTile - 1) / kTile;
  { debug_plan_kernel<<<nblk((long long)B * nT * nT, 256), 256, 0, s>>>(B, N, causal, key_len, E_lo, E_hi, classes, segs); note_launch(1); }
  return cudaGetLastError();
}

}  // namespace relpos
