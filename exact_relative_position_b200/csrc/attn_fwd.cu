// attn_fwd.cu -- fused forward of exact relative-position attention on sm_100a
// (digest of "Fast and Exact Relative-Position Attention via Structure-Aware
// Kernels": Eq. (1)/(2), the FlashAttention-style loop of the pipeline
// section, and "constant tiles and the saturated region").
//
// One CTA owns two 128-row query tiles (Q0, Q1) of one (batch, head) and
// walks the key tiles once for both, so each K/V tile that TMA brings into
// shared memory feeds four tcgen05 GEMMs.  Warp roles:
//   warp 0       TMA producer: Q0/Q1 once, then K/V tiles (and the key
//                tile's saturated relation columns) into a 3-stage ring
//   warp 1       MMA issuer (one thread): S_g = Q_g K^T into tensor memory,
//                O_g += P_g V with P_g read from tensor memory
//   warp 2       allocates / frees the tensor-memory columns
//   warps 4..7   softmax of Q0 (thread r owns row r = TMEM lane r)
//   warps 8..11  softmax of Q1
// Tensor memory: S0 cols [0,128), S1 [128,256), O0 [256,320), O1 [320,384),
// P0 [384,448), P1 [448,512).  A softmax warpgroup releases S_g as soon as
// it has read it into registers, so the GEMM of the next key tile runs while
// it computes; its 16-bit P_g (two keys per column) goes back to tensor
// memory, where the PV GEMM reads it as its A operand.  Shared memory then
// only carries the operands TMA brings in.
//
// Relation terms are added to the scores in registers.  A key tile whose
// every offset saturates (CONST_LO / CONST_HI: two comparisons of the tile's
// offset range with E_lo / E_hi) adds one per-row constant tau (Z^Q_i,sat +
// b_sat) and one per-column vector tau Z^K_j,sat staged with the K/V tile and
// broadcast; a BAND tile gathers Z^Q[i, e], Z^K[j, e] and b[e] per score with
// e = clamp(j - i, E_lo, E_hi) - E_lo.  The online softmax runs in base 2 and
// only rescales O when the running row maximum grows by more than 8 (a
// factor 256), which keeps every P <= 256 and the result exact.
#include <cudaTypedefs.h>

#include "band.cuh"
#include "kernels.cuh"
#include "sm100.cuh"
#include "warp_mma.cuh"

namespace relpos {

namespace {

using namespace sm100;

constexpr int kBQ = 128;          // rows per query tile (one softmax warpgroup)
constexpr int kBK = 128;          // keys per key tile (the tile-plan edge)
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = 128 * 128;   // one [128 x 64] 16-bit tile
constexpr uint32_t kOffQ = 0;
// A K/V stage: K tile, V tile, then the key tile's two saturated relation
// columns tau log2e Z^K[j, 0] and [j, R_exp - 1] (128 floats each).
constexpr uint32_t kColvBytes = 2 * kBK * 4;
constexpr uint32_t kStageBytes = 2 * kTileBytes + 1024;   // keeps every K/V tile 1024-byte aligned
constexpr uint32_t kOffKV = 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffKV + kStages * kStageBytes;
constexpr uint32_t kOffAbort = kOffBar + 256;
constexpr uint32_t kOffTmem = kOffAbort + 16;
constexpr uint32_t kSmemBytes = kOffTmem + 16 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;              // log2 of the largest P allowed before rescaling O

// barrier slots (8 bytes each)
constexpr int kBarQ = 0;
constexpr int kBarKvFull = 1;
constexpr int kBarKvEmpty = kBarKvFull + kStages;
constexpr int kBarSFull = kBarKvEmpty + kStages;   // 2: S_g written (MMA commit)
constexpr int kBarSFree = kBarSFull + 2;           // 2: S_g read into registers (128 arrivals)
constexpr int kBarPReady = kBarSFree + 2;          // 2: P_g written to tensor memory (128 arrivals)
constexpr int kBarPFree = kBarPReady + 2;          // 2: PV_g done: P_g buffer and O_g free (MMA commit)
constexpr int kBarDrain = kBarPFree + 2;

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


template <typename OutT> struct RowStore;
template <> struct RowStore<float> {
  static __device__ __forceinline__ void row(float* dst, const float* v) {
#pragma unroll
    for (int c = 0; c < 64; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
  }
};
template <typename T> struct RowStore {
  static __device__ __forceinline__ void row(T* dst, const float* v) {
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      uint4 u;
      u.x = DT<T>::pack(v[c], v[c + 1]);
      u.y = DT<T>::pack(v[c + 2], v[c + 3]);
      u.z = DT<T>::pack(v[c + 4], v[c + 5]);
      u.w = DT<T>::pack(v[c + 6], v[c + 7]);
      *reinterpret_cast<uint4*>(dst + c) = u;
    }
  }
};

template <typename T, typename OutT, bool AQ, bool AK, bool BIAS, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const Plan p, const Tensors t, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + kOffAbort);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sg + kOffTmem);
  auto bar = [&](int slot) { return sb + kOffBar + 8u * (uint32_t)slot; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  // causal: query tile pairs in descending order, the longest rows (most key
  // tiles) first, so that the last wave holds the shortest ones
  const int qpair = abs(p.qrev_pair - (int)blockIdx.x);
  const int N = p.N, q0 = qpair * (2 * kBQ);
  const SeqRows sr = seq_rows(p, b);   // this sequence's rows (the dense layout: all N)
  // keys j >= nkv are masked: the sequence length (packed), or the clamped key length
  const int nkv = p.packed ? sr.len : (p.padding ? iclamp(p.key_len[b], 0, N) : N);
  int kend = nkv;
  if (p.causal) kend = imin(kend, imin(q0 + 2 * kBQ, N));
  // nothing to do for query tiles past the sequence (packed batches)
  const int nkt = (kend > 0 && q0 < sr.len) ? (kend + kBK - 1) / kBK : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKvFull + s), 1);
      mbar_init(bar(kBarKvEmpty + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(kBarSFull + g), 1);
      mbar_init(bar(kBarSFree + g), 128);
      mbar_init(bar(kBarPReady + g), 128);
      mbar_init(bar(kBarPFree + g), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Register split: the launch gives every thread 168 registers (384 x 168 =
  // 64512); warpgroup 0 (producer, MMA issuer, allocator) drops to 56 and the
  // two softmax warpgroups take 224: 128 x 56 + 256 x 224 = 64512.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0 && nkt > 0) {
      // ---------------------------------------------------------- TMA producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(bar(kBarQ), 2 * kTileBytes);
      int c1, c2;
      tma_rows(p, sr, bh, h, q0, c1, c2);
      tma_load_3d(sb + kOffQ, &tmQ, bar(kBarQ), 0, c1, c2);
      tma_rows(p, sr, bh, h, q0 + kBQ, c1, c2);
      tma_load_3d(sb + kOffQ + kTileBytes, &tmQ, bar(kBarQ), 0, c1, c2);
      int issued = 0;
#pragma unroll 1
      for (int it = 0; it < nkt; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait(bar(kBarKvEmpty + s), ((it / kStages) - 1) & 1, abort_flag, p.wait_ns)) break;
        const uint32_t dst = sb + kOffKV + (uint32_t)s * kStageBytes;
        mbar_expect_tx(bar(kBarKvFull + s), 2 * kTileBytes + (AK ? kColvBytes : 0u));
        tma_rows(p, sr, bh, h, it * kBK, c1, c2);
        tma_load_3d(dst, &tmK, bar(kBarKvFull + s), 0, c1, c2);
        tma_load_3d(dst + kTileBytes, &tmV, bar(kBarKvFull + s), 0, c1, c2);
        if (AK) {
          const float* src = t.zk_sat + (size_t)bh * 2 * p.nT * kBK + (size_t)it * kBK;
          bulk_load(dst + 2 * kTileBytes, src, kBK * 4, bar(kBarKvFull + s));
          bulk_load(dst + 2 * kTileBytes + kBK * 4, src + (size_t)p.nT * kBK, kBK * 4, bar(kBarKvFull + s));
        }
        issued = it + 1;
      }
      // every load issued has landed before the CTA can exit (after an abort
      // the consumers may never have waited for them); each stage's last fill
      // is the latest phase of its barrier
      mbar_drain(bar(kBarQ), 0);
      for (int it = imax(0, issued - kStages); it < issued; ++it)
        mbar_drain(bar(kBarKvFull + it % kStages), (it / kStages) & 1);
    } else if (warp == 1 && lane == 0 && nkt > 0) {
      // ---------------------------------------------------------- MMA issuer
      // order per key tile t: S_0(t+1), S_1(t+1) as soon as S_g(t) has been
      // read, then PV_0(t), PV_1(t) as soon as P_g(t) is in shared memory
      const bool bf = t.is_bf16 != 0;
      const uint32_t id_qk = idesc_f16(bf, 128, 128, false, false);
      const uint32_t id_pv = idesc_f16(bf, 128, 64, false, true);
      // descriptors are built once; a K step inside a 128-byte swizzle atom
      // advances the start address by 32 bytes (+2 in the descriptor), a V
      // step by 16 keys = 2048 bytes (+128), a P step across atoms by 16 KB
      const uint64_t dq0 = sdesc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sb + kOffKV, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sb + kOffKV + kTileBytes, 8192, 1024);
      constexpr uint64_t kTile16 = kTileBytes >> 4, kStage16 = kStageBytes >> 4;
      auto issue_qk = [&](int g, int s) {
        const uint64_t a = dq0 + (uint64_t)g * kTile16;
        const uint64_t k = dk0 + (uint64_t)s * kStage16;
        const uint32_t d = tmem + (uint32_t)g * 128;
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk) mma_ss(d, a + 2 * kk, k + 2 * kk, id_qk, kk > 0);
      };
      // keys 16 kk .. 16 kk + 15 of P_g are its columns 8 kk .. 8 kk + 7
      auto issue_pv = [&](int g, int s, bool acc) {
        const uint64_t v = dv0 + (uint64_t)s * kStage16;
        const uint32_t pt = tmem + 384 + (uint32_t)g * 64;
        const uint32_t d = tmem + 256 + (uint32_t)g * 64;
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ts(d, pt + 8 * kk, v + 128 * kk, id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, p.wait_ns) && mbar_wait(bar(kBarKvFull + 0), 0, abort_flag, p.wait_ns);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(bar(kBarSFull + 0));
        issue_qk(1, 0);
        mma_commit(bar(kBarSFull + 1));
#pragma unroll 1
        for (int it = 0; it < nkt && ok; ++it) {
          const int s = it % kStages;
          if (it + 1 < nkt) {
            const int sn = (it + 1) % kStages;
            ok = mbar_wait(bar(kBarKvFull + sn), ((it + 1) / kStages) & 1, abort_flag, p.wait_ns);
            for (int g = 0; g < 2 && ok; ++g) {
              ok = mbar_wait(bar(kBarSFree + g), it & 1, abort_flag, p.wait_ns);
              if (!ok) break;
              tc_fence_after();
              issue_qk(g, sn);
              mma_commit(bar(kBarSFull + g));
            }
          }
          for (int g = 0; g < 2 && ok; ++g) {
            ok = mbar_wait(bar(kBarPReady + g), it & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_pv(g, s, it > 0);
            mma_commit(bar(kBarPFree + g));
          }
          if (ok) mma_commit(bar(kBarKvEmpty + s));
        }
      }
      {
        // drain: wait (bounded, ignoring the abort flag) until every issued MMA is
        // done, also when only the compute warps gave up, so that tensor memory is
        // never freed under a running MMA
        mma_commit(bar(kBarDrain));
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    // ------------------------------------------------------------ softmax
    const int g = (warp - 4) >> 2;
    const int wl = warp & 3;
    const int r = wl * 32 + lane;
    const int qtile = (q0 >> 7) + g;
    const int i = q0 + g * kBQ + r;
    const bool rok = i < sr.len;
    const uint32_t t_lane = (uint32_t)(wl * 32) << 16;
    const uint32_t tS = tmem + t_lane + (uint32_t)g * 128;
    const uint32_t tO = tmem + t_lane + 256 + (uint32_t)g * 64;
    const uint32_t tP = tmem + t_lane + 384 + (uint32_t)g * 64;
    const float sc = p.tau * kLog2e;
    // projection group of this query tile (the last one for a tile past N,
    // whose rows are all discarded); rows past N read row 0 (in bounds)
    const GroupInfo gi = p.gq[imin(qtile, p.nT - 1)];
    const int rrow = rok ? i - qtile * kBQ : 0;
    const float* zq_row = AQ ? t.zq + (size_t)bh * p.zq_head + gi.base + (long long)rrow * gi.S - gi.e0 : nullptr;
    float crow_lo = 0.f, crow_hi = 0.f;
    if (rok) {
      // saturated columns e = 0 / R_exp - 1 (present in the row's group whenever a
      // CONST tile can occur for it)
      if (AQ) {
        if (gi.e0 == 0) crow_lo += __ldg(zq_row);
        if (gi.e0 + gi.W >= p.Rexp) crow_hi += __ldg(zq_row + p.Rexp - 1);
      }
      if (BIAS) {
        crow_lo += __ldg(t.b_exp + (size_t)h * p.Rexp);
        crow_hi += __ldg(t.b_exp + (size_t)h * p.Rexp + p.Rexp - 1);
      }
    }
    crow_lo *= sc;
    crow_hi *= sc;
    const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int it = 0; it < nkt; ++it) {
      const int j0 = it * kBK;
      const int cls = tile_class(qtile, it, N, nkv, p.causal, p.E_lo, p.E_hi);
      const bool is_const = cls == RELPOS_TILE_CONST_LO || cls == RELPOS_TILE_CONST_HI;
      const int stage = it % kStages;
      const float* cv = reinterpret_cast<const float*>(sg + kOffKV + (uint32_t)stage * kStageBytes + 2 * kTileBytes) +
                        (cls == RELPOS_TILE_CONST_LO ? 0 : kBK);
      // every decision before a tcgen05.ld/st (warp-collective) is warp-uniform;
      // S ready implies the stage's TMA data landed, and waiting on the stage's
      // own barrier as well makes its saturated columns visible to these threads
      const bool got_s = mbar_wait(bar(kBarSFull + g), it & 1, abort_flag, p.wait_ns) &&
                         (!AK || mbar_wait(bar(kBarKvFull + stage), (it / kStages) & 1, abort_flag, p.wait_ns));
      if (!__all_sync(0xffffffffu, got_s)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      tmem_ld32(tS + 0, reinterpret_cast<uint32_t*>(x) + 0);
      tmem_ld32(tS + 32, reinterpret_cast<uint32_t*>(x) + 32);
      tmem_ld32(tS + 64, reinterpret_cast<uint32_t*>(x) + 64);
      tmem_ld32(tS + 96, reinterpret_cast<uint32_t*>(x) + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kBarSFree + g));    // the next key tile's S_g may now be written
      // x holds the scaled score (without the row constant rowc) in base 2;
      // for a saturated tile without key-side terms the scale is applied in
      // the exponent instead (xs = sc) to save one pass
      float rowc = 0.f, xs = 1.f;
      if (is_const) {
        rowc = cls == RELPOS_TILE_CONST_LO ? crow_lo : crow_hi;
        if (AK) {
          const float2 sc2 = make_float2(sc, sc);
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(cv + c);
            const float2 a = ffma2(make_float2(x[c], x[c + 1]), sc2, make_float2(v4.x, v4.y));
            const float2 b2 = ffma2(make_float2(x[c + 2], x[c + 3]), sc2, make_float2(v4.z, v4.w));
            x[c] = a.x; x[c + 1] = a.y; x[c + 2] = b2.x; x[c + 3] = b2.y;
          }
        } else {
          xs = sc;
        }
      } else {
        const float* zk_tile = nullptr;
        int zS = 0, ek0 = 0, ek1 = 0;
        if (AK) {
          const GroupInfo gk = p.gk[it];
          zk_tile = t.zk + (size_t)bh * p.zk_head + gk.base - gk.e0;
          zS = gk.S;
          ek0 = gk.e0;
          ek1 = gk.e0 + gk.W - 1;
        }
        // the float4 gather pays in the forward where q.aQ is the only per-row
        // gather (the identity map's Transformer-XL layer); beside the aK gather
        // its extra registers cost more than it saves
        if (AQ && !AK)
          band_terms_q_vec<AK, BIAS, 128>(x, p.E_lo, p.E_hi, i, lane, j0, 0, zq_row, gi.e0, gi.e0 + gi.W - 1, zk_tile,
                                          zS, imin(kBK, N - j0) - 1, ek0, ek1, bexp, sc);
        else
          band_terms_q<AQ, AK, BIAS, 128>(x, p.E_lo, p.E_hi, i, j0, 0, zq_row, gi.e0, gi.e0 + gi.W - 1, zk_tile, zS,
                                          imin(kBK, N - j0) - 1, ek0, ek1, bexp, sc);
      }
      const bool need_mask = (j0 + kBK > nkv) || (p.causal && j0 + kBK - 1 > q0 + g * kBQ);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = j0 + c;
          if (j >= nkv || (p.causal && j > i)) x[c] = -INFINITY;
        }
      }
      // 8 independent partial maxima (three-input max) keep the chains short
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = max3(x[u], x[u + 8], x[u + 16]);
#pragma unroll
      for (int c = 24; c < 128; c += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = max3(pm[u], x[c + u], c + 8 + u < 128 ? x[c + 8 + u] : pm[u]);
      }
      float mx = max3(max3(pm[0], pm[1], pm[2]), max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx = mx * xs + rowc;
      const float m_new = fmaxf(m_run, mx);
      // lazy rescale: only rows whose maximum grew by more than the threshold
      // move their reference point; O is touched by the whole warp once
      // PV of the previous key tile is done
      const bool grow = m_new > m_run + kRescaleThreshold;
      const float alpha = grow ? fast_exp2(m_run - m_new) : 1.f;
      bool pfree_seen = it == 0;
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        const bool got = mbar_wait(bar(kBarPFree + g), (it - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        pfree_seen = true;
        tc_fence_after();
        uint32_t ov[64];
        tmem_ld32(tO + 0, ov);
        tmem_ld32(tO + 32, ov + 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
        tmem_st32(tO + 0, ov);
        tmem_st32(tO + 32, ov + 32);
        tmem_wait_st();
      }
      if (grow) {
        l_run *= alpha;
        m_run = m_new;
      }
      // p = 2^(x * xs + rowc - m_run), packed two keys per word; the words go
      // to row r of P_g in tensor memory once the previous PV has read P_g,
      // so that PV overlaps these exponentials
      const float msub = m_run == -INFINITY ? 0.f : m_run - rowc;
      const float2 xs2 = make_float2(xs, xs), ms2 = make_float2(-msub, -msub);
      float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float ps[2] = {0.f, 0.f};
      uint32_t pk[64];
      uint32_t km[4] = {0u, 0u, 0u, 0u};   // dropout keep bits of the 128 keys
      if (DROP) {
        keep_mask64(p, bh, i, j0, true, *reinterpret_cast<uint32_t(*)[2]>(km));
        keep_mask64(p, bh, i, j0 + 64, true, *reinterpret_cast<uint32_t(*)[2]>(km + 2));
      }
#pragma unroll
      for (int w = 0; w < 64; ++w) {
        const float2 z = ffma2(make_float2(x[2 * w], x[2 * w + 1]), xs2, ms2);
        const float2 e = make_float2(fast_exp2(z.x), fast_exp2(z.y));
        pk[w] = DT<T>::pack(e.x, e.y);
        // bf16 keeps 8 bits: sum what PV really uses; fp16's rounding is small
        // enough to sum the fp32 values and spare the conversions.  The row sum
        // (hence LSE) is that of the undropped P.
        if (DT<T>::kCoarse) ps[w & 1] += DT<T>::pair_sum(pk[w]);
        else ps2[w & 1] = fadd2(ps2[w & 1], e);
        if (DROP) {
          // PV sees P o M; the epilogue scales O by 1 / (1 - p')
          const uint32_t kb = (km[w >> 4] >> (2 * (w & 15))) & 3u;
          pk[w] = DT<T>::pack((kb & 1u) ? e.x : 0.f, (kb & 2u) ? e.y : 0.f);
        }
      }
      l_run += DT<T>::kCoarse ? ps[0] + ps[1] : (ps2[0].x + ps2[1].x) + (ps2[0].y + ps2[1].y);
      if (!pfree_seen) {
        const bool got = mbar_wait(bar(kBarPFree + g), (it - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st32(tP, pk);
      tmem_st32(tP + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarPReady + g));
    }
    // ------------------------------------------------------------ epilogue
    float ov[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) ov[c] = 0.f;
    const bool got_o = nkt > 0 && ok && mbar_wait(bar(kBarPFree + g), (nkt - 1) & 1, abort_flag, p.wait_ns);
    if (__all_sync(0xffffffffu, got_o)) {
      tc_fence_after();
      uint32_t u[64];
      tmem_ld32(tO + 0, u);
      tmem_ld32(tO + 32, u + 32);
      tmem_wait_ld();
      // dropout: the kept P went to PV unscaled (the same 16-bit values the row
      // sum holds); 1 / (1 - p') is applied here
      const float inv = l_run > 0.f ? (DROP ? p.drop_scale : 1.f) / l_run : 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) ov[c] = __uint_as_float(u[c]) * inv;
    }
    if (rok) {
      OutT* O = static_cast<OutT*>(t.o) + act_row(p, sr, b, h, i) * 64;
      RowStore<OutT>::row(O, ov);
      t.lse[lse_index(p, sr, b, h, i)] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag && t.status) *t.status = kStatusTimeout;
}

}  // namespace

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// A 16-bit activation tensor viewed as 3-D for TMA, 128-row boxes with
// 128-byte swizzle: dense [B H, N, 64] as {64, N, B H}, rows past N read as
// zero; packed [T, H, 64] as {64, H, T} (box 64 x 1 x 128, monotonic
// strides), rows past T read as zero.  Either box lands in shared memory as
// 128 rows of 128 bytes.  Coordinates: tma_rows.
bool make_rows_map(CUtensorMap* m, const void* base, const Plan& p, bool bf16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)p.N, (cuuint64_t)p.B * p.H};
  cuuint64_t strides[2] = {128, (cuuint64_t)p.N * 128};
  cuuint32_t box[3] = {64, 128, 1};
  if (p.packed) {
    dims[1] = (cuuint64_t)p.H;
    dims[2] = (cuuint64_t)p.T;
    strides[1] = (cuuint64_t)p.H * 128;
    box[1] = 1;
    box[2] = 128;
  }
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <typename T, typename OutT>
cudaError_t launch_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  const int mask = (t.aq_exp ? 1 : 0) | (t.ak_exp ? 2 : 0) | (t.b_exp ? 4 : 0);
  void (*kern)(const Plan, const Tensors, const CUtensorMap, const CUtensorMap, const CUtensorMap) = nullptr;
  switch (mask + (p.dropout ? 8 : 0)) {
    case 0: kern = fwd_sm100_kernel<T, OutT, false, false, false, false>; break;
    case 1: kern = fwd_sm100_kernel<T, OutT, true, false, false, false>; break;
    case 2: kern = fwd_sm100_kernel<T, OutT, false, true, false, false>; break;
    case 3: kern = fwd_sm100_kernel<T, OutT, true, true, false, false>; break;
    case 4: kern = fwd_sm100_kernel<T, OutT, false, false, true, false>; break;
    case 5: kern = fwd_sm100_kernel<T, OutT, true, false, true, false>; break;
    case 6: kern = fwd_sm100_kernel<T, OutT, false, true, true, false>; break;
    case 7: kern = fwd_sm100_kernel<T, OutT, true, true, true, false>; break;
    case 8: kern = fwd_sm100_kernel<T, OutT, false, false, false, true>; break;
    case 9: kern = fwd_sm100_kernel<T, OutT, true, false, false, true>; break;
    case 10: kern = fwd_sm100_kernel<T, OutT, false, true, false, true>; break;
    case 11: kern = fwd_sm100_kernel<T, OutT, true, true, false, true>; break;
    case 12: kern = fwd_sm100_kernel<T, OutT, false, false, true, true>; break;
    case 13: kern = fwd_sm100_kernel<T, OutT, true, false, true, true>; break;
    case 14: kern = fwd_sm100_kernel<T, OutT, false, true, true, true>; break;
    default: kern = fwd_sm100_kernel<T, OutT, true, true, true, true>; break;
  }
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  const bool bf = t.is_bf16 != 0;
  if (!make_rows_map(&mq, t.q, p, bf) || !make_rows_map(&mk, t.k, p, bf) || !make_rows_map(&mv, t.v, p, bf))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + 2 * kBQ - 1) / (2 * kBQ), BH);
  { kern<<<grid, kThreads, kSmemBytes, s>>>(p, t, mq, mk, mv); note_launch(1); }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward(const Plan& p, const Tensors& t, cudaStream_t s) {
  if (t.is_bf16) {
    return t.o_f32 ? launch_typed<__nv_bfloat16, float>(p, t, s) : launch_typed<__nv_bfloat16, __nv_bfloat16>(p, t, s);
  }
  return t.o_f32 ? launch_typed<__half, float>(p, t, s) : launch_typed<__half, __half>(p, t, s);
}

}  // namespace relpos
