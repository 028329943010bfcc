// attn_bwd_sm100.cu -- two-pass backward of exact relative-position attention
// on sm_100a (digest of "Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels": backward section, Eq. (4), "constant tiles and
// the saturated region").
//
//   prep         D_i = sum_c dO_ic O_ic and LSE_i log2 e, padded to whole tiles
//   Q-parallel   one CTA per 128 query rows: S = Q K^T and dP = dO V^T on
//                tcgen05 into tensor memory, P = 2^(S' - LSE'), dS = P (dP - D)
//                in registers, dQ += dS K on tcgen05; the query-side relation
//                gradient is written by offset (one key per interior offset,
//                so a plain store by the row's owner) and the two saturated
//                offsets are summed on chip and stored once per row.
//   K-parallel   one CTA per 128 keys: S^T = K Q^T, dP^T = V dO^T,
//                dV += P^T dO, dK += dS^T Q, and the key-side relation
//                gradient by offset in the same single-writer way.
// No gradient entry has two writers: no atomics, fixed summation order.
//
// Pipelining (both passes): the score and dP GEMMs of tile t+1 are issued as
// soon as the compute warps have read tile t's S and dP out of tensor memory.
// Two compute warps share each row of the tile (its tensor-memory lane), one
// per 64-column half, and write the 16-bit P / dS operands of the next GEMMs
// back into tensor memory, where the TS-form GEMMs read them as their A
// operand.  Every mbarrier wait is bounded (see sm100.cuh).
#include <cudaTypedefs.h>

#include "band.cuh"
#include "kernels.cuh"
#include "sm100.cuh"
#include "warp_mma.cuh"

namespace relpos {

namespace {

using namespace sm100;

constexpr int kT = 128;                       // rows / keys per tile
constexpr uint32_t kTileBytes = 128 * 128;    // one [128 x 64] 16-bit tile
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}


// ------------------------------------------------------------------ prep
// dsum[bh][i] = sum_c dO_ic O_ic and lse2[bh][i] = LSE_i log2 e for i < N;
// rows past N (up to a whole tile) get D = 0 and LSE = +inf (so P = 0).  A
// row whose keys were all masked (LSE = -inf) also gets +inf.
template <typename OT, typename T>
__global__ void __launch_bounds__(256) prep_sm100_kernel(const Plan p, const OT* __restrict__ o,
                                                         const T* __restrict__ dout, const float* __restrict__ lse,
                                                         float* __restrict__ dsum, float* __restrict__ lse2,
                                                         int npad, long long BH) {
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gt >> 3;
  const int part = (int)(gt & 7);
  const long long bh = row / npad;
  const int i = (int)(row - bh * npad);
  const int b = (int)(bh / p.H), h = (int)(bh - (long long)b * p.H);
  SeqRows sr;
  sr.row0 = 0;
  sr.len = 0;
  if (bh < BH) sr = seq_rows(p, b);
  float acc = 0.f;
  // rows past the sequence get D = 0 and LSE = +inf, so P = 0 in both passes
  const bool ok = bh < BH && i < sr.len;
  if (ok) {
    const size_t off = (size_t)act_row(p, sr, b, h, i) * 64 + part * 8;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc += (float)o[off + c] * (float)dout[off + c];
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (bh < BH && part == 0) {
    dsum[row] = acc;
    float l2 = INFINITY;
    if (ok) {
      const float l = lse[lse_index(p, sr, b, h, i)];
      if (l != -INFINITY) l2 = l * kLog2e;
    }
    lse2[row] = l2;
  }
}

// ------------------------------------------------------------------ Q-parallel
namespace qp {
constexpr int kThreads = 384;                 // warps 0..3: TMA, MMA, TMEM alloc, idle; 4..11 compute
constexpr int kRegLaunch = 168, kRegLow = 72, kRegHigh = 208;
static_assert(128 * kRegLow + 256 * kRegHigh <= kThreads * kRegLaunch, "register split exceeds the launch");
constexpr int kStages = 4;
constexpr uint32_t kColvBytes = 2 * kT * 4;
constexpr uint32_t kStageBytes = 2 * kTileBytes + 1024;   // K, V, saturated key columns
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffDO = kTileBytes;
constexpr uint32_t kOffKV = 2 * kTileBytes;
// warp-private staging areas of BAND tiles: 16-bit dS rows for the by-offset store
constexpr uint32_t kOffStage = kOffKV + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffStage + 8 * kStageWarpBytes;
constexpr uint32_t kOffAbort = kOffBar + 256;
constexpr uint32_t kOffTmem = kOffAbort + 16;
constexpr uint32_t kOffSat = kOffTmem + 16;          // [128 rows][2] saturated sums of column half 1
constexpr uint32_t kSmemBytes = kOffSat + 1024 + 1024;
// tensor memory: S [0,128), dS buffers [128,192) and [192,256) (16-bit, two
// keys per column: the A operand of dQ += dS K; compute half hc owns columns
// 32 hc .. 32 hc + 31 of each), dP [256,384), dQ [384,448).  dS is double-
// buffered so that writing dS(t + 1) waits for dQ(t - 1), not dQ(t).
constexpr uint32_t kTmDS = 128, kTmDP = 256, kTmDQ = 384;
// barriers
constexpr int kBarQ = 0, kBarKvFull = 1, kBarKvEmpty = kBarKvFull + kStages, kBarSFull = kBarKvEmpty + kStages,
              kBarSFree = kBarSFull + 1, kBarDpFull = kBarSFree + 1, kBarDpFree = kBarDpFull + 1,
              // DsReady / DsFree: one per dS buffer.  With two buffers the compute
              // warps can finish tile t + 1 before the MMA issuer has waited for
              // tile t; per-buffer barriers keep every waiter within one phase.
              kBarDsReady = kBarDpFree + 1, kBarDsFree = kBarDsReady + 2, kBarDrain = kBarDsFree + 2;
}  // namespace qp

template <typename T, bool AQ, bool AK, bool BIAS, bool DZQ, bool DQ32, bool DROP>
__global__ void __launch_bounds__(qp::kThreads, 1)
    dq_sm100_kernel(const Plan p, const Tensors t, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmDO) {
  using namespace qp;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + kOffAbort);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sg + kOffTmem);
  auto bar = [&](int slot) { return sb + kOffBar + 8u * (uint32_t)slot; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // causal: query tiles in descending order, the longest rows first (the
  // K-parallel pass already starts with its longest key tiles)
  const int qt = abs(p.qrev - (int)blockIdx.x);
  const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, q0 = qt * kT;
  const int npad = p.nT * kT;
  const SeqRows sr = seq_rows(p, b);   // this sequence's rows (the dense layout: all N)
  // keys j >= nkv are masked: the sequence length (packed), or the clamped key length
  const int nkv = p.packed ? sr.len : (p.padding ? iclamp(p.key_len[b], 0, N) : N);
  int kend = nkv;
  if (p.causal) kend = imin(kend, imin(q0 + kT, N));
  // nothing to do for a query tile past the sequence (packed batches)
  const int nkt = (kend > 0 && q0 < sr.len) ? (kend + kT - 1) / kT : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKvFull + s), 1);
      mbar_init(bar(kBarKvEmpty + s), 1);
    }
    mbar_init(bar(kBarSFull), 1);
    mbar_init(bar(kBarSFree), 256);
    mbar_init(bar(kBarDpFull), 1);
    mbar_init(bar(kBarDpFree), 256);
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(kBarDsReady + u), 256);
      mbar_init(bar(kBarDsFree + u), 1);
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
  // 64512); warpgroup 0 (producer, MMA issuer, allocator) drops to kRegLow
  // and the two compute warpgroups take kRegHigh (the sum fits: static_assert).
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow) : "memory");
    if (warp == 0) {
      if (lane == 0 && nkt > 0) {
        // ------------------------------------------------------------ TMA producer
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmDO);
        mbar_expect_tx(bar(kBarQ), 2 * kTileBytes);
        int c1, c2;
        tma_rows(p, sr, bh, h, q0, c1, c2);
        tma_load_3d(sb + kOffQ, &tmQ, bar(kBarQ), 0, c1, c2);
        tma_load_3d(sb + kOffDO, &tmDO, bar(kBarQ), 0, c1, c2);
        int issued = 0;
  #pragma unroll 1
        for (int it = 0; it < nkt; ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(bar(kBarKvEmpty + s), ((it / kStages) - 1) & 1, abort_flag, p.wait_ns)) break;
          const uint32_t dst = sb + kOffKV + (uint32_t)s * kStageBytes;
          mbar_expect_tx(bar(kBarKvFull + s), 2 * kTileBytes + (AK ? kColvBytes : 0u));
          tma_rows(p, sr, bh, h, it * kT, c1, c2);
          tma_load_3d(dst, &tmK, bar(kBarKvFull + s), 0, c1, c2);
          tma_load_3d(dst + kTileBytes, &tmV, bar(kBarKvFull + s), 0, c1, c2);
          if (AK) {
            const float* src = t.zk_sat + (size_t)bh * 2 * npad + (size_t)it * kT;
            bulk_load(dst + 2 * kTileBytes, src, kT * 4, bar(kBarKvFull + s));
            bulk_load(dst + 2 * kTileBytes + kT * 4, src + npad, kT * 4, bar(kBarKvFull + s));
          }
          issued = it + 1;
        }
        // no load may still be landing when the CTA exits (see the forward)
        mbar_drain(bar(kBarQ), 0);
        for (int it = imax(0, issued - kStages); it < issued; ++it)
          mbar_drain(bar(kBarKvFull + it % kStages), (it / kStages) & 1);
      }
    } else if (warp == 1) {
      if (lane == 0 && nkt > 0) {
        // ------------------------------------------------------------ MMA issuer
        // per tile t: S(t+1) once S(t) has been read, dP(t+1) once dP(t) has
        // been read, dQ += dS(t) K(t) once dS(t) is in its tensor-memory buffer
        const bool bf = t.is_bf16 != 0;
        const uint32_t id_s = idesc_f16(bf, 128, 128, false, false);
        const uint32_t id_dq = idesc_f16(bf, 128, 64, false, true);
        const uint64_t dq0 = sdesc_sw128(sb + kOffQ, 16, 1024);
        const uint64_t ddo0 = sdesc_sw128(sb + kOffDO, 16, 1024);
        const uint64_t dk0 = sdesc_sw128(sb + kOffKV, 16, 1024);
        const uint64_t dv0 = sdesc_sw128(sb + kOffKV + kTileBytes, 16, 1024);
        const uint64_t dkmn0 = sdesc_sw128(sb + kOffKV, 8192, 1024);
        constexpr uint64_t kStage16 = kStageBytes >> 4;
        auto issue_s = [&](int s) {
          const uint64_t kd = dk0 + (uint64_t)s * kStage16;
  #pragma unroll 1
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem, dq0 + 2 * kk, kd + 2 * kk, id_s, kk > 0);
        };
        auto issue_dp = [&](int s) {
          const uint64_t vd = dv0 + (uint64_t)s * kStage16;
  #pragma unroll 1
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kTmDP, ddo0 + 2 * kk, vd + 2 * kk, id_s, kk > 0);
        };
        // keys 16 kk .. 16 kk + 15 of dS are columns 8 kk .. 8 kk + 7 of its buffer
        auto issue_dq = [&](int s, int db, bool acc) {
          const uint64_t kd = dkmn0 + (uint64_t)s * kStage16;
          const uint32_t a = tmem + kTmDS + 64u * (uint32_t)db;
  #pragma unroll 1
          for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + kTmDQ, a + 8 * kk, kd + 128 * kk, id_dq, (acc || kk > 0) ? 1u : 0u);
        };
        bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, p.wait_ns) && mbar_wait(bar(kBarKvFull + 0), 0, abort_flag, p.wait_ns);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          mma_commit(bar(kBarSFull));
          issue_dp(0);
          mma_commit(bar(kBarDpFull));
        }
  #pragma unroll 1
        for (int it = 0; it < nkt && ok; ++it) {
          const int s = it % kStages, s1 = (it + 1) % kStages;
          if (it + 1 < nkt) {
            ok = mbar_wait(bar(kBarKvFull + s1), ((it + 1) / kStages) & 1, abort_flag, p.wait_ns) &&
                 mbar_wait(bar(kBarSFree), it & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_s(s1);
            mma_commit(bar(kBarSFull));
            ok = mbar_wait(bar(kBarDpFree), it & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_dp(s1);
            mma_commit(bar(kBarDpFull));
          }
          ok = mbar_wait(bar(kBarDsReady + (it & 1)), (it >> 1) & 1, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_dq(s, it & 1, it > 0);
          mma_commit(bar(kBarDsFree + (it & 1)));
          mma_commit(bar(kBarKvEmpty + s));
        }
        {
          // drain (bounded): no MMA may still run when tensor memory is freed
          mma_commit(bar(kBarDrain));
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh) : "memory");
    // -------------------------------------------------------------- compute
    // warps 4..7 take key columns 0..63 of the tile, warps 8..11 columns
    // 64..127, both for rows r = (warp & 3) * 32 + lane (the tensor-memory lane)
    const int hc = (warp - 4) >> 2;
    const int cb = 64 * hc;
    const int r = (warp & 3) * 32 + lane;
    const int i = q0 + r;
    const bool rok = i < sr.len;
    const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
    const float sc = p.tau * kLog2e;
    const size_t prow = (size_t)bh * npad + q0 + r;
    const float lse2 = t.lse2[prow];
    const float dval = t.dsum[prow];
    // saturated-offset row constants tau log2e (Z^Q[i, sat] + b_sat) - LSE_i log2e
    // (-inf for rows without a probability)
    const float crow_lo = (AQ || BIAS) ? t.zq_sat[(size_t)bh * 2 * npad + q0 + r] : 0.f;
    const float crow_hi = (AQ || BIAS) ? t.zq_sat[(size_t)bh * 2 * npad + npad + q0 + r] : 0.f;
    // projection group of this query tile; rows past N use row 0 (in bounds)
    const GroupInfo gi = p.gq[qt];
    const int rrow = rok ? r : 0;
    T* dzq_base = DZQ ? static_cast<T*>(t.dzq) + (size_t)bh * p.zq_head + gi.base : nullptr;
    const int nrows_q = imin(kT, N - q0);
    const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
    T* stg = reinterpret_cast<T*>(sg + kOffStage + (uint32_t)(warp - 4) * kStageWarpBytes);
    const float* zq_row = AQ ? t.zq + (size_t)bh * p.zq_head + gi.base + (long long)rrow * gi.S - gi.e0 : nullptr;
    float sat_lo = 0.f, sat_hi = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int it = 0; it < nkt; ++it) {
      const int j0 = it * kT;
      // class of this half's 64 keys: the two halves of a tile on the edge of
      // the band often differ (one BAND, one CONST).  Bias-only variants keep
      // the tile's class (their band is wider than a half for the maps here,
      // and the extra live values make that variant spill).
      const int cls = (AQ || AK) ? half_class(qt, it, hc, true, N, nkv, p.causal, p.E_lo, p.E_hi)
                                 : tile_class(qt, it, N, nkv, p.causal, p.E_lo, p.E_hi);
      const bool is_const = cls == RELPOS_TILE_CONST_LO || cls == RELPOS_TILE_CONST_HI;
      const int stage = it % kStages;
      const float* cv = reinterpret_cast<const float*>(sg + kOffKV + (uint32_t)stage * kStageBytes + 2 * kTileBytes) +
                        (cls == RELPOS_TILE_CONST_LO ? 0 : kT) + cb;
      const bool got_s = mbar_wait(bar(kBarSFull), it & 1, abort_flag, p.wait_ns) &&
                         (!(AK && is_const) || mbar_wait(bar(kBarKvFull + stage), (it / kStages) & 1, abort_flag, p.wait_ns));
      if (!__all_sync(0xffffffffu, got_s)) { ok = false; break; }
      tc_fence_after();
      float x[64];
      {
        const uint32_t ts = tmem + t_lane + cb;
        tmem_ld32(ts + 0, reinterpret_cast<uint32_t*>(x) + 0);
        tmem_ld32(ts + 32, reinterpret_cast<uint32_t*>(x) + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(kBarSFree));   // S(t + 1) may now be written
      // P = 2^(S tau log2e + relation terms - LSE log2e)
      if (is_const) {
        const float off = (AQ || BIAS) ? (cls == RELPOS_TILE_CONST_LO ? crow_lo : crow_hi) : -lse2;
        // paired fp32 arithmetic: one instruction per two scores
        const float2 sc2 = make_float2(sc, sc), off2 = make_float2(off, off);
        if (AK) {
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(cv + c);
            const float2 z0 = ffma2(make_float2(x[c], x[c + 1]), sc2, fadd2(make_float2(v4.x, v4.y), off2));
            const float2 z1 = ffma2(make_float2(x[c + 2], x[c + 3]), sc2, fadd2(make_float2(v4.z, v4.w), off2));
            x[c] = fast_exp2(z0.x);
            x[c + 1] = fast_exp2(z0.y);
            x[c + 2] = fast_exp2(z1.x);
            x[c + 3] = fast_exp2(z1.y);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 z = ffma2(make_float2(x[c], x[c + 1]), sc2, off2);
            x[c] = fast_exp2(z.x);
            x[c + 1] = fast_exp2(z.y);
          }
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
        if (AQ)
          band_terms_q_vec<AK, BIAS, 64>(x, p.E_lo, p.E_hi, i, lane, j0, cb, zq_row, gi.e0, gi.e0 + gi.W - 1, zk_tile,
                                         zS, imin(kT, N - j0) - 1, ek0, ek1, bexp, sc);
        else
          band_terms_q<AQ, AK, BIAS, 64>(x, p.E_lo, p.E_hi, i, j0, cb, zq_row, gi.e0, gi.e0 + gi.W - 1, zk_tile, zS,
                                         imin(kT, N - j0) - 1, ek0, ek1, bexp, sc);
        const float2 nl2 = make_float2(-lse2, -lse2);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 z = fadd2(make_float2(x[c], x[c + 1]), nl2);
          x[c] = fast_exp2(z.x);
          x[c + 1] = fast_exp2(z.y);
        }
      }
      const bool need_mask = (j0 + kT > nkv) || (p.causal && j0 + kT - 1 > q0);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int j = j0 + cb + c;
          if (j >= nkv || (p.causal && j > i)) x[c] = 0.f;
        }
      }
      // dS = P (dP - D) for this thread's 64 keys; written as the 16-bit A
      // operand of dQ += dS K
      const bool got_dp = mbar_wait(bar(kBarDpFull), it & 1, abort_flag, p.wait_ns);
      if (!__all_sync(0xffffffffu, got_dp)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t dp[64];
        const uint32_t td = tmem + t_lane + kTmDP + cb;
        tmem_ld32(td, dp);
        tmem_ld32(td + 32, dp + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(kBarDpFree));     // dP(t + 1) may now be written
        if (DROP) {
          // dropout: dS = P o (M / (1 - p') o dP - D)
          uint32_t km[2];
          keep_mask64(p, bh, i, j0 + cb, true, km);
#pragma unroll
          for (int w = 0; w < 32; ++w) {
            const uint32_t kb = (km[w >> 4] >> (2 * (w & 15))) & 3u;
            dp[2 * w] = __float_as_uint((kb & 1u) ? __uint_as_float(dp[2 * w]) * p.drop_scale : 0.f);
            dp[2 * w + 1] = __float_as_uint((kb & 2u) ? __uint_as_float(dp[2 * w + 1]) * p.drop_scale : 0.f);
          }
        }
        if (!DZQ || is_const) {
          float2 ssum = make_float2(0.f, 0.f);
          const float2 nd2 = make_float2(-dval, -dval);
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 ds = fmul2(make_float2(x[c], x[c + 1]),
                                    fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nd2));
            x[c] = ds.x;
            x[c + 1] = ds.y;
            if (DZQ) ssum = fadd2(ssum, ds);
          }
          if (DZQ) {
            if (cls == RELPOS_TILE_CONST_LO) sat_lo += ssum.x + ssum.y;
            else sat_hi += ssum.x + ssum.y;
          }
        } else if (j0 + cb - (i - lane) - 31 > p.E_lo && j0 + cb + 63 - (i - lane) < p.E_hi) {
          // every offset of the warp's 32 rows x 64 keys interior (warp-uniform):
          // nothing saturated to sum, all entries stored below
          const float2 nd2 = make_float2(-dval, -dval);
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 ds = fmul2(make_float2(x[c], x[c + 1]),
                                    fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nd2));
            x[c] = ds.x;
            x[c + 1] = ds.y;
          }
        } else {
          // saturated cells summed here; the interior ones are stored below.
          // Kept keys are cc <= ckeep (cc = key - j0); low-saturated cc <= clo, high cc >= chi.
          int ckeep = rok ? imin(nkv - 1 - j0, 127) : -1;
          if (p.causal) ckeep = imin(ckeep, i - j0);
          const int clo = imin(p.E_lo + i - j0, ckeep);
          const int chi = imax(p.E_hi + i - j0, p.E_lo + i - j0 + 1);
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int cc = cb + c;
            const float ds = x[c] * (__uint_as_float(dp[c]) - dval);
            x[c] = ds;
            sat_lo += cc <= clo ? ds : 0.f;
            sat_hi += (cc >= chi && cc <= ckeep) ? ds : 0.f;
          }
        }
      }
      // dS buffer (t & 1) is free once dQ(t - 2) has read it
      if (it > 1) {
        const bool got = mbar_wait(bar(kBarDsFree + (it & 1)), ((it >> 1) - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
      }
      // this half's 64 keys of dS, two per tensor-memory column
      {
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) pk[u] = DT<T>::pack(x[2 * u], x[2 * u + 1]);
        tmem_st32(tmem + t_lane + kTmDS + 64u * (uint32_t)(it & 1) + 32 * hc, pk);
        if (DZQ && !is_const) {
          // BAND tile: the same 16-bit values also go to the warp's staging
          // area (its own rows) for the coalesced by-offset store below
          __syncwarp();
          const uint32_t row16 = smem_u32(stg) + (uint32_t)(lane * kDsPitch) * 2u;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) st_shared_v4(row16 + 16u * ch, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        tmem_wait_st();
      }
      if (DZQ && !is_const) {
        __syncwarp();
        dz_band_store<T>(stg, (warp & 3) * 32, lane, false, q0, j0, cb, nrows_q, nkv, N,
                         p.causal, p.E_lo, p.E_hi, dzq_base, gi.S, gi.e0);
      }
      tc_fence_before();
      mbar_arrive(bar(kBarDsReady + (it & 1)));
    }
    // -------------------------------------------------------------- epilogue
    if (DZQ) {
      // combine the two column halves' saturated sums; half 0 writes them
      float* sat = reinterpret_cast<float*>(sg + kOffSat);
      if (hc == 1) {
        sat[2 * r] = sat_lo;
        sat[2 * r + 1] = sat_hi;
      }
      named_bar_sync(1, 256);
      if (hc == 0 && rok)
        *reinterpret_cast<float2*>(t.dzq_sat + 2 * prow) = make_float2(sat_lo + sat[2 * r], sat_hi + sat[2 * r + 1]);
    }
    // dQ: half hc stores head-dim columns [32 hc, 32 hc + 32) of its row
    float dq[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) dq[c] = 0.f;
    // the last dQ GEMM's commit covers every earlier one
    const bool got_q = nkt > 0 && ok && mbar_wait(bar(kBarDsFree + ((nkt - 1) & 1)), ((nkt - 1) >> 1) & 1, abort_flag, p.wait_ns);
    if (__all_sync(0xffffffffu, got_q)) {
      tc_fence_after();
      uint32_t u[32];
      tmem_ld32(tmem + t_lane + kTmDQ + 32 * hc, u);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) dq[c] = __uint_as_float(u[c]) * p.tau;
    }
    if (rok) {
      if (DQ32) {
        // the fp32 accumulator keeps the workspace's dense layout
        float* dst = t.dq_acc + ((size_t)bh * N + i) * 64 + 32 * hc;
#pragma unroll
        for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(dq[c], dq[c + 1], dq[c + 2], dq[c + 3]);
      } else {
        T* dst = static_cast<T*>(t.dq) + act_row(p, sr, b, h, i) * 64 + 32 * hc;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint4 w;
          w.x = DT<T>::pack(dq[c], dq[c + 1]);
          w.y = DT<T>::pack(dq[c + 2], dq[c + 3]);
          w.z = DT<T>::pack(dq[c + 4], dq[c + 5]);
          w.w = DT<T>::pack(dq[c + 6], dq[c + 7]);
          *reinterpret_cast<uint4*>(dst + c) = w;
        }
      }
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

// ------------------------------------------------------------------ K-parallel
namespace kp {
constexpr int kThreads = 384;                 // warps 0..3: TMA, MMA, TMEM alloc, idle; 4..11 compute
constexpr int kRegLaunch = 168, kRegLow = 88, kRegHigh = 208;
static_assert(128 * kRegLow + 256 * kRegHigh <= kThreads * kRegLaunch, "register split exceeds the launch");
constexpr int kStages = 3;
// a stage: Q tile, dO tile, then LSE log2e, D and the two saturated query
// columns (tau log2e (Z^Q[i, sat] + b_sat)) of the query tile, 128 floats each
constexpr uint32_t kVecBytes = 4 * kT * 4;
constexpr uint32_t kStageBytes = 2 * kTileBytes + 2048;
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kTileBytes;
constexpr uint32_t kOffQD = 2 * kTileBytes;
// warp-private staging areas of BAND tiles: 16-bit dS^T rows for the by-offset store
constexpr uint32_t kOffStage = kOffQD + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffStage + 8 * kStageWarpBytes;
constexpr uint32_t kOffAbort = kOffBar + 256;
constexpr uint32_t kOffTmem = kOffAbort + 16;
constexpr uint32_t kOffSat = kOffTmem + 16;          // [128 keys][2] saturated sums of column half 1
constexpr uint32_t kSmemBytes = kOffSat + 1024 + 1024;
// tensor memory: S^T [0,128), P^T [128,192), dS^T [192,256), dP^T [256,384),
// dV [384,448), dK [448,512).  P^T and dS^T are 16-bit, two queries per
// column; compute half hc (queries 64 hc .. 64 hc + 63) owns columns
// 32 hc .. 32 hc + 31 of each.  They are the A operands of dV += P^T dO and
// dK += dS^T Q.  Every region a GEMM reads is rewritten only after a commit
// that follows that GEMM (PFree, DsFree), and every region the compute warps
// read is rewritten by a GEMM only after their arrival (SFree, DpFree).
constexpr uint32_t kTmP = 128, kTmDS = 192, kTmDP = 256, kTmDV = 384, kTmDK = 448;
constexpr int kBarKV = 0, kBarQsFull = 1, kBarQsEmpty = kBarQsFull + kStages, kBarSFull = kBarQsEmpty + kStages,
              kBarSFree = kBarSFull + 1, kBarDpFull = kBarSFree + 1, kBarDpFree = kBarDpFull + 1,
              kBarPReady = kBarDpFree + 1, kBarPFree = kBarPReady + 1, kBarDsReady = kBarPFree + 1,
              kBarDsFree = kBarDsReady + 1, kBarDrain = kBarDsFree + 1;
}  // namespace kp

// VEC (with aK, for a wide interior band): the BAND tiles' k.aK gathers of a
// key's own Z^K row read aligned float4 pieces where a chunk is all interior
// (band_terms_k_vec); a narrow band, as Shaw clip 64's, has few such chunks and
// keeps the plain gather (a separate instantiation, chosen by the host).
template <typename T, bool AQ, bool AK, bool BIAS, bool DZK, bool DK32, bool DROP, bool VEC>
__global__ void __launch_bounds__(kp::kThreads, 1)
    dkdv_sm100_kernel(const Plan p, const Tensors t, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmDO) {
  using namespace kp;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + kOffAbort);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sg + kOffTmem);
  auto bar = [&](int slot) { return sb + kOffBar + 8u * (uint32_t)slot; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, k0 = kt * kT;
  const int npad = p.nT * kT;
  const SeqRows sr = seq_rows(p, b);   // this sequence's rows (the dense layout: all N)
  // keys j >= nkv are masked: the sequence length (packed), or the clamped key length
  const int nkv = p.packed ? sr.len : (p.padding ? iclamp(p.key_len[b], 0, N) : N);
  const int qt0 = p.causal ? kt : 0;            // queries i >= j only under the causal mask
  const int nq = k0 < nkv ? p.nT - qt0 : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarKV), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarQsFull + s), 1);
      mbar_init(bar(kBarQsEmpty + s), 1);
    }
    mbar_init(bar(kBarSFull), 1);
    mbar_init(bar(kBarSFree), 256);
    mbar_init(bar(kBarDpFull), 1);
    mbar_init(bar(kBarDpFree), 256);
    mbar_init(bar(kBarPReady), 256);
    mbar_init(bar(kBarPFree), 1);
    mbar_init(bar(kBarDsReady), 256);
    mbar_init(bar(kBarDsFree), 1);
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
  // 64512); warpgroup 0 (producer, MMA issuer, allocator) drops to kRegLow
  // and the two compute warpgroups take kRegHigh (the sum fits: static_assert).
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow) : "memory");
    if (warp == 0) {
      if (lane == 0 && nq > 0) {
        // ------------------------------------------------------------ TMA producer
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmDO);
        mbar_expect_tx(bar(kBarKV), 2 * kTileBytes);
        int c1, c2;
        tma_rows(p, sr, bh, h, k0, c1, c2);
        tma_load_3d(sb + kOffK, &tmK, bar(kBarKV), 0, c1, c2);
        tma_load_3d(sb + kOffV, &tmV, bar(kBarKV), 0, c1, c2);
        int issued = 0;
  #pragma unroll 1
        for (int it = 0; it < nq; ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(bar(kBarQsEmpty + s), ((it / kStages) - 1) & 1, abort_flag, p.wait_ns)) break;
          const int qb = (qt0 + it) * kT;
          const uint32_t dst = sb + kOffQD + (uint32_t)s * kStageBytes;
          const uint32_t fb = bar(kBarQsFull + s);
          mbar_expect_tx(fb, 2 * kTileBytes + ((AQ || BIAS) ? kVecBytes : kVecBytes / 2));
          tma_rows(p, sr, bh, h, qb, c1, c2);
          tma_load_3d(dst, &tmQ, fb, 0, c1, c2);
          tma_load_3d(dst + kTileBytes, &tmDO, fb, 0, c1, c2);
          const size_t vo = (size_t)bh * npad + qb;
          bulk_load(dst + 2 * kTileBytes, t.lse2 + vo, kT * 4, fb);
          bulk_load(dst + 2 * kTileBytes + kT * 4, t.dsum + vo, kT * 4, fb);
          if (AQ || BIAS) {
            const float* src = t.zq_sat + (size_t)bh * 2 * npad + qb;
            bulk_load(dst + 2 * kTileBytes + 2 * kT * 4, src, kT * 4, fb);
            bulk_load(dst + 2 * kTileBytes + 3 * kT * 4, src + npad, kT * 4, fb);
          }
          issued = it + 1;
        }
        // no load may still be landing when the CTA exits (see the forward)
        mbar_drain(bar(kBarKV), 0);
        for (int it = imax(0, issued - kStages); it < issued; ++it)
          mbar_drain(bar(kBarQsFull + it % kStages), (it / kStages) & 1);
      }
    } else if (warp == 1) {
      if (lane == 0 && nq > 0) {
        // ------------------------------------------------------------ MMA issuer
        const bool bf = t.is_bf16 != 0;
        const uint32_t id_s = idesc_f16(bf, 128, 128, false, false);
        const uint32_t id_g = idesc_f16(bf, 128, 64, false, true);
        const uint64_t dk = sdesc_sw128(sb + kOffK, 16, 1024);
        const uint64_t dv = sdesc_sw128(sb + kOffV, 16, 1024);
        const uint64_t dq0 = sdesc_sw128(sb + kOffQD, 16, 1024);
        const uint64_t ddo0 = sdesc_sw128(sb + kOffQD + kTileBytes, 16, 1024);
        const uint64_t dqmn0 = sdesc_sw128(sb + kOffQD, 8192, 1024);
        const uint64_t ddomn0 = sdesc_sw128(sb + kOffQD + kTileBytes, 8192, 1024);
        constexpr uint64_t kStage16 = kStageBytes >> 4;
        auto issue_s = [&](int s) {
          const uint64_t qd = dq0 + (uint64_t)s * kStage16;
  #pragma unroll 1
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem, dk + 2 * kk, qd + 2 * kk, id_s, kk > 0);
        };
        auto issue_dp = [&](int s) {
          const uint64_t od = ddo0 + (uint64_t)s * kStage16;
  #pragma unroll 1
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kTmDP, dv + 2 * kk, od + 2 * kk, id_s, kk > 0);
        };
        // D[keys x 64] (+)= A[keys x queries] (tensor memory at a, queries
        // 16 kk .. 16 kk + 15 in columns 8 kk .. 8 kk + 7) * B[queries x 64] (MN-major)
        auto issue_g = [&](uint32_t d, uint32_t a, uint64_t bmn, bool acc) {
  #pragma unroll 1
          for (int kk = 0; kk < 8; ++kk) mma_ts(d, a + 8 * kk, bmn + 128 * kk, id_g, (acc || kk > 0) ? 1u : 0u);
        };
        bool ok = mbar_wait(bar(kBarKV), 0, abort_flag, p.wait_ns) && mbar_wait(bar(kBarQsFull + 0), 0, abort_flag, p.wait_ns);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          mma_commit(bar(kBarSFull));
          issue_dp(0);
          mma_commit(bar(kBarDpFull));
        }
        // per tile t: S(t+1) once S(t) has been read, dV(t) once P^T(t) is
        // written, dP(t+1) once dP(t) has been read, dK(t) once dS^T(t) is written
  #pragma unroll 1
        for (int it = 0; it < nq && ok; ++it) {
          const int s = it % kStages, s1 = (it + 1) % kStages;
          if (it + 1 < nq) {
            ok = mbar_wait(bar(kBarQsFull + s1), ((it + 1) / kStages) & 1, abort_flag, p.wait_ns) &&
                 mbar_wait(bar(kBarSFree), it & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_s(s1);
            mma_commit(bar(kBarSFull));
          }
          ok = mbar_wait(bar(kBarPReady), it & 1, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_g(tmem + kTmDV, tmem + kTmP, ddomn0 + (uint64_t)s * kStage16, it > 0);
          mma_commit(bar(kBarPFree));
          if (it + 1 < nq) {
            ok = mbar_wait(bar(kBarDpFree), it & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_dp(s1);
            mma_commit(bar(kBarDpFull));
          }
          ok = mbar_wait(bar(kBarDsReady), it & 1, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_g(tmem + kTmDK, tmem + kTmDS, dqmn0 + (uint64_t)s * kStage16, it > 0);
          mma_commit(bar(kBarDsFree));
          mma_commit(bar(kBarQsEmpty + s));
        }
        {
          // drain (bounded): no MMA may still run when tensor memory is freed
          mma_commit(bar(kBarDrain));
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh) : "memory");
    // -------------------------------------------------------------- compute
    // warps 4..7 take query columns 0..63 of the tile, warps 8..11 columns
    // 64..127, both for keys r = (warp & 3) * 32 + lane (the tensor-memory lane)
    const int hc = (warp - 4) >> 2;
    const int cb = 64 * hc;
    const int r = (warp & 3) * 32 + lane;
    const int j = k0 + r;
    const bool jok = j < sr.len;
    const bool jkeep = j < nkv;                  // keys past key_len are masked for every query
    const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
    const float sc = p.tau * kLog2e;
    // saturated-offset row constants tau log2e Z^K[j, sat] (zero past N)
    const float rowk_lo = AK ? t.zk_sat[(size_t)bh * 2 * npad + k0 + r] : 0.f;
    const float rowk_hi = AK ? t.zk_sat[(size_t)bh * 2 * npad + npad + k0 + r] : 0.f;
    // projection group of this key tile; keys past N use row 0 (in bounds)
    const GroupInfo gk = p.gk[kt];
    const int krow = jok ? r : 0;
    T* dzk_base = DZK ? static_cast<T*>(t.dzk) + (size_t)bh * p.zk_head + gk.base : nullptr;
    const int nrows_k = imin(kT, N - k0);
    const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
    T* stg = reinterpret_cast<T*>(sg + kOffStage + (uint32_t)(warp - 4) * kStageWarpBytes);
    const float* zk_row = AK ? t.zk + (size_t)bh * p.zk_head + gk.base + (long long)krow * gk.S - gk.e0 : nullptr;
    float sat_lo = 0.f, sat_hi = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int it = 0; it < nq; ++it) {
      const int qi = qt0 + it, qb = qi * kT;
      // class of this half's 64 queries (bias-only variants: the tile's class)
      const int cls = (AQ || AK) ? half_class(qi, kt, hc, false, N, nkv, p.causal, p.E_lo, p.E_hi)
                                 : tile_class(qi, kt, N, nkv, p.causal, p.E_lo, p.E_hi);
      const bool is_const = cls == RELPOS_TILE_CONST_LO || cls == RELPOS_TILE_CONST_HI;
      const int stage = it % kStages;
      const float* vec = reinterpret_cast<const float*>(sg + kOffQD + (uint32_t)stage * kStageBytes + 2 * kTileBytes);
      const float* lse2v = vec + cb;
      const float* dvec = vec + kT + cb;
      const float* cvq = vec + (cls == RELPOS_TILE_CONST_LO ? 2 * kT : 3 * kT) + cb;
      // the stage's own barrier makes its TMA-written vectors visible to these threads
      const bool got_s = mbar_wait(bar(kBarSFull), it & 1, abort_flag, p.wait_ns) &&
                         mbar_wait(bar(kBarQsFull + stage), (it / kStages) & 1, abort_flag, p.wait_ns);
      if (!__all_sync(0xffffffffu, got_s)) { ok = false; break; }
      tc_fence_after();
      float x[64];
      {
        const uint32_t ts = tmem + t_lane + cb;
        tmem_ld32(ts + 0, reinterpret_cast<uint32_t*>(x) + 0);
        tmem_ld32(ts + 32, reinterpret_cast<uint32_t*>(x) + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(kBarSFree));   // S(t + 1) may now be written
      // P^T = 2^(S^T tau log2e + relation terms - LSE_i log2e), column c = query qb + cb + c
      if (is_const) {
        const float rowk = cls == RELPOS_TILE_CONST_LO ? rowk_lo : rowk_hi;
        // paired fp32 arithmetic: one instruction per two scores
        const float2 sc2 = make_float2(sc, sc), rk2 = make_float2(rowk, rowk);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          // per query: the staged saturated column already holds its relation terms
          // minus LSE log2e; without them it is -LSE log2e
          float2 w0, w1;
          if (AQ || BIAS) {
            const float4 c4 = *reinterpret_cast<const float4*>(cvq + c);
            w0 = fadd2(rk2, make_float2(c4.x, c4.y));
            w1 = fadd2(rk2, make_float2(c4.z, c4.w));
          } else {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2v + c);
            w0 = fadd2(rk2, make_float2(-l4.x, -l4.y));
            w1 = fadd2(rk2, make_float2(-l4.z, -l4.w));
          }
          const float2 z0 = ffma2(make_float2(x[c], x[c + 1]), sc2, w0);
          const float2 z1 = ffma2(make_float2(x[c + 2], x[c + 3]), sc2, w1);
          x[c] = fast_exp2(z0.x);
          x[c + 1] = fast_exp2(z0.y);
          x[c + 2] = fast_exp2(z1.x);
          x[c + 3] = fast_exp2(z1.y);
        }
      } else {
        const float* zq_tile = nullptr;
        int zS = 0, eq0 = 0, eq1 = 0;
        if (AQ) {
          const GroupInfo gq = p.gq[qi];
          zq_tile = t.zq + (size_t)bh * p.zq_head + gq.base - gq.e0;
          zS = gq.S;
          eq0 = gq.e0;
          eq1 = gq.e0 + gq.W - 1;
        }
        if (AK && VEC)
          band_terms_k_vec<AQ, BIAS, 64>(x, p.E_lo, p.E_hi, j, qb, cb, zk_row, gk.e0, gk.e0 + gk.W - 1, zq_tile, zS,
                                         imin(kT, N - qb) - 1, eq0, eq1, bexp, sc);
        else
          band_terms_k<AQ, AK, BIAS, 64>(x, p.E_lo, p.E_hi, j, qb, cb, zk_row, gk.e0, gk.e0 + gk.W - 1, zq_tile, zS,
                                         imin(kT, N - qb) - 1, eq0, eq1, bexp, sc);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2v + c);
          const float2 z0 = fadd2(make_float2(x[c], x[c + 1]), make_float2(-l4.x, -l4.y));
          const float2 z1 = fadd2(make_float2(x[c + 2], x[c + 3]), make_float2(-l4.z, -l4.w));
          x[c] = fast_exp2(z0.x);
          x[c + 1] = fast_exp2(z0.y);
          x[c + 2] = fast_exp2(z1.x);
          x[c + 3] = fast_exp2(z1.y);
        }
      }
      const bool need_mask = !jkeep || (p.causal && k0 + kT - 1 > qb);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          if (!jkeep || (p.causal && j > qb + cb + c)) x[c] = 0.f;
        }
      }
      // P^T, two queries per column, once dV(t - 1) has read P^T(t - 1)
      if (it > 0) {
        const bool got = mbar_wait(bar(kBarPFree), (it - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
      }
      // dropout: keep bits of this half's 64 queries for this key (bit c of km)
      uint32_t km[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      if (DROP) keep_mask64(p, bh, j, qb + cb, false, km);
      auto kept = [&](int c) { return ((km[c >> 5] >> (c & 31)) & 1u) != 0u; };
      {
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          if (DROP)   // dV sees P^T o M; the epilogue scales dV by 1 / (1 - p')
            pk[u] = DT<T>::pack(kept(2 * u) ? x[2 * u] : 0.f, kept(2 * u + 1) ? x[2 * u + 1] : 0.f);
          else
            pk[u] = DT<T>::pack(x[2 * u], x[2 * u + 1]);
        }
        tmem_st32(tmem + t_lane + kTmP + 32 * hc, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(kBarPReady));
      // dS^T = P^T (dP^T - D_i): the A operand of dK += dS^T Q, and the
      // key-side relation gradient of this key row
      const bool got_dp = mbar_wait(bar(kBarDpFull), it & 1, abort_flag, p.wait_ns);
      if (!__all_sync(0xffffffffu, got_dp)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t dp[64];
        const uint32_t td = tmem + t_lane + kTmDP + cb;
        tmem_ld32(td, dp);
        tmem_ld32(td + 32, dp + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(kBarDpFree));   // dP(t + 1) may now be written
        if (DROP) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            dp[c] = __float_as_uint(kept(c) ? __uint_as_float(dp[c]) * p.drop_scale : 0.f);
        }
        if (!DZK || is_const) {
          float2 ssum = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c);
            const float2 ds0 = fmul2(make_float2(x[c], x[c + 1]),
                                     fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                           make_float2(-d4.x, -d4.y)));
            const float2 ds1 = fmul2(make_float2(x[c + 2], x[c + 3]),
                                     fadd2(make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3])),
                                           make_float2(-d4.z, -d4.w)));
            x[c] = ds0.x; x[c + 1] = ds0.y; x[c + 2] = ds1.x; x[c + 3] = ds1.y;
            if (DZK) ssum = fadd2(ssum, fadd2(ds0, ds1));
          }
          if (DZK) {
            if (cls == RELPOS_TILE_CONST_LO) sat_lo += ssum.x + ssum.y;
            else sat_hi += ssum.x + ssum.y;
          }
        } else if ((j - lane) - (qb + cb + 63) > p.E_lo && (j - lane) + 31 - (qb + cb) < p.E_hi) {
          // every offset of the warp's 32 keys x 64 queries interior (warp-uniform)
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c);
            const float2 ds0 = fmul2(make_float2(x[c], x[c + 1]),
                                     fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                           make_float2(-d4.x, -d4.y)));
            const float2 ds1 = fmul2(make_float2(x[c + 2], x[c + 3]),
                                     fadd2(make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3])),
                                           make_float2(-d4.z, -d4.w)));
            x[c] = ds0.x; x[c + 1] = ds0.y; x[c + 2] = ds1.x; x[c + 3] = ds1.y;
          }
        } else {
          // column cc = query qb + cc of this key row: kept for
          // ckeep_lo <= cc <= ckeep_hi; delta = j - qb - cc is low-saturated
          // for cc >= clo and high-saturated (and not low) for cc <= chi
          const int ckeep_lo = p.causal ? imax(j - qb, 0) : 0;
          const int ckeep_hi = jkeep ? imin(N - 1 - qb, 127) : -1;
          const int clo = j - qb - p.E_lo;
          const int chi = imin(j - qb - p.E_hi, clo - 1);
          const int lo_beg = imax(clo, ckeep_lo), hi_end = imin(chi, ckeep_hi);
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c);
            const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int cc = cb + c + u;
              const float ds = x[c + u] * (__uint_as_float(dp[c + u]) - dd[u]);
              x[c + u] = ds;
              sat_lo += (cc >= lo_beg && cc <= ckeep_hi) ? ds : 0.f;
              sat_hi += (cc <= hi_end && cc >= ckeep_lo) ? ds : 0.f;
            }
          }
        }
      }
      // dS^T, two queries per column, once dK(t - 1) has read dS^T(t - 1)
      if (it > 0) {
        const bool got = mbar_wait(bar(kBarDsFree), (it - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) pk[u] = DT<T>::pack(x[2 * u], x[2 * u + 1]);
        tmem_st32(tmem + t_lane + kTmDS + 32 * hc, pk);
        if (DZK && !is_const) {
          // BAND tile: the same 16-bit values also go to the warp's staging
          // area (its own rows) for the coalesced by-offset store below
          __syncwarp();
          const uint32_t row16 = smem_u32(stg) + (uint32_t)(lane * kDsPitch) * 2u;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) st_shared_v4(row16 + 16u * ch, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        tmem_wait_st();
      }
      if (DZK && !is_const) {
        __syncwarp();
        dz_band_store<T>(stg, (warp & 3) * 32, lane, true, k0, qb, cb, nrows_k, nkv, N,
                         p.causal, p.E_lo, p.E_hi, dzk_base, gk.S, gk.e0);
      }
      tc_fence_before();
      mbar_arrive(bar(kBarDsReady));
    }
    // -------------------------------------------------------------- epilogue
    if (DZK) {
      // combine the two column halves' saturated sums; half 0 writes them
      float* sat = reinterpret_cast<float*>(sg + kOffSat);
      if (hc == 1) {
        sat[2 * r] = sat_lo;
        sat[2 * r + 1] = sat_hi;
      }
      named_bar_sync(1, 256);
      if (hc == 0 && jok)
        *reinterpret_cast<float2*>(t.dzk_sat + 2 * ((size_t)bh * npad + k0 + r)) =
            make_float2(sat_lo + sat[2 * r], sat_hi + sat[2 * r + 1]);
    }
    // dV and dK: half hc stores head-dim columns [32 hc, 32 hc + 32) of its key
    float dv[32], dk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) dv[c] = dk[c] = 0.f;
    const bool got_o = nq > 0 && ok && mbar_wait(bar(kBarDsFree), (nq - 1) & 1, abort_flag, p.wait_ns);
    if (__all_sync(0xffffffffu, got_o)) {
      tc_fence_after();
      uint32_t u[32];
      tmem_ld32(tmem + t_lane + kTmDV + 32 * hc, u);
      tmem_wait_ld();
      const float vs = DROP ? p.drop_scale : 1.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) dv[c] = __uint_as_float(u[c]) * vs;
      tmem_ld32(tmem + t_lane + kTmDK + 32 * hc, u);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) dk[c] = __uint_as_float(u[c]) * p.tau;
    }
    if (jok) {
      const size_t o = (size_t)act_row(p, sr, b, h, j) * 64 + 32 * hc;
      T* vdst = static_cast<T*>(t.dv) + o;
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
        uint4 w;
        w.x = DT<T>::pack(dv[c], dv[c + 1]);
        w.y = DT<T>::pack(dv[c + 2], dv[c + 3]);
        w.z = DT<T>::pack(dv[c + 4], dv[c + 5]);
        w.w = DT<T>::pack(dv[c + 6], dv[c + 7]);
        *reinterpret_cast<uint4*>(vdst + c) = w;
      }
      if (DK32) {
        // the fp32 accumulator keeps the workspace's dense layout
        float* dst = t.dk_acc + ((size_t)bh * N + j) * 64 + 32 * hc;
#pragma unroll
        for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(dk[c], dk[c + 1], dk[c + 2], dk[c + 3]);
      } else {
        T* dst = static_cast<T*>(t.dk) + o;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint4 w;
          w.x = DT<T>::pack(dk[c], dk[c + 1]);
          w.y = DT<T>::pack(dk[c + 2], dk[c + 3]);
          w.z = DT<T>::pack(dk[c + 4], dk[c + 5]);
          w.w = DT<T>::pack(dk[c + 6], dk[c + 7]);
          *reinterpret_cast<uint4*>(dst + c) = w;
        }
      }
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

// ---------------------------------------------------------------- host side
template <typename K>
cudaError_t launch4(K kern, dim3 grid, int threads, uint32_t smem, const Plan& p, const Tensors& t,
                    const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, const CUtensorMap& d,
                    cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  { kern<<<grid, threads, smem, s>>>(p, t, a, b, c, d); note_launch(1); }
  return cudaGetLastError();
}

struct Maps {
  CUtensorMap q, k, v, dout;
};

bool make_maps(const Plan& p, const Tensors& t, Maps& m) {
  const bool bf = t.is_bf16 != 0;
  return make_rows_map(&m.q, t.q, p, bf) && make_rows_map(&m.k, t.k, p, bf) && make_rows_map(&m.v, t.v, p, bf) &&
         make_rows_map(&m.dout, t.dout, p, bf);
}

template <typename T>
cudaError_t dq_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  Maps m;
  if (!make_maps(p, t, m)) return cudaErrorInvalidValue;
  const bool aq = t.aq_exp, ak = t.ak_exp, bb = t.b_exp;
  const dim3 grid(p.nT, p.B * p.H);
#define RP_DQ(A, K_, B_)                                                                                       \
  if (aq == A && ak == K_ && bb == B_)                                                                         \
    return p.dropout ? launch4(dq_sm100_kernel<T, A, K_, B_, (A || B_), A, true>, grid, qp::kThreads,          \
                               qp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s)                                 \
                     : launch4(dq_sm100_kernel<T, A, K_, B_, (A || B_), A, false>, grid, qp::kThreads,         \
                               qp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s);
  RP_DQ(false, false, false) RP_DQ(true, false, false) RP_DQ(false, true, false) RP_DQ(true, true, false)
  RP_DQ(false, false, true) RP_DQ(true, false, true) RP_DQ(false, true, true) RP_DQ(true, true, true)
#undef RP_DQ
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dk_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  Maps m;
  if (!make_maps(p, t, m)) return cudaErrorInvalidValue;
  const bool aq = t.aq_exp, ak = t.ak_exp, bb = t.b_exp;
  const dim3 grid(p.nT, p.B * p.H);
  // the float4 k.aK gather for an interior band wider than two tiles
  const bool wide = p.E_hi - p.E_lo + 1 > 2 * kT;
#define RP_DK(A, K_, B_)                                                                                           \
  if (aq == A && ak == K_ && bb == B_) {                                                                           \
    if (K_ && wide)                                                                                                \
      return p.dropout ? launch4(dkdv_sm100_kernel<T, A, K_, B_, K_, K_, true, K_>, grid, kp::kThreads,          \
                                 kp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s)                                 \
                       : launch4(dkdv_sm100_kernel<T, A, K_, B_, K_, K_, false, K_>, grid, kp::kThreads,         \
                                 kp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s);                                \
    return p.dropout ? launch4(dkdv_sm100_kernel<T, A, K_, B_, K_, K_, true, false>, grid, kp::kThreads,         \
                               kp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s)                                   \
                     : launch4(dkdv_sm100_kernel<T, A, K_, B_, K_, K_, false, false>, grid, kp::kThreads,        \
                               kp::kSmemBytes, p, t, m.q, m.k, m.v, m.dout, s);                                  \
  }
  RP_DK(false, false, false) RP_DK(true, false, false) RP_DK(false, true, false) RP_DK(true, true, false)
  RP_DK(false, false, true) RP_DK(true, false, true) RP_DK(false, true, true) RP_DK(true, true, true)
#undef RP_DK
  return cudaErrorInvalidValue;
}

inline unsigned nblocks(long long n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t launch_bwd_prep(const Plan& p, const Tensors& t, cudaStream_t s) {
  const long long BH = (long long)p.B * p.H;
  const int npad = p.nT * kT;
  const unsigned blocks = nblocks(BH * npad * 8, 256);
  if (t.is_bf16) {
    if (t.o_f32) {
      prep_sm100_kernel<float, __nv_bfloat16><<<blocks, 256, 0, s>>>(p, (const float*)t.o,
                                                                      (const __nv_bfloat16*)t.dout, t.lse, t.dsum,
                                                                      t.lse2, npad, BH);
    } else {
      prep_sm100_kernel<__nv_bfloat16, __nv_bfloat16><<<blocks, 256, 0, s>>>(
          p, (const __nv_bfloat16*)t.o, (const __nv_bfloat16*)t.dout, t.lse, t.dsum, t.lse2, npad, BH);
    }
  } else {
    if (t.o_f32) {
      prep_sm100_kernel<float, __half><<<blocks, 256, 0, s>>>(p, (const float*)t.o, (const __half*)t.dout, t.lse,
                                                               t.dsum, t.lse2, npad, BH);
    } else {
      prep_sm100_kernel<__half, __half><<<blocks, 256, 0, s>>>(p, (const __half*)t.o, (const __half*)t.dout, t.lse,
                                                                t.dsum, t.lse2, npad, BH);
    }
  }
  note_launch(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const Plan& p, const Tensors& t, cudaStream_t s) {
  return t.is_bf16 ? dq_typed<__nv_bfloat16>(p, t, s) : dq_typed<__half>(p, t, s);
}

cudaError_t launch_bwd_dkdv(const Plan& p, const Tensors& t, cudaStream_t s) {
  return t.is_bf16 ? dk_typed<__nv_bfloat16>(p, t, s) : dk_typed<__half>(p, t, s);
}

}  // namespace relpos
