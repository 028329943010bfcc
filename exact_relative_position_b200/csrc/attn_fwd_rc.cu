// attn_fwd_rc.cu -- forward of exact relative-position attention with the
// query-side projection recomputed inside every tile instead of read from a
// stored Z^Q (digest of "Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels": the ablation's "projection precompute" row and
// the limitations section -- storing the identity map's projection is
// quadratic, recomputing it per tile makes the forward's memory linear at
// the cost of more tensor work).
//
// Terms: q.aQ and the bias b (the Transformer-XL form, whose identity map is
// the one that needs this mode); the key-side term k.aK is not supported here.
//
// One CTA owns one 128-row query tile of one (batch, head).  Warp roles:
//   warp 0       TMA producer: Q once; per key tile K and V into a 2-stage
//                ring; per BAND tile the window of the expanded table aQ_exp
//                that the tile's offsets reach (256 rows, single buffer)
//   warp 1       MMA issuer (one thread): S = Q K^T; for a BAND tile also
//                Zt = Q Aw^T (M = 128, N = 256), the tile's projection;
//                O += P V with P read from tensor memory
//   warp 2       allocates / frees the tensor-memory columns
//   warps 4..7   softmax (thread r owns row r = TMEM lane r)
// Tensor memory: S [0,128), O [128,192), P [192,256), Zt [256,512).
//
// Window of key tile (qi, kj): offsets d0 .. d0 + 255 with d0 = j0 - i0 - 127,
// so cell (r, c) of the tile (offset j0 + c - i0 - r) sits in column
// c - r + 127 of Zt: row r needs a skewed run of 128 of its own 256 columns.
// Each softmax warp copies the 160 columns its 32 rows can reach from tensor
// memory into a warp-private shared-memory area (row pitch 164 floats: the
// 16-byte stores of a row are conflict-free and so are the skewed 4-byte
// reads, lane l reading word l * 163 + const), and every thread reads its own
// run from there.  Offsets outside (E_lo, E_hi) take the row's two saturated
// values q_i.aQ_exp[0] and q_i.aQ_exp[R_exp - 1], computed once per CTA.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "sm100.cuh"
#include "warp_mma.cuh"

namespace relpos {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

namespace {

using namespace sm100;

constexpr int kT = 128;
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr int kWinRows = 256;                     // offsets per projection window (N of the Zt GEMM)
constexpr uint32_t kTileBytes = 128 * 128;        // one [128 x 64] 16-bit tile
constexpr uint32_t kWinBytes = kWinRows * 128;    // [256 x 64] 16-bit window
constexpr int kSkPitch = 164;                     // floats per row of a warp's skew area
constexpr int kSkCols = 160;                      // columns of Zt a warp's rows can reach
constexpr uint32_t kSkWarpBytes = 32u * kSkPitch * 4u;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kTileBytes;                              // stages of (K, V)
constexpr uint32_t kOffWin = kOffKV + kStages * 2 * kTileBytes;     // 1024-aligned
constexpr uint32_t kOffSk = kOffWin + kWinBytes;
constexpr uint32_t kOffBar = kOffSk + 4 * kSkWarpBytes;
constexpr uint32_t kOffAbort = kOffBar + 256;
constexpr uint32_t kOffTmem = kOffAbort + 16;
constexpr uint32_t kSmemBytes = kOffTmem + 16 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS = 0, kTmO = 128, kTmP = 192, kTmZ = 256;
constexpr float kRescaleThreshold = 8.0f;
static_assert(kSmemBytes <= 232448, "shared memory of the recompute forward exceeds the per-block limit");
static_assert((kOffWin & 1023u) == 0 && (kOffKV & 1023u) == 0, "TMA tiles must be 1024-byte aligned");

// barrier slots (8 bytes each)
constexpr int kBarQ = 0;
constexpr int kBarKvFull = 1;
constexpr int kBarKvEmpty = kBarKvFull + kStages;
constexpr int kBarWinFull = kBarKvEmpty + kStages;   // window landed (TMA)
constexpr int kBarWinEmpty = kBarWinFull + 1;        // Zt GEMM done reading the window (MMA commit)
constexpr int kBarSFull = kBarWinEmpty + 1;          // S written (MMA commit)
constexpr int kBarSFree = kBarSFull + 1;             // S read (128 arrivals)
constexpr int kBarZFull = kBarSFree + 1;             // Zt written (MMA commit)
constexpr int kBarZFree = kBarZFull + 1;             // Zt copied out (128 arrivals)
constexpr int kBarPReady = kBarZFree + 1;            // P written (128 arrivals)
constexpr int kBarPFree = kBarPReady + 1;            // PV done (MMA commit)
constexpr int kBarDrain = kBarPFree + 1;

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// is key tile kj of query tile qi a BAND tile (the only ones that need Zt)?
__device__ __forceinline__ bool band_tile(const Plan& p, int qi, int kj, int nkv) {
  return tile_class(qi, kj, p.N, nkv, p.causal, p.E_lo, p.E_hi) == RELPOS_TILE_BAND;
}

template <typename OutT> struct RowStoreRc;
template <> struct RowStoreRc<float> {
  static __device__ __forceinline__ void row(float* dst, const float* v) {
#pragma unroll
    for (int c = 0; c < 64; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
  }
};
template <typename T> struct RowStoreRc {
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

// SAT: a window offset can lie outside [E_lo, E_hi] (every map but the identity
// map), so saturated cells take the row's saturated values instead of Zt.
template <typename T, typename OutT, bool AQ, bool BIAS, bool DROP, bool SAT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_rc_kernel(const Plan p, const Tensors t, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmA) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + kOffAbort);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sg + kOffTmem);
  auto bar = [&](int slot) { return sb + kOffBar + 8u * (uint32_t)slot; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // causal: query tiles in descending order, the longest rows first
  const int qt = abs(p.qrev - (int)blockIdx.x);
  const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, i0 = qt * kT;
  const SeqRows sr = seq_rows(p, b);   // this sequence's rows (the dense layout: all N)
  // keys j >= nkv are masked: the sequence length (packed), or the clamped key length
  const int nkv = p.packed ? sr.len : (p.padding ? iclamp(p.key_len[b], 0, N) : N);
  int kend = nkv;
  if (p.causal) kend = imin(kend, imin(i0 + kT, N));
  // nothing to do for a query tile past the sequence (packed batches)
  const int nkt = (kend > 0 && i0 < sr.len) ? (kend + kT - 1) / kT : 0;
  const int hq = t.table_per_head ? h : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKvFull + s), 1);
      mbar_init(bar(kBarKvEmpty + s), 1);
    }
    mbar_init(bar(kBarWinFull), 1);
    mbar_init(bar(kBarWinEmpty), 1);
    mbar_init(bar(kBarSFull), 1);
    mbar_init(bar(kBarSFree), 128);
    mbar_init(bar(kBarZFull), 1);
    mbar_init(bar(kBarZFree), 128);
    mbar_init(bar(kBarPReady), 128);
    mbar_init(bar(kBarPFree), 1);
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

  if (warp < 4) {
    if (warp == 0 && lane == 0 && nkt > 0) {
      // ---------------------------------------------------------- TMA producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (AQ) prefetch_tmap(&tmA);
      mbar_expect_tx(bar(kBarQ), kTileBytes);
      int c1, c2;
      tma_rows(p, sr, bh, h, i0, c1, c2);
      tma_load_3d(sb + kOffQ, &tmQ, bar(kBarQ), 0, c1, c2);
      int issued = 0, nwin = 0;
#pragma unroll 1
      for (int it = 0; it < nkt; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait(bar(kBarKvEmpty + s), ((it / kStages) - 1) & 1, abort_flag, p.wait_ns)) break;
        const uint32_t dst = sb + kOffKV + (uint32_t)s * 2 * kTileBytes;
        mbar_expect_tx(bar(kBarKvFull + s), 2 * kTileBytes);
        tma_rows(p, sr, bh, h, it * kT, c1, c2);
        tma_load_3d(dst, &tmK, bar(kBarKvFull + s), 0, c1, c2);
        tma_load_3d(dst + kTileBytes, &tmV, bar(kBarKvFull + s), 0, c1, c2);
        issued = it + 1;
        if (AQ && band_tile(p, qt, it, nkv)) {
          // the previous window has been read by its Zt GEMM
          if (nwin > 0 && !mbar_wait(bar(kBarWinEmpty), (nwin - 1) & 1, abort_flag, p.wait_ns)) break;
          // expanded rows of offsets j0 - i0 - 127 .. + 255; rows outside [0, R_exp) read as zero
          // (their offsets saturate and take the row's saturated values instead)
          const int e_w0 = it * kT - i0 - 127 - p.E_lo;
          mbar_expect_tx(bar(kBarWinFull), kWinBytes);
          tma_load_3d(sb + kOffWin, &tmA, bar(kBarWinFull), 0, e_w0, hq);
          ++nwin;
        }
      }
      // every load issued has landed before the CTA can exit
      mbar_drain(bar(kBarQ), 0);
      for (int it = imax(0, issued - kStages); it < issued; ++it)
        mbar_drain(bar(kBarKvFull + it % kStages), (it / kStages) & 1);
      if (nwin > 0) mbar_drain(bar(kBarWinFull), (nwin - 1) & 1);
    } else if (warp == 1 && lane == 0 && nkt > 0) {
      // ---------------------------------------------------------- MMA issuer
      const bool bf = t.is_bf16 != 0;
      const uint32_t id_qk = idesc_f16(bf, 128, 128, false, false);
      const uint32_t id_qa = idesc_f16(bf, 128, kWinRows, false, false);
      const uint32_t id_pv = idesc_f16(bf, 128, 64, false, true);
      const uint64_t dq = sdesc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sb + kOffKV, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sb + kOffKV + kTileBytes, 8192, 1024);
      const uint64_t dw = sdesc_sw128(sb + kOffWin, 16, 1024);
      constexpr uint64_t kStage16 = (2 * kTileBytes) >> 4;
      auto issue_qk = [&](int s) {
        const uint64_t k = dk0 + (uint64_t)s * kStage16;
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kTmS, dq + 2 * kk, k + 2 * kk, id_qk, kk > 0);
      };
      auto issue_qa = [&]() {
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kTmZ, dq + 2 * kk, dw + 2 * kk, id_qa, kk > 0);
      };
      auto issue_pv = [&](int s, bool acc) {
        const uint64_t v = dv0 + (uint64_t)s * kStage16;
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + kTmO, tmem + kTmP + 8 * kk, v + 128 * kk, id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      // S(t) and, for a BAND tile, Zt(t): S once the previous S has been read,
      // Zt once the previous Zt has been copied out and its window has landed
      int nband = 0;
      auto issue_tile = [&](int it) -> bool {
        const int s = it % kStages;
        if (!mbar_wait(bar(kBarKvFull + s), (it / kStages) & 1, abort_flag, p.wait_ns)) return false;
        if (it > 0 && !mbar_wait(bar(kBarSFree), (it - 1) & 1, abort_flag, p.wait_ns)) return false;
        tc_fence_after();
        issue_qk(s);
        mma_commit(bar(kBarSFull));
        if (AQ && band_tile(p, qt, it, nkv)) {
          if (!mbar_wait(bar(kBarWinFull), nband & 1, abort_flag, p.wait_ns)) return false;
          if (nband > 0 && !mbar_wait(bar(kBarZFree), (nband - 1) & 1, abort_flag, p.wait_ns)) return false;
          tc_fence_after();
          issue_qa();
          mma_commit(bar(kBarZFull));
          mma_commit(bar(kBarWinEmpty));
          ++nband;
        }
        return true;
      };
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, p.wait_ns) && issue_tile(0);
#pragma unroll 1
      for (int it = 0; it < nkt && ok; ++it) {
        if (it + 1 < nkt) {
          ok = issue_tile(it + 1);
          if (!ok) break;
        }
        ok = mbar_wait(bar(kBarPReady), it & 1, abort_flag, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(it % kStages, it > 0);
        mma_commit(bar(kBarPFree));
        mma_commit(bar(kBarKvEmpty + it % kStages));
      }
      {
        // drain (bounded): no MMA may still run when tensor memory is freed
        mma_commit(bar(kBarDrain));
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wl = warp & 3;
    const int r = wl * 32 + lane;
    const int i = i0 + r;
    const bool rok = i < sr.len;
    const uint32_t t_lane = (uint32_t)(wl * 32) << 16;
    const uint32_t tS = tmem + t_lane + kTmS;
    const uint32_t tO = tmem + t_lane + kTmO;
    const uint32_t tP = tmem + t_lane + kTmP;
    const uint32_t tZ = tmem + t_lane + kTmZ + (uint32_t)(96 - 32 * wl);   // first column this warp reaches
    const float sc = p.tau * kLog2e;
    // the row's saturated projections q_i.aQ_exp[0] and q_i.aQ_exp[R_exp - 1]
    // (rows past the sequence use its last row, in bounds; their results are discarded)
    float zq_lo = 0.f, zq_hi = 0.f;
    if (AQ && sr.len > 0) {
      const T* qrow = static_cast<const T*>(t.q) + act_row(p, sr, b, h, imin(i, sr.len - 1)) * 64;
      const T* alo = static_cast<const T*>(t.aq_exp) + (size_t)hq * t.aq_hs;
      const T* ahi = alo + (size_t)(p.Rexp - 1) * 64;
#pragma unroll 8
      for (int c = 0; c < 64; ++c) {
        const float qv = DT<T>::to_f(qrow[c]);
        zq_lo = fmaf(qv, DT<T>::to_f(alo[c]), zq_lo);
        zq_hi = fmaf(qv, DT<T>::to_f(ahi[c]), zq_hi);
      }
    }
    const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
    float crow_lo = zq_lo, crow_hi = zq_hi;
    if (BIAS) {
      crow_lo += __ldg(bexp);
      crow_hi += __ldg(bexp + p.Rexp - 1);
    }
    crow_lo *= sc;
    crow_hi *= sc;
    float* sk = reinterpret_cast<float*>(sg + kOffSk + (uint32_t)wl * kSkWarpBytes);
    const uint32_t sk_row = smem_u32(sk) + (uint32_t)(lane * kSkPitch) * 4u;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int nband = 0;
    for (int it = 0; it < nkt; ++it) {
      const int j0 = it * kT;
      const int cls = tile_class(qt, it, N, nkv, p.causal, p.E_lo, p.E_hi);
      const bool is_const = cls == RELPOS_TILE_CONST_LO || cls == RELPOS_TILE_CONST_HI;
      // every decision before a tcgen05.ld/st (warp-collective) is warp-uniform
      const bool got_s = mbar_wait(bar(kBarSFull), it & 1, abort_flag, p.wait_ns);
      if (!__all_sync(0xffffffffu, got_s)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      tmem_ld32(tS + 0, reinterpret_cast<uint32_t*>(x) + 0);
      tmem_ld32(tS + 32, reinterpret_cast<uint32_t*>(x) + 32);
      tmem_ld32(tS + 64, reinterpret_cast<uint32_t*>(x) + 64);
      tmem_ld32(tS + 96, reinterpret_cast<uint32_t*>(x) + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kBarSFree));    // the next key tile's S may now be written
      float rowc = 0.f, xs = 1.f;
      if (is_const) {
        // saturated tile: one row constant, the scale applied in the exponent
        rowc = cls == RELPOS_TILE_CONST_LO ? crow_lo : crow_hi;
        xs = sc;
      } else {
        if (AQ) {
          // copy the 160 columns of Zt this warp's rows reach into its skew area
          const bool got_z = mbar_wait(bar(kBarZFull), nband & 1, abort_flag, p.wait_ns);
          if (!__all_sync(0xffffffffu, got_z)) { ok = false; break; }
          ++nband;
          tc_fence_after();
          __syncwarp();
#pragma unroll 1
          for (int ch = 0; ch < kSkCols / 32; ++ch) {
            uint32_t zv[32];
            tmem_ld32(tZ + 32 * ch, zv);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              st_shared_v4(sk_row + (uint32_t)(32 * ch + 4 * q4) * 4u, zv[4 * q4], zv[4 * q4 + 1], zv[4 * q4 + 2],
                           zv[4 * q4 + 3]);
          }
          tc_fence_before();
          mbar_arrive(bar(kBarZFree));   // the next BAND tile's Zt may now be written
          __syncwarp();
        }
        // cell (r, c) has offset d = j0 + c - i; its projection sits at column
        // c - lane + 31 of this lane's row of the skew area
        const int dbase = j0 - i;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
#pragma unroll
          for (int c = c0; c < c0 + 32; ++c) {
            const int d = dbase + c;
            float rel = 0.f;
            if (AQ) {
              const float zin = sk[lane * kSkPitch + c - lane + 31];
              rel = SAT ? (d <= p.E_lo ? zq_lo : (d >= p.E_hi ? zq_hi : zin)) : zin;
            }
            if (BIAS) rel += __ldg(bexp + iclamp(d, p.E_lo, p.E_hi) - p.E_lo);
            x[c] = (x[c] + rel) * sc;
          }
          // keep the compiler from hoisting every chunk's loads at once (register pressure)
          asm volatile("" ::: "memory");
        }
        __syncwarp();   // every lane has read the skew area before the next tile rewrites it
      }
      const bool need_mask = (j0 + kT > nkv) || (p.causal && j0 + kT - 1 > i0);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = j0 + c;
          if (j >= nkv || (p.causal && j > i)) x[c] = -INFINITY;
        }
      }
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = max3(x[u], x[u + 8], x[u + 16]);
#pragma unroll
      for (int c = 24; c < 128; c += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = max3(pm[u], x[c + u], c + 8 + u < 128 ? x[c + 8 + u] : pm[u]);
      }
      float mx = max3(max3(pm[0], pm[1], pm[2]), max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx = mx * xs + rowc;   // xs > 0 (tau > 0)
      const float m_new = fmaxf(m_run, mx);
      const bool grow = m_new > m_run + kRescaleThreshold;
      const float alpha = grow ? fast_exp2(m_run - m_new) : 1.f;
      bool pfree_seen = it == 0;
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        const bool got = mbar_wait(bar(kBarPFree), (it - 1) & 1, abort_flag, p.wait_ns);
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
      const float msub = m_run == -INFINITY ? 0.f : m_run - rowc;
      const float2 xs2 = make_float2(xs, xs), ms2 = make_float2(-msub, -msub);
      float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float ps[2] = {0.f, 0.f};
      uint32_t pk[64];
      uint32_t km[4] = {0u, 0u, 0u, 0u};
      if (DROP) {
        keep_mask64(p, bh, i, j0, true, *reinterpret_cast<uint32_t(*)[2]>(km));
        keep_mask64(p, bh, i, j0 + 64, true, *reinterpret_cast<uint32_t(*)[2]>(km + 2));
      }
#pragma unroll
      for (int w = 0; w < 64; ++w) {
        const float2 z = ffma2(make_float2(x[2 * w], x[2 * w + 1]), xs2, ms2);
        const float2 e = make_float2(fast_exp2(z.x), fast_exp2(z.y));
        pk[w] = DT<T>::pack(e.x, e.y);
        if (DT<T>::kCoarse) ps[w & 1] += DT<T>::pair_sum(pk[w]);
        else ps2[w & 1] = fadd2(ps2[w & 1], e);
        if (DROP) {
          const uint32_t kb = (km[w >> 4] >> (2 * (w & 15))) & 3u;
          pk[w] = DT<T>::pack((kb & 1u) ? e.x : 0.f, (kb & 2u) ? e.y : 0.f);
        }
      }
      l_run += DT<T>::kCoarse ? ps[0] + ps[1] : (ps2[0].x + ps2[1].x) + (ps2[0].y + ps2[1].y);
      if (!pfree_seen) {
        const bool got = mbar_wait(bar(kBarPFree), (it - 1) & 1, abort_flag, p.wait_ns);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st32(tP, pk);
      tmem_st32(tP + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarPReady));
    }
    // ------------------------------------------------------------ epilogue
    float ov[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) ov[c] = 0.f;
    const bool got_o = nkt > 0 && ok && mbar_wait(bar(kBarPFree), (nkt - 1) & 1, abort_flag, p.wait_ns);
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
      RowStoreRc<OutT>::row(O, ov);
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

// [Hq, R_exp, 64] 16-bit expanded table viewed as 3-D for TMA: 256-row boxes,
// 128-byte swizzle, rows outside [0, R_exp) read as zero.
bool make_table_map(CUtensorMap* m, const void* base, int Hq, int Rexp, long long head_stride_elems, bool bf16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)Rexp, (cuuint64_t)Hq};
  cuuint64_t strides[2] = {128, (cuuint64_t)head_stride_elems * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kWinRows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T, typename OutT, bool SAT>
cudaError_t launch_rc_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  using K = void (*)(const Plan, const Tensors, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                     const CUtensorMap);
  const int mask = (t.aq_exp ? 1 : 0) | (t.b_exp ? 2 : 0) | (p.dropout ? 4 : 0);
  K kern = nullptr;
  switch (mask) {
    case 0: kern = fwd_rc_kernel<T, OutT, false, false, false, SAT>; break;
    case 1: kern = fwd_rc_kernel<T, OutT, true, false, false, SAT>; break;
    case 2: kern = fwd_rc_kernel<T, OutT, false, true, false, SAT>; break;
    case 3: kern = fwd_rc_kernel<T, OutT, true, true, false, SAT>; break;
    case 4: kern = fwd_rc_kernel<T, OutT, false, false, true, SAT>; break;
    case 5: kern = fwd_rc_kernel<T, OutT, true, false, true, SAT>; break;
    case 6: kern = fwd_rc_kernel<T, OutT, false, true, true, SAT>; break;
    default: kern = fwd_rc_kernel<T, OutT, true, true, true, SAT>; break;
  }
  CUtensorMap mq, mk, mv, ma;
  const int BH = p.B * p.H;
  const bool bf = t.is_bf16 != 0;
  if (!make_rows_map(&mq, t.q, p, bf) || !make_rows_map(&mk, t.k, p, bf) || !make_rows_map(&mv, t.v, p, bf))
    return cudaErrorInvalidValue;
  memset(&ma, 0, sizeof(ma));
  if (t.aq_exp && !make_table_map(&ma, t.aq_exp, t.table_per_head ? p.H : 1, p.Rexp, t.aq_hs, bf))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nT, BH);
  { kern<<<grid, kThreads, kSmemBytes, s>>>(p, t, mq, mk, mv, ma); note_launch(1); }
  return cudaGetLastError();
}

}  // namespace

template <bool SAT>
cudaError_t launch_rc_sat(const Plan& p, const Tensors& t, cudaStream_t s) {
  if (t.is_bf16) {
    return t.o_f32 ? launch_rc_typed<__nv_bfloat16, float, SAT>(p, t, s)
                   : launch_rc_typed<__nv_bfloat16, __nv_bfloat16, SAT>(p, t, s);
  }
  return t.o_f32 ? launch_rc_typed<__half, float, SAT>(p, t, s) : launch_rc_typed<__half, __half, SAT>(p, t, s);
}

cudaError_t launch_forward_recompute(const Plan& p, const Tensors& t, cudaStream_t s) {
  if (t.ak_exp) return cudaErrorInvalidValue;   // the key-side term needs the stored projection
  // the identity map's expanded range is every reachable offset: no window cell saturates
  const bool exact_window = p.E_lo == 1 - p.N && p.E_hi == p.N - 1 && p.Rexp == 2 * p.N - 1;
  return exact_window ? launch_rc_sat<false>(p, t, s) : launch_rc_sat<true>(p, t, s);
}

}  // namespace relpos
