// attn_bwd.cu -- two-pass backward of exact relative-position attention
// (digest of "Fast and Exact Relative-Position Attention via Structure-Aware
// Kernels": backward section and Eq. (4)).
//
//   prep:        D_i = sum_c dO_ic O_ic
//   Q-parallel:  one CTA per 128 query rows recomputes S and P from LSE,
//                dP = dO V^T, dS = P (dP - D), dQ = tau dS K, and writes the
//                query-side relation gradient by offset: for an interior
//                offset the entry dZ^Q[i, e] has exactly one key, so it is a
//                plain store by the CTA that owns row i; the two saturated
//                rows are summed in registers and stored once per row.
//   K-parallel:  one CTA per 128 keys recomputes S^T and P^T, dV = P^T dO,
//                dK = tau dS^T Q and the key-side dZ^K the same way.
// No entry has two writers, so no atomics are needed and every sum has a
// fixed order.
#include "kernels.cuh"
#include "warp_mma.cuh"

namespace relpos {

namespace {

constexpr int kThreads = 256;

template <typename OutT> struct St2;
template <> struct St2<float> {
  static __device__ __forceinline__ void two(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
};
template <> struct St2<__half> {
  static __device__ __forceinline__ void two(__half* p, float a, float b) { *reinterpret_cast<__half2*>(p) = __floats2half2_rn(a, b); }
};
template <> struct St2<__nv_bfloat16> {
  static __device__ __forceinline__ void two(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
  }
};

// ------------------------------------------------------------------ prep
template <typename OT, typename T>
__global__ void __launch_bounds__(256) prep_kernel(const OT* __restrict__ o, const T* __restrict__ dout,
                                                   float* __restrict__ dsum, long long rows) {
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gt >> 3;
  const int part = (int)(gt & 7);
  float acc = 0.f;
  if (row < rows) {
    const OT* orow = o + row * 64 + part * 8;
    const T* drow = dout + row * 64 + part * 8;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc += (float)orow[c] * (float)drow[c];
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (row < rows && part == 0) dsum[row] = acc;
}

// ------------------------------------------------------------------ Q-parallel
constexpr int kSmemDq = 2 * 128 * 128 + 2 * 2 * 64 * 128;

template <typename T, bool AQ, bool AK, bool BIAS, bool DZQ, bool DQ32>
__global__ void __launch_bounds__(kThreads) dq_kernel(const Plan p, const Tensors t) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, q0 = qt * 128;
  const size_t off = (size_t)bh * N * 64;
  const T* Q = static_cast<const T*>(t.q) + off;
  const T* K = static_cast<const T*>(t.k) + off;
  const T* V = static_cast<const T*>(t.v) + off;
  const T* dO = static_cast<const T*>(t.dout) + off;
  const uint32_t sQ = smem_u32(smem), sdO = sQ + 128 * 128, sKV = sdO + 128 * 128;

  const int nkv = p.padding ? p.key_len[b] : N;
  int kend = nkv;
  if (p.causal) kend = imin(kend, imin(q0 + 128, N));
  const int ntiles = kend > 0 ? (kend + 63) / 64 : 0;

  load_tile_async<128, kThreads>(sQ, Q, q0, N, tid);
  load_tile_async<128, kThreads>(sdO, dO, q0, N, tid);
  if (ntiles > 0) {
    load_tile_async<64, kThreads>(sKV, K, 0, N, tid);
    load_tile_async<64, kThreads>(sKV + 64 * 128, V, 0, N, tid);
  }
  cp_async_commit();

  const int g = lane >> 2, tq = lane & 3;
  int irow[2] = {q0 + warp * 16 + g, q0 + warp * 16 + g + 8};
  float lse2[2], dval[2];
  const float* zq_row[2] = {nullptr, nullptr};
  float* dzq_row[2] = {nullptr, nullptr};
  {
    const GroupInfo gi = p.gq[qt];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int i = irow[hf];
      const bool ok = i < N;
      const float l = ok ? t.lse[(size_t)bh * N + i] : -INFINITY;
      lse2[hf] = l == -INFINITY ? INFINITY : l * kLog2e;   // +inf makes every P of a dead row 0
      dval[hf] = ok ? t.dsum[(size_t)bh * N + i] : 0.f;
      const long long ro = gi.base + (long long)(i - q0) * gi.S - gi.e0;
      if (AQ) zq_row[hf] = t.zq + (size_t)bh * p.zq_head + ro;
      if (DZQ) dzq_row[hf] = t.dzq + (size_t)bh * p.zq_head + ro;
    }
  }
  const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
  const float sc = p.tau * kLog2e;

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float sat_lo[2] = {0.f, 0.f}, sat_hi[2] = {0.f, 0.f};
  uint32_t qa[4][4], da[4][4];

  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) {
      const uint32_t sb = sKV + (uint32_t)((it + 1) & 1) * (2 * 64 * 128);
      load_tile_async<64, kThreads>(sb, K, (it + 1) * 64, N, tid);
      load_tile_async<64, kThreads>(sb + 64 * 128, V, (it + 1) * 64, N, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
      load_a_frags(sQ, warp * 16, lane, qa);
      load_a_frags(sdO, warp * 16, lane, da);
    }
    const uint32_t sK = sKV + (uint32_t)(it & 1) * (2 * 64 * 128);
    const uint32_t sV = sK + 64 * 128;
    const int k0 = it * 64;

    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
    }
    mma_abt<T, 8>(s, qa, sK, 0, lane);
    mma_abt<T, 8>(dp, da, sV, 0, lane);

    const float* zk_tile = nullptr;
    int zk_S = 0;
    if (AK) {
      const int kg = k0 / kTile;
      const GroupInfo gi = p.gk[kg];
      zk_tile = t.zk + (size_t)bh * p.zk_head + gi.base - gi.e0 + (long long)(k0 - kg * kTile) * gi.S;
      zk_S = gi.S;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int hf = r >> 1;
        const int cj = nt * 8 + 2 * tq + (r & 1);
        const int i = irow[hf], j = k0 + cj;
        const bool inr = (i < N) && (j < N);
        const bool keep = inr && (j < nkv) && !(p.causal && j > i);
        const int delta = j - i;
        const int e = iclamp(delta, p.E_lo, p.E_hi) - p.E_lo;
        float pv = 0.f;
        if (keep) {
          float rel = 0.f;
          if (AQ) rel += __ldg(zq_row[hf] + e);
          if (AK) rel += __ldg(zk_tile + (long long)cj * zk_S + e);
          if (BIAS) rel += __ldg(bexp + e);
          pv = exp2f((s[nt][r] + rel) * sc - lse2[hf]);
        }
        const float ds = pv * (dp[nt][r] - dval[hf]);
        s[nt][r] = ds;
        if (DZQ && keep) {   // masked cells have dS = 0 and may lie outside the group's columns
          const float val = p.tau * ds;
          if (delta <= p.E_lo) sat_lo[hf] += val;
          else if (delta >= p.E_hi) sat_hi[hf] += val;
          else dzq_row[hf][e] = val;
        }
      }
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      pa[kk][0] = DT<T>::pack(s[2 * kk][0], s[2 * kk][1]);
      pa[kk][1] = DT<T>::pack(s[2 * kk][2], s[2 * kk][3]);
      pa[kk][2] = DT<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[kk][3] = DT<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    }
    mma_ab<T, 4>(acc, pa, sK, 0, lane);
    __syncthreads();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int i = irow[hf];
    if (DZQ) {
      float lo = sat_lo[hf], hi = sat_hi[hf];
      lo += __shfl_xor_sync(0xffffffffu, lo, 1);
      lo += __shfl_xor_sync(0xffffffffu, lo, 2);
      hi += __shfl_xor_sync(0xffffffffu, hi, 1);
      hi += __shfl_xor_sync(0xffffffffu, hi, 2);
      if (i < N && tq == 0) {
        const GroupInfo gi = p.gq[qt];
        if (p.Rexp == 1) {
          dzq_row[hf][0] = lo + hi;
        } else {
          if (gi.e0 == 0) dzq_row[hf][0] = lo;
          if (p.Rexp - 1 < gi.e0 + gi.W) dzq_row[hf][p.Rexp - 1] = hi;
        }
      }
    }
    if (i < N) {
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const float a0 = acc[dt][2 * hf] * p.tau, a1 = acc[dt][2 * hf + 1] * p.tau;
        if (DQ32) St2<float>::two(t.dq_acc + off + (size_t)i * 64 + dt * 8 + 2 * tq, a0, a1);
        else St2<T>::two(static_cast<T*>(t.dq) + off + (size_t)i * 64 + dt * 8 + 2 * tq, a0, a1);
      }
    }
  }
}

// ------------------------------------------------------------------ K-parallel
constexpr int kSmemDk = 2 * 128 * 128 + 2 * 2 * 64 * 128;

template <typename T, bool AQ, bool AK, bool BIAS, bool DZK, bool DK32>
__global__ void __launch_bounds__(kThreads) dkdv_kernel(const Plan p, const Tensors t) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kt = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, k0 = kt * 128;
  const size_t off = (size_t)bh * N * 64;
  const T* Q = static_cast<const T*>(t.q) + off;
  const T* K = static_cast<const T*>(t.k) + off;
  const T* V = static_cast<const T*>(t.v) + off;
  const T* dO = static_cast<const T*>(t.dout) + off;
  const uint32_t sK = smem_u32(smem), sV = sK + 128 * 128, sQD = sV + 128 * 128;

  const int nkv = p.padding ? p.key_len[b] : N;
  const int qstart = p.causal ? (k0 / 64) * 64 : 0;
  const int ntiles = (k0 < nkv && qstart < N) ? (N - qstart + 63) / 64 : 0;

  load_tile_async<128, kThreads>(sK, K, k0, N, tid);
  load_tile_async<128, kThreads>(sV, V, k0, N, tid);
  if (ntiles > 0) {
    load_tile_async<64, kThreads>(sQD, Q, qstart, N, tid);
    load_tile_async<64, kThreads>(sQD + 64 * 128, dO, qstart, N, tid);
  }
  cp_async_commit();

  const int g = lane >> 2, tq = lane & 3;
  const int jrow[2] = {k0 + warp * 16 + g, k0 + warp * 16 + g + 8};
  const float* zk_row[2] = {nullptr, nullptr};
  float* dzk_row[2] = {nullptr, nullptr};
  {
    const GroupInfo gi = p.gk[kt];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const long long ro = gi.base + (long long)(jrow[hf] - k0) * gi.S - gi.e0;
      if (AK) zk_row[hf] = t.zk + (size_t)bh * p.zk_head + ro;
      if (DZK) dzk_row[hf] = t.dzk + (size_t)bh * p.zk_head + ro;
    }
  }
  const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
  const float* lse = t.lse + (size_t)bh * N;
  const float* dsum = t.dsum + (size_t)bh * N;
  const float sc = p.tau * kLog2e;

  float dk[8][4], dv[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  float sat_lo[2] = {0.f, 0.f}, sat_hi[2] = {0.f, 0.f};
  uint32_t ka[4][4], va[4][4];

  for (int it = 0; it < ntiles; ++it) {
    const int qb = qstart + it * 64;
    if (it + 1 < ntiles) {
      const uint32_t sb = sQD + (uint32_t)((it + 1) & 1) * (2 * 64 * 128);
      load_tile_async<64, kThreads>(sb, Q, qb + 64, N, tid);
      load_tile_async<64, kThreads>(sb + 64 * 128, dO, qb + 64, N, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
      load_a_frags(sK, warp * 16, lane, ka);
      load_a_frags(sV, warp * 16, lane, va);
    }
    const uint32_t sQ = sQD + (uint32_t)(it & 1) * (2 * 64 * 128);
    const uint32_t sD = sQ + 64 * 128;

    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
    }
    mma_abt<T, 8>(s, ka, sQ, 0, lane);     // S^T = K Q^T
    mma_abt<T, 8>(dp, va, sD, 0, lane);    // dP^T = V dO^T

    const float* zq_tile = nullptr;
    int zq_S = 0;
    if (AQ) {
      const int qg = qb / kTile;
      const GroupInfo gi = p.gq[qg];
      zq_tile = t.zq + (size_t)bh * p.zq_head + gi.base - gi.e0 + (long long)(qb - qg * kTile) * gi.S;
      zq_S = gi.S;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int ci = nt * 8 + 2 * tq + c;
        const int i = qb + ci;
        const bool iok = i < N;
        const float l = iok ? __ldg(lse + i) : -INFINITY;
        const float l2 = l == -INFINITY ? INFINITY : l * kLog2e;
        const float dd = iok ? __ldg(dsum + i) : 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = 2 * hf + c;
          const int j = jrow[hf];
          const bool inr = iok && (j < N);
          const bool keep = inr && (j < nkv) && !(p.causal && j > i);
          const int delta = j - i;
          const int e = iclamp(delta, p.E_lo, p.E_hi) - p.E_lo;
          float pv = 0.f;
          if (keep) {
            float rel = 0.f;
            if (AQ) rel += __ldg(zq_tile + (long long)ci * zq_S + e);
            if (AK) rel += __ldg(zk_row[hf] + e);
            if (BIAS) rel += __ldg(bexp + e);
            pv = exp2f((s[nt][r] + rel) * sc - l2);
          }
          const float ds = pv * (dp[nt][r] - dd);
          s[nt][r] = pv;
          dp[nt][r] = ds;
          if (DZK && keep) {
            const float val = p.tau * ds;
            if (delta <= p.E_lo) sat_lo[hf] += val;
            else if (delta >= p.E_hi) sat_hi[hf] += val;
            else dzk_row[hf][e] = val;
          }
        }
      }
    }
    uint32_t pa[4][4], sa[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      pa[kk][0] = DT<T>::pack(s[2 * kk][0], s[2 * kk][1]);
      pa[kk][1] = DT<T>::pack(s[2 * kk][2], s[2 * kk][3]);
      pa[kk][2] = DT<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[kk][3] = DT<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      sa[kk][0] = DT<T>::pack(dp[2 * kk][0], dp[2 * kk][1]);
      sa[kk][1] = DT<T>::pack(dp[2 * kk][2], dp[2 * kk][3]);
      sa[kk][2] = DT<T>::pack(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
      sa[kk][3] = DT<T>::pack(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
    }
    mma_ab<T, 4>(dv, pa, sD, 0, lane);   // dV += P^T dO
    mma_ab<T, 4>(dk, sa, sQ, 0, lane);   // dK += dS^T Q
    __syncthreads();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int j = jrow[hf];
    if (DZK) {
      float lo = sat_lo[hf], hi = sat_hi[hf];
      lo += __shfl_xor_sync(0xffffffffu, lo, 1);
      lo += __shfl_xor_sync(0xffffffffu, lo, 2);
      hi += __shfl_xor_sync(0xffffffffu, hi, 1);
      hi += __shfl_xor_sync(0xffffffffu, hi, 2);
      if (j < N && tq == 0) {
        const GroupInfo gi = p.gk[kt];
        if (p.Rexp == 1) {
          dzk_row[hf][0] = lo + hi;
        } else {
          if (gi.e0 == 0) dzk_row[hf][0] = lo;
          if (p.Rexp - 1 < gi.e0 + gi.W) dzk_row[hf][p.Rexp - 1] = hi;
        }
      }
    }
    if (j < N) {
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const float a0 = dk[dt][2 * hf] * p.tau, a1 = dk[dt][2 * hf + 1] * p.tau;
        if (DK32) St2<float>::two(t.dk_acc + off + (size_t)j * 64 + dt * 8 + 2 * tq, a0, a1);
        else St2<T>::two(static_cast<T*>(t.dk) + off + (size_t)j * 64 + dt * 8 + 2 * tq, a0, a1);
        St2<T>::two(static_cast<T*>(t.dv) + off + (size_t)j * 64 + dt * 8 + 2 * tq, dv[dt][2 * hf], dv[dt][2 * hf + 1]);
      }
    }
  }
}

template <typename K>
cudaError_t launch_k(K kern, dim3 grid, int smem, const Plan& p, const Tensors& t, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  { kern<<<grid, kThreads, smem, s>>>(p, t); note_launch(1); }
  return cudaGetLastError();
}

template <typename T>
cudaError_t dq_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  const bool aq = t.aq_exp, ak = t.ak_exp, bb = t.b_exp;
  const bool dz = aq || bb;   // dZ^Q feeds daQ and db
  dim3 grid(p.nT, p.B * p.H);
#define RP_DQ(A, K_, B_) \
  if (aq == A && ak == K_ && bb == B_) return launch_k(dq_kernel<T, A, K_, B_, (A || B_), A>, grid, kSmemDq, p, t, s);
  RP_DQ(false, false, false) RP_DQ(true, false, false) RP_DQ(false, true, false) RP_DQ(true, true, false)
  RP_DQ(false, false, true) RP_DQ(true, false, true) RP_DQ(false, true, true) RP_DQ(true, true, true)
#undef RP_DQ
  (void)dz;
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dk_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  const bool aq = t.aq_exp, ak = t.ak_exp, bb = t.b_exp;
  dim3 grid(p.nT, p.B * p.H);
#define RP_DK(A, K_, B_) \
  if (aq == A && ak == K_ && bb == B_) return launch_k(dkdv_kernel<T, A, K_, B_, K_, K_>, grid, kSmemDk, p, t, s);
  RP_DK(false, false, false) RP_DK(true, false, false) RP_DK(false, true, false) RP_DK(true, true, false)
  RP_DK(false, false, true) RP_DK(true, false, true) RP_DK(false, true, true) RP_DK(true, true, true)
#undef RP_DK
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_bwd_prep(const Plan& p, const Tensors& t, cudaStream_t s) {
  const long long rows = (long long)p.B * p.H * p.N;
  const long long threads = rows * 8;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (t.is_bf16) {
    if (t.o_f32) { prep_kernel<float, __nv_bfloat16><<<blocks, 256, 0, s>>>((const float*)t.o, (const __nv_bfloat16*)t.dout, t.dsum, rows); note_launch(1); }
    else { prep_kernel<__nv_bfloat16, __nv_bfloat16><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)t.o, (const __nv_bfloat16*)t.dout, t.dsum, rows); note_launch(1); }
  } else {
    if (t.o_f32) { prep_kernel<float, __half><<<blocks, 256, 0, s>>>((const float*)t.o, (const __half*)t.dout, t.dsum, rows); note_launch(1); }
    else { prep_kernel<__half, __half><<<blocks, 256, 0, s>>>((const __half*)t.o, (const __half*)t.dout, t.dsum, rows); note_launch(1); }
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const Plan& p, const Tensors& t, cudaStream_t s) {
  return t.is_bf16 ? dq_typed<__nv_bfloat16>(p, t, s) : dq_typed<__half>(p, t, s);
}

cudaError_t launch_bwd_dkdv(const Plan& p, const Tensors& t, cudaStream_t s) {
  return t.is_bf16 ? dk_typed<__nv_bfloat16>(p, t, s) : dk_typed<__half>(p, t, s);
}

}  // namespace relpos
