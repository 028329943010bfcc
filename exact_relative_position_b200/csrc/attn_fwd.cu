// attn_fwd.cu -- fused forward of exact relative-position attention
// (digest of "Fast and Exact Relative-Position Attention via Structure-Aware
// Kernels": Eq. (1)/(2) and the FlashAttention-style outer loop over query
// tiles with an online softmax over key tiles).
//
// One CTA owns 128 query rows of one (batch, head).  Q stays in registers as
// tensor-core fragments; K/V tiles of 64 keys stream through a two-stage
// cp.async ring.  Each score gets tau * (Z^Q[i,e] + Z^K[j,e] + b[e]) added in
// registers, e = clamp(j - i, E_lo, E_hi) - E_lo being the expanded relation
// row, before the base-2 online softmax.  No N x N tensor touches memory.
#include "kernels.cuh"
#include "warp_mma.cuh"

namespace relpos {

namespace {

constexpr int kBM = 128;   // query rows per CTA (8 warps x 16)
constexpr int kBN = 64;    // keys per inner step
constexpr int kThreads = 256;
constexpr int kSmem = kBM * 128 + 2 * 2 * kBN * 128;   // Q + 2 stages of (K, V)

template <typename OutT> struct Store;
template <> struct Store<float> {
  static __device__ __forceinline__ void two(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
};
template <> struct Store<__half> {
  static __device__ __forceinline__ void two(__half* p, float a, float b) { *reinterpret_cast<__half2*>(p) = __floats2half2_rn(a, b); }
};
template <> struct Store<__nv_bfloat16> {
  static __device__ __forceinline__ void two(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
  }
};

template <typename T, typename OutT, bool AQ, bool AK, bool BIAS>
__global__ void __launch_bounds__(kThreads) fwd_kernel(const Plan p, const Tensors t) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int N = p.N, q0 = qt * kBM;
  const size_t off = (size_t)bh * N * 64;
  const T* Q = static_cast<const T*>(t.q) + off;
  const T* K = static_cast<const T*>(t.k) + off;
  const T* V = static_cast<const T*>(t.v) + off;

  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + kBM * 128;

  const int nkv = p.padding ? p.key_len[b] : N;
  int kend = nkv;
  if (p.causal) kend = imin(kend, imin(q0 + kBM, N));
  const int ntiles = kend > 0 ? (kend + kBN - 1) / kBN : 0;

  load_tile_async<kBM, kThreads>(sQ, Q, q0, N, tid);
  if (ntiles > 0) {
    load_tile_async<kBN, kThreads>(sKV, K, 0, N, tid);
    load_tile_async<kBN, kThreads>(sKV + kBN * 128, V, 0, N, tid);
  }
  cp_async_commit();

  // Per-thread rows: hf = 0 -> row g, hf = 1 -> row g + 8 of the warp's 16.
  const int g = lane >> 2, tq = lane & 3;
  int irow[2];
  const float* zq_row[2] = {nullptr, nullptr};
  irow[0] = q0 + warp * 16 + g;
  irow[1] = irow[0] + 8;
  if (AQ) {
    const GroupInfo gi = p.gq[qt];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
      zq_row[hf] = t.zq + (size_t)bh * p.zq_head + gi.base + (long long)(irow[hf] - q0) * gi.S - gi.e0;
  }
  const float* bexp = BIAS ? t.b_exp + (size_t)h * p.Rexp : nullptr;
  const float sc = p.tau * kLog2e;

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  uint32_t qa[4][4];

  for (int it = 0; it < ntiles; ++it) {
    const int stage = it & 1;
    if (it + 1 < ntiles) {
      const uint32_t sb = sKV + (uint32_t)((it + 1) & 1) * (2 * kBN * 128);
      load_tile_async<kBN, kThreads>(sb, K, (it + 1) * kBN, N, tid);
      load_tile_async<kBN, kThreads>(sb + kBN * 128, V, (it + 1) * kBN, N, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) load_a_frags(sQ, warp * 16, lane, qa);
    const uint32_t sK = sKV + (uint32_t)stage * (2 * kBN * 128);
    const uint32_t sV = sK + kBN * 128;
    const int k0 = it * kBN;

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    mma_abt<T, 8>(s, qa, sK, 0, lane);

    // Key-side projection rows of this key tile (64 keys lie in one 128-group).
    const float* zk_tile = nullptr;
    if (AK) {
      const int kg = k0 / kTile;
      const GroupInfo gi = p.gk[kg];
      zk_tile = t.zk + (size_t)bh * p.zk_head + gi.base - gi.e0 + (long long)(k0 - kg * kTile) * gi.S;
      // element for key k0 + c at expanded row e: zk_tile[c * S + e]
    }
    const int zk_S = AK ? p.gk[k0 / kTile].S : 0;

    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int hf = r >> 1;
        const int cj = nt * 8 + 2 * tq + (r & 1);
        const int i = irow[hf], j = k0 + cj;
        float x = -INFINITY;
        const bool keep = (i < N) && (j < nkv) && !(p.causal && j > i);
        if (keep) {
          const int e = iclamp(j - i, p.E_lo, p.E_hi) - p.E_lo;
          float rel = 0.f;
          if (AQ) rel += __ldg(zq_row[hf] + e);
          if (AK) rel += __ldg(zk_tile + (long long)cj * zk_S + e);
          if (BIAS) rel += __ldg(bexp + e);
          x = (s[nt][r] + rel) * sc;
        }
        s[nt][r] = x;
        mx[hf] = fmaxf(mx[hf], x);
      }
    }
    float alpha[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 1));
      mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 2));
      const float m_new = fmaxf(m_run[hf], mx[hf]);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      alpha[hf] = exp2f(m_run[hf] - m_use);
      m_run[hf] = m_new;
      mx[hf] = m_use;
      l_run[hf] *= alpha[hf];
    }
#pragma unroll
    for (int dt = 0; dt < 8; ++dt) {
      o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
      o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pv = exp2f(s[nt][r] - mx[r >> 1]);
        s[nt][r] = pv;
        l_run[r >> 1] += pv;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      pa[kk][0] = DT<T>::pack(s[2 * kk][0], s[2 * kk][1]);
      pa[kk][1] = DT<T>::pack(s[2 * kk][2], s[2 * kk][3]);
      pa[kk][2] = DT<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[kk][3] = DT<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    }
    mma_ab<T, 4>(o, pa, sV, 0, lane);
    __syncthreads();
  }
  cp_async_wait<0>();

  OutT* O = static_cast<OutT*>(t.o) + off;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float l = l_run[hf];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int i = irow[hf];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (i < N) {
#pragma unroll
      for (int dt = 0; dt < 8; ++dt)
        Store<OutT>::two(O + (size_t)i * 64 + dt * 8 + 2 * tq, o[dt][2 * hf] * inv, o[dt][2 * hf + 1] * inv);
      if (tq == 0) t.lse[(size_t)bh * N + i] = l > 0.f ? (m_run[hf] + log2f(l)) * kLn2 : -INFINITY;
    }
  }
}

template <typename T, typename OutT>
cudaError_t launch_typed(const Plan& p, const Tensors& t, cudaStream_t s) {
  const int mask = (t.aq_exp ? 1 : 0) | (t.ak_exp ? 2 : 0) | (t.b_exp ? 4 : 0);
  void (*kern)(const Plan, const Tensors) = nullptr;
  switch (mask) {
    case 0: kern = fwd_kernel<T, OutT, false, false, false>; break;
    case 1: kern = fwd_kernel<T, OutT, true, false, false>; break;
    case 2: kern = fwd_kernel<T, OutT, false, true, false>; break;
    case 3: kern = fwd_kernel<T, OutT, true, true, false>; break;
    case 4: kern = fwd_kernel<T, OutT, false, false, true>; break;
    case 5: kern = fwd_kernel<T, OutT, true, false, true>; break;
    case 6: kern = fwd_kernel<T, OutT, false, true, true>; break;
    default: kern = fwd_kernel<T, OutT, true, true, true>; break;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + kBM - 1) / kBM, p.B * p.H);
  { kern<<<grid, kThreads, kSmem, s>>>(p, t); note_launch(1); }
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
