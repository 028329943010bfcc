// api.cu -- the C ABI (include/relpos_attn.h): argument validation, the host
// planner (expanded offset range, projection group geometry, workspace
// layout) and the launch sequence of the forward and backward passes.
//
// Forward  (digest of "Fast and Exact Relative-Position Attention via
//           Structure-Aware Kernels", pipeline section):
//   tables -> projection Z^Q, Z^K over reachable columns -> fused attention.
// Backward (two-pass backward, Eq. (4)):
//   tables -> projection -> D -> Q-parallel pass (dQ, dZ^Q) -> K-parallel pass
//   (dK, dV, dZ^K) -> relation GEMMs, split sums and bucket fold.
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "kernels.cuh"
#include "sm100.cuh"

#define RELPOS_EXPORT extern "C" __attribute__((visibility("default")))

namespace relpos {
static std::atomic<long long> g_kernel_launches{0};
void note_launch(int n) { g_kernel_launches += n; }
}  // namespace relpos

using namespace relpos;

namespace {
int cuda_fail(cudaError_t e);
}

int relpos::cuda_status(cudaError_t e) { return cuda_fail(e); }

namespace {

// ---- optional per-phase event timing (relpos_profile_start / _stop)
enum Phase { PH_TABLES, PH_PROJ, PH_FWD, PH_PREP, PH_DQ, PH_DKDV, PH_FOLD, PH_RELGRAD, PH_BWD_ATTN, PH_COUNT };
const char* const kPhaseNames[PH_COUNT] = {"tables",  "projection", "fwd_attention", "bwd_prep",     "bwd_dq",
                                           "bwd_dkdv", "fold_ranges", "relation_grads", "bwd_attention"};
// Duration a -> b, or a -> the later of b and c when c is set (two streams).
struct PhaseEvent {
  int phase, kernels;
  cudaEvent_t a, b, c;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<PhaseEvent> g_prof_events;

template <typename F>
cudaError_t run_phase(int ph, cudaStream_t s, F&& f) {
  if (!g_prof_on.load()) return f();
  cudaEvent_t a = nullptr, b = nullptr;
  if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return f();
  const long long before = g_kernel_launches.load();
  cudaEventRecord(a, s);
  const cudaError_t e = f();
  cudaEventRecord(b, s);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_events.push_back({ph, (int)(g_kernel_launches.load() - before), a, b, nullptr});
  return e;
}

// "bwd_attention": both backward passes, which run concurrently on two
// streams, from the start of the first to the end of the later one.
struct PairTimer {
  cudaEvent_t a = nullptr, b = nullptr, c = nullptr;
  PairTimer() {
    if (!g_prof_on.load()) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess ||
        cudaEventCreate(&c) != cudaSuccess) {
      cudaGetLastError();
      a = b = c = nullptr;
    }
  }
  void start(cudaStream_t s) { if (a) cudaEventRecord(a, s); }
  void end_first(cudaStream_t s) { if (b) cudaEventRecord(b, s); }
  void end_second(cudaStream_t s) { if (c) cudaEventRecord(c, s); }
  void commit(int kernels) {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_events.push_back({PH_BWD_ATTN, kernels, a, b, c});
  }
};

// Extra streams per device, created once (non-blocking, never destroyed):
// 0 carries the K-parallel backward pass, 1 and 2 the relation-gradient row
// updates of the query and the key side.  A fork records an event on the
// caller's stream and makes the side stream wait for it; join does the
// reverse, so work issued on the side stream in between is ordered before
// anything the caller issues afterwards (also under stream capture).  If the
// side stream or the events cannot be created the fork degrades to the
// caller's stream alone.
// A thread that sets single-stream mode gets no side stream: its forks
// degrade to the caller's stream and create no streams or events.
constexpr int kSideStreams = 3;
thread_local bool g_single_stream = false;
cudaStream_t side_stream(int which) {
  static std::mutex mu;
  static cudaStream_t streams[64][kSideStreams] = {};
  int dev = 0;
  if (g_single_stream || which < 0 || which >= kSideStreams) return nullptr;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  cudaStream_t& st = streams[dev][which];
  if (!st && cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    st = nullptr;
  }
  return st;
}

class Fork {
 public:
  explicit Fork(cudaStream_t s, int which = 0) : s_(s), side_(s) {
    cudaStream_t s2 = side_stream(which);
    if (!s2 || cudaEventCreateWithFlags(&fork_, cudaEventDisableTiming) != cudaSuccess) return;
    if (cudaEventCreateWithFlags(&join_, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(fork_, s) != cudaSuccess || cudaStreamWaitEvent(s2, fork_, 0) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    side_ = s2;
  }
  cudaStream_t side() const { return side_; }
  cudaError_t join() {
    cudaError_t e = cudaSuccess;
    if (side_ != s_) {
      e = cudaEventRecord(join_, side_);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s_, join_, 0);
    }
    return e;
  }
  ~Fork() {
    if (fork_) cudaEventDestroy(fork_);
    if (join_) cudaEventDestroy(join_);
  }

 private:
  cudaStream_t s_, side_;
  cudaEvent_t fork_ = nullptr, join_ = nullptr;
};

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return RELPOS_ERR_CUDA;
}

constexpr int kMaxN = 1 << 22;

// Limit of the fused kernels' bounded waits for launches planned from now on
// (0: the built-in 2 s).  Process-wide; only tests lower it.
std::atomic<unsigned long long> g_wait_limit_ns{0};

int check_map(const relpos_map_desc* m) {
  if (!m) return RELPOS_ERR_INVALID_ARG;
  switch (m->kind) {
    case RELPOS_MAP_TRUNCATED:
      return (m->clip >= 0 && m->clip <= kMaxN) ? RELPOS_OK : RELPOS_ERR_INVALID_ARG;
    case RELPOS_MAP_IDENTITY:
      return RELPOS_OK;
    case RELPOS_MAP_BUCKET_T5: {
      const int h = m->bidirectional ? m->num_buckets / 2 : m->num_buckets;
      if (m->num_buckets < 2 || m->num_buckets > 65536 || h < 2) return RELPOS_ERR_INVALID_ARG;
      if (m->max_distance <= h / 2) return RELPOS_ERR_INVALID_ARG;
      return RELPOS_OK;
    }
    case RELPOS_MAP_BUCKET_LOG:
    case RELPOS_MAP_BUCKET_LOG_REVERSED: {
      if (m->num_buckets < 2 || m->num_buckets > 65536) return RELPOS_ERR_INVALID_ARG;
      if (m->max_distance - 1 <= m->num_buckets / 2) return RELPOS_ERR_INVALID_ARG;
      return RELPOS_OK;
    }
    default:
      return RELPOS_ERR_UNSUPPORTED;
  }
}

int rows_of(const relpos_map_desc& m, int N) {
  switch (m.kind) {
    case RELPOS_MAP_TRUNCATED: return 2 * m.clip + 1;
    case RELPOS_MAP_IDENTITY: return 2 * N - 1;
    case RELPOS_MAP_BUCKET_T5: return m.num_buckets;
    default: return 2 * m.num_buckets;
  }
}

// Leading / trailing runs of offsets that share one row (see header).
void bounds_of(const relpos_map_desc& m, int N, int* lo, int* hi) {
  if (m.kind == RELPOS_MAP_IDENTITY) { *lo = 1 - N; *hi = N - 1; return; }
  if (m.kind == RELPOS_MAP_TRUNCATED) {
    *lo = std::max(-m.clip, 1 - N);
    *hi = std::min(m.clip, N - 1);
    if (*hi < *lo) *hi = *lo;
    // clip 0: every offset maps to row 0; the leading run covers everything
    if (m.clip == 0) { *lo = N - 1; *hi = N - 1; }
    return;
  }
  const int p0 = phi_of(m, N, 1 - N);
  int d = 1 - N;
  while (d + 1 <= N - 1 && phi_of(m, N, d + 1) == p0) ++d;
  *lo = d;
  const int p1 = phi_of(m, N, N - 1);
  d = N - 1;
  while (d - 1 >= 1 - N && phi_of(m, N, d - 1) == p1) --d;
  *hi = std::max(d, *lo);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
  size_t status, zksat, gq, gk, phi, fold_lo, fold_hi, bexp, aqe, ake, zq, zk, fwd_end;
  size_t dsum, lse2, zqsat, dzq, dzk, dzqs, dzks, dqacc, dkacc, daqp, dakp, dbp, bwd_end;
  int R, Hq, expand, nsq, nsk, nsb;
  int recompute;   // projection = RECOMPUTE: Z^Q lives in the backward-only part
};

int make_plan(const relpos_fwd_args* a, Plan* p, Layout* L) {
  if (!a) return RELPOS_ERR_INVALID_ARG;
  if (a->d != kHeadDim) return RELPOS_ERR_UNSUPPORTED;
  if (a->dtype != RELPOS_F16 && a->dtype != RELPOS_BF16) return RELPOS_ERR_UNSUPPORTED;
  if (a->out_dtype != a->dtype && a->out_dtype != RELPOS_F32) return RELPOS_ERR_UNSUPPORTED;
  if (a->B < 1 || a->H < 1 || a->N < 1 || a->N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  if ((long long)a->B * a->H > 65535) return RELPOS_ERR_INVALID_ARG;
  if (a->mask & ~(RELPOS_MASK_CAUSAL | RELPOS_MASK_KEY_PADDING)) return RELPOS_ERR_UNSUPPORTED;
  // tau > 0 and finite: the kernels fold tau into the base-2 exponent and take
  // row maxima of the scaled scores, which assumes a positive scale
  if (!(a->tau > 0.f) || a->tau > 3.0e38f) return RELPOS_ERR_INVALID_ARG;
  int st = check_map(&a->map);
  if (st) return st;
  if (a->projection != RELPOS_PROJECTION_RETAINED && a->projection != RELPOS_PROJECTION_RECOMPUTE)
    return RELPOS_ERR_INVALID_ARG;
  if (a->projection == RELPOS_PROJECTION_RECOMPUTE && a->ak) return RELPOS_ERR_UNSUPPORTED;
  memset(p, 0, sizeof(*p));
  memset(L, 0, sizeof(*L));
  const int N = a->N;
  p->B = a->B; p->H = a->H; p->N = N;
  bounds_of(a->map, N, &p->E_lo, &p->E_hi);
  p->Rexp = p->E_hi - p->E_lo + 1;
  p->nT = (N + kTile - 1) / kTile;
  p->grouped = p->Rexp > N + kTile - 1;
  p->causal = (a->mask & RELPOS_MASK_CAUSAL) != 0;
  // causal: the forward and Q-parallel grids take query tiles (pairs) longest first
  p->qrev = p->causal ? p->nT - 1 : 0;
  p->qrev_pair = p->causal ? (N + 2 * kTile - 1) / (2 * kTile) - 1 : 0;
  p->padding = (a->mask & RELPOS_MASK_KEY_PADDING) != 0;
  p->tau = a->tau;
  if (!(a->dropout_p >= 0.f && a->dropout_p < 1.f)) return RELPOS_ERR_INVALID_ARG;
  p->dropout = a->dropout_p > 0.f;
  // 8-bit uniforms: the realised rate is p rounded up to a multiple of 1/256,
  // and the kept cells are scaled by the reciprocal of its keep probability
  p->drop_thresh = (uint32_t)ceil((double)a->dropout_p * 256.0);
  p->drop_scale = p->dropout ? (float)(256.0 / (256.0 - (double)p->drop_thresh)) : 1.f;
  p->seed_lo = (uint32_t)(a->dropout_seed & 0xFFFFFFFFull);
  p->seed_hi = (uint32_t)(a->dropout_seed >> 32);
  p->drop_offset = a->dropout_offset;
  if (a->cu_seqlens) {
    // packed variable-length batch: the sequence lengths mask the keys
    if ((a->mask & RELPOS_MASK_KEY_PADDING) || a->total_tokens < 1) return RELPOS_ERR_INVALID_ARG;
    p->packed = 1;
    p->T = a->total_tokens;
    p->cu = a->cu_seqlens;
  }
  {
    const unsigned long long lim = g_wait_limit_ns.load();
    p->wait_ns = lim ? lim : (unsigned long long)sm100::kTimeoutNs;
  }
  const bool aq = a->aq != nullptr, ak = a->ak != nullptr, bb = a->b != nullptr;
  const long long zq_head = head_elems(*p, 0), zk_head = head_elems(*p, 1);
  p->zq_head = (aq || bb) ? zq_head : 0;
  p->zk_head = ak ? zk_head : 0;
  L->R = rows_of(a->map, N);
  L->Hq = a->table_per_head ? a->H : 1;
  L->expand = a->map.kind == RELPOS_MAP_BUCKET_T5 || a->map.kind == RELPOS_MAP_BUCKET_LOG ||
              a->map.kind == RELPOS_MAP_BUCKET_LOG_REVERSED;
  L->recompute = a->projection == RELPOS_PROJECTION_RECOMPUTE;
  const size_t BH = (size_t)a->B * a->H;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = up256(off + bytes); return o; };
  L->status = take(sizeof(int));
  L->gq = take(sizeof(GroupInfo) * p->nT);
  L->gk = take(sizeof(GroupInfo) * p->nT);
  L->phi = take(sizeof(int) * p->Rexp);
  L->fold_lo = take(sizeof(int) * L->R);
  L->fold_hi = take(sizeof(int) * L->R);
  L->bexp = bb ? take(sizeof(float) * a->H * p->Rexp) : 0;
  L->aqe = (aq && L->expand) ? take((size_t)2 * L->Hq * p->Rexp * 64) : 0;
  L->ake = (ak && L->expand) ? take((size_t)2 * L->Hq * p->Rexp * 64) : 0;
  L->zq = (aq && !L->recompute) ? take(sizeof(float) * BH * p->zq_head) : 0;
  L->zk = ak ? take(sizeof(float) * BH * p->zk_head) : 0;
  L->zksat = ak ? take(sizeof(float) * BH * 2 * (size_t)p->nT * kTile) : 0;
  L->fwd_end = off;
  // a recomputing forward stores no projection; its backward rebuilds Z^Q here
  if (aq && L->recompute) L->zq = take(sizeof(float) * BH * p->zq_head);
  const size_t npad = (size_t)p->nT * kTile;
  L->dsum = take(sizeof(float) * BH * npad);
  L->lse2 = take(sizeof(float) * BH * npad);
  L->zqsat = (aq || bb) ? take(sizeof(float) * BH * 2 * npad) : 0;
  // relation gradients: 16-bit interior entries, fp32 saturated-offset sums per row
  L->dzq = (aq || bb) ? take(2 * BH * p->zq_head) : 0;
  L->dzk = ak ? take(2 * BH * p->zk_head) : 0;
  L->dzqs = (aq || bb) ? take(sizeof(float) * BH * npad * 2) : 0;
  L->dzks = ak ? take(sizeof(float) * BH * npad * 2) : 0;
  L->dqacc = aq ? take(sizeof(float) * BH * N * 64) : 0;
  L->dkacc = ak ? take(sizeof(float) * BH * N * 64) : 0;
  const int nE = (p->Rexp + 255) / 256;   // expanded-row blocks of the table-gradient kernel
  const long long items = a->table_per_head ? (long long)a->B * p->nT : (long long)BH * p->nT;
  auto pick = [](long long want, long long items_) {
    long long s = std::max(1LL, want);
    s = std::min(s, items_);
    s = std::min(s, 256LL);
    return (int)std::max(1LL, s);
  };
  L->nsq = pick(148LL / ((long long)nE * L->Hq), items);   // one table-gradient CTA per SM
  // a grouped map (the identity map) gives the table-gradient blocks very uneven
  // work: an offset block near the diagonal is stored by every query group, one
  // far from it by a few.  Eight splits spread the long blocks' items.
  if (p->grouped) L->nsq = std::max(L->nsq, pick(8, items));
  L->nsk = L->nsq;
  // with per-head aQ tables the bias gradient comes out of the aQ table-gradient
  // pass, on its splits
  L->nsb = (aq && a->table_per_head) ? L->nsq
                                     : pick(592LL / ((long long)((p->Rexp + 255) / 256) * a->H), (long long)a->B * p->nT);
  L->daqp = aq ? take(sizeof(float) * (size_t)L->nsq * L->Hq * p->Rexp * 64) : 0;
  L->dakp = ak ? take(sizeof(float) * (size_t)L->nsk * L->Hq * p->Rexp * 64) : 0;
  L->dbp = bb ? take(sizeof(float) * (size_t)L->nsb * a->H * p->Rexp) : 0;
  L->bwd_end = off;
  return RELPOS_OK;
}

int check_fwd_ptrs(const relpos_fwd_args* a) {
  if (!a->q || !a->k || !a->v || !a->o || !a->lse) return RELPOS_ERR_INVALID_ARG;
  if ((a->mask & RELPOS_MASK_KEY_PADDING) && !a->key_len) return RELPOS_ERR_INVALID_ARG;
  const void* al[] = {a->q, a->k, a->v, a->o, a->aq, a->ak};
  for (const void* x : al)
    if (x && !aligned16(x)) return RELPOS_ERR_INVALID_ARG;
  return RELPOS_OK;
}

// Resolve workspace regions and the expanded-table pointers; launch the
// table builder and the projections (shared by forward and backward).
// Pointers into the workspace for a call with these arguments; when `build`
// is set, also (re)computes the tables, group records and projections there
// (the forward always builds; the backward skips it when the caller declares
// the forward's state still in the workspace).
int prepare(const relpos_fwd_args* a, Plan& p, const Layout& L, uint8_t* ws, Tensors& t, cudaStream_t s,
            bool build = true, bool build_projection = true) {
  memset(&t, 0, sizeof(t));
  GroupInfo* gq = reinterpret_cast<GroupInfo*>(ws + L.gq);
  GroupInfo* gk = reinterpret_cast<GroupInfo*>(ws + L.gk);
  p.gq = gq;
  p.gk = gk;
  p.key_len = a->key_len;
  t.q = a->q; t.k = a->k; t.v = a->v;
  t.o = a->o; t.o_f32 = a->out_dtype == RELPOS_F32; t.lse = a->lse;
  t.is_bf16 = a->dtype == RELPOS_BF16;
  t.table_per_head = a->table_per_head;
  t.R = L.R;
  t.status = reinterpret_cast<int*>(ws + L.status);
  {
    const cudaError_t e0 = cudaMemsetAsync(t.status, 0, sizeof(int), s);
    if (e0 != cudaSuccess) return cuda_fail(e0);
  }
  int* phi_exp = reinterpret_cast<int*>(ws + L.phi);
  t.phi_exp = phi_exp;
  t.fold_lo = reinterpret_cast<int*>(ws + L.fold_lo);
  t.fold_hi = reinterpret_cast<int*>(ws + L.fold_hi);
  if (a->b) t.b_exp = reinterpret_cast<float*>(ws + L.bexp);
  // expanded-table row e <-> offset E_lo + e
  // truncated / identity maps use the caller's table in place: expanded row e is
  // table row phi(E_lo) + e (consecutive rows; for clip 0 the single row 0)
  long long row0 = 0;
  if (a->map.kind == RELPOS_MAP_TRUNCATED || a->map.kind == RELPOS_MAP_IDENTITY)
    row0 = phi_of(a->map, a->N, p.E_lo);
  const size_t esz = 2;
  if (a->aq) {
    if (L.expand) { t.aq_exp = ws + L.aqe; t.aq_hs = (long long)p.Rexp * 64; }
    else { t.aq_exp = static_cast<const uint8_t*>(a->aq) + row0 * 64 * esz; t.aq_hs = (long long)L.R * 64; }
    t.zq = reinterpret_cast<float*>(ws + L.zq);
  }
  if (a->ak) {
    if (L.expand) { t.ak_exp = ws + L.ake; t.ak_hs = (long long)p.Rexp * 64; }
    else { t.ak_exp = static_cast<const uint8_t*>(a->ak) + row0 * 64 * esz; t.ak_hs = (long long)L.R * 64; }
    t.zk = reinterpret_cast<float*>(ws + L.zk);
    t.zk_sat = reinterpret_cast<float*>(ws + L.zksat);
  }
  cudaError_t e = cudaSuccess;
  if (build) {
    e = run_phase(PH_TABLES, s, [&] {
      return launch_build_tables(p, a->map, gq, gk, phi_exp, L.R, a->aq, a->ak, a->table_per_head, ws + L.aqe,
                                 ws + L.ake, a->b, const_cast<float*>(t.b_exp), t.is_bf16, L.expand, s);
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (build_projection && (a->aq || a->ak)) {
    // Z^Q on the caller's stream, Z^K and its saturated columns beside it
    e = run_phase(PH_PROJ, s, [&] {
      Fork aux(s, 1);
      cudaError_t e1 = launch_projection(p, t, s, aux.side());
      if (e1 == cudaSuccess && a->ak) e1 = launch_saturated_columns(p, t, aux.side());
      const cudaError_t ej = aux.join();
      return e1 != cudaSuccess ? e1 : ej;
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return RELPOS_OK;
}

}  // namespace

namespace relpos {
void set_single_stream(bool on) { g_single_stream = on; }
}  // namespace relpos

RELPOS_EXPORT int relpos_table_rows(const relpos_map_desc* map, int32_t N, int32_t* R_out) {
  if (!map || !R_out || N < 1 || N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  *R_out = rows_of(*map, N);
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_expanded_bounds(const relpos_map_desc* map, int32_t N, int32_t* e_lo, int32_t* e_hi) {
  if (!map || !e_lo || !e_hi || N < 1 || N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  bounds_of(*map, N, e_lo, e_hi);
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_workspace_size(const relpos_fwd_args* a, size_t* fwd_bytes, size_t* bwd_bytes) {
  Plan p;
  Layout L;
  const int st = make_plan(a, &p, &L);
  if (st) return st;
  if (fwd_bytes) *fwd_bytes = L.fwd_end;
  if (bwd_bytes) *bwd_bytes = L.bwd_end;
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_attn_fwd(const relpos_fwd_args* a, void* workspace, size_t ws_bytes, relpos_stream_t stream) {
  Plan p;
  Layout L;
  int st = make_plan(a, &p, &L);
  if (st) return st;
  st = check_fwd_ptrs(a);
  if (st) return st;
  if (!workspace || ws_bytes < L.fwd_end || (reinterpret_cast<uintptr_t>(workspace) & 255)) return RELPOS_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Tensors t;
  // a recomputing forward builds the tables only; its kernel projects per tile
  st = prepare(a, p, L, static_cast<uint8_t*>(workspace), t, s, true, !L.recompute);
  if (st) return st;
  const cudaError_t e = run_phase(PH_FWD, s, [&] {
    return L.recompute ? launch_forward_recompute(p, t, s) : launch_forward(p, t, s);
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_attn_bwd(const relpos_bwd_args* g, void* workspace, size_t ws_bytes, relpos_stream_t stream) {
  if (!g) return RELPOS_ERR_INVALID_ARG;
  const relpos_fwd_args* a = &g->fwd;
  Plan p;
  Layout L;
  int st = make_plan(a, &p, &L);
  if (st) return st;
  st = check_fwd_ptrs(a);
  if (st) return st;
  if (!g->dout || !g->dq || !g->dk || !g->dv) return RELPOS_ERR_INVALID_ARG;
  if ((a->aq && !g->daq) || (a->ak && !g->dak) || (a->b && !g->db)) return RELPOS_ERR_INVALID_ARG;
  const void* al[] = {g->dout, g->dq, g->dk, g->dv, g->daq, g->dak, g->db};
  for (const void* x : al)
    if (x && !aligned16(x)) return RELPOS_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < L.bwd_end || (reinterpret_cast<uintptr_t>(workspace) & 255)) return RELPOS_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (g->reuse_forward_workspace != 0 && g->reuse_forward_workspace != 1) return RELPOS_ERR_INVALID_ARG;
  Tensors t;
  // reuse: the forward's tables (and, retained, its projections) are in the workspace;
  // after a recomputing forward the projection is always rebuilt
  st = prepare(a, p, L, ws, t, s, /*build=*/g->reuse_forward_workspace == 0,
               /*build_projection=*/g->reuse_forward_workspace == 0 || L.recompute);
  if (st) return st;
  t.dout = g->dout;
  t.dsum = reinterpret_cast<float*>(ws + L.dsum);
  t.lse2 = reinterpret_cast<float*>(ws + L.lse2);
  t.dq = g->dq; t.dk = g->dk; t.dv = g->dv;
  t.daq = g->daq; t.dak = g->dak; t.db = g->db;
  const size_t BH = (size_t)a->B * a->H;
  cudaError_t e;
  if (a->aq || a->b) {
    t.dzq = ws + L.dzq;
    t.dzq_sat = reinterpret_cast<float*>(ws + L.dzqs);
    e = cudaMemsetAsync(t.dzq, 0, 2 * BH * p.zq_head, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (a->ak) {
    t.dzk = ws + L.dzk;
    t.dzk_sat = reinterpret_cast<float*>(ws + L.dzks);
    e = cudaMemsetAsync(t.dzk, 0, 2 * BH * p.zk_head, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (a->aq) { t.dq_acc = reinterpret_cast<float*>(ws + L.dqacc); t.daq_part = reinterpret_cast<float*>(ws + L.daqp); }
  if (a->ak) { t.dk_acc = reinterpret_cast<float*>(ws + L.dkacc); t.dak_part = reinterpret_cast<float*>(ws + L.dakp); }
  if (a->b) t.db_part = reinterpret_cast<float*>(ws + L.dbp);
  t.nsplit_q = L.nsq; t.nsplit_k = L.nsk; t.nsplit_b = L.nsb;
  if ((e = run_phase(PH_PREP, s, [&] { return launch_bwd_prep(p, t, s); })) != cudaSuccess) return cuda_fail(e);
  if (a->aq || a->b) {
    // the saturated row constants fold in LSE log2e, so they follow the prep
    t.zq_sat = reinterpret_cast<float*>(ws + L.zqsat);
    if ((e = run_phase(PH_PROJ, s, [&] { return launch_saturated_rows(p, t, s); })) != cudaSuccess) return cuda_fail(e);
  }
  const bool terms = a->aq || a->ak || a->b;
  if (terms) {
    e = run_phase(PH_FOLD, s, [&] { return launch_fold_ranges(p, t.phi_exp, L.R, t.fold_lo, t.fold_hi, s); });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  // The Q-parallel pass (then the query-side relation gradients) stays on the
  // caller's stream; the K-parallel pass (then the key side) runs on a second
  // stream forked from it, so that its CTAs fill the SMs the other pass leaves
  // idle in its last partial wave.  The caller's stream waits for both.
  Fork fork(s);
  cudaStream_t s2 = fork.side();
  cudaError_t e2 = cudaSuccess;
  PairTimer pair;
  pair.start(s);
  e = run_phase(PH_DQ, s, [&] { return launch_bwd_dq(p, t, s); });
  pair.end_first(s);
  e2 = run_phase(PH_DKDV, s2, [&] { return launch_bwd_dkdv(p, t, s2); });
  pair.end_second(s2);
  pair.commit(2);
  // each side's dQ / dK row update runs beside its table-gradient kernels
  auto relgrad = [&](int side, cudaStream_t st) {
    return run_phase(PH_RELGRAD, st, [&] {
      Fork aux(st, 1 + side);
      const cudaError_t el = launch_relgrad(p, t, side, st, aux.side());
      const cudaError_t ea = aux.join();
      return el != cudaSuccess ? el : ea;
    });
  };
  if (terms && e == cudaSuccess) e = relgrad(0, s);
  if (a->ak && e2 == cudaSuccess) e2 = relgrad(1, s2);
  const cudaError_t ej = fork.join();
  if (e != cudaSuccess) return cuda_fail(e);
  if (e2 != cudaSuccess) return cuda_fail(e2);
  if (ej != cudaSuccess) return cuda_fail(ej);
  return RELPOS_OK;
}

static_assert(sizeof(relpos_group_info) == sizeof(GroupInfo), "relpos_group_info mirrors GroupInfo");
static_assert(offsetof(relpos_group_info, base) == offsetof(GroupInfo, base), "relpos_group_info mirrors GroupInfo");

RELPOS_EXPORT int relpos_debug_projection(const relpos_fwd_args* a_in, void* workspace, size_t ws_bytes,
                                          relpos_stream_t stream, relpos_projection_layout* layout) {
  if (!a_in) return RELPOS_ERR_INVALID_ARG;
  // the stored projection is the retained mode's
  relpos_fwd_args args = *a_in;
  args.projection = RELPOS_PROJECTION_RETAINED;
  const relpos_fwd_args* a = &args;
  Plan p;
  Layout L;
  int st = make_plan(a, &p, &L);
  if (st) return st;
  if (!layout || !a->q || !a->k) return RELPOS_ERR_INVALID_ARG;
  if ((a->mask & RELPOS_MASK_KEY_PADDING) && !a->key_len) return RELPOS_ERR_INVALID_ARG;
  const void* al[] = {a->q, a->k, a->aq, a->ak};
  for (const void* x : al)
    if (x && !aligned16(x)) return RELPOS_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < L.fwd_end || (reinterpret_cast<uintptr_t>(workspace) & 255)) return RELPOS_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Tensors t;
  st = prepare(a, p, L, static_cast<uint8_t*>(workspace), t, s);
  if (st) return st;
  const cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  layout->E_lo = p.E_lo;
  layout->E_hi = p.E_hi;
  layout->R_exp = p.Rexp;
  layout->nT = p.nT;
  layout->grouped = p.grouped;
  layout->pad = 0;
  layout->zq_offset = a->aq ? (int64_t)L.zq : -1;
  layout->zk_offset = a->ak ? (int64_t)L.zk : -1;
  layout->zq_head = a->aq ? p.zq_head : 0;
  layout->zk_head = a->ak ? p.zk_head : 0;
  layout->gq_offset = (int64_t)L.gq;
  layout->gk_offset = (int64_t)L.gk;
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store((unsigned long long)ns);
  return RELPOS_OK;
}

RELPOS_EXPORT const char* relpos_status_string(int status) {
  switch (status) {
    case RELPOS_OK: return "ok";
    case RELPOS_ERR_INVALID_ARG: return "invalid argument";
    case RELPOS_ERR_UNSUPPORTED: return "unsupported configuration";
    case RELPOS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case RELPOS_ERR_CUDA: return "CUDA error (see relpos_last_cuda_error)";
    case RELPOS_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

RELPOS_EXPORT int relpos_last_cuda_error(void) { return g_last_cuda_error; }

RELPOS_EXPORT int relpos_check_workspace(const void* workspace, relpos_stream_t stream, int32_t* device_status) {
  if (!workspace) return RELPOS_ERR_INVALID_ARG;
  int st = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (device_status) *device_status = st;
  return st == 0 ? RELPOS_OK : RELPOS_ERR_TIMEOUT;
}

RELPOS_EXPORT int relpos_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& ev : g_prof_events) {
    cudaEventDestroy(ev.a);
    cudaEventDestroy(ev.b);
    if (ev.c) cudaEventDestroy(ev.c);
  }
  g_prof_events.clear();
  g_prof_on = true;
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_profile_stop(relpos_phase_stat* stats, int32_t max_stats, int32_t* n_stats) {
  g_prof_on = false;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  relpos_phase_stat agg[PH_COUNT];
  memset(agg, 0, sizeof(agg));
  int status = RELPOS_OK;
  for (auto& ev : g_prof_events) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(ev.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, ev.a, ev.b);
    if (e == cudaSuccess && ev.c) {
      float ms2 = 0.f;
      e = cudaEventSynchronize(ev.c);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms2, ev.a, ev.c);
      ms = std::max(ms, ms2);
    }
    if (e != cudaSuccess) status = cuda_fail(e);
    agg[ev.phase].calls += 1;
    agg[ev.phase].kernels += ev.kernels;
    agg[ev.phase].total_ms += ms;
    cudaEventDestroy(ev.a);
    cudaEventDestroy(ev.b);
    if (ev.c) cudaEventDestroy(ev.c);
  }
  g_prof_events.clear();
  int n = 0;
  for (int ph = 0; ph < PH_COUNT; ++ph) {
    if (agg[ph].calls == 0) continue;
    strncpy(agg[ph].name, kPhaseNames[ph], sizeof(agg[ph].name) - 1);
    if (stats && n < max_stats) stats[n] = agg[ph];
    ++n;
  }
  if (n_stats) *n_stats = n;
  return status;
}

RELPOS_EXPORT int64_t relpos_kernel_launches(void) { return g_kernel_launches.load(); }

// ---------------------------------------------------------------- data-parallel exchange
namespace relpos {
namespace {
// out[i] = ((p[0][i] + p[1][i]) + p[2][i]) + ... : one thread per entry, rows
// added in ascending order, so the bits do not depend on the launch shape.
// out may be row 0 of p (each entry is read before it is written).
__global__ void sum_partials_kernel(const float* p, int world, long long n, float* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float acc = p[i];
    for (int r = 1; r < world; ++r) acc = __fadd_rn(acc, p[(long long)r * n + i]);
    out[i] = acc;
  }
}
}  // namespace
}  // namespace relpos

RELPOS_EXPORT int relpos_sum_partials(const float* partials, int32_t world, int64_t n, float* out,
                                      relpos_stream_t stream) {
  using namespace relpos;
  if (world < 1 || n < 0) return RELPOS_ERR_INVALID_ARG;
  if (n == 0) return RELPOS_OK;
  if (!partials || !out || (reinterpret_cast<uintptr_t>(partials) & 3) || (reinterpret_cast<uintptr_t>(out) & 3))
    return RELPOS_ERR_INVALID_ARG;
  // out is row 0 or lies outside rows 1 .. world - 1
  const float* rows_end = partials + (long long)world * n;
  if (out != partials && out + n > partials && out < rows_end) return RELPOS_ERR_INVALID_ARG;
  const long long blocks = (n + 255) / 256;
  const int grid = (int)(blocks < 148 * 8 ? blocks : 148 * 8);
  sum_partials_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(partials, world, n, out);
  note_launch(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RELPOS_OK : cuda_fail(e);
}

RELPOS_EXPORT int relpos_debug_phi(const relpos_map_desc* map, int32_t N, int32_t* phi_host) {
  if (!map || !phi_host || N < 1 || N > 46340) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  std::vector<int> by_delta(2 * (size_t)N - 1);
  for (int d = 1 - N; d <= N - 1; ++d) by_delta[d + N - 1] = phi_of(*map, N, d);
  for (int i = 0; i < N; ++i)
    for (int j = 0; j < N; ++j) phi_host[(size_t)i * N + j] = by_delta[j - i + N - 1];
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_debug_phi_device(const relpos_map_desc* map, int32_t N, int32_t* phi_dev, relpos_stream_t stream) {
  if (!map || !phi_dev || N < 1 || N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_debug_phi(*map, N, phi_dev, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? RELPOS_OK : cuda_fail(e);
}

RELPOS_EXPORT int relpos_debug_tile_plan(const relpos_map_desc* map, int32_t B, int32_t N, int32_t mask,
                                         const int32_t* key_len_host, int32_t* classes_host, int32_t* segs_host) {
  if (!map || !classes_host || !segs_host || B < 1 || N < 1 || N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  if (mask & ~(RELPOS_MASK_CAUSAL | RELPOS_MASK_KEY_PADDING)) return RELPOS_ERR_UNSUPPORTED;
  if ((mask & RELPOS_MASK_KEY_PADDING) && !key_len_host) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  int lo, hi;
  bounds_of(*map, N, &lo, &hi);
  const int nT = (N + kTile - 1) / kTile;
  const int causal = (mask & RELPOS_MASK_CAUSAL) != 0;
  for (int b = 0; b < B; ++b) {
    const int nkv = (mask & RELPOS_MASK_KEY_PADDING) ? iclamp(key_len_host[b], 0, N) : N;
    for (int qi = 0; qi < nT; ++qi) {
      for (int kj = 0; kj < nT; ++kj)
        classes_host[((size_t)b * nT + qi) * nT + kj] = tile_class(qi, kj, N, nkv, causal, lo, hi);
      int sg[4];
      tile_segments(qi, nT, N, nkv, causal, lo, hi, sg);
      for (int c = 0; c < 4; ++c) segs_host[((size_t)b * nT + qi) * 4 + c] = sg[c];
    }
  }
  return RELPOS_OK;
}

RELPOS_EXPORT int relpos_debug_tile_plan_device(const relpos_map_desc* map, int32_t B, int32_t N, int32_t mask,
                                                const int32_t* key_len_dev, int32_t* classes_dev, int32_t* segs_dev,
                                                relpos_stream_t stream) {
  if (!map || !classes_dev || !segs_dev || B < 1 || N < 1 || N > kMaxN) return RELPOS_ERR_INVALID_ARG;
  if (mask & ~(RELPOS_MASK_CAUSAL | RELPOS_MASK_KEY_PADDING)) return RELPOS_ERR_UNSUPPORTED;
  if ((mask & RELPOS_MASK_KEY_PADDING) && !key_len_dev) return RELPOS_ERR_INVALID_ARG;
  const int st = check_map(map);
  if (st) return st;
  int lo, hi;
  bounds_of(*map, N, &lo, &hi);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_debug_tile_plan(B, N, (mask & RELPOS_MASK_CAUSAL) != 0,
                                         (mask & RELPOS_MASK_KEY_PADDING) ? key_len_dev : nullptr, lo, hi,
                                         classes_dev, segs_dev, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? RELPOS_OK : cuda_fail(e);
}
