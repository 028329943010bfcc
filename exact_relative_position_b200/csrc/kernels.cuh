// kernels.cuh -- launch wrappers of the library's kernels (one translation
// unit per kernel family) and the parameter blocks they take.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace relpos {

// Device pointers of one forward/backward call, resolved into the workspace.
struct Tensors {
  const void *q, *k, *v;
  const void *aq_exp, *ak_exp;   // expanded tables, [Hq][Rexp][64] (Hq = H or 1), or null
  int table_per_head;
  long long aq_hs, ak_hs;        // head stride (elements) of the expanded tables when per head
  const float* b_exp;            // [H][Rexp] or null
  float *zq, *zk;                // projections (grouped layout), or null
  float* zk_sat;                 // [B*H][2][nT*128]: tau log2e Z^K[j, 0] and Z^K[j, R_exp-1], zero past N
  void* o;
  int o_f32;
  float* lse;
  // backward
  const void* dout;
  float* dsum;                   // D_i = sum_c dO_ic O_ic, [B*H][nT*128] (0 past N)
  float* lse2;                   // LSE_i log2 e, [B*H][nT*128] (+inf past N and for rows with every key masked)
  float* zq_sat;                 // [B*H][2][nT*128]: tau log2e (Z^Q[i, sat] + b_sat) - LSE_i log2e, sat = 0, R_exp-1
  void *dzq, *dzk;               // offset-sharded relation gradients: the 16-bit dS of each interior
                                 // offset (tau not applied), same layout as zq/zk, zero elsewhere
  float *dzq_sat, *dzk_sat;      // [B*H][nT*128][2]: each row's sums of dS over its cells at the low /
                                 // high saturated offset (tau not applied)
  void *dq, *dk, *dv;
  float *dq_acc, *dk_acc;        // fp32 [B,H,N,64] before the relation-GEMM epilogue (or null)
  float *daq_part, *dak_part;    // [nsplit][Hq][Rexp][64] partial table gradients
  float* db_part;                // [nsplit][H][Rexp]
  int nsplit_q, nsplit_k, nsplit_b;
  float *daq_exp, *dak_exp, *db_exp_grad;   // summed expanded-table gradients
  const int* phi_exp;            // [Rexp] expanded row -> original table row
  int* fold_lo;                  // [R] first expanded row of each table row
  int* fold_hi;                  // [R] one past its last expanded row
  int R;
  float *daq, *dak, *db;         // final outputs
  int is_bf16;
  int* status;                   // device status word (0 = ok; set when a kernel's bounded wait expires)
};

// Records e as this thread's last CUDA error and returns RELPOS_ERR_CUDA.
// Thread-local: while on, the library issues everything on the caller's stream
// (no side streams or events are created).
void set_single_stream(bool on);
int cuda_status(cudaError_t e);

// Counts kernel launches (process-wide, reported by relpos_kernel_launches).
void note_launch(int n);

cudaError_t launch_build_tables(const Plan& p, const relpos_map_desc& map, GroupInfo* gq, GroupInfo* gk,
                                int* phi_exp, int R, const void* aq, const void* ak, int table_per_head,
                                void* aq_exp, void* ak_exp, const float* b, float* b_exp, int is_bf16,
                                int expand_tables, cudaStream_t s);
cudaError_t launch_fold_ranges(const Plan& p, const int* phi_exp, int R, int* fold_lo, int* fold_hi, cudaStream_t s);
cudaError_t launch_projection(const Plan& p, const Tensors& t, cudaStream_t s, cudaStream_t key_stream);
cudaError_t launch_saturated_columns(const Plan& p, const Tensors& t, cudaStream_t s);
cudaError_t launch_saturated_rows(const Plan& p, const Tensors& t, cudaStream_t s);

// A 16-bit activation tensor ([B, H, N, 64] dense or [T, H, 64] packed) viewed
// as 3-D for TMA with 128-row boxes; coordinates from tma_rows (common.cuh).
bool make_rows_map(CUtensorMap* m, const void* base, const Plan& p, bool bf16);
cudaError_t launch_forward(const Plan& p, const Tensors& t, cudaStream_t s);
// Forward with Z^Q recomputed per tile (q.aQ and b terms only).
cudaError_t launch_forward_recompute(const Plan& p, const Tensors& t, cudaStream_t s);
cudaError_t launch_bwd_prep(const Plan& p, const Tensors& t, cudaStream_t s);
cudaError_t launch_bwd_dq(const Plan& p, const Tensors& t, cudaStream_t s);
cudaError_t launch_bwd_dkdv(const Plan& p, const Tensors& t, cudaStream_t s);
// side 0: query-side relation gradients (dQ += dZ^Q aQ_exp, daQ, db);
// side 1: key side (dK += dZ^K aK_exp, daK).  The dQ / dK row update goes to
// rows_stream and the table gradients to s (the two share no outputs); the
// caller orders rows_stream after s's earlier work and joins it back.
cudaError_t launch_relgrad(const Plan& p, const Tensors& t, int side, cudaStream_t s, cudaStream_t rows_stream);
cudaError_t launch_debug_phi(const relpos_map_desc& map, int N, int* out, cudaStream_t s);
cudaError_t launch_debug_tile_plan(int B, int N, int causal, const int* key_len, int E_lo, int E_hi,
                                   int* classes, int* segs, cudaStream_t s);

}  // namespace relpos
