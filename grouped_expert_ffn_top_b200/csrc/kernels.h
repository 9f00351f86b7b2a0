// Internal launchers of the MoE layer library (host side, no validation:
// the C ABI in api.cu checks every argument before calling these).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kRouteThreads = 256;
constexpr int kRouteTokensPerBlock = 256;

// error message and launch count of the C ABI (api.cu)
int report_error(int code, const char* msg);
void count_launches(int n);

// routing (route.cu)
cudaError_t launch_router_logits(const void* x, const void* Wr, const float* b, int dtype,
                                 int64_t T, int d, int E, float* z, cudaStream_t s);
cudaError_t launch_route(const float* z, int64_t T, int E, int k, int G, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int64_t* offsets, int32_t* group_counts,
                         int64_t* group_offsets, int32_t* row_of_pair, int32_t* pair_of_row,
                         int32_t* block_counts, int32_t* block_base, unsigned* err,
                         cudaStream_t s);
cudaError_t route_set_smem_limits();
cudaError_t launch_route_bwd(const float* dg, const float* w, const int32_t* idx, int64_t T,
                             int E, int k, float* dz, cudaStream_t s);

// dispatch / combine (dispatch.cu)
cudaError_t launch_permute(const void* x, int dtype, int64_t T, int d, int k,
                           const int32_t* row_of_pair, void* xp, cudaStream_t s);
cudaError_t launch_combine(const void* yp, const float* w, const int32_t* row_of_pair, int dtype,
                           int64_t T, int d, int k, void* Y, cudaStream_t s);
cudaError_t launch_combine_bwd(const void* dY, const void* yp, const float* w,
                               const int32_t* row_of_pair, int dtype, int64_t T, int d, int k,
                               void* dyp, float* dg, cudaStream_t s);
cudaError_t launch_permute_bwd(const void* dxp, const int32_t* row_of_pair, const float* dz,
                               const void* Wr, const int32_t* idx, int dtype, int64_t T, int d,
                               int E, int k, void* dX, cudaStream_t s);
// expert-parallel regroup of received rows (1 launch)
cudaError_t launch_ep_regroup(const int32_t* recv, int G, int El, int32_t* row_map,
                              int64_t* local_offsets, cudaStream_t s);
int router_bwd_max_items(int64_t rows, int E);
// gather: `xp` is x [T, d] and dispatch row r is read as x[pair_of_row[r] / k]
cudaError_t launch_router_bwd(const void* xp, const float* dz, const int32_t* pair_of_row,
                              const int64_t* offsets, int dtype, int64_t rows, int d, int E, int k,
                              float* dWr, float* db, int accumulate, float* partial, cudaStream_t s,
                              bool gather = false);

// grouped expert FFN (grouped_gemm_sm100.cu, grouped_simt.cu)
// Gathered dispatch rows: with gather_rows set, `xp` points at x [gather_T, d]
// and dispatch row r of the expert input is x[gather_rows[r] / gather_k]
// (gather_rows = pair_of_row), read in place instead of from a permuted copy.
struct RowGather {
  const int32_t* rows = nullptr;
  int k = 1;
  int64_t T = 0;
};
struct FfnFwdArgs {
  const void *xp, *Wg, *Wu, *Wd;
  const int64_t* offsets;
  int64_t rows;
  int E, d, f;
  void *h1, *h2, *a, *yp;
  unsigned* err;
  RowGather gather;
};
struct FfnBwdArgs {
  const void *xp, *Wg, *Wu, *Wd, *h1, *h2, *a, *dyp;
  const int64_t* offsets;
  int64_t rows;
  int E, d, f;
  void* dxp;
  float *dWg, *dWu, *dWd;
  void *dh1, *dh2;  // [rows, f]: written by dgrad, read by wgrad
  unsigned* err;
  int accumulate;   // wgrad: 1 adds to dW, 0 writes dW (zero for experts with no rows)
  RowGather gather; // wgrad: xp's rows gathered from x
};

cudaError_t launch_selftest_wait_timeout(unsigned* err, long long limit, cudaStream_t s);

// Auxiliary load-balancing loss (aux_loss.cu).
int aux_blocks(int64_t T);                 // per-block partials of the forward
int dense_router_chunks(int64_t T);        // token chunks of the dense router backward
cudaError_t launch_aux_loss(const float* z, const int32_t* counts, int64_t T, int E, int k,
                            float alpha, float* importance, float* loss, float* entropy,
                            float* partial, cudaStream_t s);  // 2 launches
cudaError_t launch_aux_loss_bwd(const float* z, const int32_t* counts, int64_t T, int E, int k,
                                float alpha, float dloss, float* dz, cudaStream_t s);  // 1 launch
cudaError_t launch_router_bwd_dense(const void* x, const void* Wr, const float* dz, int dtype,
                                    int64_t T, int d, int E, void* dX, float* dWr, float* db,
                                    int accumulate, float* partial, cudaStream_t s);  // 2 or 3
cudaError_t launch_ffn_fwd_bf16(const FfnFwdArgs& a, cudaStream_t s);
// The gate/up GEMM alone, storing whichever of h1, h2, a are set (1 launch).
cudaError_t launch_ffn_gateup_bf16(const FfnFwdArgs& a, cudaStream_t s);
cudaError_t launch_ffn_gateup_f32(const FfnFwdArgs& a, cudaStream_t s);
cudaError_t launch_ffn_dgrad_bf16(const FfnBwdArgs& a, cudaStream_t s);  // 2 launches
cudaError_t launch_ffn_wgrad_bf16(const FfnBwdArgs& a, cudaStream_t s);  // 1 launch
cudaError_t launch_ffn_fwd_f32(const FfnFwdArgs& a, cudaStream_t s);
cudaError_t launch_ffn_dgrad_f32(const FfnBwdArgs& a, cudaStream_t s);   // 2 launches
cudaError_t launch_ffn_wgrad_f32(const FfnBwdArgs& a, cudaStream_t s);   // 1 launch

}  // namespace moe
