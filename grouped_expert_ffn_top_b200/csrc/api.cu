// The C ABI (include/moe.h): argument checks, workspace carving and launches.
// Every check runs before anything is launched, so a rejected call changes
// nothing on the device.
#include <stdarg.h>
#include <atomic>
#include <stdio.h>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char g_msg[512] = "";
std::atomic<int64_t> g_launches{0};

void counted(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Adds the launches of a call that succeeded; passes the status through.
int launched(int rc, int n) {
  if (rc == MOE_OK) counted(n);
  return rc;
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool dtype_ok(int dtype) { return dtype == MOE_F32 || dtype == MOE_BF16; }
size_t elem_bytes(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }
size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common checks of the row-wise passes (permute / combine and their backward).
int check_rows(const char* fn, int dtype, int64_t T, int d, int k) {
  if (!dtype_ok(dtype)) return fail(MOE_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, dtype);
  if (T < 0 || d < 1 || k < 1) return fail(MOE_ERR_INVALID_ARG, "%s: T=%lld d=%d k=%d", fn,
                                           static_cast<long long>(T), d, k);
  if (k > 32) return fail(MOE_ERR_UNSUPPORTED, "%s: k=%d > 32", fn, k);
  if (d % 8 != 0) return fail(MOE_ERR_UNSUPPORTED, "%s: d=%d is not a multiple of 8", fn, d);
  if (T * k >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "%s: T*k=%lld rows exceed int32", fn,
                static_cast<long long>(T * k));
  return MOE_OK;
}

int check_ffn(const char* fn, int dtype, int64_t rows, int E, int d, int f) {
  if (!dtype_ok(dtype)) return fail(MOE_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, dtype);
  if (rows < 0 || E < 1 || d < 1 || f < 1)
    return fail(MOE_ERR_INVALID_ARG, "%s: rows=%lld E=%d d=%d f=%d", fn,
                static_cast<long long>(rows), E, d, f);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "%s: E=%d > %d", fn, E, MOE_MAX_EXPERTS);
  if (rows >= (int64_t(1) << 31)) return fail(MOE_ERR_UNSUPPORTED, "%s: rows exceed int32", fn);
  // bf16: 16-byte rows for TMA (the last K block and the last column tile
  // past d or f are zero-filled and masked); fp32 (CUDA cores): 16-byte vectors
  const int q = dtype == MOE_BF16 ? 8 : 4;
  if (d % q != 0 || f % q != 0)
    return fail(MOE_ERR_UNSUPPORTED, "%s: d=%d and f=%d must be multiples of %d for this dtype",
                fn, d, f, q);
  if (static_cast<int64_t>(E) * (d > f ? d : f) >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "%s: E*max(d,f) exceeds int32", fn);
  return MOE_OK;
}

}  // namespace

// accumulate = 0 on an empty batch: the requested gradient is zero. Null
// buffers are skipped.
static cudaError_t zero_grads(cudaStream_t stream, size_t bytes0, float* g0, size_t bytes1 = 0,
                              float* g1 = nullptr, size_t bytes2 = 0, float* g2 = nullptr) {
  float* g[3] = {g0, g1, g2};
  size_t n[3] = {bytes0, bytes1, bytes2};
  for (int i = 0; i < 3; ++i) {
    if (!g[i]) continue;
    cudaError_t e = cudaMemsetAsync(g[i], 0, n[i], stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

namespace moe {
// Records the message moe_last_error() returns, for entry points defined in
// other files of the library; returns `code`.
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }
// Adds `n` kernel launches to the count moe_launch_count() returns.
void count_launches(int n) { counted(n); }
}  // namespace moe

extern "C" {

const char* moe_last_error(void) { return g_msg; }

int moe_version(void) { return 1; }

int64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_selftest_wait_timeout(void* ws, long long limit_cycles, cudaStream_t stream) {
  if (!ws || !aligned16(ws)) return fail(MOE_ERR_INVALID_ARG, "moe_selftest_wait_timeout: workspace");
  if (limit_cycles < 1000) limit_cycles = 1000;
  if (limit_cycles > 4000000000LL) limit_cycles = 4000000000LL;
  return launched(cuda_status(moe::launch_selftest_wait_timeout(static_cast<unsigned*>(ws),
                                                                limit_cycles, stream),
                              "moe_selftest_wait_timeout"), 1);
}

int moe_get_error(void* ws, cudaStream_t stream) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "moe_get_error: null workspace");
  unsigned h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(unsigned), stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e, "moe_get_error");
  return static_cast<int>(h & 0x7fffffffu);
}

// ------------------------------------------------------------------ routing

int moe_router_logits(const void* x, const void* Wr, const float* b, int dtype, int64_t T, int d,
                      int E, float* logits, cudaStream_t stream) {
  if (!dtype_ok(dtype)) return fail(MOE_ERR_UNSUPPORTED, "moe_router_logits: dtype %d", dtype);
  if (T < 0 || d < 1 || E < 1) return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: sizes");
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "moe_router_logits: E=%d", E);
  if (d % 8 != 0) return fail(MOE_ERR_UNSUPPORTED, "moe_router_logits: d=%d not a multiple of 8", d);
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !logits) return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: null pointer");
  if (!aligned16(x) || !aligned16(Wr))
    return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: x and Wr must be 16-byte aligned");
  return launched(cuda_status(moe::launch_router_logits(x, Wr, b, dtype, T, d, E, logits, stream),
                              "moe_router_logits"), 1);
}

size_t moe_route_workspace_bytes(int64_t T, int E) {
  if (T < 0 || E < 1) return 0;
  const int64_t nb = (T + moe::kRouteTokensPerBlock - 1) / moe::kRouteTokensPerBlock;
  return moe::kWsHeader + 2 * align256(sizeof(int32_t) * static_cast<size_t>(nb) * E);
}

int moe_route(const float* logits, int64_t T, int E, int k, int ep_groups, int32_t* topk_idx,
              float* topk_w, int32_t* expert_counts, int64_t* expert_offsets,
              int32_t* group_counts, int64_t* group_offsets, int32_t* row_of_pair,
              int32_t* pair_of_row, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E || ep_groups < 1)
    return fail(MOE_ERR_INVALID_ARG, "moe_route: T=%lld E=%d k=%d ep_groups=%d",
                static_cast<long long>(T), E, k, ep_groups);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "moe_route: E=%d > %d", E, MOE_MAX_EXPERTS);
  if (k > 32) return fail(MOE_ERR_UNSUPPORTED, "moe_route: k=%d > 32", k);
  if (E % ep_groups != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_route: E=%d is not divisible by ep_groups=%d", E,
                ep_groups);
  if (T * k >= (int64_t(1) << 31)) return fail(MOE_ERR_UNSUPPORTED, "moe_route: T*k exceeds int32");
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w || !expert_counts || !expert_offsets || !group_counts ||
      !group_offsets || !row_of_pair || !pair_of_row || !ws)
    return fail(MOE_ERR_INVALID_ARG, "moe_route: null pointer");
  if (ws_bytes < moe_route_workspace_bytes(T, E) || !aligned16(ws))
    return fail(MOE_ERR_WORKSPACE, "moe_route: workspace needs %zu bytes (got %zu), 16-aligned",
                moe_route_workspace_bytes(T, E), ws_bytes);
  const int64_t nb = (T + moe::kRouteTokensPerBlock - 1) / moe::kRouteTokensPerBlock;
  uint8_t* base = static_cast<uint8_t*>(ws);
  unsigned* err = reinterpret_cast<unsigned*>(base);
  int32_t* block_counts = reinterpret_cast<int32_t*>(base + moe::kWsHeader);
  int32_t* block_base = reinterpret_cast<int32_t*>(
      base + moe::kWsHeader + align256(sizeof(int32_t) * static_cast<size_t>(nb) * E));
  if (E > 768) {
    cudaError_t e = moe::route_set_smem_limits();
    if (e != cudaSuccess) return cuda_status(e, "moe_route");
  }
  return cuda_status(moe::launch_route(logits, T, E, k, ep_groups, topk_idx, topk_w, expert_counts,
                                       expert_offsets, group_counts, group_offsets, row_of_pair,
                                       pair_of_row, block_counts, block_base, err, stream),
                     "moe_route") == MOE_OK ? launched(MOE_OK, 3) : MOE_ERR_CUDA;
}

int moe_route_bwd(const float* dg, const float* topk_w, const int32_t* topk_idx, int64_t T, int E,
                  int k, float* dlogits, cudaStream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "moe_route_bwd: sizes");
  if (k > 32) return fail(MOE_ERR_UNSUPPORTED, "moe_route_bwd: k=%d > 32", k);
  if (T == 0) return MOE_OK;
  if (!dg || !topk_w || !topk_idx || !dlogits)
    return fail(MOE_ERR_INVALID_ARG, "moe_route_bwd: null pointer");
  return launched(cuda_status(moe::launch_route_bwd(dg, topk_w, topk_idx, T, E, k, dlogits, stream),
                              "moe_route_bwd"), 1);
}

// ----------------------------------------------------------------- dispatch

int moe_permute(const void* x, int dtype, int64_t T, int d, int k, const int32_t* row_of_pair,
                void* xp, cudaStream_t stream) {
  int rc = check_rows("moe_permute", dtype, T, d, k);
  if (rc != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  if (!x || !row_of_pair || !xp) return fail(MOE_ERR_INVALID_ARG, "moe_permute: null pointer");
  if (!aligned16(x) || !aligned16(xp)) return fail(MOE_ERR_INVALID_ARG, "moe_permute: 16-byte alignment");
  return launched(cuda_status(moe::launch_permute(x, dtype, T, d, k, row_of_pair, xp, stream),
                              "moe_permute"), 1);
}

int moe_unpermute_combine(const void* yp, const float* topk_w, const int32_t* row_of_pair,
                          int dtype, int64_t T, int d, int k, void* Y, cudaStream_t stream) {
  int rc = check_rows("moe_unpermute_combine", dtype, T, d, k);
  if (rc != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  if (!yp || !topk_w || !row_of_pair || !Y)
    return fail(MOE_ERR_INVALID_ARG, "moe_unpermute_combine: null pointer");
  if (!aligned16(yp) || !aligned16(Y))
    return fail(MOE_ERR_INVALID_ARG, "moe_unpermute_combine: 16-byte alignment");
  return launched(cuda_status(moe::launch_combine(yp, topk_w, row_of_pair, dtype, T, d, k, Y, stream),
                              "moe_unpermute_combine"), 1);
}

int moe_unpermute_combine_bwd(const void* dY, const void* yp, const float* topk_w,
                              const int32_t* row_of_pair, int dtype, int64_t T, int d, int k,
                              void* dyp, float* dg, cudaStream_t stream) {
  int rc = check_rows("moe_unpermute_combine_bwd", dtype, T, d, k);
  if (rc != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  if (!dY || !yp || !topk_w || !row_of_pair || !dyp || !dg)
    return fail(MOE_ERR_INVALID_ARG, "moe_unpermute_combine_bwd: null pointer");
  if (!aligned16(dY) || !aligned16(yp) || !aligned16(dyp))
    return fail(MOE_ERR_INVALID_ARG, "moe_unpermute_combine_bwd: 16-byte alignment");
  return launched(cuda_status(moe::launch_combine_bwd(dY, yp, topk_w, row_of_pair, dtype, T, d, k,
                                                      dyp, dg, stream),
                              "moe_unpermute_combine_bwd"), 1);
}

int moe_permute_bwd(const void* dxp, const int32_t* row_of_pair, const float* dlogits,
                    const void* Wr, const int32_t* topk_idx, int dtype, int64_t T, int d, int E,
                    int k, void* dX, cudaStream_t stream) {
  int rc = check_rows("moe_permute_bwd", dtype, T, d, k);
  if (rc != MOE_OK) return rc;
  if (E < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "moe_permute_bwd: E=%d k=%d", E, k);
  if (T == 0) return MOE_OK;
  if (!dxp || !row_of_pair || !dX || (dlogits && (!Wr || !topk_idx)))
    return fail(MOE_ERR_INVALID_ARG, "moe_permute_bwd: null pointer");
  if (!aligned16(dxp) || !aligned16(dX) || (dlogits && !aligned16(Wr)))
    return fail(MOE_ERR_INVALID_ARG, "moe_permute_bwd: 16-byte alignment");
  return cuda_status(moe::launch_permute_bwd(dxp, row_of_pair, dlogits, Wr, topk_idx, dtype, T, d,
                                             E, k, dX, stream),
                     "moe_permute_bwd") == MOE_OK ? launched(MOE_OK, 1) : MOE_ERR_CUDA;
}

int moe_ep_regroup(const int32_t* recv_counts, int G, int El, int32_t* row_map,
                   int64_t* local_offsets, cudaStream_t stream) {
  if (G < 1 || El < 1 || !recv_counts || !row_map || !local_offsets)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_regroup: G=%d El=%d or null pointer", G, El);
  if (static_cast<int64_t>(G) * El > MOE_MAX_EXPERTS)
    return fail(MOE_ERR_UNSUPPORTED, "moe_ep_regroup: G*El=%lld > %d", static_cast<long long>(G) * El,
                MOE_MAX_EXPERTS);
  return cuda_status(moe::launch_ep_regroup(recv_counts, G, El, row_map, local_offsets, stream),
                     "moe_ep_regroup") == MOE_OK ? launched(MOE_OK, 1) : MOE_ERR_CUDA;
}

size_t moe_router_bwd_workspace_bytes(int64_t rows, int d, int E) {
  if (rows < 0 || d < 1 || E < 1) return 0;
  const size_t items = static_cast<size_t>(moe::router_bwd_max_items(rows, E));
  return moe::kWsHeader + align256(sizeof(float) * items * (static_cast<size_t>(d) + 1));
}

}  // extern "C"

// xp, or with `gather` x [T, d] read through pair_of_row
static int router_bwd_impl(const char* fn, bool gather, const void* xp, const float* dlogits,
                           const int32_t* pair_of_row, const int64_t* expert_offsets, int dtype,
                           int64_t T, int d, int E, int k, float* dWr, float* db, int accumulate,
                           void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = check_rows(fn, dtype, T, d, k);
  if (rc != MOE_OK) return rc;
  if (E < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "%s: E=%d k=%d", fn, E, k);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "%s: E=%d", fn, E);
  if (accumulate != 0 && accumulate != 1)
    return fail(MOE_ERR_INVALID_ARG, "%s: accumulate=%d (0 or 1)", fn, accumulate);
  if (T == 0) {
    if (accumulate) return MOE_OK;
    if (!dWr) return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
    return cuda_status(zero_grads(stream, sizeof(float) * static_cast<size_t>(E) * d, dWr,
                                  sizeof(float) * E, db),
                       fn);
  }
  if (!xp || !dlogits || !pair_of_row || !expert_offsets || !dWr || !ws)
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
  const int64_t rows = T * k;
  if (ws_bytes < moe_router_bwd_workspace_bytes(rows, d, E) || !aligned16(ws) || !aligned16(xp))
    return fail(MOE_ERR_WORKSPACE, "%s: workspace needs %zu bytes (16-byte aligned)", fn,
                moe_router_bwd_workspace_bytes(rows, d, E));
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + moe::kWsHeader);
  return launched(cuda_status(moe::launch_router_bwd(xp, dlogits, pair_of_row, expert_offsets,
                                                      dtype, rows, d, E, k, dWr, db, accumulate,
                                                      partial, stream, gather),
                              fn), 2);
}

extern "C" {

int moe_router_bwd(const void* xp, const float* dlogits, const int32_t* pair_of_row,
                   const int64_t* expert_offsets, int dtype, int64_t T, int d, int E, int k,
                   float* dWr, float* db, int accumulate, void* ws, size_t ws_bytes,
                   cudaStream_t stream) {
  return router_bwd_impl("moe_router_bwd", false, xp, dlogits, pair_of_row, expert_offsets, dtype,
                         T, d, E, k, dWr, db, accumulate, ws, ws_bytes, stream);
}

int moe_router_bwd_gather(const void* x, const float* dlogits, const int32_t* pair_of_row,
                          const int64_t* expert_offsets, int dtype, int64_t T, int d, int E, int k,
                          float* dWr, float* db, int accumulate, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  return router_bwd_impl("moe_router_bwd_gather", true, x, dlogits, pair_of_row, expert_offsets,
                         dtype, T, d, E, k, dWr, db, accumulate, ws, ws_bytes, stream);
}

// ------------------------------------------------------------ grouped FFN

// --------------------------------------------------- auxiliary balance loss

size_t moe_aux_loss_workspace_bytes(int64_t T, int E) {
  if (T < 0 || E < 1) return 0;
  return moe::kWsHeader + align256(sizeof(float) * static_cast<size_t>(moe::aux_blocks(T)) * (E + 1));
}

int moe_aux_loss(const float* logits, const int32_t* expert_counts, int64_t T, int E, int k,
                 float alpha, float* importance, float* loss, float* entropy, void* ws,
                 size_t ws_bytes, cudaStream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E)
    return fail(MOE_ERR_INVALID_ARG, "moe_aux_loss: T=%lld E=%d k=%d", static_cast<long long>(T), E, k);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "moe_aux_loss: E=%d", E);
  if (!importance || !loss) return fail(MOE_ERR_INVALID_ARG, "moe_aux_loss: null pointer");
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(importance, 0, sizeof(float) * E, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(loss, 0, sizeof(float), stream);
    if (e == cudaSuccess && entropy) e = cudaMemsetAsync(entropy, 0, sizeof(float), stream);
    return cuda_status(e, "moe_aux_loss");
  }
  if (!logits || !expert_counts || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_aux_loss: null pointer");
  if (ws_bytes < moe_aux_loss_workspace_bytes(T, E) || !aligned16(ws))
    return fail(MOE_ERR_WORKSPACE, "moe_aux_loss: workspace needs %zu bytes (16-byte aligned)",
                moe_aux_loss_workspace_bytes(T, E));
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + moe::kWsHeader);
  return launched(cuda_status(moe::launch_aux_loss(logits, expert_counts, T, E, k, alpha,
                                                   importance, loss, entropy, partial, stream),
                              "moe_aux_loss"), 2);
}

int moe_aux_loss_bwd(const float* logits, const int32_t* expert_counts, int64_t T, int E, int k,
                     float alpha, float dloss, float* dlogits_aux, cudaStream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E)
    return fail(MOE_ERR_INVALID_ARG, "moe_aux_loss_bwd: T=%lld E=%d k=%d", static_cast<long long>(T), E, k);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "moe_aux_loss_bwd: E=%d", E);
  if (T == 0) return MOE_OK;
  if (!logits || !expert_counts || !dlogits_aux)
    return fail(MOE_ERR_INVALID_ARG, "moe_aux_loss_bwd: null pointer");
  return launched(cuda_status(moe::launch_aux_loss_bwd(logits, expert_counts, T, E, k, alpha, dloss,
                                                       dlogits_aux, stream),
                              "moe_aux_loss_bwd"), 1);
}

size_t moe_router_bwd_dense_workspace_bytes(int64_t T, int d, int E) {
  if (T < 0 || d < 1 || E < 1) return 0;
  const size_t chunks = static_cast<size_t>(moe::dense_router_chunks(T));
  return moe::kWsHeader + align256(sizeof(float) * chunks * E * (static_cast<size_t>(d) + 1));
}

int moe_router_bwd_dense(const void* x, const void* Wr, const float* dz, int dtype, int64_t T,
                         int d, int E, void* dX, float* dWr, float* db, int accumulate, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  if (!dtype_ok(dtype)) return fail(MOE_ERR_UNSUPPORTED, "moe_router_bwd_dense: dtype %d", dtype);
  if (T < 0 || d < 1 || E < 1)
    return fail(MOE_ERR_INVALID_ARG, "moe_router_bwd_dense: T=%lld d=%d E=%d",
                static_cast<long long>(T), d, E);
  if (d % 4 != 0) return fail(MOE_ERR_UNSUPPORTED, "moe_router_bwd_dense: d=%d (multiple of 4)", d);
  if (E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED, "moe_router_bwd_dense: E=%d", E);
  if (accumulate != 0 && accumulate != 1)
    return fail(MOE_ERR_INVALID_ARG, "moe_router_bwd_dense: accumulate=%d (0 or 1)", accumulate);
  if (!dWr) return fail(MOE_ERR_INVALID_ARG, "moe_router_bwd_dense: null pointer");
  if (T == 0) {
    if (accumulate) return MOE_OK;
    return cuda_status(zero_grads(stream, sizeof(float) * static_cast<size_t>(E) * d, dWr,
                                  sizeof(float) * E, db),
                       "moe_router_bwd_dense");
  }
  if (!x || !Wr || !dz || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_router_bwd_dense: null pointer");
  if (ws_bytes < moe_router_bwd_dense_workspace_bytes(T, d, E) || !aligned16(ws))
    return fail(MOE_ERR_WORKSPACE, "moe_router_bwd_dense: workspace needs %zu bytes (16-byte aligned)",
                moe_router_bwd_dense_workspace_bytes(T, d, E));
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + moe::kWsHeader);
  return launched(cuda_status(moe::launch_router_bwd_dense(x, Wr, dz, dtype, T, d, E, dX, dWr, db,
                                                           accumulate, partial, stream),
                              "moe_router_bwd_dense"), dX ? 3 : 2);
}

size_t moe_grouped_ffn_fwd_workspace_bytes(int64_t rows, int E, int d, int f, int dtype) {
  (void)rows; (void)E; (void)d; (void)f; (void)dtype;
  return moe::kWsHeader;
}

}  // extern "C"

// The expert input of a grouped-FFN call: xp [rows, d], or x [T, d] read
// through pair_of_row (rows = T k; dispatch row r is x[pair_of_row[r] / k]).
static int check_gather(const char* fn, const moe::RowGather& g, int dtype, int64_t rows, int d) {
  if (!g.rows) return MOE_OK;
  int rc = check_rows(fn, dtype, g.T, d, g.k);
  if (rc != MOE_OK) return rc;
  if (g.T * g.k != rows)
    return fail(MOE_ERR_INVALID_ARG, "%s: rows=%lld != T*k=%lld", fn, static_cast<long long>(rows),
                static_cast<long long>(g.T * g.k));
  return MOE_OK;
}

static int ffn_fwd_impl(const char* fn, const void* xp, const moe::RowGather& g, const void* Wg,
                        const void* Wu, const void* Wd, int dtype, const int64_t* expert_offsets,
                        int64_t rows, int E, int d, int f, void* h1, void* h2, void* a, void* yp,
                        void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = check_ffn(fn, dtype, rows, E, d, f);
  if (rc == MOE_OK) rc = check_gather(fn, g, dtype, rows, d);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!xp || !Wg || !Wu || !Wd || !expert_offsets || !a || !yp || !ws || (!h1) != (!h2))
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
  const void* ptrs[] = {xp, Wg, Wu, Wd, h1, h2, a, yp, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "%s: 16-byte alignment", fn);
  if (ws_bytes < moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dtype))
    return fail(MOE_ERR_WORKSPACE, "%s: workspace too small", fn);
  moe::FfnFwdArgs args{xp, Wg, Wu, Wd, expert_offsets, rows, E, d, f, h1, h2, a, yp,
                       static_cast<unsigned*>(ws), g};
  cudaError_t e = dtype == MOE_BF16 ? moe::launch_ffn_fwd_bf16(args, stream)
                                    : moe::launch_ffn_fwd_f32(args, stream);
  return launched(cuda_status(e, fn), 2);
}

static int ffn_recompute_impl(const char* fn, const void* xp, const moe::RowGather& g,
                              const void* Wg, const void* Wu, int dtype,
                              const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                              void* h1, void* h2, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = check_ffn(fn, dtype, rows, E, d, f);
  if (rc == MOE_OK) rc = check_gather(fn, g, dtype, rows, d);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!xp || !Wg || !Wu || !expert_offsets || !h1 || !h2 || !ws)
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
  const void* ptrs[] = {xp, Wg, Wu, h1, h2, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "%s: 16-byte alignment", fn);
  if (ws_bytes < moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dtype))
    return fail(MOE_ERR_WORKSPACE, "%s: workspace too small", fn);
  moe::FfnFwdArgs args{xp, Wg, Wu, nullptr, expert_offsets, rows, E, d, f, h1, h2, nullptr, nullptr,
                       static_cast<unsigned*>(ws), g};
  cudaError_t e = dtype == MOE_BF16 ? moe::launch_ffn_gateup_bf16(args, stream)
                                    : moe::launch_ffn_gateup_f32(args, stream);
  return launched(cuda_status(e, fn), 1);
}

static int ffn_bwd_impl(const char* fn, const void* xp, const moe::RowGather& g, const void* Wg,
                        const void* Wu, const void* Wd, const void* h1, const void* h2,
                        const void* a, const void* dyp, int dtype, const int64_t* expert_offsets,
                        int64_t rows, int E, int d, int f, void* dxp, float* dWg, float* dWu,
                        float* dWd, int accumulate, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
  int rc = check_ffn(fn, dtype, rows, E, d, f);
  if (rc == MOE_OK) rc = check_gather(fn, g, dtype, rows, d);
  if (rc != MOE_OK) return rc;
  if (accumulate != 0 && accumulate != 1)
    return fail(MOE_ERR_INVALID_ARG, "%s: accumulate=%d (0 or 1)", fn, accumulate);
  if (rows == 0) {
    if (accumulate) return MOE_OK;
    if (!dWg || !dWu || !dWd) return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
    const size_t n = sizeof(float) * static_cast<size_t>(E) * f * d;
    return cuda_status(zero_grads(stream, n, dWg, n, dWu, n, dWd), fn);
  }
  if (!xp || !Wg || !Wu || !Wd || !h1 || !h2 || !a || !dyp || !expert_offsets || !dxp || !dWg ||
      !dWu || !dWd || !ws)
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
  const void* ptrs[] = {xp, Wg, Wu, Wd, h1, h2, a, dyp, dxp, dWg, dWu, dWd, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "%s: 16-byte alignment", fn);
  if (ws_bytes < moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dtype))
    return fail(MOE_ERR_WORKSPACE, "%s: workspace needs %zu bytes (got %zu)", fn,
                moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dtype), ws_bytes);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t h = align256(static_cast<size_t>(rows) * f * elem_bytes(dtype));
  moe::FfnBwdArgs args{xp, Wg, Wu, Wd, h1, h2, a, dyp, expert_offsets, rows, E, d, f, dxp,
                       dWg, dWu, dWd, base + moe::kWsHeader, base + moe::kWsHeader + h,
                       static_cast<unsigned*>(ws), accumulate, g};
  cudaError_t e = dtype == MOE_BF16 ? moe::launch_ffn_dgrad_bf16(args, stream)
                                    : moe::launch_ffn_dgrad_f32(args, stream);
  if (e == cudaSuccess) {
    counted(2);
    e = dtype == MOE_BF16 ? moe::launch_ffn_wgrad_bf16(args, stream)
                          : moe::launch_ffn_wgrad_f32(args, stream);
  }
  return launched(cuda_status(e, fn), 1);
}

static int ffn_wgrad_impl(const char* fn, const void* xp, const moe::RowGather& g, const void* a,
                          const void* dyp, const void* dh1, const void* dh2, int dtype,
                          const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                          float* dWg, float* dWu, float* dWd, int accumulate, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  int rc = check_ffn(fn, dtype, rows, E, d, f);
  if (rc == MOE_OK) rc = check_gather(fn, g, dtype, rows, d);
  if (rc != MOE_OK) return rc;
  if (accumulate != 0 && accumulate != 1)
    return fail(MOE_ERR_INVALID_ARG, "%s: accumulate=%d (0 or 1)", fn, accumulate);
  if (rows == 0) {
    if (accumulate) return MOE_OK;
    if (!dWg || !dWu || !dWd) return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
    const size_t n = sizeof(float) * static_cast<size_t>(E) * f * d;
    return cuda_status(zero_grads(stream, n, dWg, n, dWu, n, dWd), fn);
  }
  if (!xp || !a || !dyp || !dh1 || !dh2 || !expert_offsets || !dWg || !dWu || !dWd || !ws)
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", fn);
  const void* ptrs[] = {xp, a, dyp, dh1, dh2, dWg, dWu, dWd, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "%s: 16-byte alignment", fn);
  if (ws_bytes < moe_grouped_ffn_wgrad_workspace_bytes(E, dtype))
    return fail(MOE_ERR_WORKSPACE, "%s: workspace needs %zu bytes (got %zu)", fn,
                moe_grouped_ffn_wgrad_workspace_bytes(E, dtype), ws_bytes);
  moe::FfnBwdArgs args{xp, nullptr, nullptr, nullptr, nullptr, nullptr, a, dyp, expert_offsets,
                       rows, E, d, f, nullptr, dWg, dWu, dWd, const_cast<void*>(dh1),
                       const_cast<void*>(dh2), static_cast<unsigned*>(ws), accumulate, g};
  cudaError_t e = dtype == MOE_BF16 ? moe::launch_ffn_wgrad_bf16(args, stream)
                                    : moe::launch_ffn_wgrad_f32(args, stream);
  return launched(cuda_status(e, fn), 1);
}

static moe::RowGather row_gather(const int32_t* pair_of_row, int64_t T, int k) {
  moe::RowGather g;
  g.rows = pair_of_row;
  g.k = k;
  g.T = T;
  return g;
}

extern "C" {

int moe_grouped_ffn_fwd(const void* xp, const void* Wg, const void* Wu, const void* Wd, int dtype,
                        const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                        void* h1, void* h2, void* a, void* yp, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
  return ffn_fwd_impl("moe_grouped_ffn_fwd", xp, moe::RowGather{}, Wg, Wu, Wd, dtype,
                      expert_offsets, rows, E, d, f, h1, h2, a, yp, ws, ws_bytes, stream);
}

int moe_grouped_ffn_fwd_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                               const void* Wg, const void* Wu, const void* Wd, int dtype,
                               const int64_t* expert_offsets, int E, int d, int f, void* h1,
                               void* h2, void* a, void* yp, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  if (!pair_of_row && T > 0) return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_fwd_gather: null pointer");
  return ffn_fwd_impl("moe_grouped_ffn_fwd_gather", x, row_gather(pair_of_row, T, k), Wg, Wu, Wd,
                      dtype, expert_offsets, T * k, E, d, f, h1, h2, a, yp, ws, ws_bytes, stream);
}

int moe_grouped_ffn_recompute(const void* xp, const void* Wg, const void* Wu, int dtype,
                              const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                              void* h1, void* h2, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return ffn_recompute_impl("moe_grouped_ffn_recompute", xp, moe::RowGather{}, Wg, Wu, dtype,
                            expert_offsets, rows, E, d, f, h1, h2, ws, ws_bytes, stream);
}

int moe_grouped_ffn_recompute_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                                     const void* Wg, const void* Wu, int dtype,
                                     const int64_t* expert_offsets, int E, int d, int f, void* h1,
                                     void* h2, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!pair_of_row && T > 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_recompute_gather: null pointer");
  return ffn_recompute_impl("moe_grouped_ffn_recompute_gather", x, row_gather(pair_of_row, T, k),
                            Wg, Wu, dtype, expert_offsets, T * k, E, d, f, h1, h2, ws, ws_bytes,
                            stream);
}

size_t moe_grouped_ffn_bwd_workspace_bytes(int64_t rows, int E, int d, int f, int dtype) {
  (void)d;
  if (rows < 0 || E < 1 || f < 1 || !dtype_ok(dtype)) return 0;
  const size_t h = align256(static_cast<size_t>(rows) * f * elem_bytes(dtype));
  return moe::kWsHeader + 2 * h;
}

size_t moe_grouped_ffn_wgrad_workspace_bytes(int E, int dtype) {
  if (E < 1 || !dtype_ok(dtype)) return 0;
  return moe::kWsHeader;
}

int moe_grouped_ffn_bwd(const void* xp, const void* Wg, const void* Wu, const void* Wd,
                        const void* h1, const void* h2, const void* a, const void* dyp, int dtype,
                        const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                        void* dxp, float* dWg, float* dWu, float* dWd, int accumulate, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  return ffn_bwd_impl("moe_grouped_ffn_bwd", xp, moe::RowGather{}, Wg, Wu, Wd, h1, h2, a, dyp,
                      dtype, expert_offsets, rows, E, d, f, dxp, dWg, dWu, dWd, accumulate, ws,
                      ws_bytes, stream);
}

int moe_grouped_ffn_bwd_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                               const void* Wg, const void* Wu, const void* Wd, const void* h1,
                               const void* h2, const void* a, const void* dyp, int dtype,
                               const int64_t* expert_offsets, int E, int d, int f, void* dxp,
                               float* dWg, float* dWu, float* dWd, int accumulate, void* ws,
                               size_t ws_bytes, cudaStream_t stream) {
  if (!pair_of_row && T > 0) return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_bwd_gather: null pointer");
  return ffn_bwd_impl("moe_grouped_ffn_bwd_gather", x, row_gather(pair_of_row, T, k), Wg, Wu, Wd,
                      h1, h2, a, dyp, dtype, expert_offsets, T * k, E, d, f, dxp, dWg, dWu, dWd,
                      accumulate, ws, ws_bytes, stream);
}

int moe_grouped_ffn_dgrad(const void* Wg, const void* Wu, const void* Wd, const void* h1,
                          const void* h2, const void* dyp, int dtype, const int64_t* expert_offsets,
                          int64_t rows, int E, int d, int f, void* dh1, void* dh2, void* dxp,
                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = check_ffn("moe_grouped_ffn_dgrad", dtype, rows, E, d, f);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!Wg || !Wu || !Wd || !h1 || !h2 || !dyp || !expert_offsets || !dh1 || !dh2 || !dxp || !ws)
    return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_dgrad: null pointer");
  const void* ptrs[] = {Wg, Wu, Wd, h1, h2, dyp, dh1, dh2, dxp, ws};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_dgrad: 16-byte alignment");
  if (ws_bytes < moe::kWsHeader) return fail(MOE_ERR_WORKSPACE, "moe_grouped_ffn_dgrad: workspace");
  moe::FfnBwdArgs args{nullptr, Wg, Wu, Wd, h1, h2, nullptr, dyp, expert_offsets, rows, E, d, f,
                       dxp, nullptr, nullptr, nullptr, dh1, dh2, static_cast<unsigned*>(ws), 1};
  cudaError_t e = dtype == MOE_BF16 ? moe::launch_ffn_dgrad_bf16(args, stream)
                                    : moe::launch_ffn_dgrad_f32(args, stream);
  return launched(cuda_status(e, "moe_grouped_ffn_dgrad"), 2);
}

int moe_grouped_ffn_wgrad(const void* xp, const void* a, const void* dyp, const void* dh1,
                          const void* dh2, int dtype, const int64_t* expert_offsets, int64_t rows,
                          int E, int d, int f, float* dWg, float* dWu, float* dWd, int accumulate,
                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  return ffn_wgrad_impl("moe_grouped_ffn_wgrad", xp, moe::RowGather{}, a, dyp, dh1, dh2, dtype,
                        expert_offsets, rows, E, d, f, dWg, dWu, dWd, accumulate, ws, ws_bytes,
                        stream);
}

int moe_grouped_ffn_wgrad_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                                 const void* a, const void* dyp, const void* dh1, const void* dh2,
                                 int dtype, const int64_t* expert_offsets, int E, int d, int f,
                                 float* dWg, float* dWu, float* dWd, int accumulate, void* ws,
                                 size_t ws_bytes, cudaStream_t stream) {
  if (!pair_of_row && T > 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_wgrad_gather: null pointer");
  return ffn_wgrad_impl("moe_grouped_ffn_wgrad_gather", x, row_gather(pair_of_row, T, k), a, dyp,
                        dh1, dh2, dtype, expert_offsets, T * k, E, d, f, dWg, dWu, dWd, accumulate,
                        ws, ws_bytes, stream);
}

}  // extern "C"
