/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE layer hot path.
 *
 * The layer is the one the expert-parallel MoE training runtimes on the
 * pages run on every step: expert routing, EP token dispatch, grouped expert
 * compute, and the combine that restores full source-order outputs, forward
 * and backward, with uneven and empty work per expert and per microbatch.
 *   - "EP token dispatch, grouped expert compute": leap-finetune PR #26
 *     "Add MoE expert parallel training runtime", Summary / Major changes.
 *   - "grouped-GEMM": ART issue #917 "Support combined expert and data
 *     parallelism in TrainerRank", Related.
 *   - expert-routing communication, expert communication groups, full
 *     source-order outputs, accumulation, uneven or empty work, explicit
 *     errors for unsupported cases: ART issue #917, intro, Desired behavior
 *     and Acceptance.
 * The pages give no formulas; the arithmetic below is the plainest reading
 * (a dropless top-k softmax-gated mixture of SwiGLU experts):
 *   z      = x Wr^T + b                             router logits
 *   S_t    = the k largest z[t,:], ties to the lower expert index, in
 *            descending order (slot j holds the j-th largest)
 *   g_t    = softmax(z[t, S_t])                     gate weights, sum to 1
 *   h1 = xp Wg_e^T, h2 = xp Wu_e^T, a = silu(h1) * h2, yp = a Wd_e^T
 *   Y_t    = sum_j g_{t,j} yp[row(t,j)]
 * and the backward is the exact gradient of that with S_t held fixed.
 *
 * Conventions (every entry point):
 *   - Pointers are DEVICE pointers unless stated otherwise, owned by the
 *     caller. The library never allocates device memory. Scratch memory is
 *     a caller buffer `ws` of at least the size the matching
 *     *_workspace_bytes function returns; it must be zero-filled once after
 *     allocation (its first bytes hold the device error word).
 *   - Tensors are dense row-major; the last listed dimension is contiguous.
 *   - `dtype` selects the element type of activations and weights:
 *     MOE_BF16 (bf16 storage, fp32 accumulation, tcgen05 tensor cores) or
 *     MOE_F32 (fp32 throughout, CUDA cores). Logits, gate weights and every
 *     gradient of a parameter are fp32.
 *   - Index arrays are int32; offsets are int64.
 *   - Every call is asynchronous on `stream`, performs no host
 *     synchronisation and no allocation. moe_get_error is the one call that
 *     synchronises.
 *   - T = 0 (an empty microbatch) is valid everywhere: the call returns
 *     MOE_OK, launches nothing and leaves every output and accumulator as it
 *     was (except that a parameter gradient requested with accumulate = 0 is
 *     set to zero, the gradient of an empty batch).
 *   - Gradients of parameters go to fp32 buffers: with accumulate = 1 they
 *     are added (+=, gradient accumulation over microbatches), with
 *     accumulate = 0 they are written (=, the first microbatch of a step;
 *     the buffer's old contents are not read). Activation gradients
 *     overwrite.
 *   - Return value: MOE_OK, or a negative MOE_ERR_* code with a message
 *     available from moe_last_error() (thread-local). Arguments are checked
 *     before anything is launched; a rejected call changes nothing.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_F32 0
#define MOE_BF16 1

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null pointer, negative size, k < 1, k > E */
#define MOE_ERR_UNSUPPORTED (-2) /* shape or dtype outside the supported set  */
#define MOE_ERR_WORKSPACE (-3)   /* ws too small or misaligned                */
#define MOE_ERR_CUDA (-4)        /* a CUDA call or launch failed              */

/* Bits of the device error word returned by moe_get_error. */
#define MOE_DEVERR_NONFINITE_LOGIT 1u /* a token's gate softmax was undefined   */
#define MOE_DEVERR_TIMEOUT 2u         /* a bounded wait inside a kernel gave up   */

/* Limits of this build. */
#define MOE_MAX_EXPERTS 1024

/* Message of the last failed call on this host thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Library ABI version (increments on any signature change). */
MOE_API int moe_version(void);

/* Number of kernels this library has launched in the process so far (all
 * devices, all threads). A diagnostic: differences around a region count the
 * library's launches in it. */
MOE_API int64_t moe_launch_count(void);

/* Self-test of the kernels' failure detection: launches one block that
 * waits on an mbarrier nothing ever arrives at, with the same bounded wait
 * the grouped GEMMs use, giving up after `limit_cycles` SM cycles (clamped to
 * [1e3, 4e9]). It then raises MOE_DEVERR_TIMEOUT in the ws error word and
 * returns normally, so the CUDA context stays usable; moe_get_error(ws)
 * reports it. ws: a zeroed workspace of at least 256 bytes. */
MOE_API int moe_selftest_wait_timeout(void* ws, long long limit_cycles, cudaStream_t stream);

/* Synchronises `stream`, returns the device error word accumulated in `ws`
 * by the calls that used it since the last moe_get_error (0 = no error), and
 * clears it. Returns MOE_ERR_CUDA (< 0) if the synchronisation fails. */
MOE_API int moe_get_error(void* ws, cudaStream_t stream);

/* ------------------------------------------------------------ routing */

/* Router logits z[t,e] = sum_i x[t,i] Wr[e,i] + b[e], in fp32: one fused
 * multiply-add per element in ascending i, then one add of b[e]. This fixed
 * order makes the logits, and therefore the top-k, bit-reproducible.
 * (Expert-routing step: ART issue #917, intro.)
 *   x       [T, d]   dtype      activations
 *   Wr      [E, d]   dtype      router weight
 *   b       [E]      fp32       router bias (may be NULL: no bias)
 *   logits  [T, E]   fp32       output
 * Errors: INVALID_ARG for null x/Wr/logits with T > 0, d, E < 1, or x, Wr
 * not 16-byte aligned; UNSUPPORTED for E > MOE_MAX_EXPERTS or d not a
 * multiple of 8. */
MOE_API int moe_router_logits(const void* x, const void* Wr, const float* b, int dtype,
                      int64_t T, int d, int E, float* logits, cudaStream_t stream);

/* Workspace of moe_route, in bytes. */
MOE_API size_t moe_route_workspace_bytes(int64_t T, int E);

/* Top-k softmax routing and the dispatch layout, all on the device.
 * Selection: per token the k largest logits, ties to the lower expert index,
 * NaN below every number, slots in descending order. Gate weights: softmax
 * over the k selected logits (they sum to 1), exp(z_j - m) / sum_i
 * exp(z_i - m) with m the largest selected logit; a selected -inf next to a
 * finite m gets exactly 0. Where that softmax is undefined -- m is +inf, every
 * selected logit is -inf, or a selected logit is NaN -- the token's weights
 * are 1/k each and MOE_DEVERR_NONFINITE_LOGIT is raised in the ws error word.
 * Layout (EP token dispatch, leap-finetune PR #26 Summary; expert
 * communication groups, ART issue #917 Desired behavior): pair (t,j) gets
 * row row_of_pair[t*k+j]; rows are sorted by (expert, token), both
 * ascending, so expert e owns rows [expert_offsets[e], expert_offsets[e+1])
 * in token order (stable, dropless, no padding). Experts are split into
 * `ep_groups` contiguous blocks of E/ep_groups (the destination groups an
 * all-to-all would send to); group g owns rows
 * [group_offsets[g], group_offsets[g+1]).
 *   logits         [T, E]        fp32  input
 *   topk_idx       [T, k]        int32 output, selected experts
 *   topk_w         [T, k]        fp32  output, gate weights
 *   expert_counts  [E]           int32 output
 *   expert_offsets [E+1]         int64 output, exclusive prefix sum
 *   group_counts   [ep_groups]   int32 output
 *   group_offsets  [ep_groups+1] int64 output
 *   row_of_pair    [T*k]         int32 output
 *   pair_of_row    [T*k]         int32 output, inverse permutation
 * For T = 0 nothing is written (as for every call), so a caller that reads
 * the counts of an empty microbatch zeroes them itself.
 * Errors: INVALID_ARG (null pointer, k < 1, k > E, ep_groups < 1),
 * UNSUPPORTED (E > MOE_MAX_EXPERTS, k > 32, E % ep_groups != 0,
 * T*k >= 2^31), WORKSPACE (ws_bytes < moe_route_workspace_bytes or ws not
 * 16-byte aligned). */
MOE_API int moe_route(const float* logits, int64_t T, int E, int k, int ep_groups,
              int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
              int64_t* expert_offsets, int32_t* group_counts, int64_t* group_offsets,
              int32_t* row_of_pair, int32_t* pair_of_row,
              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Largest ceil(T/256) * E that moe_route_noalloc accepts. */
#define MOE_ROUTE_NOALLOC_MAX_SLOTS 262144

/* moe_route for callers that cannot allocate device memory. (The pages have
 * no counterpart of this entry point; it exists for integration.)
 * moe_route asks the caller for a workspace; some callers cannot provide one:
 * code running inside another library or runtime that owns all device memory,
 * hosts that plan every byte ahead and forbid new allocations, or paths where
 * a cudaMalloc would synchronise the device. This variant keeps its scratch
 * (per-block expert counts and bases) in a fixed array compiled into the
 * library -- 2 MiB per GPU that loads the library, held until the process
 * exits -- and calls no cudaMalloc, cudaFree or other allocating routine.
 * Same arguments, outputs and results as moe_route, except:
 *   - no workspace; ceil(T/256) * E must not exceed MOE_ROUTE_NOALLOC_MAX_SLOTS
 *     (MOE_ERR_UNSUPPORTED otherwise: use moe_route);
 *   - err_flags: device pointer to a caller-zeroed unsigned int that the
 *     kernels OR MOE_DEVERR_* bits into, or NULL to not report them.
 * The first call on each device looks up the array's device address (with
 * that device current); make it before any stream capture. The address is
 * kept per device ordinal and looked up again when the device's primary
 * context changes (after cudaDeviceReset the array lives at a new address
 * in the new context). All calls on a
 * device share the array: calls that overlap on the GPU (other streams,
 * other host threads) race, so the caller must serialise them. Nothing has
 * to be cleared between calls. */
MOE_API int moe_route_noalloc(const float* logits, int64_t T, int E, int k, int ep_groups,
                              int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                              int64_t* expert_offsets, int32_t* group_counts,
                              int64_t* group_offsets, int32_t* row_of_pair, int32_t* pair_of_row,
                              unsigned int* err_flags, cudaStream_t stream);

/* ---------------------------------------------------------- dispatch */

/* Permute (dispatch copy): xp[row_of_pair[t*k+j], :] = x[t, :].
 *   x [T, d] dtype; row_of_pair [T*k] int32; xp [T*k, d] dtype output.
 * Errors: INVALID_ARG, UNSUPPORTED (d not a multiple of 8). */
MOE_API int moe_permute(const void* x, int dtype, int64_t T, int d, int k,
                const int32_t* row_of_pair, void* xp, cudaStream_t stream);

/* Workspace of moe_grouped_ffn_fwd, in bytes. */
MOE_API size_t moe_grouped_ffn_fwd_workspace_bytes(int64_t rows, int E, int d, int f, int dtype);

/* Grouped SwiGLU expert FFN, forward (grouped expert compute,
 * leap-finetune PR #26 Summary; grouped-GEMM, ART issue #917). Rows
 * [expert_offsets[e], expert_offsets[e+1]) of xp go through expert e:
 *   h1 = xp Wg_e^T, h2 = xp Wu_e^T, a = silu(h1) * h2, yp = a Wd_e^T.
 * The offsets are read on the device: an expert with no rows costs nothing
 * and no host synchronisation is needed.
 *   xp [rows, d]; Wg, Wu [E, f, d]; Wd [E, d, f]   dtype inputs
 *   expert_offsets [E+1] int64 (from moe_route), expert_offsets[E] == rows
 *   h1, h2, a [rows, f]; yp [rows, d]              dtype outputs
 *     (h1, h2 and a are saved for the backward; h1 and h2 may both be NULL:
 *     then they are not stored, 2 rows * f elements less written, and the
 *     backward rebuilds them with moe_grouped_ffn_recompute; activation
 *     checkpointing)
 * Errors: INVALID_ARG; UNSUPPORTED (bf16 needs d and f multiples of 8,
 * fp32 needs multiples of 4; E > MOE_MAX_EXPERTS); WORKSPACE. */
MOE_API int moe_grouped_ffn_fwd(const void* xp, const void* Wg, const void* Wu, const void* Wd,
                        int dtype, const int64_t* expert_offsets, int64_t rows, int E,
                        int d, int f, void* h1, void* h2, void* a, void* yp,
                        void* ws, size_t ws_bytes, cudaStream_t stream);

/* Fused dispatch (the permute folded into the expert GEMMs' operand loads;
 * EP token dispatch, leap-finetune PR #26 "Add MoE expert parallel training
 * runtime", Summary): moe_grouped_ffn_fwd with the expert input read in place
 * from the tokens instead of from the permuted copy xp. Dispatch row r of the
 * expert input is x[pair_of_row[r] / k], exactly the row moe_permute copies
 * to xp[r], so every output is bitwise that of moe_permute followed by
 * moe_grouped_ffn_fwd; xp is neither written nor read.
 *   x [T, d] dtype; pair_of_row [T*k] int32 (moe_route's output); rows = T*k;
 *   every other argument and error as moe_grouped_ffn_fwd (k in 1..32).
 * The bf16 path gathers the rows with 16-byte cp.async copies into the
 * GEMM's swizzled operand stages (the weights still arrive by TMA). It saves
 * the copy xp but runs slower than moe_permute + moe_grouped_ffn_fwd on
 * large d and f: the GEMM reads each row once per 128 output columns, and
 * row-sized gathers deliver those reads at a fraction of the tiled TMA rate. */
MOE_API int moe_grouped_ffn_fwd_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                                       const void* Wg, const void* Wu, const void* Wd, int dtype,
                                       const int64_t* expert_offsets, int E, int d, int f,
                                       void* h1, void* h2, void* a, void* yp, void* ws,
                                       size_t ws_bytes, cudaStream_t stream);

/* Unpermute and weighted combine (full source-order outputs, ART issue
 * #917 Desired behavior):
 *   Y[t, :] = sum_{j<k} topk_w[t,j] * yp[row_of_pair[t*k+j], :]
 * summed in fp32 with j ascending, rounded once to dtype.
 *   yp [T*k, d] dtype; topk_w [T, k] fp32; row_of_pair [T*k]; Y [T, d] dtype.
 * Errors: INVALID_ARG, UNSUPPORTED (d not a multiple of 8). */
MOE_API int moe_unpermute_combine(const void* yp, const float* topk_w, const int32_t* row_of_pair,
                          int dtype, int64_t T, int d, int k, void* Y, cudaStream_t stream);

/* --------------------------------------------------------- backward */

/* Combine backward:
 *   dyp[row_of_pair[t*k+j], :] = topk_w[t,j] * dY[t, :]
 *   dg[t, j] = sum_i dY[t,i] * yp[row_of_pair[t*k+j], i]   (fp32)
 *   dY [T, d] dtype; yp [T*k, d] dtype; dyp [T*k, d] dtype; dg [T, k] fp32. */
MOE_API int moe_unpermute_combine_bwd(const void* dY, const void* yp, const float* topk_w,
                              const int32_t* row_of_pair, int dtype, int64_t T, int d, int k,
                              void* dyp, float* dg, cudaStream_t stream);

/* Route backward through the softmax over the selected logits:
 *   dlogits[t, S_j] = g_j * (dg_j - sum_m g_m dg_m), and 0 for every expert
 *   not selected by token t.
 *   dg, topk_w [T, k] fp32; topk_idx [T, k] int32; dlogits [T, E] fp32 output. */
MOE_API int moe_route_bwd(const float* dg, const float* topk_w, const int32_t* topk_idx,
                  int64_t T, int E, int k, float* dlogits, cudaStream_t stream);

/* Activation checkpointing: recomputes h1 = xp Wg_e^T and h2 = xp Wu_e^T of
 * a forward that did not store them (the same kernel and order as
 * moe_grouped_ffn_fwd, so they are bitwise the values it would have stored).
 * a is not written. Arguments and errors as moe_grouped_ffn_fwd; ws needs
 * moe_grouped_ffn_fwd_workspace_bytes() bytes. */
MOE_API int moe_grouped_ffn_recompute(const void* xp, const void* Wg, const void* Wu, int dtype,
                                      const int64_t* expert_offsets, int64_t rows, int E, int d,
                                      int f, void* h1, void* h2, void* ws, size_t ws_bytes,
                                      cudaStream_t stream);

/* moe_grouped_ffn_recompute with the expert input gathered from x through
 * pair_of_row (rows = T*k), as moe_grouped_ffn_fwd_gather. */
MOE_API int moe_grouped_ffn_recompute_gather(const void* x, const int32_t* pair_of_row, int64_t T,
                                             int k, const void* Wg, const void* Wu, int dtype,
                                             const int64_t* expert_offsets, int E, int d, int f,
                                             void* h1, void* h2, void* ws, size_t ws_bytes,
                                             cudaStream_t stream);

/* Workspace of moe_grouped_ffn_bwd, in bytes (holds dh1 and dh2). */
MOE_API size_t moe_grouped_ffn_bwd_workspace_bytes(int64_t rows, int E, int d, int f, int dtype);

/* Grouped SwiGLU expert FFN, backward. Per expert e over its rows:
 *   da  = dyp Wd_e;  dh1 = da * h2 * silu'(h1);  dh2 = da * silu(h1)
 *   dxp = dh1 Wg_e + dh2 Wu_e                           (overwritten)
 *   dWg_e += dh1^T xp;  dWu_e += dh2^T xp;  dWd_e += dyp^T a   (fp32)
 * with silu'(u) = s (1 + u (1 - s)), s = sigmoid(u). accumulate = 1: the
 * products are added to dW, and an expert with no rows leaves its gradients
 * untouched; accumulate = 0: dW is overwritten with the products (zero for
 * an expert with no rows) and never read.
 *   xp, dyp [rows, d]; h1, h2, a [rows, f]; Wg, Wu [E, f, d]; Wd [E, d, f]
 *   dxp [rows, d] dtype output; dWg, dWu [E, f, d], dWd [E, d, f] fp32.
 * Errors: as moe_grouped_ffn_fwd. */
MOE_API int moe_grouped_ffn_bwd(const void* xp, const void* Wg, const void* Wu, const void* Wd,
                        const void* h1, const void* h2, const void* a, const void* dyp,
                        int dtype, const int64_t* expert_offsets, int64_t rows, int E, int d,
                        int f, void* dxp, float* dWg, float* dWu, float* dWd, int accumulate,
                        void* ws, size_t ws_bytes, cudaStream_t stream);

/* moe_grouped_ffn_bwd with xp (the weight gradients' dWg, dWu operand) read
 * in place from x through pair_of_row (rows = T*k), as
 * moe_grouped_ffn_fwd_gather; bitwise the results of moe_grouped_ffn_bwd on
 * moe_permute's xp. dxp stays in dispatch-row order. */
MOE_API int moe_grouped_ffn_bwd_gather(const void* x, const int32_t* pair_of_row, int64_t T, int k,
                                       const void* Wg, const void* Wu, const void* Wd,
                                       const void* h1, const void* h2, const void* a,
                                       const void* dyp, int dtype, const int64_t* expert_offsets,
                                       int E, int d, int f, void* dxp, float* dWg, float* dWu,
                                       float* dWd, int accumulate, void* ws, size_t ws_bytes,
                                       cudaStream_t stream);

/* The two halves of moe_grouped_ffn_bwd, for callers that keep dh1 / dh2
 * themselves (and may schedule the weight gradient apart from the data
 * gradient). Same arithmetic as moe_grouped_ffn_bwd.
 * moe_grouped_ffn_dgrad: data gradients
 *   dh1, dh2 [rows, f] dtype outputs (the SwiGLU backward of da = dyp Wd_e)
 *   dxp [rows, d] dtype output (= dh1 Wg_e + dh2 Wu_e)
 * moe_grouped_ffn_wgrad: weight gradients in fp32, added or written as the
 * accumulate flag says (as moe_grouped_ffn_bwd)
 *   dWg_e (+)= dh1^T xp; dWu_e (+)= dh2^T xp; dWd_e (+)= dyp^T a
 * ws of moe_grouped_ffn_dgrad needs moe_grouped_ffn_fwd_workspace_bytes()
 * bytes (its error word); ws of moe_grouped_ffn_wgrad needs
 * moe_grouped_ffn_wgrad_workspace_bytes(E, dtype) bytes. */
/* Workspace of moe_grouped_ffn_wgrad and moe_grouped_ffn_wgrad_gather, in
 * bytes (its error word). Calls that overlap on the GPU need their own. */
MOE_API size_t moe_grouped_ffn_wgrad_workspace_bytes(int E, int dtype);
MOE_API int moe_grouped_ffn_dgrad(const void* Wg, const void* Wu, const void* Wd, const void* h1,
                                  const void* h2, const void* dyp, int dtype,
                                  const int64_t* expert_offsets, int64_t rows, int E, int d, int f,
                                  void* dh1, void* dh2, void* dxp, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);
MOE_API int moe_grouped_ffn_wgrad(const void* xp, const void* a, const void* dyp, const void* dh1,
                                  const void* dh2, int dtype, const int64_t* expert_offsets,
                                  int64_t rows, int E, int d, int f, float* dWg, float* dWu,
                                  float* dWd, int accumulate, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);
/* moe_grouped_ffn_wgrad with xp gathered from x through pair_of_row
 * (rows = T*k), as moe_grouped_ffn_fwd_gather. */
MOE_API int moe_grouped_ffn_wgrad_gather(const void* x, const int32_t* pair_of_row, int64_t T,
                                         int k, const void* a, const void* dyp, const void* dh1,
                                         const void* dh2, int dtype, const int64_t* expert_offsets,
                                         int E, int d, int f, float* dWg, float* dWu, float* dWd,
                                         int accumulate, void* ws, size_t ws_bytes,
                                         cudaStream_t stream);

/* Permute backward, with the router's input gradient folded in:
 *   dX[t, :] = sum_{j<k} dxp[row_of_pair[t*k+j], :]
 *            + sum_{j<k} dlogits[t, S_j] * Wr[S_j, :]      (if dlogits != NULL)
 * summed in fp32 (j ascending), rounded once to dtype; dX is overwritten.
 * The router term reads only the k selected columns of dlogits: it equals
 * dlogits[t,:] Wr when dlogits is zero off the selection, which
 * moe_route_bwd guarantees.
 *   dxp [T*k, d] dtype; row_of_pair [T*k]; dlogits [T, E] fp32 or NULL;
 *   Wr [E, d] dtype (ignored if dlogits is NULL); topk_idx [T, k];
 *   dX [T, d] dtype output. */
MOE_API int moe_permute_bwd(const void* dxp, const int32_t* row_of_pair, const float* dlogits,
                    const void* Wr, const int32_t* topk_idx, int dtype, int64_t T, int d,
                    int E, int k, void* dX, cudaStream_t stream);

/* Expert-parallel regroup (expert communication groups, ART issue #917
 * "Support combined expert and data parallelism in TrainerRank", Desired
 * behavior; EP token dispatch, leap-finetune PR #26 Summary). After the
 * dispatch all-to-all, a rank holds rows from G source ranks, each source's
 * rows grouped by this rank's El local experts in expert order (the R4 group
 * layout of moe_route on the sender). This call builds, on the device, the
 * map that sorts them by (local expert, source rank, arrival):
 *   recv_counts   [G, El] int32  rows received from source s for local expert e
 *   row_map       [sum recv_counts] int32 output: received row i goes to
 *                 row row_map[i] (a scatter for moe_permute with k = 1; its
 *                 inverse gather is moe_permute_bwd with k = 1)
 *   local_offsets [El+1] int64 output: local expert e owns sorted rows
 *                 [local_offsets[e], local_offsets[e+1]) (the expert_offsets
 *                 of the grouped FFN calls on this rank)
 * row_map must hold sum(recv_counts) entries (at least one); the counts are
 * read on the device only, so no host synchronisation is needed.
 * Errors: INVALID_ARG (null pointer, G or El < 1), UNSUPPORTED
 * (G * El > MOE_MAX_EXPERTS). */
MOE_API int moe_ep_regroup(const int32_t* recv_counts, int G, int El, int32_t* row_map,
                           int64_t* local_offsets, cudaStream_t stream);

/* Workspace of moe_router_bwd, in bytes (rows = T*k). */
MOE_API size_t moe_router_bwd_workspace_bytes(int64_t rows, int d, int E);

/* Router weight gradients (fp32, deterministic order; added with
 * accumulate = 1, written with accumulate = 0):
 *   dWr[e, :] (+)= sum_t dlogits[t, e] x[t, :];   db[e] (+)= sum_t dlogits[t, e]
 * (router backward of z = x Wr^T + b). The sums run over the dispatch rows
 * instead of all tokens: expert e's rows [expert_offsets[e],
 * expert_offsets[e+1]) hold exactly the tokens that selected e, and xp holds
 * their x rows, so
 *   dWr[e, :] += sum_{r in e} dlogits[pair_of_row[r] / k, e] xp[r, :].
 * This equals the sum over all tokens when dlogits is zero off the selection,
 * which moe_route_bwd guarantees; it reads xp once instead of computing a
 * T x E x d product.
 *   xp [T*k, d] dtype (moe_permute's output); dlogits [T, E] fp32;
 *   pair_of_row [T*k], expert_offsets [E+1] (moe_route's outputs);
 *   dWr [E, d] fp32; db [E] fp32 (may be NULL). An expert no token selected
 * keeps its rows (accumulate = 1) or gets zeros (accumulate = 0). */
MOE_API int moe_router_bwd(const void* xp, const float* dlogits, const int32_t* pair_of_row,
                           const int64_t* expert_offsets, int dtype, int64_t T, int d, int E,
                           int k, float* dWr, float* db, int accumulate, void* ws,
                           size_t ws_bytes, cudaStream_t stream);
/* moe_router_bwd reading dispatch row r as x[pair_of_row[r] / k] (x [T, d])
 * instead of xp[r]: the same values in the same order, so bitwise the same
 * dWr and db, without the permuted copy. */
MOE_API int moe_router_bwd_gather(const void* x, const float* dlogits, const int32_t* pair_of_row,
                                  const int64_t* expert_offsets, int dtype, int64_t T, int d,
                                  int E, int k, float* dWr, float* db, int accumulate, void* ws,
                                  size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------
 * Auxiliary load-balancing loss of the router and routing metrics.
 * The pages name MoE losses and metrics without a formula (leap-finetune
 * PR #26 "Add MoE expert parallel training runtime", its MoE-loss tests);
 * the reading taken is the Switch-style balance loss:
 *   p[t,e] = softmax over all E experts of logits[t,:]
 *   f_e    = expert_counts[e] / (T k)      (fraction of routed pairs)
 *   P_e    = (1/T) sum_t p[t,e]            (importance)
 *   loss   = alpha * E * sum_e f_e P_e
 *   entropy = (1/T) sum_t -sum_e p[t,e] ln p[t,e]   (mean routing entropy)
 * f counts routed pairs and is constant in the logits. Sums run in a fixed
 * order (deterministic). */

/* Workspace of moe_aux_loss, in bytes: per-block partial sums. */
MOE_API size_t moe_aux_loss_workspace_bytes(int64_t T, int E);

/* logits [T, E] fp32, expert_counts [E] int32 (moe_route's outputs);
 * importance [E] fp32, loss [1] fp32, entropy [1] fp32 (may be NULL):
 * device outputs. T = 0 writes zeros. Errors: MOE_ERR_INVALID_ARG (null
 * pointers, k < 1, k > E), MOE_ERR_UNSUPPORTED (E > MOE_MAX_EXPERTS). */
MOE_API int moe_aux_loss(const float* logits, const int32_t* expert_counts, int64_t T, int E,
                         int k, float alpha, float* importance, float* loss, float* entropy,
                         void* ws, size_t ws_bytes, cudaStream_t stream);

/* Gradient of dloss * loss in the logits, the counts held fixed:
 *   dlogits_aux[t,j] = dloss * alpha * E / T * p[t,j] * (f_j - sum_e f_e p[t,e])
 * written (not added) to dlogits_aux [T, E] fp32. It is dense: carry it to
 * x, Wr and b with moe_router_bwd_dense. */
MOE_API int moe_aux_loss_bwd(const float* logits, const int32_t* expert_counts, int64_t T, int E,
                             int k, float alpha, float dloss, float* dlogits_aux,
                             cudaStream_t stream);

/* Workspace of moe_router_bwd_dense, in bytes (per-chunk partial sums of
 * dWr and db: 4 (E d + E) bytes per 256 tokens). */
MOE_API size_t moe_router_bwd_dense_workspace_bytes(int64_t T, int d, int E);

/* Router backward for a dense logit gradient dz (for example the balance
 * loss's; moe_permute_bwd and moe_router_bwd use only the selected columns):
 *   dX[t,:] += sum_e dz[t,e] Wr[e,:]      (dX in the activation dtype, one
 *                                          rounding of the fp32 sum; may be NULL)
 *   dWr[e,:] (+)= sum_t dz[t,e] x[t,:];   db[e] (+)= sum_t dz[t,e]
 * added (accumulate = 1) or written (accumulate = 0); db may be NULL.
 *   x [T, d] dtype, Wr [E, d] dtype, dz [T, E] fp32. fp32 sums in a fixed
 * order. d must be a multiple of 4. */
MOE_API int moe_router_bwd_dense(const void* x, const void* Wr, const float* dz, int dtype,
                                 int64_t T, int d, int E, void* dX, float* dWr, float* db,
                                 int accumulate, void* ws, size_t ws_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
