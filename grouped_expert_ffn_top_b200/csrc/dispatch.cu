// HBM-bound passes of the layer: permute (dispatch copy), unpermute-combine,
// their backward, and the router's weight gradient.
// (EP token dispatch: leap-finetune PR #26 Summary; full source-order outputs:
// ART issue #917 Desired behavior.)
//
// Each token is handled by one warp that moves whole rows with 16-byte
// vectors: a row of d elements is d/8 (bf16) or d/4 (fp32) vectors, spread
// over the 32 lanes, so every warp-wide access is 512 contiguous bytes. Each
// source row is read once and each destination row written once, which is
// the algorithmic minimum of these passes.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kWarpsPerBlock = 8;

// Row indices (and weights) of token t's k pairs, broadcast to every lane.
template <int KMAX>
struct PairRows {
  int64_t row[KMAX];
  float w[KMAX];
};

template <int KMAX>
__device__ __forceinline__ PairRows<KMAX> load_pairs(const int32_t* __restrict__ rop,
                                                     const float* __restrict__ w, int64_t t,
                                                     int k) {
  const int lane = threadIdx.x & 31;
  int r = 0;
  float g = 0.0f;
  if (lane < k) {
    r = rop[t * k + lane];
    if (w) g = w[t * k + lane];
  }
  PairRows<KMAX> p;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    p.row[j] = __shfl_sync(0xffffffffu, r, j);
    p.w[j] = __shfl_sync(0xffffffffu, g, j);
  }
  return p;
}

// ------------------------------------------------------------------ permute
// xp[row_of_pair[t*k+j]] = x[t]: x is read once, each of the k copies written once.
template <typename T, int KMAX>
__global__ void __launch_bounds__(256) permute_kernel(const T* __restrict__ x, int64_t Ttok,
                                                      int d, int k,
                                                      const int32_t* __restrict__ rop,
                                                      T* __restrict__ xp) {
  constexpr int VE = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= Ttok) return;
  const PairRows<KMAX> p = load_pairs<KMAX>(rop, nullptr, t, k);
  const int nvec = d / VE;
  const T* src = x + t * d;
#pragma unroll 4
  for (int v = lane; v < nvec; v += 32) {
    const Vec16<T> val = ld16_stream(src + v * VE);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) st16(xp + p.row[j] * d + v * VE, val);
  }
}

// ------------------------------------------------------------------ combine
// Y[t] = sum_j w[t,j] yp[row_of_pair[t*k+j]], fp32, j ascending.
template <typename T, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ yp,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ rop,
                                                      int64_t Ttok, int d, int k,
                                                      T* __restrict__ Y) {
  constexpr int VE = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= Ttok) return;
  const PairRows<KMAX> p = load_pairs<KMAX>(rop, w, t, k);
  const int nvec = d / VE;
#pragma unroll 2
  for (int v = lane; v < nvec; v += 32) {
    Vec16<T> in[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) in[j] = ld16_stream(yp + p.row[j] * d + v * VE);
    float acc[VE];
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
#pragma unroll
        for (int q = 0; q < VE; ++q) acc[q] = __fmaf_rn(p.w[j], in[j].get(q), acc[q]);
      }
    Vec16<T> o;
#pragma unroll
    for (int q = 0; q < VE; ++q) o.set(q, acc[q]);
    st16(Y + t * d + v * VE, o);
  }
}

// -------------------------------------------------------- combine backward
// dyp[row] = w[t,j] dY[t];  dg[t,j] = <dY[t], yp[row]>.
template <typename T, int KMAX>
__global__ void __launch_bounds__(256) combine_bwd_kernel(const T* __restrict__ dY,
                                                          const T* __restrict__ yp,
                                                          const float* __restrict__ w,
                                                          const int32_t* __restrict__ rop,
                                                          int64_t Ttok, int d, int k,
                                                          T* __restrict__ dyp,
                                                          float* __restrict__ dg) {
  constexpr int VE = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= Ttok) return;
  const PairRows<KMAX> p = load_pairs<KMAX>(rop, w, t, k);
  const int nvec = d / VE;
  float dot[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) dot[j] = 0.0f;
  for (int v = lane; v < nvec; v += 32) {
    const Vec16<T> g = ld16_stream(dY + t * d + v * VE);
    Vec16<T> in[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) in[j] = ld16_stream(yp + p.row[j] * d + v * VE);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
        Vec16<T> o;
#pragma unroll
        for (int q = 0; q < VE; ++q) {
          const float gq = g.get(q);
          dot[j] = __fmaf_rn(gq, in[j].get(q), dot[j]);
          o.set(q, p.w[j] * gq);
        }
        st16(dyp + p.row[j] * d + v * VE, o);
      }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    float s = dot[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0 && j < k) dg[t * k + j] = s;
  }
}

// -------------------------------------------------------- permute backward
// dX[t] = sum_j dxp[row_of_pair[t*k+j]] + sum_j dz[t, S_j] Wr[S_j]   (fp32 sum)
template <typename T, int KMAX>
__global__ void __launch_bounds__(256) permute_bwd_kernel(const T* __restrict__ dxp,
                                                          const int32_t* __restrict__ rop,
                                                          const float* __restrict__ dz,
                                                          const T* __restrict__ Wr,
                                                          const int32_t* __restrict__ idx,
                                                          int64_t Ttok, int d, int E, int k,
                                                          T* __restrict__ dX) {
  constexpr int VE = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= Ttok) return;
  const PairRows<KMAX> p = load_pairs<KMAX>(rop, nullptr, t, k);
  int ej = 0;
  float zj = 0.0f;
  if (dz && lane < k) {
    ej = idx[t * k + lane];
    zj = dz[t * E + ej];
  }
  int64_t wrow[KMAX];
  float zsel[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    wrow[j] = static_cast<int64_t>(__shfl_sync(0xffffffffu, ej, j)) * d;
    zsel[j] = __shfl_sync(0xffffffffu, zj, j);
  }
  const int nvec = d / VE;
#pragma unroll 2
  for (int v = lane; v < nvec; v += 32) {
    Vec16<T> in[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) in[j] = ld16_stream(dxp + p.row[j] * d + v * VE);
    float acc[VE];
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
#pragma unroll
        for (int q = 0; q < VE; ++q) acc[q] += in[j].get(q);
      }
    if (dz) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) {
          const Vec16<T> wr = ld16(Wr + wrow[j] + v * VE);
#pragma unroll
          for (int q = 0; q < VE; ++q) acc[q] = __fmaf_rn(zsel[j], wr.get(q), acc[q]);
        }
    }
    Vec16<T> o;
#pragma unroll
    for (int q = 0; q < VE; ++q) o.set(q, acc[q]);
    st16(dX + t * d + v * VE, o);
  }
}

// ------------------------------------------------------------- launchers

#define MOE_KSWITCH(k, CALL) \
  do {                       \
    if ((k) <= 1) {          \
      CALL(1);               \
    } else if ((k) <= 2) {   \
      CALL(2);               \
    } else if ((k) <= 4) {   \
      CALL(4);               \
    } else if ((k) <= 8) {   \
      CALL(8);               \
    } else if ((k) <= 16) {  \
      CALL(16);              \
    } else {                 \
      CALL(32);              \
    }                        \
  } while (0)

static unsigned warp_grid(int64_t T) {
  return static_cast<unsigned>((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

template <typename T>
static void permute_t(const T* x, int64_t Tn, int d, int k, const int32_t* rop, T* xp,
                      cudaStream_t s) {
#define CALL(KM) permute_kernel<T, KM><<<warp_grid(Tn), 256, 0, s>>>(x, Tn, d, k, rop, xp)
  MOE_KSWITCH(k, CALL);
#undef CALL
}

cudaError_t launch_permute(const void* x, int dtype, int64_t T, int d, int k,
                           const int32_t* row_of_pair, void* xp, cudaStream_t s) {
  if (dtype == MOE_BF16)
    permute_t(static_cast<const bf16*>(x), T, d, k, row_of_pair, static_cast<bf16*>(xp), s);
  else
    permute_t(static_cast<const float*>(x), T, d, k, row_of_pair, static_cast<float*>(xp), s);
  return cudaGetLastError();
}

template <typename T>
static void combine_t(const T* yp, const float* w, const int32_t* rop, int64_t Tn, int d, int k,
                      T* Y, cudaStream_t s) {
#define CALL(KM) combine_kernel<T, KM><<<warp_grid(Tn), 256, 0, s>>>(yp, w, rop, Tn, d, k, Y)
  MOE_KSWITCH(k, CALL);
#undef CALL
}

cudaError_t launch_combine(const void* yp, const float* w, const int32_t* row_of_pair, int dtype,
                           int64_t T, int d, int k, void* Y, cudaStream_t s) {
  if (dtype == MOE_BF16)
    combine_t(static_cast<const bf16*>(yp), w, row_of_pair, T, d, k, static_cast<bf16*>(Y), s);
  else
    combine_t(static_cast<const float*>(yp), w, row_of_pair, T, d, k, static_cast<float*>(Y), s);
  return cudaGetLastError();
}

template <typename T>
static void combine_bwd_t(const T* dY, const T* yp, const float* w, const int32_t* rop,
                          int64_t Tn, int d, int k, T* dyp, float* dg, cudaStream_t s) {
#define CALL(KM) \
  combine_bwd_kernel<T, KM><<<warp_grid(Tn), 256, 0, s>>>(dY, yp, w, rop, Tn, d, k, dyp, dg)
  MOE_KSWITCH(k, CALL);
#undef CALL
}

cudaError_t launch_combine_bwd(const void* dY, const void* yp, const float* w,
                               const int32_t* row_of_pair, int dtype, int64_t T, int d, int k,
                               void* dyp, float* dg, cudaStream_t s) {
  if (dtype == MOE_BF16)
    combine_bwd_t(static_cast<const bf16*>(dY), static_cast<const bf16*>(yp), w, row_of_pair, T,
                  d, k, static_cast<bf16*>(dyp), dg, s);
  else
    combine_bwd_t(static_cast<const float*>(dY), static_cast<const float*>(yp), w, row_of_pair, T,
                  d, k, static_cast<float*>(dyp), dg, s);
  return cudaGetLastError();
}

template <typename T>
static void permute_bwd_t(const T* dxp, const int32_t* rop, const float* dz, const T* Wr,
                          const int32_t* idx, int64_t Tn, int d, int E, int k, T* dX,
                          cudaStream_t s) {
#define CALL(KM)                                                                          \
  permute_bwd_kernel<T, KM><<<warp_grid(Tn), 256, 0, s>>>(dxp, rop, dz, Wr, idx, Tn, d, E, k, \
                                                          dX)
  MOE_KSWITCH(k, CALL);
#undef CALL
}

cudaError_t launch_permute_bwd(const void* dxp, const int32_t* row_of_pair, const float* dz,
                               const void* Wr, const int32_t* idx, int dtype, int64_t T, int d,
                               int E, int k, void* dX, cudaStream_t s) {
  if (dtype == MOE_BF16)
    permute_bwd_t(static_cast<const bf16*>(dxp), row_of_pair, dz, static_cast<const bf16*>(Wr),
                  idx, T, d, E, k, static_cast<bf16*>(dX), s);
  else
    permute_bwd_t(static_cast<const float*>(dxp), row_of_pair, dz, static_cast<const float*>(Wr),
                  idx, T, d, E, k, static_cast<float*>(dX), s);
  return cudaGetLastError();
}

// ------------------------------------------------------ router weight grad
//
// dWr[e, c] += sum_t dz[t, e] x[t, c]; db[e] += sum_t dz[t, e].
// Pass 1: block (column chunk of 64, token split, expert chunk of 64) sums its
// split into partial[split][e][c] (fp32). Pass 2 adds the splits in order.
// No atomics: the result does not depend on scheduling.

constexpr int kRbRows = 256;  // dispatch rows per work item
constexpr int kRbThreads = 256;

int router_bwd_max_items(int64_t rows, int E) {
  return static_cast<int>((rows + kRbRows - 1) / kRbRows) + E;
}

// First work item of each expert (expert e owns ceil(count_e / kRbRows)
// items, in expert order); s_start[E] = number of items. Whole block.
__device__ void router_items_prefix(const int64_t* __restrict__ off, int E, int* s_start) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int v = e < E ? static_cast<int>((off[e + 1] - off[e] + kRbRows - 1) / kRbRows) : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      if (e < E) s_start[e] = carry + inc - v;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) s_start[E] = carry;
  }
  __syncthreads();
}

__device__ __forceinline__ int expert_of_item(const int* s_start, int E, int item) {
  int lo = 0, hi = E - 1;  // largest e with s_start[e] <= item
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_start[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// partial[item, cols] = sum over the item's rows r (ascending) of
// dz[token(r), e] * xp[r, cols]; partial_db[item] = sum of those dz.
// Each xp row is read once, 16 bytes per thread, coalesced across the block.
// GATHER: `xp` is x [T, d] and row r is read as x[token(r)] (the same values,
// since xp[r] is a copy of x[token(r)]), so xp need not exist.
template <typename T, bool GATHER>
__global__ void __launch_bounds__(kRbThreads) router_wgrad_partial_kernel(
    const T* __restrict__ xp, const float* __restrict__ dz, const int32_t* __restrict__ por,
    const int64_t* __restrict__ off, int E, int d, int k, float* __restrict__ partial,
    float* __restrict__ partial_db) {
  constexpr int VE = Vec16<T>::N;
  __shared__ int s_start[MOE_MAX_EXPERTS + 1];
  __shared__ float s_dz[kRbRows];
  __shared__ int s_tok[GATHER ? kRbRows : 1];
  router_items_prefix(off, E, s_start);
  const int item = blockIdx.x;
  if (item >= s_start[E]) return;
  const int e = expert_of_item(s_start, E, item);
  const int64_t r0 = off[e] + static_cast<int64_t>(item - s_start[e]) * kRbRows;
  const int nrows = static_cast<int>(min(off[e + 1] - r0, static_cast<int64_t>(kRbRows)));
  for (int i = threadIdx.x; i < nrows; i += blockDim.x) {
    const int t = por[r0 + i] / k;
    s_dz[i] = dz[static_cast<int64_t>(t) * E + e];
    if (GATHER) s_tok[i] = t;
  }
  __syncthreads();
  const int c = (blockIdx.y * kRbThreads + threadIdx.x) * VE;
  if (c < d) {
    float acc[VE];
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] = 0.0f;
    const T* src = xp + (GATHER ? 0 : r0 * d) + c;
#pragma unroll 4
    for (int i = 0; i < nrows; ++i) {
      const int64_t row = GATHER ? static_cast<int64_t>(s_tok[i]) : static_cast<int64_t>(i);
      const Vec16<T> v = ld16_stream(src + row * d);
      const float g = s_dz[i];
#pragma unroll
      for (int q = 0; q < VE; ++q) acc[q] = __fmaf_rn(g, v.get(q), acc[q]);
    }
    float* dst = partial + static_cast<int64_t>(item) * d + c;
#pragma unroll
    for (int q = 0; q < VE; q += 4)
      *reinterpret_cast<float4*>(dst + q) = make_float4(acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    float sdb = 0.0f;
    for (int i = 0; i < nrows; ++i) sdb += s_dz[i];
    partial_db[item] = sdb;
  }
}

// dWr[e, c] += sum of expert e's item partials, in item order; db likewise.
__global__ void __launch_bounds__(256) router_wgrad_reduce_kernel(
    const float* __restrict__ partial, const float* __restrict__ partial_db,
    const int64_t* __restrict__ off, int E, int d, float* __restrict__ dWr, float* __restrict__ db,
    int accumulate) {
  __shared__ int s_start[MOE_MAX_EXPERTS + 1];
  router_items_prefix(off, E, s_start);
  const int64_t n = static_cast<int64_t>(E) * d;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i / d);
    const int c = static_cast<int>(i % d);
    // no token selected e: untouched when accumulating, zero when writing
    if (s_start[e + 1] == s_start[e] && accumulate) continue;
    float s = 0.0f;
    for (int it = s_start[e]; it < s_start[e + 1]; ++it) s += partial[static_cast<int64_t>(it) * d + c];
    dWr[i] = accumulate ? dWr[i] + s : s;
    if (db && c == 0) {
      float sb = 0.0f;
      for (int it = s_start[e]; it < s_start[e + 1]; ++it) sb += partial_db[it];
      db[e] = accumulate ? db[e] + sb : sb;
    }
  }
}

template <typename T>
static void launch_router_partial(bool gather, dim3 grid, const void* src, const float* dz,
                                  const int32_t* por, const int64_t* off, int E, int d, int k,
                                  float* partial, float* partial_db, cudaStream_t s) {
  if (gather)
    router_wgrad_partial_kernel<T, true><<<grid, kRbThreads, 0, s>>>(
        static_cast<const T*>(src), dz, por, off, E, d, k, partial, partial_db);
  else
    router_wgrad_partial_kernel<T, false><<<grid, kRbThreads, 0, s>>>(
        static_cast<const T*>(src), dz, por, off, E, d, k, partial, partial_db);
}

cudaError_t launch_router_bwd(const void* xp, const float* dz, const int32_t* por,
                              const int64_t* off, int dtype, int64_t rows, int d, int E, int k,
                              float* dWr, float* db, int accumulate, float* partial, cudaStream_t s,
                              bool gather) {
  const int items = router_bwd_max_items(rows, E);
  float* partial_db = partial + static_cast<int64_t>(items) * d;
  const int vec = dtype == MOE_BF16 ? 8 : 4;
  dim3 grid(items, (d + kRbThreads * vec - 1) / (kRbThreads * vec));
  if (dtype == MOE_BF16)
    launch_router_partial<bf16>(gather, grid, xp, dz, por, off, E, d, k, partial, partial_db, s);
  else
    launch_router_partial<float>(gather, grid, xp, dz, por, off, E, d, k, partial, partial_db, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = static_cast<int64_t>(E) * d;
  const unsigned blocks = static_cast<unsigned>(((n + 255) / 256) < 148 * 8 ? (n + 255) / 256 : 148 * 8);
  router_wgrad_reduce_kernel<<<blocks, 256, 0, s>>>(partial, partial_db, off, E, d, dWr, db,
                                                     accumulate);
  return cudaGetLastError();
}

// ------------------------------------------------- expert-parallel regroup
// recv [G, El]: rows this rank received from source rank s for its local
// expert e. They arrive sources ascending and, within a source, experts
// ascending, so block (s, e) starts at received row
//   A(s, e) = sum of the counts before (s, e) in row-major order,
// and its row q goes to
//   D(s, e) + q,  D(s, e) = sum_{e' < e} sum_s' recv[s', e'] + sum_{s' < s} recv[s', e],
// which sorts the rows by (local expert, source rank, arrival). Local expert
// e owns rows [local_offsets[e], local_offsets[e+1]). One block per (s, e);
// each sums the G El <= MOE_MAX_EXPERTS counts it needs.
__global__ void __launch_bounds__(256) ep_regroup_kernel(const int32_t* __restrict__ recv, int G, int El,
                                                         int32_t* __restrict__ row_map,
                                                         int64_t* __restrict__ local_offsets) {
  const int blk = blockIdx.x;
  const int s = blk / El, e = blk % El;
  int64_t a = 0, dd = 0;
  for (int i = threadIdx.x; i < G * El; i += blockDim.x) {
    const int64_t c = recv[i];
    const int si = i / El, ei = i % El;
    if (i < blk) a += c;
    if (ei < e || (ei == e && si < s)) dd += c;
  }
  __shared__ int64_t s_a[8], s_d[8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    dd += __shfl_xor_sync(0xffffffffu, dd, off);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_a[warp] = a;
    s_d[warp] = dd;
  }
  __syncthreads();
  a = 0;
  dd = 0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    a += s_a[w];
    dd += s_d[w];
  }
  const int n = recv[blk];
  for (int q = threadIdx.x; q < n; q += blockDim.x) row_map[a + q] = static_cast<int32_t>(dd + q);
  if (threadIdx.x == 0) {
    if (s == 0) local_offsets[e] = dd;
    if (blk == G * El - 1) local_offsets[El] = a + n;
  }
}

cudaError_t launch_ep_regroup(const int32_t* recv, int G, int El, int32_t* row_map,
                              int64_t* local_offsets, cudaStream_t s) {
  ep_regroup_kernel<<<G * El, 256, 0, s>>>(recv, G, El, row_map, local_offsets);
  return cudaGetLastError();
}

}  // namespace moe
