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

constexpr int kRbTile = 64;
constexpr int kRbTok = 32;

// Block: 64 experts x 64 columns of dWr, 64 threads, 8x8 register tile per
// thread; tokens of the block's split in chunks of 32, staged with 16-byte
// loads one chunk ahead (register double buffer).
template <typename T>
__global__ void __launch_bounds__(64) router_wgrad_partial_kernel(
    const T* __restrict__ x, const float* __restrict__ dz, int64_t Ttok, int d, int E,
    int64_t tok_per_split, float* __restrict__ partial, float* __restrict__ partial_db) {
  constexpr int VE = Vec16<T>::N;
  constexpr int XV = kRbTok * kRbTile / VE / 64;  // x vectors per thread per chunk
  constexpr int ZV = kRbTok * kRbTile / 4 / 64;   // dz float4 per thread per chunk
  __shared__ __align__(16) float sz[kRbTok][kRbTile];
  __shared__ __align__(16) float sx[kRbTok][kRbTile];
  const int tid = threadIdx.x;
  const int te = tid / 8, tc = tid % 8;
  const int c0 = blockIdx.x * kRbTile;
  const int split = blockIdx.y;
  const int e0 = blockIdx.z * kRbTile;
  const int64_t tb = split * tok_per_split;
  const int64_t tend = min(Ttok, tb + tok_per_split);
  const bool e_vec_ok = (E % 4 == 0);

  Vec16<T> xr[XV];
  float4 zr[ZV];
  auto load_stage = [&](int64_t t0) {
#pragma unroll
    for (int j = 0; j < XV; ++j) {
      const int vid = tid + 64 * j;
      const int tt = vid / (kRbTile / VE), cv = vid % (kRbTile / VE);
      const int64_t t = t0 + tt;
      const int c = c0 + cv * VE;
      if (t < tend && c < d) xr[j] = ld16_stream(x + t * d + c);
      else xr[j].raw = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < ZV; ++j) {
      const int vid = tid + 64 * j;
      const int tt = vid / (kRbTile / 4), ev = vid % (kRbTile / 4);
      const int64_t t = t0 + tt;
      const int e = e0 + ev * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < tend) {
        const float* src = dz + t * E + e;
        if (e_vec_ok && e + 3 < E) {
          v = __ldcs(reinterpret_cast<const float4*>(src));
        } else {
          if (e < E) v.x = src[0];
          if (e + 1 < E) v.y = src[1];
          if (e + 2 < E) v.z = src[2];
          if (e + 3 < E) v.w = src[3];
        }
      }
      zr[j] = v;
    }
  };

  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.0f;
  float dbacc = 0.0f;
  if (tb < tend) load_stage(tb);
  for (int64_t t0 = tb; t0 < tend; t0 += kRbTok) {
#pragma unroll
    for (int j = 0; j < XV; ++j) {
      const int vid = tid + 64 * j;
      const int tt = vid / (kRbTile / VE), cv = vid % (kRbTile / VE);
#pragma unroll
      for (int q = 0; q < VE; q += 4)
        *reinterpret_cast<float4*>(&sx[tt][cv * VE + q]) =
            make_float4(xr[j].get(q), xr[j].get(q + 1), xr[j].get(q + 2), xr[j].get(q + 3));
    }
#pragma unroll
    for (int j = 0; j < ZV; ++j) {
      const int vid = tid + 64 * j;
      const int tt = vid / (kRbTile / 4), ev = vid % (kRbTile / 4);
      *reinterpret_cast<float4*>(&sz[tt][ev * 4]) = zr[j];
    }
    __syncthreads();
    if (t0 + kRbTok < tend) load_stage(t0 + kRbTok);
#pragma unroll 4
    for (int tt = 0; tt < kRbTok; ++tt) {
      const float4 za = *reinterpret_cast<const float4*>(&sz[tt][te * 8]);
      const float4 zb = *reinterpret_cast<const float4*>(&sz[tt][te * 8 + 4]);
      const float4 xa = *reinterpret_cast<const float4*>(&sx[tt][tc * 8]);
      const float4 xb = *reinterpret_cast<const float4*>(&sx[tt][tc * 8 + 4]);
      const float zv[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = __fmaf_rn(zv[a], xv[c], acc[a][c]);
    }
    if (blockIdx.x == 0)
      for (int tt = 0; tt < kRbTok; ++tt) dbacc += sz[tt][tid];
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int e = e0 + te * 8 + a;
    if (e >= E) continue;
    float* dst = partial + (static_cast<int64_t>(split) * E + e) * d + c0 + tc * 8;
    if (c0 + tc * 8 + 8 <= d) {
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c0 + tc * 8 + c < d) dst[c] = acc[a][c];
    }
  }
  if (blockIdx.x == 0 && e0 + tid < E) partial_db[static_cast<int64_t>(split) * E + e0 + tid] = dbacc;
}

__global__ void router_wgrad_reduce_kernel(const float* __restrict__ partial,
                                           const float* __restrict__ partial_db, int S, int E,
                                           int d, float* __restrict__ dWr, float* __restrict__ db) {
  const int64_t n = static_cast<int64_t>(E) * d;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int q = 0; q < S; ++q) s += partial[q * n + i];
    dWr[i] += s;
    if (db && i < E) {
      float sb = 0.0f;
      for (int q = 0; q < S; ++q) sb += partial_db[static_cast<int64_t>(q) * E + i];
      db[i] += sb;
    }
  }
}

int router_bwd_splits(int64_t T, int d, int E) {
  const int64_t tiles = static_cast<int64_t>((d + kRbTile - 1) / kRbTile) * ((E + kRbTile - 1) / kRbTile);
  int64_t S = (4 * 148 + tiles - 1) / tiles;
  const int64_t max_s = (T + kRbTok - 1) / kRbTok;
  if (S > max_s) S = max_s;
  if (S < 1) S = 1;
  if (S > 1024) S = 1024;
  return static_cast<int>(S);
}

cudaError_t launch_router_bwd(const void* x, const float* dz, int dtype, int64_t T, int d, int E,
                              float* dWr, float* db, float* partial, cudaStream_t s) {
  const int S = router_bwd_splits(T, d, E);
  int64_t tps = (T + S - 1) / S;
  tps = (tps + kRbTok - 1) / kRbTok * kRbTok;
  float* partial_db = partial + static_cast<int64_t>(S) * E * d;
  dim3 grid((d + kRbTile - 1) / kRbTile, S, (E + kRbTile - 1) / kRbTile);
  if (dtype == MOE_BF16)
    router_wgrad_partial_kernel<bf16><<<grid, 64, 0, s>>>(static_cast<const bf16*>(x), dz, T, d,
                                                           E, tps, partial, partial_db);
  else
    router_wgrad_partial_kernel<float><<<grid, 64, 0, s>>>(static_cast<const float*>(x), dz, T,
                                                            d, E, tps, partial, partial_db);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = static_cast<int64_t>(E) * d;
  const unsigned blocks = static_cast<unsigned>(((n + 255) / 256) < 148 * 8 ? (n + 255) / 256 : 148 * 8);
  router_wgrad_reduce_kernel<<<blocks, 256, 0, s>>>(partial, partial_db, S, E, d, dWr, db);
  return cudaGetLastError();
}

}  // namespace moe
