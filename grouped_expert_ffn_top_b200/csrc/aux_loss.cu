// Auxiliary load-balancing loss of the router, its gradient in the logits,
// and the dense router backward that carries that gradient to x, Wr and b.
// (MoE losses and metrics: leap-finetune PR #26 "Add MoE expert parallel
// training runtime", its MoE-loss tests; the loss is read as the Switch-style
// balance loss E * sum_e f_e P_e.)
//
//   p[t,e] = softmax over all E of z[t,:];  f_e = counts[e] / (T k)
//   P_e = (1/T) sum_t p[t,e];  L = alpha E sum_e f_e P_e
//   H = (1/T) sum_t -sum_e p[t,e] ln p[t,e]
//   dz[t,j] = dL alpha E / T * p[t,j] (f_j - sum_e f_e p[t,e])
// Every sum runs in a fixed order (per-block partials, then a fixed-order
// reduction), so results do not depend on timing.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kAuxThreads = 256;  // 8 warps, 32 tokens each
constexpr int kAuxTokensPerBlock = 256;

int aux_blocks(int64_t T) { return static_cast<int>((T + kAuxTokensPerBlock - 1) / kAuxTokensPerBlock); }

// Softmax of one token's logits held S per lane (lane + 32 s): returns p in
// place. Lanes past E hold p = 0.
template <int S>
__device__ __forceinline__ void warp_softmax(float (&v)[S], int lane, int E) {
  float m = -INFINITY;
#pragma unroll
  for (int s = 0; s < S; ++s)
    if (lane + 32 * s < E) m = fmaxf(m, v[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float sum = 0.0f;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    v[s] = lane + 32 * s < E ? expf(v[s] - m) : 0.0f;
    sum += v[s];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
  for (int s = 0; s < S; ++s) v[s] = v[s] / sum;
}

// Per block of 256 tokens: sum_t p[t,e] into partial[blk][e] and the
// entropy sum into partial[blk][E]. Warps take 32 tokens each in order; the
// warps' sums are added in warp order.
template <int S>
__global__ void __launch_bounds__(kAuxThreads) aux_partial_kernel(const float* __restrict__ z,
                                                                  int64_t T, int E,
                                                                  float* __restrict__ partial) {
  extern __shared__ float s_red[];  // [8][E + 1]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kAuxThreads / 32;
  constexpr int kTokPerWarp = kAuxTokensPerBlock / kWarps;
  float acc[S];
#pragma unroll
  for (int s = 0; s < S; ++s) acc[s] = 0.0f;
  float hacc = 0.0f;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kAuxTokensPerBlock + warp * kTokPerWarp;
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int64_t t = base + q;
    if (t >= T) break;
    float v[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const int e = lane + 32 * s;
      v[s] = e < E ? z[t * E + e] : 0.0f;
    }
    warp_softmax<S>(v, lane, E);
    float h = 0.0f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
      acc[s] += v[s];
      if (v[s] > 0.0f) h -= v[s] * logf(v[s]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) h += __shfl_xor_sync(0xffffffffu, h, off);
    hacc += h;
  }
  const int row = E + 1;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int e = lane + 32 * s;
    if (e < E) s_red[warp * row + e] = acc[s];
  }
  if (lane == 0) s_red[warp * row + E] = hacc;
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    float sum = 0.0f;
    for (int w = 0; w < kWarps; ++w) sum += s_red[w * row + e];
    partial[static_cast<int64_t>(blockIdx.x) * row + e] = sum;
  }
}

// One block: importance, loss and entropy from the per-block partials.
__global__ void __launch_bounds__(1024) aux_final_kernel(const float* __restrict__ partial, int nb,
                                                         const int32_t* __restrict__ counts,
                                                         int64_t T, int E, int k, float alpha,
                                                         float* __restrict__ importance,
                                                         float* __restrict__ loss,
                                                         float* __restrict__ entropy) {
  __shared__ float s_term[1024];
  const int row = E + 1;
  const float invT = 1.0f / static_cast<float>(T);
  const float invTk = 1.0f / (static_cast<float>(T) * static_cast<float>(k));
  for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
    float term = 0.0f;
    if (e < E) {
      float s = 0.0f;
      for (int b = 0; b < nb; ++b) s += partial[static_cast<int64_t>(b) * row + e];
      const float imp = s * invT;
      importance[e] = imp;
      term = static_cast<float>(counts[e]) * invTk * imp;
    }
    s_term[e] = term;
  }
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {  // fixed-order tree over the 1024 slots
    for (int e = threadIdx.x; e < w; e += blockDim.x) s_term[e] += s_term[e + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = alpha * static_cast<float>(E) * s_term[0];
  if (entropy && threadIdx.x < 32) {
    float h = 0.0f;
    for (int b = threadIdx.x; b < nb; b += 32) h += partial[static_cast<int64_t>(b) * row + E];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) h += __shfl_xor_sync(0xffffffffu, h, off);
    if (threadIdx.x == 0) *entropy = h * invT;
  }
}

// dz[t,j] = c p[t,j] (f_j - sum_e f_e p[t,e]), one warp per token.
template <int S>
__global__ void __launch_bounds__(kAuxThreads) aux_bwd_kernel(const float* __restrict__ z,
                                                              const int32_t* __restrict__ counts,
                                                              int64_t T, int E, int k, float c,
                                                              float* __restrict__ dz) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float invTk = 1.0f / (static_cast<float>(T) * static_cast<float>(k));
  float f[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int e = lane + 32 * s;
    f[s] = e < E ? static_cast<float>(counts[e]) * invTk : 0.0f;
  }
  for (int64_t t = gw; t < T; t += nw) {
    float v[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const int e = lane + 32 * s;
      v[s] = e < E ? z[t * E + e] : 0.0f;
    }
    warp_softmax<S>(v, lane, E);
    float sf = 0.0f;
#pragma unroll
    for (int s = 0; s < S; ++s) sf += f[s] * v[s];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sf += __shfl_xor_sync(0xffffffffu, sf, off);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const int e = lane + 32 * s;
      if (e < E) dz[t * E + e] = c * v[s] * (f[s] - sf);
    }
  }
}

template <int S>
static cudaError_t launch_aux_s(const float* z, const int32_t* counts, int64_t T, int E, int k,
                                float alpha, float* importance, float* loss, float* entropy,
                                float* partial, cudaStream_t s) {
  const int nb = aux_blocks(T);
  aux_partial_kernel<S><<<nb, kAuxThreads, sizeof(float) * 8 * (E + 1), s>>>(z, T, E, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  aux_final_kernel<<<1, 1024, 0, s>>>(partial, nb, counts, T, E, k, alpha, importance, loss,
                                      entropy);
  return cudaGetLastError();
}

cudaError_t launch_aux_loss(const float* z, const int32_t* counts, int64_t T, int E, int k,
                            float alpha, float* importance, float* loss, float* entropy,
                            float* partial, cudaStream_t s) {
  const int S = (E + 31) / 32;
  if (S <= 1) return launch_aux_s<1>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
  if (S <= 2) return launch_aux_s<2>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
  if (S <= 4) return launch_aux_s<4>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
  if (S <= 8) return launch_aux_s<8>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
  if (S <= 16) return launch_aux_s<16>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
  return launch_aux_s<32>(z, counts, T, E, k, alpha, importance, loss, entropy, partial, s);
}

cudaError_t launch_aux_loss_bwd(const float* z, const int32_t* counts, int64_t T, int E, int k,
                                float alpha, float dloss, float* dz, cudaStream_t s) {
  const float c = dloss * alpha * static_cast<float>(E) / static_cast<float>(T);
  const int64_t warps = T < 148 * 64 ? T : 148 * 64;
  const unsigned blocks = static_cast<unsigned>((warps * 32 + kAuxThreads - 1) / kAuxThreads);
  const int S = (E + 31) / 32;
#define MOE_AUX_BWD(SV) aux_bwd_kernel<SV><<<blocks, kAuxThreads, 0, s>>>(z, counts, T, E, k, c, dz)
  if (S <= 1) MOE_AUX_BWD(1);
  else if (S <= 2) MOE_AUX_BWD(2);
  else if (S <= 4) MOE_AUX_BWD(4);
  else if (S <= 8) MOE_AUX_BWD(8);
  else if (S <= 16) MOE_AUX_BWD(16);
  else MOE_AUX_BWD(32);
#undef MOE_AUX_BWD
  return cudaGetLastError();
}

// ----------------------------------------------------- dense router backward
//
// The balance loss's logit gradient dz is dense over the experts, so its
// router backward is two small dense products, dX += dz Wr ([T, E] x [E, d])
// and dWr (+)= dz^T x ([E, T] x [T, d]) with db (+)= the column sums of dz,
// on fp32 FFMA register tiles fed from operands staged as fp32 in shared
// memory. Each output is summed in a fixed order (e ascending for dX; tokens
// ascending inside 256-token chunks, then the chunks in order, for dWr), so
// the result does not depend on scheduling. Experts are staged EC at a time
// (16 when E <= 16, else 32), so no FMA runs on padding experts beyond the
// last chunk's. A thread's 8 columns are two groups of 4, c0 + 4 tx and
// c0 + 64 + 4 tx, so each quarter-warp's 16-byte shared loads cover 128
// contiguous bytes.

constexpr int kDenseTokens = 64;   // tokens per dX block and per dWr staging step
constexpr int kDenseCols = 128;    // columns per block
constexpr int kDenseChunk = 256;   // tokens per dWr partial

int dense_router_chunks(int64_t T) {
  return static_cast<int>((T + kDenseChunk - 1) / kDenseChunk);
}

// Elements i .. i + 3 of a row as floats, zero at or past n. VEC: one 8-byte
// (bf16) or 16-byte (fp32) load; the row start and i are multiples of 4
// elements and the base is aligned to 4 elements (checked at launch).
template <typename T, bool VEC>
__device__ __forceinline__ float4 load4(const T* row, int i, int n) {
  if (VEC && i + 4 <= n) {
    if constexpr (sizeof(T) == 2) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(row + i));
      const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      return make_float4(lo.x, lo.y, hi.x, hi.y);
    } else {
      return __ldg(reinterpret_cast<const float4*>(row + i));
    }
  }
  float v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) v[q] = i + q < n ? to_f32(row[i + q]) : 0.0f;
  return make_float4(v[0], v[1], v[2], v[3]);
}

// row[i + q] = row[i + q] + a[q] (one rounding to T) for q < 4, i + q < n.
template <typename T, bool VEC>
__device__ __forceinline__ void add4(T* row, int i, int n, const float (&a)[4]) {
  if (VEC && i + 4 <= n) {
    if constexpr (sizeof(T) == 2) {
      uint2* p = reinterpret_cast<uint2*>(row + i);
      uint2 u = *p;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
      const float2 lo = __bfloat1622float2(h[0]), hi = __bfloat1622float2(h[1]);
      h[0] = __floats2bfloat162_rn(lo.x + a[0], lo.y + a[1]);
      h[1] = __floats2bfloat162_rn(hi.x + a[2], hi.y + a[3]);
      *p = u;
    } else {
      float4* p = reinterpret_cast<float4*>(row + i);
      float4 u = *p;
      u.x += a[0]; u.y += a[1]; u.z += a[2]; u.w += a[3];
      *p = u;
    }
    return;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (i + q < n) row[i + q] = from_f32<T>(to_f32(row[i + q]) + a[q]);
}

// dX[t, i] += sum_e dz[t,e] Wr[e,i]. Block: 64 tokens x 128 columns, 128
// threads, each 8 tokens x 8 columns.
template <typename T, int EC, bool VEC>
__global__ void __launch_bounds__(128) dense_dx_kernel(const float* __restrict__ dz,
                                                       const T* __restrict__ Wr, int64_t Ttok,
                                                       int d, int E, T* __restrict__ dX) {
  __shared__ __align__(16) float s_dz[EC][kDenseTokens + 4];  // [e][token]
  __shared__ __align__(16) float s_w[EC][kDenseCols + 4];     // [e][column]
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // columns 4 tx, 64 + 4 tx; tokens 8 ty ..
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kDenseTokens;
  const int i0 = blockIdx.y * kDenseCols;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.0f;
  for (int e0 = 0; e0 < E; e0 += EC) {
    for (int idx = tid; idx < kDenseTokens * EC; idx += 128) {
      const int tt = idx / EC, ee = idx % EC;  // consecutive threads: consecutive e
      const int64_t t = t0 + tt;
      const int e = e0 + ee;
      s_dz[ee][tt] = (t < Ttok && e < E) ? dz[t * E + e] : 0.0f;
    }
    for (int idx = tid; idx < EC * (kDenseCols / 4); idx += 128) {
      const int ee = idx / (kDenseCols / 4), c4 = 4 * (idx % (kDenseCols / 4));
      const int e = e0 + ee;
      *reinterpret_cast<float4*>(&s_w[ee][c4]) =
          e < E ? load4<T, VEC>(Wr + static_cast<int64_t>(e) * d, i0 + c4, d) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const int ee_end = min(EC, E - e0);
    for (int ee = 0; ee < ee_end; ++ee) {
      const float4 za = *reinterpret_cast<const float4*>(&s_dz[ee][ty * 8]);
      const float4 zb = *reinterpret_cast<const float4*>(&s_dz[ee][ty * 8 + 4]);
      const float4 wa = *reinterpret_cast<const float4*>(&s_w[ee][tx * 4]);
      const float4 wb = *reinterpret_cast<const float4*>(&s_w[ee][64 + tx * 4]);
      const float zv[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
      const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = __fmaf_rn(zv[a], wv[c], acc[a][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t t = t0 + ty * 8 + a;
    if (t >= Ttok) continue;
    T* row = dX + t * d;
    const float lo[4] = {acc[a][0], acc[a][1], acc[a][2], acc[a][3]};
    const float hi[4] = {acc[a][4], acc[a][5], acc[a][6], acc[a][7]};
    add4<T, VEC>(row, i0 + tx * 4, d, lo);
    add4<T, VEC>(row, i0 + 64 + tx * 4, d, hi);
  }
}

// partial[chunk][e][i] = sum_{t in chunk} dz[t,e] x[t,i] and, for the first
// column tile, partial_db[chunk][e] = sum_{t in chunk} dz[t,e]. Block: one
// 256-token chunk x EC experts x 128 columns, 128 threads, each EC / 8
// experts x 8 columns; tokens in steps of 64, summed in token order.
template <typename T, int EC, bool VEC>
__global__ void __launch_bounds__(128) dense_dwr_partial_kernel(const T* __restrict__ x,
                                                                const float* __restrict__ dz,
                                                                int64_t Ttok, int d, int E,
                                                                float* __restrict__ partial,
                                                                float* __restrict__ partial_db) {
  constexpr int RE = EC / 8;
  __shared__ __align__(16) float s_dz[kDenseTokens][EC + 4];       // [token][e]
  __shared__ __align__(16) float s_x[kDenseTokens][kDenseCols + 4];  // [token][column]
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // columns 4 tx, 64 + 4 tx; experts RE ty ..
  const int chunk = blockIdx.x;
  const int i0 = blockIdx.y * kDenseCols;
  const int e0 = blockIdx.z * EC;
  float acc[RE][8];
  float accb[RE];
#pragma unroll
  for (int a = 0; a < RE; ++a) {
    accb[a] = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.0f;
  }
  const int64_t tbeg = static_cast<int64_t>(chunk) * kDenseChunk;
  const int64_t tend = min(tbeg + kDenseChunk, Ttok);
  for (int64_t ts = tbeg; ts < tend; ts += kDenseTokens) {
    for (int idx = tid; idx < kDenseTokens * EC; idx += 128) {
      const int tt = idx / EC, ee = idx % EC;
      const int64_t t = ts + tt;
      const int e = e0 + ee;
      s_dz[tt][ee] = (t < tend && e < E) ? dz[t * E + e] : 0.0f;
    }
    for (int idx = tid; idx < kDenseTokens * (kDenseCols / 4); idx += 128) {
      const int tt = idx / (kDenseCols / 4), c4 = 4 * (idx % (kDenseCols / 4));
      const int64_t t = ts + tt;
      *reinterpret_cast<float4*>(&s_x[tt][c4]) =
          t < tend ? load4<T, VEC>(x + t * d, i0 + c4, d) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    for (int tt = 0; tt < kDenseTokens; ++tt) {
      float zv[RE];
      if constexpr (RE == 4) {
        const float4 z4 = *reinterpret_cast<const float4*>(&s_dz[tt][ty * 4]);
        zv[0] = z4.x; zv[1] = z4.y; zv[2] = z4.z; zv[3] = z4.w;
      } else {
#pragma unroll
        for (int a = 0; a < RE; ++a) zv[a] = s_dz[tt][ty * RE + a];
      }
      const float4 xa = *reinterpret_cast<const float4*>(&s_x[tt][tx * 4]);
      const float4 xb = *reinterpret_cast<const float4*>(&s_x[tt][64 + tx * 4]);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int a = 0; a < RE; ++a) {
        accb[a] += zv[a];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = __fmaf_rn(zv[a], xv[c], acc[a][c]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < RE; ++a) {
    const int e = e0 + ty * RE + a;
    if (e >= E) continue;
    float* prow = partial + (static_cast<int64_t>(chunk) * E + e) * d;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = i0 + 64 * h + tx * 4;
      if (i + 4 <= d) {
        *reinterpret_cast<float4*>(prow + i) =
            make_float4(acc[a][4 * h], acc[a][4 * h + 1], acc[a][4 * h + 2], acc[a][4 * h + 3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (i + q < d) prow[i + q] = acc[a][4 * h + q];
      }
    }
    if (blockIdx.y == 0 && tx == 0) partial_db[static_cast<int64_t>(chunk) * E + e] = accb[a];
  }
}

// dWr[e,i] (+)= sum over chunks in order; db likewise.
__global__ void __launch_bounds__(256) dense_dwr_reduce_kernel(const float* __restrict__ partial,
                                                               const float* __restrict__ partial_db,
                                                               int nchunk, int d, int E,
                                                               float* __restrict__ dWr,
                                                               float* __restrict__ db,
                                                               int accumulate) {
  const int64_t n = static_cast<int64_t>(E) * d;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; id < n + E;
       id += stride) {
    if (id < n) {
      float s = 0.0f;
      for (int c = 0; c < nchunk; ++c) s += partial[static_cast<int64_t>(c) * n + id];
      dWr[id] = accumulate ? dWr[id] + s : s;
    } else if (db) {
      const int e = static_cast<int>(id - n);
      float s = 0.0f;
      for (int c = 0; c < nchunk; ++c) s += partial_db[static_cast<int64_t>(c) * E + e];
      db[e] = accumulate ? db[e] + s : s;
    }
  }
}

template <typename T, int EC, bool VEC>
static cudaError_t launch_dense_e(const T* x, const T* Wr, const float* dz, int64_t Ttok, int d,
                                  int E, T* dX, float* partial, float* partial_db, cudaStream_t s) {
  const unsigned gy = static_cast<unsigned>((d + kDenseCols - 1) / kDenseCols);
  if (dX) {
    dense_dx_kernel<T, EC, VEC><<<dim3(static_cast<unsigned>((Ttok + kDenseTokens - 1) / kDenseTokens), gy),
                                  128, 0, s>>>(dz, Wr, Ttok, d, E, dX);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dense_dwr_partial_kernel<T, EC, VEC><<<dim3(static_cast<unsigned>(dense_router_chunks(Ttok)), gy,
                                              static_cast<unsigned>((E + EC - 1) / EC)),
                                         128, 0, s>>>(x, dz, Ttok, d, E, partial, partial_db);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_dense_t(const T* x, const T* Wr, const float* dz, int64_t Ttok, int d,
                                  int E, T* dX, float* dWr, float* db, int accumulate,
                                  float* partial, cudaStream_t s) {
  const int nchunk = dense_router_chunks(Ttok);
  float* partial_db = partial + static_cast<int64_t>(nchunk) * E * d;
  // vector accesses of 4 elements need every row start aligned to them (d is
  // a multiple of 4) and so the base pointers
  const uintptr_t al = 4 * sizeof(T) - 1;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(Wr) |
                     reinterpret_cast<uintptr_t>(dX)) & al) == 0;
  cudaError_t e;
  if (E <= 16)
    e = vec ? launch_dense_e<T, 16, true>(x, Wr, dz, Ttok, d, E, dX, partial, partial_db, s)
            : launch_dense_e<T, 16, false>(x, Wr, dz, Ttok, d, E, dX, partial, partial_db, s);
  else
    e = vec ? launch_dense_e<T, 32, true>(x, Wr, dz, Ttok, d, E, dX, partial, partial_db, s)
            : launch_dense_e<T, 32, false>(x, Wr, dz, Ttok, d, E, dX, partial, partial_db, s);
  if (e != cudaSuccess) return e;
  const int64_t n = static_cast<int64_t>(E) * d + E;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256 < 148 * 8 ? (n + 255) / 256 : 148 * 8);
  dense_dwr_reduce_kernel<<<blocks, 256, 0, s>>>(partial, partial_db, nchunk, d, E, dWr, db,
                                                 accumulate);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd_dense(const void* x, const void* Wr, const float* dz, int dtype,
                                    int64_t T, int d, int E, void* dX, float* dWr, float* db,
                                    int accumulate, float* partial, cudaStream_t s) {
  if (dtype == MOE_BF16)
    return launch_dense_t(static_cast<const bf16*>(x), static_cast<const bf16*>(Wr), dz, T, d, E,
                          static_cast<bf16*>(dX), dWr, db, accumulate, partial, s);
  return launch_dense_t(static_cast<const float*>(x), static_cast<const float*>(Wr), dz, T, d, E,
                        static_cast<float*>(dX), dWr, db, accumulate, partial, s);
}

}  // namespace moe
