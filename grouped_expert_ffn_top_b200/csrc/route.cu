// Routing kernels: router logits, top-k softmax, the per-expert histogram /
// scan / stable scatter that builds the dispatch layout, and the route
// backward. (Expert routing and EP token dispatch: ART issue #917 intro and
// Desired behavior; leap-finetune PR #26 Summary.)
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ------------------------------------------------------------ router logits
//
// z[t,e] = fma-chain over i = 0..d-1 of x[t,i] * Wr[e,i], then + b[e], in fp32.
// Block tile: 64 tokens x TE experts, NT threads in 8 token groups of 8
// tokens and NT / 8 expert groups; thread tile: 8 tokens x TE / (NT / 8)
// experts. Operands are staged as fp32 in shared memory, i-major, in chunks
// of 64 i, loaded with 16-byte vector loads one chunk ahead (register double
// buffer) and written transposed; each 32-float half of a staged row is
// followed by 16 bytes of padding, so that the 16-byte operand loads of the
// token and expert groups fall in distinct banks. Within a chunk the next
// step's operands load into a second register set while the current step's
// FMAs issue. The i loop is
// sequential for every output, which is what makes the result bit-identical
// to the fixed-order definition.

constexpr int kLogitTokens = 64;
constexpr int kLogitChunk = 64;

// padded column of element c of a staged row: 4 floats after every 32
__device__ __forceinline__ int logit_pad(int c) { return c + ((c >> 5) << 2); }

template <typename T, int TE, int NT>
__global__ void __launch_bounds__(NT) router_logits_kernel(const T* __restrict__ x,
                                                           const T* __restrict__ Wr,
                                                           const float* __restrict__ b,
                                                           int64_t Ttok, int d, int E,
                                                           float* __restrict__ z) {
  constexpr int VE = Vec16<T>::N;                  // elements per 16-byte vector
  constexpr int VPR = kLogitChunk / VE;            // vectors per row chunk
  constexpr int XPT = kLogitTokens * VPR / NT;     // x vectors per thread
  constexpr int WPT = TE * VPR / NT;               // Wr vectors per thread
  constexpr int EG = NT / 8;                       // expert groups
  constexpr int RE = TE / EG;                      // experts per thread
  constexpr int XROW = kLogitTokens + kLogitTokens / 32 * 4;
  constexpr int WROW = TE + (TE + 31) / 32 * 4;
  static_assert(XPT >= 1 && kLogitTokens * VPR % NT == 0, "x staging");
  static_assert(WPT >= 1 && TE * VPR % NT == 0, "Wr staging");
  static_assert(RE >= 1 && TE % EG == 0, "thread tile");
  __shared__ __align__(16) float xs[kLogitChunk][XROW];
  __shared__ __align__(16) float ws[kLogitChunk][WROW];
  const int tid = threadIdx.x;
  const int tx = tid % EG;  // expert group
  const int ty = tid / EG;  // token group
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kLogitTokens;
  const int e0 = blockIdx.y * TE;
  // x staging: thread tid loads token tid % 64, vectors (tid / 64) * XPT ..
  const int xt = tid % kLogitTokens;
  const int xv0 = (tid / kLogitTokens) * XPT;
  const int64_t my_t = t0 + xt;

  Vec16<T> xr[XPT], wr[WPT];
  auto load_stage = [&](int i0) {
#pragma unroll
    for (int v = 0; v < XPT; ++v) {
      const int i = i0 + (xv0 + v) * VE;
      if (my_t < Ttok && i < d) xr[v] = ld16_stream(x + my_t * d + i);
      else xr[v].raw = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < WPT; ++j) {
      const int vid = tid + NT * j;
      const int ee = vid % TE, v = vid / TE;
      const int e = e0 + ee, i = i0 + v * VE;
      if (e < E && i < d) wr[j] = ld16(Wr + static_cast<int64_t>(e) * d + i);
      else wr[j].raw = make_uint4(0u, 0u, 0u, 0u);
    }
  };

  float acc[8][RE];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < RE; ++c) acc[a][c] = 0.0f;

  load_stage(0);
  for (int i0 = 0; i0 < d; i0 += kLogitChunk) {
#pragma unroll
    for (int v = 0; v < XPT; ++v)
#pragma unroll
      for (int q = 0; q < VE; ++q) xs[(xv0 + v) * VE + q][logit_pad(xt)] = xr[v].get(q);
#pragma unroll
    for (int j = 0; j < WPT; ++j) {
      const int vid = tid + NT * j;
      const int ee = vid % TE, v = vid / TE;
#pragma unroll
      for (int q = 0; q < VE; ++q) ws[v * VE + q][logit_pad(ee)] = wr[j].get(q);
    }
    __syncthreads();
    if (i0 + kLogitChunk < d) load_stage(i0 + kLogitChunk);
    const int iend = min(kLogitChunk, d - i0);
    // two register sets alternate: step ii + 1 loads into one while step
    // ii's FMAs read the other
    float xa[8], wa[RE], xb[8], wb[RE];
    auto load_step = [&](int ii, float (&xv)[8], float (&wv)[RE]) {
      const float4 x0 = *reinterpret_cast<const float4*>(&xs[ii][logit_pad(ty * 8)]);
      const float4 x1 = *reinterpret_cast<const float4*>(&xs[ii][logit_pad(ty * 8) + 4]);
      xv[0] = x0.x; xv[1] = x0.y; xv[2] = x0.z; xv[3] = x0.w;
      xv[4] = x1.x; xv[5] = x1.y; xv[6] = x1.z; xv[7] = x1.w;
      if constexpr (RE % 4 == 0) {
#pragma unroll
        for (int c = 0; c < RE; c += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(&ws[ii][logit_pad(tx * RE + c)]);
          wv[c] = w4.x; wv[c + 1] = w4.y; wv[c + 2] = w4.z; wv[c + 3] = w4.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < RE; ++c) wv[c] = ws[ii][logit_pad(tx * RE + c)];
      }
    };
    // with two experts per thread (the tiles for E <= 16 and E <= 32), both
    // chains of a token in one packed instruction (__ffma2_rn rounds each
    // component as __fmaf_rn does, so the chains are the same): 14-18%
    // faster at d = 4096, E = 16; with 8 per thread the packed form measured
    // 5-20% slower
    auto fma_step = [&](const float (&xv)[8], const float (&wv)[RE]) {
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        if constexpr (RE == 2) {
          const float2 xx = make_float2(xv[a], xv[a]);
#pragma unroll
          for (int c = 0; c < RE; c += 2) {
            const float2 r = __ffma2_rn(xx, make_float2(wv[c], wv[c + 1]),
                                        make_float2(acc[a][c], acc[a][c + 1]));
            acc[a][c] = r.x;
            acc[a][c + 1] = r.y;
          }
        } else {
#pragma unroll
          for (int c = 0; c < RE; ++c) acc[a][c] = __fmaf_rn(xv[a], wv[c], acc[a][c]);
        }
      }
    };
    load_step(0, xa, wa);
    int ii = 0;
    for (; ii + 1 < iend; ii += 2) {
      load_step(ii + 1, xb, wb);
      fma_step(xa, wa);
      if (ii + 2 < iend) load_step(ii + 2, xa, wa);
      fma_step(xb, wb);
    }
    if (ii < iend) fma_step(xa, wa);  // odd chunk length (fp32 rows)
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t t = t0 + ty * 8 + a;
    if (t >= Ttok) continue;
#pragma unroll
    for (int c = 0; c < RE; ++c) {
      const int e = e0 + tx * RE + c;
      if (e < E) z[t * E + e] = __fadd_rn(acc[a][c], b ? b[e] : 0.0f);
    }
  }
}

// Small batches (T E <= kLogitSmallOutputs): one warp per logit. The chain
// of d dependent FMAs is the logit's time, so one lane runs it over the
// token's x row and the expert's Wr row staged as fp32 in the warp's shared
// memory, kSmallCols columns at a time; before each chunk's chain the warp
// issues the 16-byte loads of the next chunk into registers, which land while
// the chain runs, and stores them after it. Same order of operations as the
// tiled kernel above, same result bits.
constexpr int64_t kLogitSmallOutputs = 4096;
constexpr int kSmallCols = 512;
constexpr int kSmallWarps = 4;

template <typename T>
__global__ void __launch_bounds__(32 * kSmallWarps) router_logits_small_kernel(
    const T* __restrict__ x, const T* __restrict__ Wr, const float* __restrict__ b, int64_t Ttok,
    int d, int E, float* __restrict__ z) {
  constexpr int VE = Vec16<T>::N;           // elements per 16-byte vector
  constexpr int VPL = kSmallCols / VE / 32;  // vectors per lane per row and chunk
  __shared__ __align__(16) float st[kSmallWarps][2][kSmallCols];  // [warp][x, Wr][column]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t o = static_cast<int64_t>(blockIdx.x) * kSmallWarps + warp;
  if (o >= Ttok * E) return;  // whole warps only: no block-wide barrier below
  const int64_t t = o / E;
  const int e = static_cast<int>(o % E);
  const T* xr = x + t * d;
  const T* wr = Wr + static_cast<int64_t>(e) * d;
  Vec16<T> px[VPL], pw[VPL];
  auto gload = [&](int i0) {
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int c = i0 + (lane + 32 * j) * VE;
      if (c < d) {
        px[j] = ld16(xr + c);
        pw[j] = ld16(wr + c);
      } else {
        px[j].raw = pw[j].raw = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  auto sstore = [&]() {
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int c = (lane + 32 * j) * VE;
#pragma unroll
      for (int q = 0; q < VE; ++q) {
        st[warp][0][c + q] = px[j].get(q);
        st[warp][1][c + q] = pw[j].get(q);
      }
    }
  };
  float acc = 0.0f;
  gload(0);
  for (int i0 = 0; i0 < d; i0 += kSmallCols) {
    sstore();
    __syncwarp();
    if (i0 + kSmallCols < d) gload(i0 + kSmallCols);
    if (lane == 0) {
      const float* xs = st[warp][0];
      const float* ws = st[warp][1];
      const int n = min(kSmallCols, d - i0);  // a multiple of 8 (d is)
#pragma unroll 4
      for (int i = 0; i < n; i += 4) {
        const float4 xv = *reinterpret_cast<const float4*>(xs + i);
        const float4 wv = *reinterpret_cast<const float4*>(ws + i);
        acc = __fmaf_rn(xv.x, wv.x, acc);
        acc = __fmaf_rn(xv.y, wv.y, acc);
        acc = __fmaf_rn(xv.z, wv.z, acc);
        acc = __fmaf_rn(xv.w, wv.w, acc);
      }
    }
    __syncwarp();
  }
  if (lane == 0) z[o] = __fadd_rn(acc, b ? b[e] : 0.0f);
}

template <typename T>
static cudaError_t launch_router_logits_t(const T* x, const T* Wr, const float* b, int64_t Ttok,
                                          int d, int E, float* z, cudaStream_t s) {
  const unsigned gx = static_cast<unsigned>((Ttok + kLogitTokens - 1) / kLogitTokens);
  if (Ttok * E <= kLogitSmallOutputs) {
    const unsigned blocks = static_cast<unsigned>((Ttok * E + kSmallWarps - 1) / kSmallWarps);
    router_logits_small_kernel<T><<<blocks, 32 * kSmallWarps, 0, s>>>(x, Wr, b, Ttok, d, E, z);
  } else if (E <= 8) {
    router_logits_kernel<T, 8, 64><<<dim3(gx, 1), 64, 0, s>>>(x, Wr, b, Ttok, d, E, z);
  } else if (E <= 16) {
    // 8 tokens x 2 experts per thread: twice the FMAs per shared-memory load
    // of the 8 x 1 tile with 128 threads
    router_logits_kernel<T, 16, 64><<<dim3(gx, 1), 64, 0, s>>>(x, Wr, b, Ttok, d, E, z);
  } else if (E <= 32) {
    router_logits_kernel<T, 32, 128><<<dim3(gx, 1), 128, 0, s>>>(x, Wr, b, Ttok, d, E, z);
  } else {
    router_logits_kernel<T, 64, 64><<<dim3(gx, (E + 63) / 64), 64, 0, s>>>(x, Wr, b, Ttok, d,
                                                                           E, z);
  }
  return cudaGetLastError();
}

cudaError_t launch_router_logits(const void* x, const void* Wr, const float* b, int dtype,
                                 int64_t T, int d, int E, float* z, cudaStream_t s) {
  if (dtype == MOE_BF16)
    return launch_router_logits_t(static_cast<const bf16*>(x), static_cast<const bf16*>(Wr), b, T,
                                  d, E, z, s);
  return launch_router_logits_t(static_cast<const float*>(x), static_cast<const float*>(Wr), b, T,
                                d, E, z, s);
}

// ------------------------------------------------------------------- top-k
//
// One warp per token. Lane l holds the logits of experts l, l+32, ...; k
// rounds of a warp arg-max pick the experts in ranking order (larger logit
// first, NaN after every number, lower index on equal keys). The block's 256
// tokens are also counted per expert (shared-memory histogram) for the scan.

struct Cand {
  float v;
  int idx;  // INT_MAX when the slot is empty or already taken
};

__device__ __forceinline__ bool ranks_before(const Cand& a, const Cand& b) {
  const bool ea = a.idx == INT_MAX, eb = b.idx == INT_MAX;
  if (ea != eb) return eb;
  const bool na = isnan(a.v), nb = isnan(b.v);
  if (na != nb) return nb;
  if (!na && a.v != b.v) return a.v > b.v;
  return a.idx < b.idx;
}

template <int S, int NT>  // S = ceil(E / 32) logits per lane, NT threads per block
__global__ void __launch_bounds__(NT) topk_softmax_kernel(
    const float* __restrict__ z, int64_t Ttok, int E, int k, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, int32_t* __restrict__ block_counts, unsigned* err) {
  extern __shared__ int s_hist[];  // [E]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();

  const int64_t tok_base = static_cast<int64_t>(blockIdx.x) * kRouteTokensPerBlock;
  constexpr int kTokPerWarp = kRouteTokensPerBlock / (NT / 32);
  // the next token's logits load while this one is ranked
  float vn[S];
  auto load_token = [&](int64_t t) {
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const int e = lane + 32 * s;
      vn[s] = (t < Ttok && e < E) ? z[t * E + e] : 0.0f;
    }
  };
  load_token(tok_base + warp * kTokPerWarp);
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int64_t t = tok_base + warp * kTokPerWarp + q;
    if (t >= Ttok) break;
    float v[S];
    bool taken[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      v[s] = vn[s];
      taken[s] = lane + 32 * s >= E;
    }
    if (q + 1 < kTokPerWarp) load_token(t + 1);
    float my_val = 0.0f;  // lane j keeps the j-th selected logit
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
      Cand best{0.0f, INT_MAX};
#pragma unroll
      for (int s = 0; s < S; ++s) {
        Cand c{v[s], taken[s] ? INT_MAX : lane + 32 * s};
        if (ranks_before(c, best)) best = c;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        Cand o;
        o.v = __shfl_xor_sync(0xffffffffu, best.v, off);
        o.idx = __shfl_xor_sync(0xffffffffu, best.idx, off);
        if (ranks_before(o, best)) best = o;
      }
      // every lane now holds the same winner; its owner marks it taken
      if ((best.idx & 31) == lane) {
#pragma unroll
        for (int s = 0; s < S; ++s)
          if (lane + 32 * s == best.idx) taken[s] = true;
      }
      if (lane == j) {
        my_val = best.v;
        my_idx = best.idx;
      }
    }
    // softmax over the k selected logits (fp32), exp(z_j - m) / sum with m
    // the largest selected logit; a selected -inf next to a finite m gets
    // exactly 0. It is undefined only when m is not finite (+inf - +inf, or
    // every selected logit -inf) or a selected logit is NaN (NaN ranks last,
    // so the k-th is then NaN): those tokens get 1/k and raise the flag.
    const bool active = lane < k;
    const float m = __shfl_sync(0xffffffffu, my_val, 0);
    const float last = __shfl_sync(0xffffffffu, my_val, k - 1);
    const bool defined = isfinite(m) && !isnan(last);
    float ex = (active && defined) ? expf(my_val - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (active) {
      const float w = defined ? ex / sum : 1.0f / static_cast<float>(k);
      topk_idx[t * k + lane] = my_idx;
      topk_w[t * k + lane] = w;
      atomicAdd(&s_hist[my_idx], 1);
    }
    if (!defined && lane == 0) raise_error(err, kErrNonfiniteLogit);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_counts[static_cast<int64_t>(blockIdx.x) * E + e] = s_hist[e];
}

// --------------------------------------------------------------------- scan
//
// One block. totals[e] = sum over blocks; offsets = exclusive scan of totals;
// block_base[b][e] = offsets[e] + sum_{b' < b} block_counts[b'][e]; group
// counts and offsets from contiguous expert blocks.

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

__global__ void __launch_bounds__(1024) route_scan_kernel(
    const int32_t* __restrict__ block_counts, int nb, int E, int G,
    int32_t* __restrict__ block_base, int32_t* __restrict__ counts, int64_t* __restrict__ offsets,
    int32_t* __restrict__ group_counts, int64_t* __restrict__ group_offsets) {
  __shared__ int s_tot[MOE_MAX_EXPERTS];
  __shared__ int s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int s_warp[32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  // per-expert totals
  for (int e = warp; e < E; e += nwarps) {
    int s = 0;
    for (int b = lane; b < nb; b += 32) s += block_counts[static_cast<int64_t>(b) * E + e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) s_tot[e] = s;
  }
  __syncthreads();
  // exclusive scan of the totals over experts (E <= 1024 = blockDim)
  {
    const int e = threadIdx.x;
    const int v = e < E ? s_tot[e] : 0;
    const int inc = warp_incl_scan(v);
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      int wv = lane < nwarps ? s_warp[lane] : 0;
      int winc = warp_incl_scan(wv);
      s_warp[lane] = winc - wv;
    }
    __syncthreads();
    const int excl = inc - v + s_warp[warp];
    if (e < E) {
      s_off[e] = excl;
      counts[e] = v;
      offsets[e] = excl;
    }
    if (e == E - 1) {
      s_off[E] = excl + v;
      offsets[E] = excl + v;
    }
  }
  __syncthreads();
  // absolute per-block bases
  for (int e = warp; e < E; e += nwarps) {
    int carry = s_off[e];
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int b = b0 + lane;
      const int v = b < nb ? block_counts[static_cast<int64_t>(b) * E + e] : 0;
      const int inc = warp_incl_scan(v);
      if (b < nb) block_base[static_cast<int64_t>(b) * E + e] = carry + inc - v;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
  }
  // groups: contiguous blocks of E/G experts
  const int per = E / G;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    group_counts[g] = s_off[(g + 1) * per] - s_off[g * per];
    group_offsets[g] = s_off[g * per];
  }
  if (threadIdx.x == 0) group_offsets[G] = s_off[E];
}

// ------------------------------------------------------------------ scatter
//
// One thread per token. In each warp, bit l of mask[warp][e] says lane l's
// token selected e; the pair's rank among earlier tokens of the same expert
// is (earlier warps of the block) + popc(mask & lanes below). Tokens are
// visited in order inside a warp and warps in order inside a block, so rows
// come out sorted by token within each expert: a stable, deterministic order
// with no atomics deciding it.

__global__ void __launch_bounds__(kRouteThreads) route_scatter_kernel(
    const int32_t* __restrict__ topk_idx, int64_t Ttok, int E, int k,
    const int32_t* __restrict__ block_base, int32_t* __restrict__ row_of_pair,
    int32_t* __restrict__ pair_of_row) {
  extern __shared__ unsigned s_mem[];
  constexpr int W = kRouteThreads / 32;
  unsigned* mask = s_mem;                                   // [W][E]
  int* wbase = reinterpret_cast<int*>(s_mem + W * E);       // [W][E]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < W * E; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteTokensPerBlock + threadIdx.x;
  const bool valid = t < Ttok;
  if (valid)
    for (int j = 0; j < k; ++j) atomicOr(&mask[warp * E + topk_idx[t * k + j]], 1u << lane);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < W; ++w) {
      wbase[w * E + e] = run;
      run += __popc(mask[w * E + e]);
    }
  }
  __syncthreads();
  if (!valid) return;
  const unsigned below = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[t * k + j];
    const int row = block_base[static_cast<int64_t>(blockIdx.x) * E + e] + wbase[warp * E + e] +
                    __popc(mask[warp * E + e] & below);
    row_of_pair[t * k + j] = row;
    pair_of_row[row] = static_cast<int32_t>(t * k + j);
  }
}

// 1024 threads (8 tokens per warp) while a lane's logits fit in a few
// registers (E <= 128), else 256.
template <int SV>
static void launch_topk(int nb, size_t smem, cudaStream_t s, const float* z, int64_t T, int E,
                        int k, int32_t* topk_idx, float* topk_w, int32_t* block_counts,
                        unsigned* err) {
  if constexpr (SV <= 4)
    topk_softmax_kernel<SV, 1024><<<nb, 1024, smem, s>>>(z, T, E, k, topk_idx, topk_w,
                                                          block_counts, err);
  else
    topk_softmax_kernel<SV, kRouteThreads><<<nb, kRouteThreads, smem, s>>>(z, T, E, k, topk_idx,
                                                                           topk_w, block_counts, err);
}

cudaError_t launch_route(const float* z, int64_t T, int E, int k, int G, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int64_t* offsets, int32_t* group_counts,
                         int64_t* group_offsets, int32_t* row_of_pair, int32_t* pair_of_row,
                         int32_t* block_counts, int32_t* block_base, unsigned* err,
                         cudaStream_t s) {
  const int nb = static_cast<int>((T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock);
  const size_t hist_smem = sizeof(int) * E;
  const int S = (E + 31) / 32;
  if (S <= 1) launch_topk<1>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  else if (S <= 2) launch_topk<2>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  else if (S <= 4) launch_topk<4>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  else if (S <= 8) launch_topk<8>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  else if (S <= 16) launch_topk<16>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  else launch_topk<32>(nb, hist_smem, s, z, T, E, k, topk_idx, topk_w, block_counts, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_scan_kernel<<<1, 1024, 0, s>>>(block_counts, nb, E, G, block_base, counts, offsets,
                                        group_counts, group_offsets);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t scatter_smem = sizeof(unsigned) * 2 * (kRouteThreads / 32) * E;
  route_scatter_kernel<<<nb, kRouteThreads, scatter_smem, s>>>(topk_idx, T, E, k, block_base,
                                                               row_of_pair, pair_of_row);
  return cudaGetLastError();
}

cudaError_t route_set_smem_limits() {
  const int scatter_max = static_cast<int>(sizeof(unsigned) * 2 * (kRouteThreads / 32) *
                                           MOE_MAX_EXPERTS);
  return cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              scatter_max);
}

// ------------------------------------------------------------ route backward
//
// dz[t, S_j] = g_j (dg_j - sum_m g_m dg_m); dz = 0 off the selection.
// One warp per token; every dlogits entry is written exactly once.

__global__ void __launch_bounds__(256) route_bwd_kernel(const float* __restrict__ dg,
                                                        const float* __restrict__ w,
                                                        const int32_t* __restrict__ idx,
                                                        int64_t Ttok, int E, int k,
                                                        float* __restrict__ dz) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= Ttok) return;
  float gj = 0.0f, dgj = 0.0f;
  int ij = -1;
  if (lane < k) {
    gj = w[t * k + lane];
    dgj = dg[t * k + lane];
    ij = idx[t * k + lane];
  }
  float s = gj * dgj;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float mine = gj * (dgj - s);
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    float v = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int ie = __shfl_sync(0xffffffffu, ij, j);
      const float dv = __shfl_sync(0xffffffffu, mine, j);
      if (ie == e) v = dv;
    }
    if (e < E) dz[t * E + e] = v;
  }
}

cudaError_t launch_route_bwd(const float* dg, const float* w, const int32_t* idx, int64_t T,
                             int E, int k, float* dz, cudaStream_t s) {
  const unsigned grid = static_cast<unsigned>((T + 7) / 8);
  route_bwd_kernel<<<grid, 256, 0, s>>>(dg, w, idx, T, E, k, dz);
  return cudaGetLastError();
}

}  // namespace moe
