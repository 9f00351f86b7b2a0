// Grouped SwiGLU expert FFN in fp32 on the CUDA cores (the MOE_F32 path).
// Same arithmetic as the tensor-core path, one thread per output element with
// an fp32 sum over K in ascending order; TF32 tensor cores would not meet the
// fp32 tolerance. Rows find their expert by binary search over the device
// offsets, so empty experts cost nothing and no host synchronisation is
// needed. (Grouped expert compute: leap-finetune PR #26 Summary.)
#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ int expert_of_row(const int64_t* __restrict__ off, int E, int64_t r) {
  int lo = 0, hi = E - 1;  // largest e with off[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Row of the expert input that dispatch row r reads: r itself, or with a
// gather map the token x[gather_rows[r] / k] that xp[r] copies.
__device__ __forceinline__ int64_t input_row(const int32_t* __restrict__ grows, int gk, int64_t r) {
  return grows ? static_cast<int64_t>(grows[r] / gk) : r;
}

// h1 = xp Wg_e^T, h2 = xp Wu_e^T, a = silu(h1) h2     (one thread per (r, j))
__global__ void simt_gateup_kernel(const float* __restrict__ xp, const float* __restrict__ Wg,
                                   const float* __restrict__ Wu, const int64_t* __restrict__ off,
                                   int64_t rows, int E, int d, int f, float* __restrict__ h1,
                                   float* __restrict__ h2, float* __restrict__ a,
                                   const int32_t* __restrict__ grows, int gk) {
  const int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (id >= rows * f) return;
  const int64_t r = id / f;
  const int j = static_cast<int>(id % f);
  const int e = expert_of_row(off, E, r);
  const float* x = xp + input_row(grows, gk, r) * d;
  const float* g = Wg + (static_cast<int64_t>(e) * f + j) * d;
  const float* u = Wu + (static_cast<int64_t>(e) * f + j) * d;
  float s1 = 0.0f, s2 = 0.0f;
  for (int i = 0; i < d; ++i) {
    s1 = __fmaf_rn(x[i], g[i], s1);
    s2 = __fmaf_rn(x[i], u[i], s2);
  }
  if (h1) h1[id] = s1;  // any of the three may be skipped (checkpointing)
  if (h2) h2[id] = s2;
  if (a) a[id] = silu_f(s1) * s2;
}

// yp = a Wd_e^T     (one thread per (r, i))
__global__ void simt_down_kernel(const float* __restrict__ a, const float* __restrict__ Wd,
                                 const int64_t* __restrict__ off, int64_t rows, int E, int d,
                                 int f, float* __restrict__ yp) {
  const int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (id >= rows * d) return;
  const int64_t r = id / d;
  const int i = static_cast<int>(id % d);
  const int e = expert_of_row(off, E, r);
  const float* av = a + r * f;
  const float* w = Wd + (static_cast<int64_t>(e) * d + i) * f;
  float s = 0.0f;
  for (int j = 0; j < f; ++j) s = __fmaf_rn(av[j], w[j], s);
  yp[id] = s;
}

// da = dyp Wd_e; dh1 = da h2 silu'(h1); dh2 = da silu(h1)     (one thread per (r, j))
__global__ void simt_dgrad_down_kernel(const float* __restrict__ dyp, const float* __restrict__ Wd,
                                       const float* __restrict__ h1, const float* __restrict__ h2,
                                       const int64_t* __restrict__ off, int64_t rows, int E, int d,
                                       int f, float* __restrict__ dh1, float* __restrict__ dh2) {
  const int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (id >= rows * f) return;
  const int64_t r = id / f;
  const int j = static_cast<int>(id % f);
  const int e = expert_of_row(off, E, r);
  const float* g = dyp + r * d;
  const float* w = Wd + static_cast<int64_t>(e) * d * f + j;
  float da = 0.0f;
  for (int i = 0; i < d; ++i) da = __fmaf_rn(g[i], w[static_cast<int64_t>(i) * f], da);
  const float u = h1[id];
  const float s = sigmoid_f(u);
  dh1[id] = da * h2[id] * s * (1.0f + u * (1.0f - s));
  dh2[id] = da * u * s;
}

// dxp = dh1 Wg_e + dh2 Wu_e     (one thread per (r, i))
__global__ void simt_dgrad_gateup_kernel(const float* __restrict__ dh1,
                                         const float* __restrict__ dh2,
                                         const float* __restrict__ Wg, const float* __restrict__ Wu,
                                         const int64_t* __restrict__ off, int64_t rows, int E,
                                         int d, int f, float* __restrict__ dxp) {
  const int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (id >= rows * d) return;
  const int64_t r = id / d;
  const int i = static_cast<int>(id % d);
  const int e = expert_of_row(off, E, r);
  const float* g1 = dh1 + r * f;
  const float* g2 = dh2 + r * f;
  const float* wg = Wg + static_cast<int64_t>(e) * f * d + i;
  const float* wu = Wu + static_cast<int64_t>(e) * f * d + i;
  float s = 0.0f;
  for (int j = 0; j < f; ++j) {
    s = __fmaf_rn(g1[j], wg[static_cast<int64_t>(j) * d], s);
    s = __fmaf_rn(g2[j], wu[static_cast<int64_t>(j) * d], s);
  }
  dxp[id] = s;
}

// dWg_e[j,i] (+)= sum_r dh1[r,j] xp[r,i]; dWu_e likewise; dWd_e[i,j] (+)= sum_r dyp[r,i] a[r,j].
// One thread per (e, j, i); added when accumulating (experts without rows
// skipped), written otherwise (zero for experts without rows).
__global__ void simt_wgrad_kernel(const float* __restrict__ xp, const float* __restrict__ dyp,
                                  const float* __restrict__ a, const float* __restrict__ dh1,
                                  const float* __restrict__ dh2, const int64_t* __restrict__ off,
                                  int E, int d, int f, float* __restrict__ dWg,
                                  float* __restrict__ dWu, float* __restrict__ dWd, int accumulate,
                                  const int32_t* __restrict__ grows, int gk) {
  const int64_t id = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t per = static_cast<int64_t>(f) * d;
  if (id >= E * per) return;
  const int e = static_cast<int>(id / per);
  const int64_t r0 = off[e], r1 = off[e + 1];
  if (r1 == r0 && accumulate) return;
  const int j = static_cast<int>((id % per) / d);
  const int i = static_cast<int>(id % d);
  float sg = 0.0f, su = 0.0f, sd = 0.0f;
  for (int64_t r = r0; r < r1; ++r) {
    const float xv = xp[input_row(grows, gk, r) * d + i];
    sg = __fmaf_rn(dh1[r * f + j], xv, sg);
    su = __fmaf_rn(dh2[r * f + j], xv, su);
  }
  dWg[id] = accumulate ? dWg[id] + sg : sg;
  dWu[id] = accumulate ? dWu[id] + su : su;
  // dWd_e is [d, f]; reuse the thread for element (i', j') = (j*d+i) / f, % f
  const int64_t q = id % per;
  const int di = static_cast<int>(q / f), fj = static_cast<int>(q % f);
  for (int64_t r = r0; r < r1; ++r) sd = __fmaf_rn(dyp[r * d + di], a[r * f + fj], sd);
  float* od = dWd + static_cast<int64_t>(e) * per + q;
  *od = accumulate ? *od + sd : sd;
}

static unsigned blocks_for(int64_t n) { return static_cast<unsigned>((n + 255) / 256); }

cudaError_t launch_ffn_gateup_f32(const FfnFwdArgs& x, cudaStream_t s) {
  simt_gateup_kernel<<<blocks_for(x.rows * x.f), 256, 0, s>>>(
      static_cast<const float*>(x.xp), static_cast<const float*>(x.Wg),
      static_cast<const float*>(x.Wu), x.offsets, x.rows, x.E, x.d, x.f,
      static_cast<float*>(x.h1), static_cast<float*>(x.h2), static_cast<float*>(x.a),
      x.gather.rows, x.gather.k);
  return cudaGetLastError();
}

cudaError_t launch_ffn_fwd_f32(const FfnFwdArgs& x, cudaStream_t s) {
  const float* xp = static_cast<const float*>(x.xp);
  float* a = static_cast<float*>(x.a);
  simt_gateup_kernel<<<blocks_for(x.rows * x.f), 256, 0, s>>>(
      xp, static_cast<const float*>(x.Wg), static_cast<const float*>(x.Wu), x.offsets, x.rows,
      x.E, x.d, x.f, static_cast<float*>(x.h1), static_cast<float*>(x.h2), a, x.gather.rows,
      x.gather.k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt_down_kernel<<<blocks_for(x.rows * x.d), 256, 0, s>>>(
      a, static_cast<const float*>(x.Wd), x.offsets, x.rows, x.E, x.d, x.f,
      static_cast<float*>(x.yp));
  return cudaGetLastError();
}

cudaError_t launch_ffn_dgrad_f32(const FfnBwdArgs& x, cudaStream_t s) {
  float* dh1 = static_cast<float*>(x.dh1);
  float* dh2 = static_cast<float*>(x.dh2);
  simt_dgrad_down_kernel<<<blocks_for(x.rows * x.f), 256, 0, s>>>(
      static_cast<const float*>(x.dyp), static_cast<const float*>(x.Wd),
      static_cast<const float*>(x.h1), static_cast<const float*>(x.h2), x.offsets, x.rows, x.E,
      x.d, x.f, dh1, dh2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt_dgrad_gateup_kernel<<<blocks_for(x.rows * x.d), 256, 0, s>>>(
      dh1, dh2, static_cast<const float*>(x.Wg), static_cast<const float*>(x.Wu), x.offsets,
      x.rows, x.E, x.d, x.f, static_cast<float*>(x.dxp));
  return cudaGetLastError();
}

cudaError_t launch_ffn_wgrad_f32(const FfnBwdArgs& x, cudaStream_t s) {
  const float* dh1 = static_cast<const float*>(x.dh1);
  const float* dh2 = static_cast<const float*>(x.dh2);
  simt_wgrad_kernel<<<blocks_for(static_cast<int64_t>(x.E) * x.f * x.d), 256, 0, s>>>(
      static_cast<const float*>(x.xp), static_cast<const float*>(x.dyp),
      static_cast<const float*>(x.a), dh1, dh2, x.offsets, x.E, x.d, x.f, x.dWg, x.dWu, x.dWd,
      x.accumulate, x.gather.rows, x.gather.k);
  return cudaGetLastError();
}

}  // namespace moe
