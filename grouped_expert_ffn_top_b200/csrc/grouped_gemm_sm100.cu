// Grouped expert GEMMs on the 5th-generation tensor cores (sm_100a):
// tcgen05.mma with fp32 accumulators in TMEM, operands staged by TMA into
// 128-byte-swizzled shared memory, one persistent CTA pair (a cluster of two
// SMs sharing each MMA) per two SMs walking a tile list built on the device
// from the expert offsets (no host synchronisation; an expert with no rows
// contributes no tile, except zero tiles of a weight gradient it writes).
// (Grouped expert compute / grouped-GEMM: leap-finetune PR #26 Summary; ART
// issue #917 Related.)
//
// One kernel template serves the five GEMMs of the layer:
//   kFwdGateUp      [h1 | h2] = xp [Wg_e | Wu_e]^T, epilogue a = silu(h1) h2
//   kFwdDown        yp = a Wd_e^T
//   kBwdDgradDown   da = dyp Wd_e, epilogue dh1 = da h2 silu'(h1), dh2 = da silu(h1)
//   kBwdDgradGateUp dxp = [dh1 | dh2] [Wg_e ; Wu_e]          (K = 2f)
//   kWgrad          dWg_e^T += xp^T dh1, dWu_e^T += xp^T dh2, dWd_e^T += a^T dyp
// The first four have a ragged M (the expert's rows, tiles of 256 = 128 per
// CTA of the pair; rows of a tile past the expert's end are computed and
// discarded). kWgrad has a ragged K (the expert's rows): in the last K block
// the rows past the expert's end are zeroed in shared memory before the MMA
// reads them.
//
// Warp roles: warp 0 issues TMA loads, warp 1 allocates TMEM and issues
// tcgen05.mma (one lane of the even CTA), the remaining warps run the
// epilogue, each on its TMEM lane quarter (warp % 4). The weight gradient,
// whose fp32 stores or reductions move the most memory, uses eight epilogue
// warps: two per lane quarter, one per half of the tile's columns. Two TMEM
// accumulators let the epilogue of one tile overlap the main loop of the
// next.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace gg {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes: one swizzle row
template <int KIND>
struct Roles {
  static constexpr int kEpiWarps = KIND == 4 ? 8 : 4;  // wgrad: eight
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
};
constexpr int kMaxE = MOE_MAX_EXPERTS;
// Grouped raster of one expert's tiles: row tiles (M-ragged kinds) or M tiles
// (wgrad) are taken in groups of this many, and within a group the column
// tiles advance slowest. The persistent CTAs work on consecutive tiles at any
// moment, so the tiles in flight together share a few row tiles and a few
// column tiles: their operands stay in L2 across the group instead of being
// streamed again from HBM for every row tile. A group's row operands should
// fit in kResidentBytes of L2; when 16 row tiles of a long K range do not
// (the down projection and the gate/up input gradient at large f), the
// group has 8, which also makes the 74 tiles in flight together nearly
// square (fewest distinct operand blocks per wave). The weight gradient
// keeps the whole d-side operand of an expert (xp for dWg / dWu, dyp for
// dWd) in the group when it fits, so the long f-side operand (dh1, dh2, a)
// streams through L2 once.
constexpr int kRasterRows = 16;
constexpr int kRasterM = 8;
constexpr long long kResidentBytes = 48ll << 20;
// weight gradient: experts with fewer rows have short-K tiles (interleave_waves)
constexpr int kShortRows = 1024;
constexpr long long kWaitLimit = 2000000000LL;  // about one second of SM cycles
constexpr uint32_t kTmemCols = 512;

enum Kind : int {
  kFwdGateUp = 0,
  kFwdDown = 1,
  kBwdDgradDown = 2,
  kBwdDgradGateUp = 3,
  kWgrad = 4
};

struct Maps {
  CUtensorMap a0, a1, b0, b1, b2;
  CUtensorMap o0, o1, o2;  // TMA-stored outputs (32 x 32 boxes, 64-byte swizzle)
};

struct Params {
  const int64_t* offsets;
  int E, d, f;
  bf16* o0;
  bf16* o1;
  bf16* o2;
  const bf16* i0;
  const bf16* i1;
  float* w0;
  float* w1;
  float* w2;
  unsigned* err;
  int accumulate;  // wgrad: 1 adds to dW, 0 writes it (zero tiles for experts with no rows)
  // Gathered A rows (kernels instantiated with GATHER): dispatch row r of the
  // expert input is row grow[r] / gk of x [gT, d], the token whose copy xp[r]
  // would be; rows at or past `grows` (the tile's rows past the last expert)
  // read token 0 and are discarded like any row past the expert's end. Every
  // gathered address lies inside x: tokens are clamped to [0, gT).
  const bf16* gx;
  const int32_t* grow;
  int gk;
  int grows;
  int gT;
};

// PAIR: a cluster of two CTAs computes a 256-row tile with one
// tcgen05.mma.cta_group::2 per K step; each CTA stages its 128 rows of A and
// half of B, so per-SM operand traffic per flop drops by a third and six
// pipeline stages fit in shared memory.
template <int KIND, int BN, bool PAIR = false>
struct Traits {
  static constexpr bool A_MN = KIND == kWgrad;
  static constexpr bool B_MN = KIND == kBwdDgradDown || KIND == kBwdDgradGateUp || KIND == kWgrad;
  static constexpr int TM = PAIR ? 2 * BM : BM;  // rows of one tile
  // Kinds whose epilogue writes bf16 tiles through shared memory with TMA
  // stores: per epilogue warp, two buffers of a 32 x 32 box per output tensor
  // (the SwiGLU backward also loads h1 / h2 into them and works in place).
  static constexpr bool EPI_TMA = KIND == kFwdGateUp || KIND == kFwdDown || KIND == kBwdDgradGateUp;
  static constexpr int EPI_TENSORS = KIND == kFwdGateUp ? 3 : (KIND == kBwdDgradDown ? 2 : 1);
  static constexpr uint32_t EPI_BOX_BYTES = 32 * 32 * 2;
  static constexpr uint32_t EPI_WARP_BYTES =
      (EPI_TMA || KIND == kBwdDgradDown) ? 2 * EPI_TENSORS * EPI_BOX_BYTES : 0;
  static constexpr uint32_t EPI_BYTES = EPI_WARP_BYTES * Roles<KIND>::kEpiWarps;
  // pipeline stages: as many as fit beside the epilogue buffers and the
  // schedule of up to 1024 experts
  static constexpr int STAGES =
      (KIND == kFwdGateUp || KIND == kBwdDgradDown) ? 5 : ((PAIR || BN != 256) ? 6 : 4);
  static constexpr uint32_t A_BYTES = BM * BK * 2;                      // per CTA
  static constexpr uint32_t B_BYTES = (PAIR ? BN / 2 : BN) * BK * 2;    // per CTA
  static constexpr uint32_t STAGE_TX = (A_BYTES + B_BYTES) * (PAIR ? 2 : 1);  // all CTAs
  static constexpr uint32_t IDESC = umma_idesc_bf16(TM, BN, A_MN, B_MN);
  // Pair kinds whose tile columns run over f (dgrad down; dWg and dWu of the
  // weight gradient): when f is not a multiple of BN, a last column tile with
  // at most BN / 2 valid columns runs MMAs of half the width, each CTA staging
  // the first 64 of its B columns from the tile's midpoint instead of
  // BN / 2 past it.
  static constexpr bool NARROW = PAIR && BN == 256 && (KIND == kBwdDgradDown || KIND == kWgrad);
  static constexpr uint32_t IDESC_NARROW = umma_idesc_bf16(TM, BN / 2, A_MN, B_MN);
  // N extent of one output tile (gate/up: 128 f columns, each with its gate
  // and up accumulator, together the MMA's N = 256)
  static constexpr int NTILE = KIND == kFwdGateUp ? 128 : BN;
  static constexpr size_t BAR_BYTES = 320;
  // dynamic shared memory: alignment slack, stages, barriers, and the tile
  // schedule (expert offsets, first tile and expert of each slot) for E experts
  static constexpr size_t SMEM_FIXED =
      1024 + STAGES * static_cast<size_t>(A_BYTES + B_BYTES) + EPI_BYTES + BAR_BYTES;
  static constexpr size_t smem_bytes(int E) {
    return SMEM_FIXED + 8 * static_cast<size_t>(E + 1) + 4 * static_cast<size_t>(E + 1) +
           4 * static_cast<size_t>(E);
  }
  static_assert(KIND != kFwdGateUp || BN == 256, "gate/up pairs two 128-column accumulators");
  static_assert(2 * BN <= static_cast<int>(kTmemCols), "two accumulators must fit in TMEM");
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
};

struct TileInfo {
  int e;
  int row0;  // first row of the tile (M-ragged) or of the expert (wgrad)
  int rows;  // valid rows in the tile (M-ragged) or the expert's row count (wgrad)
  int m0;    // wgrad: first f index of the tile
  int n0;    // first output column of the tile
  int prod;  // wgrad: 0 dWg, 1 dWu, 2 dWd
  int narrow;  // half-width MMAs (Traits::NARROW)
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Tile `local` of an R x C grid in groups of G rows: (row, column) with the
// row fastest inside a group of min(G, R - first row) rows.
__device__ __forceinline__ void raster(int local, int R, int C, int G, int& row, int& col) {
  const int g = local / (G * C);
  const int rem = local - g * G * C;
  const int rg = min(G, R - g * G);
  col = rem / rg;
  row = g * G + rem % rg;
}

// Tiles of an expert with `cnt` rows. Writing weight gradients (accumulate
// = 0), an expert with no rows still has its tiles: they store zeros.
template <int KIND, int BN, bool PAIR>
__device__ __forceinline__ int tiles_of_expert(int cnt, int d, int f, int accumulate) {
  using Tr = Traits<KIND, BN, PAIR>;
  if (cnt <= 0 && (KIND != kWgrad || accumulate)) return 0;
  if (KIND == kWgrad)
    return 2 * ceil_div(d, Tr::TM) * ceil_div(f, BN) + ceil_div(f, Tr::TM) * ceil_div(d, BN);
  const int n_extent = (KIND == kFwdGateUp || KIND == kBwdDgradDown) ? f : d;
  return ceil_div(cnt, Tr::TM) * ceil_div(n_extent, Tr::NTILE);
}

// K blocks of a tile. When d or f is not a multiple of 64 the last block of
// each K range runs past it: TMA reads those columns (and the weight rows past
// the expert's matrix, through the 3D weight maps) as zero, so they add
// nothing.
template <int KIND, int BN>
__device__ __forceinline__ int num_kblocks(const TileInfo& ti, int d, int f) {
  if (KIND == kFwdGateUp || KIND == kBwdDgradDown) return ceil_div(d, BK);
  if (KIND == kFwdDown) return ceil_div(f, BK);
  if (KIND == kBwdDgradGateUp) return 2 * ceil_div(f, BK);
  return ceil_div(ti.rows, BK);  // wgrad: ragged K
}

struct Sched {
  const int64_t* off;  // [E+1] shared copy of the offsets
  const int* tstart;   // [E+1] first tile of each scheduled slot
  const int* order;    // [E] expert of each slot
  int E;
  int total;  // tiles of the launch
  int nlong;  // weight gradient: tiles of the experts with at least kShortRows rows
  int width;  // tiles in flight together (CTAs, or CTA pairs)
};

// Weight gradient: processing position g -> index in the tile list, whose
// experts run longest first, so its first nlong tiles have a long K (MMA
// bound) and the rest a short one (bound by the 256 KB fp32 store or add of
// each tile). While both parts have a whole wave of `width` tiles left, waves
// alternate between them, so each CTA pair alternates a long and a short tile
// and the short tile's epilogue runs under the long tile's main loop; the
// remaining tiles follow in list order. Experts of similar size are not
// interleaved with each other, which would only mix their operands in L2.
__device__ __forceinline__ int interleave_waves(int g, int n, int nlong, int width) {
  const int m = min(nlong / width, (n - nlong) / width);  // alternating wave pairs
  if (g < 2 * m * width) {
    const int w = g / width, pos = g - w * width;
    return (w & 1) ? nlong + (w >> 1) * width + pos : (w >> 1) * width + pos;
  }
  const int r = g - 2 * m * width;      // position among the rest
  const int along = nlong - m * width;  // long tiles left
  return r < along ? m * width + r : nlong + m * width + (r - along);
}

template <int KIND, int BN, bool PAIR>
__device__ __forceinline__ TileInfo decode_tile(const Sched& s, int tile, int d, int f) {
  using Tr = Traits<KIND, BN, PAIR>;
  if (KIND == kWgrad) tile = interleave_waves(tile, s.total, s.nlong, s.width);
  int lo = 0, hi = s.E - 1;
  while (lo < hi) {  // largest slot whose first tile is <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (s.tstart[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  TileInfo ti;
  ti.e = s.order[lo];
  const int local = tile - s.tstart[lo];
  const int base = static_cast<int>(s.off[ti.e]);
  const int cnt = static_cast<int>(s.off[ti.e + 1] - s.off[ti.e]);
  if (KIND == kWgrad) {
    // products 0, 1 (dWg, dWu): M over d, N over f; product 2 (dWd): M over f,
    // N over d. M always runs along the output's contiguous dimension.
    const int t01 = ceil_div(d, Tr::TM) * ceil_div(f, BN);
    int rem, nt;
    if (local < 2 * t01) {
      ti.prod = local / t01;
      rem = local % t01;
      nt = ceil_div(f, BN);
    } else {
      ti.prod = 2;
      rem = local - 2 * t01;
      nt = ceil_div(d, BN);
    }
    const int mt = ti.prod < 2 ? ceil_div(d, Tr::TM) : ceil_div(f, Tr::TM);
    int mi, ni;
    if (2ll * d * cnt > kResidentBytes) raster(rem, mt, nt, kRasterM, mi, ni);
    else if (ti.prod < 2) raster(rem, mt, nt, mt, mi, ni);  // M (over d) fastest
    else raster(rem, nt, mt, nt, ni, mi);                    // N (over d) fastest
    ti.m0 = mi * Tr::TM;
    ti.n0 = ni * BN;
    ti.row0 = base;
    ti.rows = cnt;
    ti.narrow = Tr::NARROW && ti.prod < 2 && f - ti.n0 <= BN / 2;
  } else {
    const int n_extent = (KIND == kFwdGateUp || KIND == kBwdDgradDown) ? f : d;
    const int nt = ceil_div(n_extent, Tr::NTILE);
    const int k_extent = (KIND == kFwdGateUp || KIND == kBwdDgradDown) ? d : (KIND == kFwdDown ? f : 2 * f);
    const int g = 2ll * kRasterRows * Tr::TM * k_extent <= kResidentBytes ? kRasterRows : kRasterRows / 2;
    int mi, ni;
    raster(local, ceil_div(cnt, Tr::TM), nt, g, mi, ni);
    ti.n0 = ni * Tr::NTILE;
    ti.row0 = base + mi * Tr::TM;
    ti.rows = min(Tr::TM, cnt - mi * Tr::TM);
    ti.m0 = 0;
    ti.prod = 0;
    ti.narrow = Tr::NARROW && f - ti.n0 <= BN / 2;
  }
  return ti;
}

// TMA loads of k block `kb` of tile `ti` into one pipeline stage.
template <int KIND, int BN>
__device__ __forceinline__ void issue_loads(const Maps& m, const TileInfo& ti, int kb, int d,
                                            int f, uint8_t* a_dst, uint8_t* b_dst,
                                            uint64_t* bar) {
  const int k0 = kb * BK;
  if (KIND == kFwdGateUp) {
    tma_load_2d(a_dst, &m.a0, bar, k0, ti.row0);
    tma_load_3d(b_dst, &m.b0, bar, k0, ti.n0, ti.e);
    tma_load_3d(b_dst + 128 * 128, &m.b1, bar, k0, ti.n0, ti.e);
  } else if (KIND == kFwdDown) {
    tma_load_2d(a_dst, &m.a0, bar, k0, ti.row0);
    tma_load_3d(b_dst, &m.b0, bar, k0, ti.n0, ti.e);
  } else if (KIND == kBwdDgradDown) {
    tma_load_2d(a_dst, &m.a0, bar, k0, ti.row0);
#pragma unroll
    for (int j = 0; j < BN / 64; ++j) tma_load_3d(b_dst + j * 8192, &m.b0, bar, ti.n0 + 64 * j, k0, ti.e);
  } else if (KIND == kBwdDgradGateUp) {
    const int half = ceil_div(f, BK);
    const bool second = kb >= half;
    const int kk = (second ? kb - half : kb) * BK;
    tma_load_2d(a_dst, second ? &m.a1 : &m.a0, bar, kk, ti.row0);
#pragma unroll
    for (int j = 0; j < BN / 64; ++j)
      tma_load_3d(b_dst + j * 8192, second ? &m.b1 : &m.b0, bar, ti.n0 + 64 * j, kk, ti.e);
  } else {  // kWgrad: A = xp (dWg, dWu) or a (dWd); B = dh1, dh2 or dyp
    const CUtensorMap* am = ti.prod == 2 ? &m.a1 : &m.a0;
    const CUtensorMap* bm = ti.prod == 0 ? &m.b0 : (ti.prod == 1 ? &m.b1 : &m.b2);
    const int r = ti.row0 + k0;
    tma_load_2d(a_dst, am, bar, ti.m0, r);
    tma_load_2d(a_dst + 8192, am, bar, ti.m0 + 64, r);
#pragma unroll
    for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * 8192, bm, bar, ti.n0 + 64 * j, r);
  }
}

// The same k block for one CTA of a pair: this CTA's 128 rows of A and its
// half of B (gate/up: CTA 0 stages the Wg rows, CTA 1 the Wu rows), counted
// on the even CTA's mbarrier at `bar`, a shared::cluster address. With
// load_a false the A operand is left to the gathered loads.
template <int KIND, int BN>
__device__ __forceinline__ void issue_loads_pair(const Maps& m, const TileInfo& ti, int kb, int d,
                                                 int f, int cta, uint8_t* a_dst, uint8_t* b_dst,
                                                 uint32_t bar, bool load_a = true) {
  const int k0 = kb * BK;
  const int arow = ti.row0 + BM * cta;
  constexpr int HALF = BN / 2;
  const int bh = ti.narrow ? HALF / 2 : HALF;  // B columns of the even CTA
  if (KIND == kFwdGateUp) {
    if (load_a) tma_load_2d_pair(a_dst, &m.a0, bar, k0, arow);
    tma_load_3d_pair(b_dst, cta == 0 ? &m.b0 : &m.b1, bar, k0, ti.n0, ti.e);
  } else if (KIND == kFwdDown) {
    tma_load_2d_pair(a_dst, &m.a0, bar, k0, arow);
    tma_load_3d_pair(b_dst, &m.b0, bar, k0, ti.n0 + HALF * cta, ti.e);
  } else if (KIND == kBwdDgradDown) {
    tma_load_2d_pair(a_dst, &m.a0, bar, k0, arow);
#pragma unroll
    for (int j = 0; j < HALF / 64; ++j)
      tma_load_3d_pair(b_dst + j * 8192, &m.b0, bar, ti.n0 + bh * cta + 64 * j, k0, ti.e);
  } else if (KIND == kBwdDgradGateUp) {
    const int half = ceil_div(f, BK);
    const bool second = kb >= half;
    const int kk = (second ? kb - half : kb) * BK;
    tma_load_2d_pair(a_dst, second ? &m.a1 : &m.a0, bar, kk, arow);
#pragma unroll
    for (int j = 0; j < HALF / 64; ++j)
      tma_load_3d_pair(b_dst + j * 8192, second ? &m.b1 : &m.b0, bar, ti.n0 + HALF * cta + 64 * j, kk, ti.e);
  } else {  // kWgrad: this CTA's 128 values of M and half of N, K rows of the expert
    const CUtensorMap* am = ti.prod == 2 ? &m.a1 : &m.a0;
    const CUtensorMap* bm = ti.prod == 0 ? &m.b0 : (ti.prod == 1 ? &m.b1 : &m.b2);
    const int r = ti.row0 + k0;
    const int mm = ti.m0 + BM * cta;
    if (load_a) {
      tma_load_2d_pair(a_dst, am, bar, mm, r);
      tma_load_2d_pair(a_dst + 8192, am, bar, mm + 64, r);
    }
#pragma unroll
    for (int j = 0; j < HALF / 64; ++j)
      tma_load_2d_pair(b_dst + j * 8192, bm, bar, ti.n0 + bh * cta + 64 * j, r);
  }
}

// Token of dispatch row r (see Params::grow).
__device__ __forceinline__ int token_of_row(const Params& p, int r) {
  const int v = r < p.grows ? __ldg(p.grow + r) / p.gk : 0;
  return min(max(v, 0), p.gT - 1);
}

// Gathered A operand of one pipeline stage, written by the 32 lanes of the
// producer warp with 16-byte cp.async copies into the 128-byte-swizzled
// layout the tiled TMA load would produce (16-byte chunk c of smem row j goes
// to chunk c ^ (j % 8); the stage is 1024-byte aligned). Each warp-wide copy
// moves four 128-byte row segments. Completion is counted on the local
// mbarrier by the caller's cp.async arrive.
//   gate/up: smem row j (0..127) = dispatch row row0 + 128 cta + j at K
//     columns k0 .. k0 + 63; lane l holds in tok[q] the token of row l + 32 q.
//   wgrad (dWg, dWu; A = x^T, M-major): smem row j (0..63) of box b = K row j
//     of the block (dispatch row row0 + k0 + j), M columns col0 + 64 b ..;
//     lane l holds in tok[q] the token of K row l + 32 q. Columns past d (the
//     last M tile when d is not a multiple of 256) feed only accumulator rows
//     the epilogue drops: they read column 0 instead.
template <int KIND>
__device__ __forceinline__ void gather_a_stage(const Params& p, int lane, uint32_t a_s, int k0,
                                               int col0, const int (&tok)[4]) {
  const char* xb = reinterpret_cast<const char*>(p.gx);
  const int c = lane & 7;
  if (KIND == kFwdGateUp) {
    const int h = lane >> 3;  // row 4 i + h of iteration i
    const uint32_t d_even = h * 128 + ((c ^ h) << 4);        // (4 i + h) % 8 = h for even i
    const uint32_t d_odd = h * 128 + ((c ^ (h + 4)) << 4);   // and 4 + h for odd i
    // K columns at or past d (the last block when d is not a multiple of 64)
    // are written as zeros without reading x
    const bool col_in = k0 + 8 * c < p.d;
    const int64_t cofs = col_in ? static_cast<int64_t>(k0 + 8 * c) * 2 : 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = __shfl_sync(0xffffffffu, tok[i >> 3], (4 * i + h) & 31);
      const uint32_t dst = a_s + i * 512 + ((i & 1) ? d_odd : d_even);
      const char* src = xb + static_cast<int64_t>(t) * p.d * 2 + cofs;
      if (col_in) cp_async_16(dst, src);
      else cp_async_16_zfill(dst, src, 0u);
    }
  } else {
    const int hh = lane >> 4;        // K row 2 i + hh of iteration i
    const int b = (lane >> 3) & 1;   // M box
    int col = col0 + 64 * b + 8 * c;
    if (col >= p.d) col = 0;
    const int64_t cofs = static_cast<int64_t>(col) * 2;
    const uint32_t dbase = b * 8192 + hh * 128;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = __shfl_sync(0xffffffffu, tok[i >> 4], (2 * i + hh) & 31);
      const uint32_t sw = static_cast<uint32_t>(c ^ ((2 * (i & 3) + hh) & 7)) << 4;
      cp_async_16(a_s + dbase + i * 256 + sw, xb + static_cast<int64_t>(t) * p.d * 2 + cofs);
    }
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
  uint4 o;
  __nv_bfloat162 t0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 t1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 t2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 t3 = __floats2bfloat162_rn(v[6], v[7]);
  o.x = *reinterpret_cast<uint32_t*>(&t0);
  o.y = *reinterpret_cast<uint32_t*>(&t1);
  o.z = *reinterpret_cast<uint32_t*>(&t2);
  o.w = *reinterpret_cast<uint32_t*>(&t3);
  return o;
}

__device__ __forceinline__ void unpack8_bf16(uint4 u, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f2 = __bfloat1622float2(h[i]);
    v[2 * i] = f2.x;
    v[2 * i + 1] = f2.y;
  }
}

__device__ __forceinline__ void store16_bf16(bf16* dst, const float* v) {
  uint4* p = reinterpret_cast<uint4*>(dst);
  p[0] = pack8_bf16(v);
  p[1] = pack8_bf16(v + 8);
}

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

// Weight-gradient epilogue of one tile for this thread's accumulator row r,
// on the columns [c0, c0 + BN / 2) of the accumulator: added to dW, or
// written (zeros for an expert with no rows, whose tile ran no MMA).
template <int BN>
__device__ __forceinline__ void epilogue_wgrad(const Params& p, const TileInfo& ti, uint32_t tacc,
                                               int r, int c0) {
  // Accumulator row m, column n is element (n, m) of the [N, M] row-major
  // output, so for each column the 32 lanes of a warp cover 32 consecutive
  // floats: one coalesced 128-byte access per column. red.global.add is
  // fire-and-forget (the add happens at L2), and each element receives
  // exactly one add or store per call, so the result is deterministic.
  const int d = p.d, f = p.f;
  const int M = ti.prod == 2 ? f : d;
  const int Nn = ti.prod == 2 ? d : f;
  const int m = ti.m0 + r;
  const bool valid = m < M;
  float* out = (ti.prod == 0 ? p.w0 : (ti.prod == 1 ? p.w1 : p.w2)) +
               static_cast<int64_t>(ti.e) * d * f + m;
  uint32_t u[16];
  const bool empty = ti.rows <= 0;
  for (int c = c0; c < c0 + BN / 2; c += 16) {
    if (empty) {
#pragma unroll
      for (int i = 0; i < 16; ++i) u[i] = 0u;
    } else {
      tmem_ld16(tacc + c, u);
      tmem_ld_wait();
    }
    if (valid && ti.n0 + c < Nn) {
      float* q = out + static_cast<int64_t>(ti.n0 + c) * M;
      const int nc = min(16, Nn - (ti.n0 + c));  // columns of this group inside the output
      if (p.accumulate) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < nc) red_add_f32(q + static_cast<int64_t>(i) * M, __uint_as_float(u[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < nc) q[static_cast<int64_t>(i) * M] = __uint_as_float(u[i]);
      }
    }
  }
}

// Epilogue of the kinds that write bf16 tiles (gate/up: h1, h2, a; down: yp;
// dgrad gate/up: dxp) for one warp: its 32 accumulator rows (tile rows
// rbase .. rbase + 31), in chunks of 32 columns. Where all 32 rows lie inside
// the expert, each chunk goes row by row into a 64-byte-swizzled shared
// buffer and one lane stores the 32 x 32 box with TMA, so the warp issues no
// scattered global stores (those stall the MMA warp's issue on the same SM).
// Rows past the expert's end belong to the next expert, so a warp with fewer
// valid rows stores its valid rows directly. Two buffers per tensor
// alternate (`ebuf`); a buffer is rewritten once its store has read it.
template <int KIND, int BN>
__device__ __forceinline__ void epilogue_tma(const Params& p, const Maps& maps, const TileInfo& ti,
                                             uint32_t tacc, int rbase, int lane, uint8_t* sbuf,
                                             int& ebuf) {
  constexpr int NT = KIND == kFwdGateUp ? 3 : 1;  // output tensors
  constexpr int W = KIND == kFwdGateUp ? 128 : BN;  // output columns of the tile
  constexpr uint32_t BOX = 32 * 32 * 2;
  const int ncols = KIND == kFwdGateUp ? p.f : p.d;
  const int valid = min(32, ti.rows - rbase);  // rows of this warp inside the expert
  if (valid <= 0) return;
  const bool full = valid == 32;
  const int64_t row = static_cast<int64_t>(ti.row0) + rbase + lane;
  const CUtensorMap* omap[3] = {&maps.o0, &maps.o1, &maps.o2};
  bf16* optr[3] = {p.o0, p.o1, p.o2};
  for (int c = 0; c < W; c += 32) {
    if (ti.n0 + c >= ncols) break;
    float o[NT][32];
    {
      uint32_t u0[16], u1[16];
      tmem_ld16(tacc + c, u0);
      tmem_ld16(tacc + c + 16, u1);
      if (KIND == kFwdGateUp) {
        uint32_t g0[16], g1[16];
        tmem_ld16(tacc + 128 + c, g0);
        tmem_ld16(tacc + 128 + c + 16, g1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float h1 = __uint_as_float(i < 16 ? u0[i] : u1[i - 16]);
          const float h2 = __uint_as_float(i < 16 ? g0[i] : g1[i - 16]);
          o[0][i] = h1;
          o[1 % NT][i] = h2;
          o[2 % NT][i] = silu_f(h1) * h2;
        }
      } else {
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[0][i] = __uint_as_float(i < 16 ? u0[i] : u1[i - 16]);
      }
    }
    if (full) {
      uint8_t* b = sbuf + ebuf * NT * BOX;
      // the store that used this buffer two chunks ago has read it
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (!optr[t]) continue;  // an output this launch does not store
        // row `lane`: four 16-byte chunks, chunk j at (j ^ ((lane >> 1) & 3)),
        // the TMA 64-byte swizzle of a 64-byte row
        uint8_t* rowp = b + t * BOX + lane * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(rowp + ((j ^ ((lane >> 1) & 3)) << 4)) = pack8_bf16(o[t] + 8 * j);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (optr[t]) tma_store_2d(omap[t], b + t * BOX, ti.n0 + c, ti.row0 + rbase);
        bulk_commit_group();
      }
      ebuf ^= 1;
    } else if (lane < valid) {
      // the chunk's columns inside the output (a multiple of 8)
      const int ncol = min(32, ncols - (ti.n0 + c));
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (!optr[t]) continue;
        bf16* dst = optr[t] + row * ncols + ti.n0 + c;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (8 * j < ncol) *reinterpret_cast<uint4*>(dst + 8 * j) = pack8_bf16(o[t] + 8 * j);
      }
    }
  }
}

// SwiGLU-backward epilogue of the dgrad-down kind for one warp: its 32 rows
// (tile rows rbase .. rbase + 31), all columns of the tile in chunks of 32.
//   dh1 = da h2 s (1 + h1 (1 - s)),  dh2 = da h1 s,  s = sigmoid(h1)
// One lane loads the chunk's h1 and h2 boxes with TMA into a 64-byte-swizzled
// buffer pair, one chunk ahead (two pairs alternate; each completes on its own
// barrier of this warp); each lane then turns its row of h1, h2 and da into
// dh1, dh2 in place, and one lane stores both boxes with TMA. Rows past the
// expert's end are loaded and computed but not stored: a warp with fewer
// valid rows writes its valid rows directly. `lphase` holds the parity of the
// next completion of each of the warp's two barriers. Returns false if a wait
// gave up (the kernel is aborting); loads it issued have landed by then.
template <int BN>
__device__ __forceinline__ bool epilogue_swiglu_bwd(const Params& p, const Maps& maps,
                                                    const TileInfo& ti, uint32_t tacc, int rbase,
                                                    int lane, uint8_t* sbuf, uint64_t* lbar,
                                                    uint32_t& lphase, volatile int* s_abort) {
  constexpr uint32_t BOX = 32 * 32 * 2;
  const int valid = min(32, ti.rows - rbase);
  if (valid <= 0) return true;
  const int nch = ceil_div(min(BN, p.f - ti.n0), 32);  // the last chunk may run past f
  const int y = ti.row0 + rbase;
  const int64_t row = static_cast<int64_t>(y) + lane;
  // buffer pair b: h1 (then dh1) at sbuf + 2 b BOX, h2 (then dh2) after it
  auto load = [&](int ch, int b) {
    if (lane == 0) {
      bulk_wait_group_read<0>();  // earlier stores from these buffers have read them
      mbar_arrive_expect_tx(&lbar[b], 2 * BOX);
      tma_load_2d(sbuf + 2 * b * BOX, &maps.a1, &lbar[b], ti.n0 + 32 * ch, y);
      tma_load_2d(sbuf + 2 * b * BOX + BOX, &maps.b1, &lbar[b], ti.n0 + 32 * ch, y);
    }
    __syncwarp();
  };
  uint32_t pend = 1u;  // buffer pairs with a load in flight
  load(0, 0);
  bool ok = true;
  for (int ch = 0; ch < nch; ++ch) {
    const int b = ch & 1;
    if (ch + 1 < nch) {
      load(ch + 1, b ^ 1);
      pend |= 1u << (b ^ 1);
    }
    uint32_t u0[16], u1[16];
    tmem_ld16(tacc + 32 * ch, u0);
    tmem_ld16(tacc + 32 * ch + 16, u1);
    tmem_ld_wait();
    if (!wait_bounded(&lbar[b], (lphase >> b) & 1u, s_abort, kWaitLimit)) {
      ok = false;
      break;
    }
    lphase ^= 1u << b;
    pend &= ~(1u << b);
    uint8_t* r1 = sbuf + 2 * b * BOX + lane * 64;
    uint8_t* r2 = r1 + BOX;
    float dh1[32], dh2[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int off = (j ^ ((lane >> 1) & 3)) << 4;  // TMA 64-byte swizzle of a 64-byte row
      float h1[8], h2[8];
      unpack8_bf16(*reinterpret_cast<const uint4*>(r1 + off), h1);
      unpack8_bf16(*reinterpret_cast<const uint4*>(r2 + off), h2);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = 8 * j + i;
        const float da = __uint_as_float(k < 16 ? u0[k] : u1[k - 16]);
        const float sg = sigmoid_f(h1[i]);
        dh1[k] = da * h2[i] * sg * (1.0f + h1[i] * (1.0f - sg));
        dh2[k] = da * h1[i] * sg;
      }
      *reinterpret_cast<uint4*>(r1 + off) = pack8_bf16(dh1 + 8 * j);
      *reinterpret_cast<uint4*>(r2 + off) = pack8_bf16(dh2 + 8 * j);
    }
    if (valid == 32) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&maps.o0, sbuf + 2 * b * BOX, ti.n0 + 32 * ch, y);
        tma_store_2d(&maps.o1, sbuf + 2 * b * BOX + BOX, ti.n0 + 32 * ch, y);
        bulk_commit_group();
      }
    } else {
      if (lane < valid) {
        const int64_t off = row * p.f + ti.n0 + 32 * ch;
        const int ncol = min(32, p.f - (ti.n0 + 32 * ch));  // a multiple of 8
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (8 * j < ncol) {
            *reinterpret_cast<uint4*>(p.o0 + off + 8 * j) = pack8_bf16(dh1 + 8 * j);
            *reinterpret_cast<uint4*>(p.o1 + off + 8 * j) = pack8_bf16(dh2 + 8 * j);
          }
      }
      __syncwarp();
    }
  }
  if (!ok) {
    // leave no TMA copy in flight into this warp's buffers
    volatile int never = 0;
    for (int b = 0; b < 2; ++b)
      if ((pend >> b) & 1u) {
        wait_bounded(&lbar[b], (lphase >> b) & 1u, &never, kWaitLimit);
        lphase ^= 1u << b;
      }
  }
  return ok;
}

// One K16 step of a stage: MMA of the stage's A and B at K offset 16 * kk.
template <typename Tr, bool PAIR>
__device__ __forceinline__ void issue_mma(uint32_t dtm, uint32_t a_addr, uint32_t b_addr, int kk,
                                          uint32_t idesc, uint32_t accumulate) {
  const uint64_t adesc = Tr::A_MN ? umma_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                  : umma_desc_sw128(a_addr + kk * 32, 16, 1024);
  const uint64_t bdesc = Tr::B_MN ? umma_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                  : umma_desc_sw128(b_addr + kk * 32, 16, 1024);
  if (PAIR) mma_bf16_pair(dtm, adesc, bdesc, idesc, accumulate);
  else mma_bf16(dtm, adesc, bdesc, idesc, accumulate);
}

// The MMA issuer's wait for a stage: its TMA loads (and, in a gathered
// kernel, the odd CTA's relayed rows) on `full`, and this CTA's own gathered
// rows on `gfull`, made visible to the tensor core's operand reads.
template <bool GATHER>
__device__ __forceinline__ bool wait_stage(uint64_t* full, uint64_t* gfull, int stage,
                                           uint32_t phase, volatile int* abort) {
  if (GATHER) {
    if (!wait_bounded(&gfull[stage], phase, abort, kWaitLimit)) return false;
    fence_proxy_async_smem();
  }
  return wait_bounded(&full[stage], phase, abort, kWaitLimit);
}

template <int KIND, int BN, bool PAIR, bool GATHER>
__global__ void __launch_bounds__(Roles<KIND>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ Maps maps, const Params p) {
  using Tr = Traits<KIND, BN, PAIR>;
  static_assert(!GATHER || (PAIR && (KIND == kFwdGateUp || KIND == kWgrad)),
                "gathered A rows: the paired gate/up and weight-gradient kernels");
  constexpr int STAGES = Tr::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Tr::A_BYTES;
  uint8_t* sEpi = sB + STAGES * Tr::B_BYTES;  // 1024-aligned: stages are multiples of 1 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + Tr::EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* lbar = drain + 1;  // [8] SwiGLU-backward epilogue loads: two per epilogue warp
  uint64_t* gfull = lbar + 8;  // [STAGES] gathered kernels: this CTA's cp.async rows landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(gfull + STAGES);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_total = const_cast<int*>(s_abort) + 1;
  int* s_nlong = s_total + 1;
  int64_t* s_off = reinterpret_cast<int64_t*>(reinterpret_cast<uint8_t*>(bars) + Tr::BAR_BYTES);
  int* s_tstart = reinterpret_cast<int*>(s_off + p.E + 1);
  int* s_order = s_tstart + p.E + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = p.E, d = p.d, f = p.f;
  // a pair shares its tiles: tile t of the pair's sequence, CTA `cta` of it
  const int cta = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = cta == 0;
  const int first_tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // gathered kernels: the even CTA's producer arrival (with the TMA
      // bytes) and the odd CTA's relay of its gathered rows
      mbar_init(&full[s], GATHER ? 2 : 1);
      mbar_init(&empty[s], 1);
      if (GATHER) mbar_init(&gfull[s], 32);  // one cp.async arrival per producer lane
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      // the even CTA's MMA waits for the epilogues of both CTAs of a pair
      mbar_init(&tempty[a], 32 * Roles<KIND>::kEpiWarps * (PAIR ? 2 : 1));
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&lbar[i], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    // only the maps this kind fills in
    tma_prefetch_desc(&maps.a0);
    tma_prefetch_desc(&maps.b0);
    if (KIND == kBwdDgradGateUp || KIND == kWgrad) tma_prefetch_desc(&maps.a1);
    if (KIND == kFwdGateUp || KIND == kBwdDgradGateUp || KIND == kWgrad) tma_prefetch_desc(&maps.b1);
    if (KIND == kWgrad) tma_prefetch_desc(&maps.b2);
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(s_tmem, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s_tmem, kTmemCols);
      tmem_relinquish();
    }
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = p.offsets[e];
  __syncthreads();
  // schedule order: wgrad tiles have ragged K, so experts go longest first
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (KIND == kWgrad) {
      const int64_t c = s_off[e + 1] - s_off[e];
      int rank = 0;
      for (int e2 = 0; e2 < E; ++e2) {
        const int64_t c2 = s_off[e2 + 1] - s_off[e2];
        rank += (c2 > c) || (c2 == c && e2 < e);
      }
      s_order[rank] = e;
    } else {
      s_order[e] = e;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int s0 = 0; s0 < E; s0 += 32) {
      const int s = s0 + lane;
      int v = 0;
      if (s < E) {
        const int e = s_order[s];
        v = tiles_of_expert<KIND, BN, PAIR>(static_cast<int>(s_off[e + 1] - s_off[e]), d, f,
                                            p.accumulate);
      }
      int inc = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
      }
      if (s < E) s_tstart[s] = carry + inc - v;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    __syncwarp();
    if (lane == 0) {
      s_tstart[E] = carry;
      *s_total = carry;
      // slots run longest first: the long tiles end at the first short expert
      int nlong = carry;
      if (KIND == kWgrad)
        for (int s = 0; s < E; ++s)
          if (s_off[s_order[s] + 1] - s_off[s_order[s]] < kShortRows) {
            nlong = s_tstart[s];
            break;
          }
      *s_nlong = nlong;
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs of a pair have their barriers initialised before either signals the other's
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = *s_total;
  const Sched sched{s_off, s_tstart, s_order, E, total, *s_nlong, tile_step};

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // last load issued on full[s], and its phase
    // loads of both CTAs of a pair complete on the even CTA's full barriers
    const uint32_t full_leader = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;
    for (int tile = first_tile; tile < total && !*s_abort; tile += tile_step) {
      const TileInfo ti = decode_tile<KIND, BN, PAIR>(sched, tile, d, f);
      const int nk = num_kblocks<KIND, BN>(ti, d, f);
      // gathered A: the tokens of this lane's rows (gate/up: rows l + 32 q of
      // the CTA's 128, the same for all k blocks of the tile; wgrad: K rows
      // l + 32 q of the k block, read one block ahead so that the loads'
      // latency hides behind the stage wait)
      const bool gath = GATHER && (KIND == kFwdGateUp || ti.prod != 2);
      int tok[4] = {0, 0, 0, 0};
      if (gath) {
        const int r0 = KIND == kFwdGateUp ? ti.row0 + BM * cta : ti.row0;
#pragma unroll
        for (int q = 0; q < (KIND == kFwdGateUp ? 4 : 2); ++q) tok[q] = token_of_row(p, r0 + lane + 32 * q);
      }
      // the TMA bytes of a stage: without the gathered A rows
      const uint32_t stage_tx = gath ? Tr::STAGE_TX - (PAIR ? 2 : 1) * Tr::A_BYTES : Tr::STAGE_TX;
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, s_abort, kWaitLimit)) break;
        uint8_t* a_dst = sA + stage * Tr::A_BYTES;
        uint8_t* b_dst = sB + stage * Tr::B_BYTES;
        const uint32_t full_addr = full_leader + 8u * static_cast<uint32_t>(stage);
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
          if (PAIR) {
            issue_loads_pair<KIND, BN>(maps, ti, kb, d, f, cta, a_dst, b_dst, full_addr, !gath);
          } else {
            issue_loads<KIND, BN>(maps, ti, kb, d, f, a_dst, b_dst, &full[stage]);
          }
        }
        if (GATHER) {
          if (gath) {
            gather_a_stage<KIND>(p, lane, smem_u32(a_dst), kb * BK, ti.m0 + BM * cta, tok);
            if (KIND == kWgrad && kb + 1 < nk) {
              tok[0] = token_of_row(p, ti.row0 + (kb + 1) * BK + lane);
              tok[1] = token_of_row(p, ti.row0 + (kb + 1) * BK + lane + 32);
            }
          }
          // every stage of a gathered kernel completes gfull (with no copies
          // of this stage the arrival waits only for earlier ones)
          cp_async_mbar_arrive_noinc(&gfull[stage]);
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (GATHER) cp_async_wait_all();
    if (*s_abort) {
      // leave no copy in flight into shared memory that is about to be freed
      // (a pair's loads all count on the even CTA's barriers)
      volatile int never = 0;
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if ((issued_mask >> s) & 1u) wait_bounded(&full[s], (issued_par >> s) & 1u, &never, kWaitLimit);
    }
  } else if (warp == 1 && leader) {
    // ------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < total && !*s_abort; tile += tile_step, ++it) {
      const TileInfo ti = decode_tile<KIND, BN, PAIR>(sched, tile, d, f);
      const int nk = num_kblocks<KIND, BN>(ti, d, f);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, s_abort, kWaitLimit)) break;
      tc_fence_after();
      const uint32_t dtm = tmem_base + acc * BN;
      const uint32_t idesc = ti.narrow ? Tr::IDESC_NARROW : Tr::IDESC;
      // Full 64-deep K blocks: four MMAs each as straight-line code (a loop
      // with a run-time bound, or a branch, between them leaves the tensor
      // pipe idle between instructions).
      const int nfull = KIND == kWgrad ? ti.rows / BK : nk;
      for (int kb = 0; kb < nfull; ++kb) {
        if (!wait_stage<GATHER>(full, gfull, stage, phase, s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(sA + stage * Tr::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Tr::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            issue_mma<Tr, PAIR>(dtm, a_addr, b_addr, kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          // the stage is free in both CTAs once these MMAs have read it
          if (PAIR) mma_commit_pair_multicast(&empty[stage], 0x3);
          else mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (KIND == kWgrad && ok && nfull < nk) {
        // ragged-K tail block: rows past the expert's end belong to the next
        // expert (or lie past the tensor). Only the 16-row MMA steps that
        // hold valid rows run, and the invalid rows inside the last of them
        // are zeroed in both operands first.
        const int kb = nfull;
        if (!wait_stage<GATHER>(full, gfull, stage, phase, s_abort)) {
          ok = false;
        } else {
          tc_fence_after();
          const int valid = ti.rows - kb * BK;
          const int ksteps = (valid + 15) / 16;
          const int zrows = ksteps * 16 - valid;
          if (zrows > 0) {
            // each 64-column box holds one 128-byte row per K row, so the rows
            // to clear are one contiguous range per box; a pair's MMA also
            // reads the odd CTA's stage, which this warp clears through
            // distributed shared memory
            const uint32_t a_st = smem_u32(sA + stage * Tr::A_BYTES);
            const uint32_t b_st = smem_u32(sB + stage * Tr::B_BYTES);
            const int chunks = zrows * 8;  // 16-byte chunks per box
            constexpr int kBoxes = 2 + static_cast<int>(Tr::B_BYTES / 8192);
            for (int peer = 0; peer < (PAIR ? 2 : 1); ++peer) {
              for (int box = 0; box < kBoxes; ++box) {
                uint32_t base = (box < 2 ? a_st + box * 8192 : b_st + (box - 2) * 8192) + valid * 128;
                if (PAIR) base = mapa_shared(base, static_cast<uint32_t>(peer));
                for (int c = lane; c < chunks; c += 32) st_cluster_zero16(base + 16u * c);
              }
            }
            if (PAIR) fence_proxy_async_cluster();
            else fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(sA + stage * Tr::A_BYTES);
            const uint32_t b_addr = smem_u32(sB + stage * Tr::B_BYTES);
            for (int kk = 0; kk < ksteps; ++kk)
              issue_mma<Tr, PAIR>(dtm, a_addr, b_addr, kk, idesc, (kb | kk) != 0 ? 1u : 0u);
            if (PAIR) mma_commit_pair_multicast(&empty[stage], 0x3);
            else mma_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
      if (lane == 0) {
        if (PAIR) mma_commit_pair_multicast(&tfull[acc], 0x3);
        else mma_commit(&tfull[acc]);
      }
      __syncwarp();
    }
    // every MMA this thread issued has completed once `drain` flips
    if (lane == 0) {
      if (PAIR) mma_commit_pair_multicast(drain, 0x1);
      else mma_commit(drain);
    }
    __syncwarp();
    volatile int never = 0;
    wait_bounded(drain, 0, &never, kWaitLimit);
  } else if (GATHER && warp == 1) {
    // --------------------------------- odd CTA: relay of its gathered rows
    // The even CTA's MMA reads this CTA's A stage too; once this CTA's
    // cp.async rows of a stage have landed, pass that on to the even CTA's
    // full barrier (in the producer's stage order).
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
    bool ok = true;
    for (int tile = first_tile; ok && tile < total && !*s_abort; tile += tile_step) {
      const TileInfo ti = decode_tile<KIND, BN, PAIR>(sched, tile, d, f);
      const int nk = num_kblocks<KIND, BN>(ti, d, f);
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_bounded(&gfull[stage], phase, s_abort, kWaitLimit)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();
        if (lane == 0) mbar_arrive_cluster(full_leader + 8u * static_cast<uint32_t>(stage));
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp >= 2) {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;
    // with eight epilogue warps each handles half of the columns
    constexpr int kSplit = Roles<KIND>::kEpiWarps / 4;
    const int c0 = ((warp - 2) >> 2) * ((KIND == kFwdGateUp ? 128 : BN) / kSplit);
    const uint32_t tempty_leader = PAIR ? mapa_shared(smem_u32(tempty), 0) : 0u;
    int ebuf = 0;         // TMA-stored epilogues: staging buffer of the next 32-column chunk
    uint32_t lphase = 0;  // SwiGLU-backward epilogue: parity of this warp's two load barriers
    int it = 0;
    for (int tile = first_tile; tile < total && !*s_abort; tile += tile_step, ++it) {
      const TileInfo ti = decode_tile<KIND, BN, PAIR>(sched, tile, d, f);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!wait_bounded(&tfull[acc], acc_phase, s_abort, kWaitLimit)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      if constexpr (Tr::EPI_TMA) {
        epilogue_tma<KIND, BN>(p, maps, ti, tacc, BM * cta + q * 32, lane,
                               sEpi + (warp - 2) * Tr::EPI_WARP_BYTES, ebuf);
      } else if constexpr (KIND == kBwdDgradDown) {
        if (!epilogue_swiglu_bwd<BN>(p, maps, ti, tacc, BM * cta + q * 32, lane,
                                     sEpi + (warp - 2) * Tr::EPI_WARP_BYTES, lbar + 2 * (warp - 2),
                                     lphase, s_abort))
          break;
      } else {
        epilogue_wgrad<BN>(p, ti, tacc, BM * cta + q * 32 + lane, c0);
      }
      tc_fence_before();
      if (PAIR) mbar_arrive_cluster(tempty_leader + 8u * static_cast<uint32_t>(acc));
      else mbar_arrive(&tempty[acc]);
    }
    // this warp's TMA stores have finished before the CTA may exit
    if (Tr::EPI_TMA || KIND == kBwdDgradDown) {
      if (lane == 0) bulk_wait_group<0>();
      __syncwarp();
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // neither CTA of a pair leaves while the other may still read its shared
  // memory or write its TMEM
  if (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0 && *s_abort) raise_error(p.err, kErrTimeout);
}

// ------------------------------------------------------------------ host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D bf16 tensor [outer, inner] (inner contiguous, row pitch `pitch` elements),
// box [box_outer, box_inner], 128-byte swizzle unless given, out-of-bounds
// reads as zero.
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 tensor [outer, mid, inner] (inner contiguous, dense), box
// [1, box_mid, box_inner], 128-byte swizzle, out-of-bounds reads as zero: the
// expert weights, so that rows past one expert's matrix read as zero rather
// than as the next expert's rows.
static bool make_map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                      uint32_t box_inner, uint32_t box_mid) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {box_inner, box_mid, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of an epilogue's TMA boxes: [rows, cols] bf16, 32 x 32 boxes, 64-byte swizzle.
static bool make_store_map(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows) {
  return make_map(m, base, cols, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

static int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int KIND, int BN, bool PAIR, bool GATHER = false>
static cudaError_t launch(const Maps& m, const Params& p, cudaStream_t s) {
  using Tr = Traits<KIND, BN, PAIR>;
  static_assert(Tr::smem_bytes(kMaxE) <= 232448, "shared memory of one CTA");
  auto kern = grouped_gemm_kernel<KIND, BN, PAIR, GATHER>;
  const size_t smem = Tr::smem_bytes(p.E);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (!PAIR) {
    kern<<<sm_count(), Roles<KIND>::kThreads, smem, s>>>(m, p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sm_count() / 2 * 2));
  cfg.blockDim = dim3(Roles<KIND>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // every pair must be resident at once: the tile sequence of a pair that
  // starts late would finish a whole wave after the others
  static int resident_pairs = 0;
  if (resident_pairs == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) != cudaSuccess)
      n = 0;
    resident_pairs = n > 0 ? n : -1;
  }
  if (resident_pairs > 0 && static_cast<unsigned>(2 * resident_pairs) < cfg.gridDim.x)
    cfg.gridDim = dim3(static_cast<unsigned>(2 * resident_pairs));
  return cudaLaunchKernelEx(&cfg, kern, m, p);
}


}  // namespace gg

// [h1 | h2] = xp [Wg_e | Wu_e]^T and a = silu(h1) h2; each of h1, h2, a is
// stored only if its pointer is set (a checkpointed forward keeps only a; its
// backward recomputes h1 and h2 alone).
cudaError_t launch_ffn_gateup_bf16(const FfnFwdArgs& a, cudaStream_t s) {
  using namespace gg;
  const uint64_t rows = static_cast<uint64_t>(a.rows), E = a.E, d = a.d, f = a.f;
  Params p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.d = a.d;
  p.f = a.f;
  p.err = a.err;
  Maps m1{};
  const bool gather = a.gather.rows != nullptr;
  // gathered: the kernel reads x [T, d] itself (the map stays valid but unused)
  if (!(gather ? make_map(&m1.a0, a.xp, d, static_cast<uint64_t>(a.gather.T), d, 64, 1)
               : make_map(&m1.a0, a.xp, d, rows, d, 64, 128)) ||
      !make_map3(&m1.b0, a.Wg, d, f, E, 64, 128) || !make_map3(&m1.b1, a.Wu, d, f, E, 64, 128))
    return cudaErrorInvalidValue;
  p.gx = static_cast<const bf16*>(a.xp);
  p.grow = a.gather.rows;
  p.gk = a.gather.k;
  p.grows = static_cast<int>(a.rows);
  p.gT = static_cast<int>(a.gather.T);
  p.o0 = static_cast<bf16*>(a.h1);
  p.o1 = static_cast<bf16*>(a.h2);
  p.o2 = static_cast<bf16*>(a.a);
  if ((a.h1 && !make_store_map(&m1.o0, a.h1, f, rows)) ||
      (a.h2 && !make_store_map(&m1.o1, a.h2, f, rows)) ||
      (a.a && !make_store_map(&m1.o2, a.a, f, rows)))
    return cudaErrorInvalidValue;
  return gather ? launch<kFwdGateUp, 256, true, true>(m1, p, s) : launch<kFwdGateUp, 256, true>(m1, p, s);
}

cudaError_t launch_ffn_fwd_bf16(const FfnFwdArgs& a, cudaStream_t s) {
  using namespace gg;
  const uint64_t rows = static_cast<uint64_t>(a.rows), E = a.E, d = a.d, f = a.f;
  cudaError_t e = launch_ffn_gateup_bf16(a, s);
  if (e != cudaSuccess) return e;
  Params p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.d = a.d;
  p.f = a.f;
  p.err = a.err;
  Maps m2{};
  // pairs: each CTA stages 128 of the tile's 256 Wd rows
  if (!make_map(&m2.a0, a.a, f, rows, f, 64, 128) || !make_map3(&m2.b0, a.Wd, f, d, E, 64, 128))
    return cudaErrorInvalidValue;
  p.o0 = static_cast<bf16*>(a.yp);
  p.o1 = p.o2 = nullptr;
  if (!make_store_map(&m2.o0, a.yp, d, rows)) return cudaErrorInvalidValue;
  return launch<kFwdDown, 256, true>(m2, p, s);
}

static gg::Params bwd_params(const FfnBwdArgs& a) {
  gg::Params p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.d = a.d;
  p.f = a.f;
  p.err = a.err;
  return p;
}

cudaError_t launch_ffn_dgrad_bf16(const FfnBwdArgs& a, cudaStream_t s) {
  using namespace gg;
  const uint64_t rows = static_cast<uint64_t>(a.rows), E = a.E, d = a.d, f = a.f;
  Params p = bwd_params(a);
  // 1. da = dyp Wd_e, SwiGLU backward in the epilogue -> dh1, dh2
  Maps m1{};
  if (!make_map(&m1.a0, a.dyp, d, rows, d, 64, 128) || !make_map3(&m1.b0, a.Wd, f, d, E, 64, 64))
    return cudaErrorInvalidValue;
  p.i0 = static_cast<const bf16*>(a.h1);
  p.i1 = static_cast<const bf16*>(a.h2);
  p.o0 = static_cast<bf16*>(a.dh1);
  p.o1 = static_cast<bf16*>(a.dh2);
  // the epilogue's h1 / h2 loads and dh1 / dh2 stores: 32 x 32 boxes
  if (!make_store_map(&m1.a1, const_cast<void*>(a.h1), f, rows) ||
      !make_store_map(&m1.b1, const_cast<void*>(a.h2), f, rows) ||
      !make_store_map(&m1.o0, a.dh1, f, rows) || !make_store_map(&m1.o1, a.dh2, f, rows))
    return cudaErrorInvalidValue;
  // 256-wide tiles even when f is not a multiple of 256 (a half-empty edge
  // tile costs less than the narrower MMA everywhere else)
  cudaError_t e = launch<kBwdDgradDown, 256, true>(m1, p, s);
  if (e != cudaSuccess) return e;
  // 2. dxp = dh1 Wg_e + dh2 Wu_e
  Maps m2{};
  if (!make_map(&m2.a0, a.dh1, f, rows, f, 64, 128) || !make_map(&m2.a1, a.dh2, f, rows, f, 64, 128) ||
      !make_map3(&m2.b0, a.Wg, d, f, E, 64, 64) || !make_map3(&m2.b1, a.Wu, d, f, E, 64, 64))
    return cudaErrorInvalidValue;
  p.i0 = p.i1 = nullptr;
  p.o0 = static_cast<bf16*>(a.dxp);
  p.o1 = nullptr;
  if (!make_store_map(&m2.o0, a.dxp, d, rows)) return cudaErrorInvalidValue;
  return launch<kBwdDgradGateUp, 256, true>(m2, p, s);
}

cudaError_t launch_ffn_wgrad_bf16(const FfnBwdArgs& a, cudaStream_t s) {
  using namespace gg;
  const uint64_t rows = static_cast<uint64_t>(a.rows), d = a.d, f = a.f;
  Params p = bwd_params(a);
  Maps m3{};
  const bool gather = a.gather.rows != nullptr;
  if (!(gather ? make_map(&m3.a0, a.xp, d, static_cast<uint64_t>(a.gather.T), d, 64, 1)
               : make_map(&m3.a0, a.xp, d, rows, d, 64, 64)) ||
      !make_map(&m3.a1, a.a, f, rows, f, 64, 64) ||
      !make_map(&m3.b0, a.dh1, f, rows, f, 64, 64) || !make_map(&m3.b1, a.dh2, f, rows, f, 64, 64) ||
      !make_map(&m3.b2, a.dyp, d, rows, d, 64, 64))
    return cudaErrorInvalidValue;
  p.w0 = a.dWg;
  p.w1 = a.dWu;
  p.w2 = a.dWd;
  p.accumulate = a.accumulate;
  p.gx = static_cast<const bf16*>(a.xp);
  p.grow = a.gather.rows;
  p.gk = a.gather.k;
  p.grows = static_cast<int>(a.rows);
  p.gT = static_cast<int>(a.gather.T);
  // CTA pairs: six stages of 32 KB per CTA hide more load latency than four
  // of 48 KB
  return gather ? launch<kWgrad, 256, true, true>(m3, p, s) : launch<kWgrad, 256, true>(m3, p, s);
}

}  // namespace moe

namespace moe {

// One block waits on an mbarrier nothing arrives at, with the bounded wait
// of the GEMM pipelines, and reports the time-out through the error word.
__global__ void selftest_wait_timeout_kernel(unsigned* err, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = sm100::wait_bounded(&bar, 0, &abort_flag, limit);
    if (!ok) raise_error(err, kErrTimeout);
  }
}

cudaError_t launch_selftest_wait_timeout(unsigned* err, long long limit, cudaStream_t s) {
  selftest_wait_timeout_kernel<<<1, 32, 0, s>>>(err, limit);
  return cudaGetLastError();
}

}  // namespace moe
