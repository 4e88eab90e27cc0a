// select_sm100.cuh - pre-pass block selector that produces the static block
// mask the prefill kernel takes (the block-sparse input), CRISP-style.
//
// What it computes (the CRISP review at rit.work, blog/crisp-sparse-attention-
// long-prefill, section "What was done", paragraphs 3-5; the constants and
// formulas are readings, the page gives none):
//   - a block-pooled estimate of the attention map: per head, qb_t = mean of
//     the query rows of tile t, kb_j = mean of the keys of block j, and
//     A[t][j] = softmax over the blocks visible from tile t of scale*qb_t.kb_j;
//   - C_struct = mean over the head's tiles of A[t][0] + A[t][last(t)] (the
//     initial positions and the local window; last(t) = the tile's last
//     visible block), which routes the head: structured when C_struct >= tau;
//   - structured path: keep block 0 and last(t), and the blocks in between
//     whose A is above their mean (the background mass);
//   - pooled path: keep the blocks with the largest A until they cover gamma
//     of the row (every block tied with the last one taken is kept too).
// Output: uint8 mask [B, Hq, nQt, nKt], 0 = selected, 1 = not (invisible
// blocks are 1): the prefill's block_mask_in convention.
//
// Three small kernels: pooled means (one CTA per tile or block; reads Q and
// K once, HBM-bound), row statistics (one warp per tile row of the map: the
// scores, kept for the next kernel, their max, normaliser and the row's
// C_struct term), selection (one warp per tile row, reading the scores back:
// the head's C_struct summed in a fixed order, the route, then the row's
// blocks; the cumulative threshold is found by bisection on the float bits of
// the map values, which picks the same set as sorting and taking a prefix).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace blasst {

struct SelectParams {
  const __nv_bfloat16* q;  // [B, Hq, Lq, d]
  const __nv_bfloat16* k;  // [B, Hkv, Lkv, d]
  float* qbar;             // [B*Hq, nQt, d]
  float* kbar;             // [B*Hkv, nKt, d]
  float* rowst;            // [B*Hq, nQt, 3]: max score, normaliser, C_struct term
  float* scores;           // [B*Hq, nQt, nKt]: scale * qb_t . kb_j of visible blocks
  uint8_t* mask;           // [B, Hq, nQt, nKt]
  float* cstruct;          // [B, Hq] or null
  int B, Hq, Hkv, Lq, Lkv, d, g;
  int Br, Bc, nQt, nKt;
  int causal, off;
  float scale, tau, gamma;
};

constexpr int SEL_MAXJ = 64;  // map values per lane: nKt <= 32 * 64 = 2048

// Last block visible from tile t (bottom-right causal alignment).
__device__ __forceinline__ int sel_last_block(const SelectParams& p, int t) {
  if (!p.causal) return p.nKt - 1;
  const int r1 = min((t + 1) * p.Br, p.Lq);
  return min((r1 - 1 + p.off) / p.Bc, p.nKt - 1);
}

// Mean of rows [r0, r1) of a [rows, d] bf16 matrix into out[d]; 128 threads,
// 16-byte loads, d / 8 threads per row.
__global__ void __launch_bounds__(128) blasst_select_pool_kernel(SelectParams p) {
  __shared__ float part[128 / 8][128];  // [row group][dim]
  const bool is_q = blockIdx.x < static_cast<unsigned>(p.B * p.Hq * p.nQt);
  int head, tile, rows, L, R;
  const __nv_bfloat16* src;
  float* dst;
  if (is_q) {
    head = blockIdx.x / p.nQt;
    tile = blockIdx.x % p.nQt;
    L = p.Lq;
    R = p.Br;
    src = p.q;
    dst = p.qbar + (static_cast<size_t>(head) * p.nQt + tile) * p.d;
  } else {
    const int id = blockIdx.x - p.B * p.Hq * p.nQt;
    head = id / p.nKt;
    tile = id % p.nKt;
    L = p.Lkv;
    R = p.Bc;
    src = p.k;
    dst = p.kbar + (static_cast<size_t>(head) * p.nKt + tile) * p.d;
  }
  const int r0 = tile * R;
  rows = min(R, L - r0);
  const int tpr = p.d / 8;          // threads per row (8 dims each)
  const int rpi = 128 / tpr;        // rows per iteration
  const int grp = threadIdx.x / tpr;
  const int c = threadIdx.x % tpr;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const __nv_bfloat16* base = src + (static_cast<size_t>(head) * L + r0) * p.d + 8 * c;
  for (int r = grp; r < rows; r += rpi) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * p.d);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(h[u]);
      acc[2 * u] += f.x;
      acc[2 * u + 1] += f.y;
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) part[grp][8 * c + u] = acc[u];
  __syncthreads();
  if (threadIdx.x < p.d) {
    float s = 0.0f;
    for (int gi = 0; gi < rpi; ++gi) s += part[gi][threadIdx.x];
    dst[threadIdx.x] = s / static_cast<float>(rows);
  }
}

__device__ __forceinline__ float sel_warp_sum(float v) {
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
  return v;
}
__device__ __forceinline__ float sel_warp_max(float v) {
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, sh));
  return v;
}

// Row statistics. One CTA per (b, hq, 8 consecutive tiles), one warp per
// tile row; the head's pooled keys are staged transposed in shared memory 32
// blocks at a time, so lane l of every warp reads block (32 c + l) without
// bank conflicts and each pooled key is read from L2 once per CTA.
__global__ void __launch_bounds__(256) blasst_select_rows_kernel(SelectParams p) {
  __shared__ __align__(16) float qs[8][128];
  __shared__ __align__(16) float kT[128][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntg = (p.nQt + 7) / 8;
  const int bh = static_cast<int>(blockIdx.x) / ntg;
  const int t0 = (static_cast<int>(blockIdx.x) % ntg) * 8;
  const int t = t0 + w;
  const bool active = t < p.nQt;
  const int hk = (bh % p.Hq) / p.g + (bh / p.Hq) * p.Hkv;
  const size_t row = static_cast<size_t>(bh) * p.nQt + t;
  if (active)
    for (int x = lane; x < p.d; x += 32) qs[w][x] = p.qbar[row * p.d + x];
  const int nvis = active ? sel_last_block(p, t) + 1 : 0;
  const int nv_max = sel_last_block(p, min(t0 + 7, p.nQt - 1)) + 1;  // nondecreasing in t
  const float4* kb4 = reinterpret_cast<const float4*>(p.kbar + static_cast<size_t>(hk) * p.nKt * p.d);
  const int d4 = p.d / 4;
  float s[SEL_MAXJ];
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) s[m] = -INFINITY;
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) {
    if (32 * m >= nv_max) break;
    __syncthreads();  // the previous chunk has been read (and qs written)
    for (int e = threadIdx.x; e < 32 * d4; e += 256) {
      const int jj = e & 31, x4 = e >> 5, j = 32 * m + jj;
      const float4 v = j < p.nKt ? kb4[static_cast<size_t>(j) * d4 + x4] : make_float4(0, 0, 0, 0);
      kT[4 * x4][jj] = v.x;
      kT[4 * x4 + 1][jj] = v.y;
      kT[4 * x4 + 2][jj] = v.z;
      kT[4 * x4 + 3][jj] = v.w;
    }
    __syncthreads();
    if (32 * m < nvis) {
      float dot = 0.0f;
      for (int x = 0; x < p.d; ++x) dot = fmaf(qs[w][x], kT[x][lane], dot);
      if (32 * m + lane < nvis) s[m] = p.scale * dot;
    }
  }
  if (!active) return;
  float* srow = p.scores + row * p.nKt;
  float mx = -INFINITY;
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) {
    if (32 * m >= nvis) break;
    if (lane + 32 * m < nvis) srow[lane + 32 * m] = s[m];
    mx = fmaxf(mx, s[m]);
  }
  mx = sel_warp_max(mx);
  float z = 0.0f;
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) {
    if (32 * m >= nvis) break;
    if (s[m] > -INFINITY) z += expf(s[m] - mx);
  }
  z = sel_warp_sum(z);
  // C_struct term: A[t][0] + A[t][last] (A[t][0] once when they coincide)
  const int jl = nvis - 1;
  float term = 0.0f;
  if (lane == 0) term += expf(s[0] - mx) / z;
  if (jl > 0 && lane == (jl & 31)) {
#pragma unroll
    for (int m = 0; m < SEL_MAXJ; ++m)
      if (m == (jl >> 5)) term += expf(s[m] - mx) / z;
  }
  term = sel_warp_sum(term);
  if (lane == 0) {
    float* st = p.rowst + row * 3;
    st[0] = mx;
    st[1] = z;
    st[2] = term;
  }
}

// Selection: one warp per (b, hq, t).
__global__ void __launch_bounds__(256) blasst_select_mask_kernel(SelectParams p) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + w;
  if (row >= static_cast<long long>(p.B) * p.Hq * p.nQt) return;
  const int bh = static_cast<int>(row / p.nQt), t = static_cast<int>(row % p.nQt);
  // the head's C_struct, summed in tile order by lane-strided partial sums
  float cs = 0.0f;
  for (int tt = lane; tt < p.nQt; tt += 32)
    cs += p.rowst[(static_cast<size_t>(bh) * p.nQt + tt) * 3 + 2];
  cs = sel_warp_sum(cs) / static_cast<float>(p.nQt);
  const bool structured = cs >= p.tau;
  if (t == 0 && lane == 0 && p.cstruct) p.cstruct[bh] = cs;
  const int nvis = sel_last_block(p, t) + 1;
  const float* srow = p.scores + static_cast<size_t>(row) * p.nKt;
  const float mx = p.rowst[static_cast<size_t>(row) * 3];
  const float z = p.rowst[static_cast<size_t>(row) * 3 + 1];
  float a[SEL_MAXJ];
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) a[m] = -1.0f;
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) {
    if (32 * m >= nvis) break;
    const int j = lane + 32 * m;
    if (j < nvis) a[m] = expf(srow[j] - mx) / z;
  }
  const int jl = nvis - 1;
  float thr;        // keep A > thr (structured) or A >= thr (pooled)
  bool strict;
  if (structured) {
    float bg = 0.0f;
#pragma unroll
    for (int m = 0; m < SEL_MAXJ; ++m) {
      if (32 * m >= nvis) break;
      const int j = lane + 32 * m;
      if (j >= 1 && j < jl) bg += a[m];
    }
    bg = sel_warp_sum(bg);
    thr = jl >= 2 ? bg / static_cast<float>(jl - 1) : INFINITY;
    strict = true;
  } else {
    // largest theta (a map value) with sum_{A >= theta} A >= gamma: bisection
    // on the bits of non-negative floats, which order like the floats
    uint32_t lo = 0u, hi = 0x7f800000u;  // mass(0) = 1 >= gamma; mass(inf) = 0
    for (int it = 0; it < 32 && hi - lo > 1u; ++it) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      const float th = __uint_as_float(mid);
      float mass = 0.0f;
#pragma unroll
      for (int m = 0; m < SEL_MAXJ; ++m) {
        if (32 * m >= nvis) break;
        if (a[m] >= th) mass += a[m];
      }
      mass = sel_warp_sum(mass);
      if (mass >= p.gamma) lo = mid;
      else hi = mid;
    }
    thr = __uint_as_float(lo);
    strict = false;
  }
  uint8_t* mrow = p.mask + static_cast<size_t>(row) * p.nKt;
#pragma unroll
  for (int m = 0; m < SEL_MAXJ; ++m) {
    const int j = lane + 32 * m;
    if (32 * m >= p.nKt) break;
    bool sel = false;
    if (j <= jl) {
      const float v = a[m];
      if (structured) sel = (j == 0 || j == jl) || (strict ? v > thr : v >= thr);
      else sel = v >= thr;
    }
    if (j < p.nKt) mrow[j] = sel ? 0 : 1;
  }
}

}  // namespace blasst
