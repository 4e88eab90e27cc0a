// decode_sm100.cuh - split-KV decode with softmax thresholding, and the
// log-sum-exp merge of the splits.
//
// Decode reads a contiguous KV cache ("В тени длинного контекста ...",
// denisavetisyan.com LongCA-bench review, closing section on the KV cache).
// The skip rule is the one of "BLASST: Dynamic BLocked Attention Sparsity via
// Softmax Thresholding" (Telegram channel seeallochnaya, post 3655,
// paragraphs 3-6 after the headline): with one query row per head, a tile is
// one row, so the test exp(m_blk - m_run) < lambda is taken per head and per
// KV block, against the running max of the split; the first block of every
// split is always computed. A block's V rows are fetched only if some head of
// the GQA group keeps the block.
//
// Work split: one CTA of 128 threads per (split, KV head, sequence), holding
// the G = Hq/Hkv query heads of the group. K blocks stream through a TMA ring
// (128-byte swizzled tiles, so a thread reading one key row is bank-conflict
// free); scores on the FMA pipes (M = G rows is far too short for the tensor
// cores, and the kernel is bound by HBM bytes, not by arithmetic).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/blasst.h"
#include "ptx_sm100.cuh"

namespace blasst {

struct DecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, d]
  float* o_parts;          // [B, Hq, S, d]
  float* lse_parts;        // [B, Hq, S]  (natural log, -inf for an empty split)
  uint8_t* mask;           // [B, Hq, nKt] or null
  blasst_stats* stats;
  int* err;
  int B, Hq, Hkv, Lkv, S, Ls, nKt;
  float scale_log2;
  float log2_lambda;
  uint64_t timeout_ns;
};

template <int D, int BC, int G>
struct DecodeCfg {
  static constexpr int NT = 128;
  static constexpr int NK = 2;          // K ring stages
  static constexpr int DBOX = D / 64;
  static constexpr int KV_BOX = BC * 128;
  static constexpr int KV_BYTES = KV_BOX * DBOX;
  static constexpr int CPR = D / 8;     // 16-byte chunks per key row
  static constexpr int KG = NT / CPR;   // key groups in the P.V phase
  static constexpr int RPT = BC / KG;   // rows per thread in the P.V phase
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  // After the last block the K/V ring is idle and holds the final reduction
  // of the KG partial O accumulators (KG x G x D fp32).
  static constexpr int RING_BYTES = (NK + 1) * KV_BYTES > KG * G * D * 4 ? (NK + 1) * KV_BYTES
                                                                         : KG * G * D * 4;
  static constexpr int OFF_Q = OFF_K + RING_BYTES;         // G x D fp32 (pre-scaled)
  static constexpr int OFF_P = OFF_Q + G * D * 4;          // G x BC fp32 weights
  // block maxima (2 x 4 warps x G, double-buffered) then block sums (4 x G)
  static constexpr int OFF_RED = OFF_P + G * BC * 4;
  static constexpr int OFF_BAR = (OFF_RED + 12 * G * 4 + 7) & ~7;
  static constexpr int NBAR = NK + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(BC % KG == 0, "rows per thread");
};

template <int D, int BC, int G>
__global__ void __launch_bounds__(128)
    blasst_decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecodeCfg<D, BC, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  float* qs = reinterpret_cast<float*>(smem + C::OFF_Q);
  float* ps = reinterpret_cast<float*>(smem + C::OFF_P);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + C::NBAR * 8);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int bhk = b * p.Hkv + hk;
  const int k0 = split * p.Ls;
  const int k1 = min(k0 + p.Ls, p.Lkv);
  const int nblk = k1 > k0 ? (k1 - k0 + BC - 1) / BC : 0;
  const bool thresholding = p.log2_lambda > -INFINITY;

  if (t == 0) {
    for (int i = 0; i < C::NBAR; ++i) ptx::mbar_init(bar(i), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  // Q rows of the group, pre-multiplied by scale*log2(e).
  for (int i = t; i < G * D; i += C::NT) {
    const int h = i / D, x = i % D;
    const int hq = hk * G + h;
    qs[i] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.Hq + hq) * D + x]) * p.scale_log2;
  }
  __syncthreads();

  auto load_tile = [&](const CUtensorMap* tm, uint32_t dst, int key0, uint32_t fb) {
    ptx::mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::DBOX; ++bx) ptx::tma_load_3d(dst + bx * C::KV_BOX, tm, bx * 64, key0, bhk, fb);
  };
  if (t == 0) {
    for (int i = 0; i < min(C::NK, nblk); ++i)
      load_tile(&tmK, sb + C::OFF_K + i * C::KV_BYTES, k0 + i * BC, bar(i));
  }

  float m[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.0f;
  }
  // P.V accumulators: thread owns chunk c (8 dims) of rows kg, kg+KG, ...
  const int c = t % C::CPR, kg = t / C::CPR;
  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[h][i] = 0.0f;

  int vphase = 0;
  unsigned long long st_vis = 0, st_skip = 0, st_vload = 0, st_flops = 0;
  bool ok = true;

  for (int i = 0; i < nblk; ++i) {
    const int key0 = k0 + i * BC;
    const int stage = i % C::NK;
    bool w = true;
    if (lane == 0) w = ptx::mbar_wait(bar(stage), (i / C::NK) & 1, abort_flag, p.timeout_ns);
    w = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    if (!w) *abort_flag = 1;
    // ---- scores: thread t <-> key t of the block --------------------------
    float s[G];
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = 0.0f;
    const bool key_ok = (t < BC) && (key0 + t < k1);
    if (t < BC) {
      const uint8_t* kst = smem + C::OFF_K + stage * C::KV_BYTES;
#pragma unroll
      for (int bx = 0; bx < C::DBOX; ++bx) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 raw = *reinterpret_cast<const uint4*>(kst + bx * C::KV_BOX + t * 128 +
                                                            ((ch ^ (t & 7)) << 4));
          const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
          float kf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kf[2 * e] = __uint_as_float(wds[e] << 16);
            kf[2 * e + 1] = __uint_as_float(wds[e] & 0xffff0000u);
          }
          const int x0 = bx * 64 + ch * 8;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float4 qa = *reinterpret_cast<const float4*>(qs + h * D + x0);
            const float4 qb = *reinterpret_cast<const float4*>(qs + h * D + x0 + 4);
            float a = s[h];
            a = fmaf(qa.x, kf[0], a);
            a = fmaf(qa.y, kf[1], a);
            a = fmaf(qa.z, kf[2], a);
            a = fmaf(qa.w, kf[3], a);
            a = fmaf(qb.x, kf[4], a);
            a = fmaf(qb.y, kf[5], a);
            a = fmaf(qb.z, kf[6], a);
            a = fmaf(qb.w, kf[7], a);
            s[h] = a;
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (!key_ok) s[h] = -INFINITY;
    // ---- block max per head -------------------------------------------------
    float* redm = red + (i & 1) * 4 * G;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = s[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) redm[warp * G + h] = v;
    }
    __syncthreads();  // K stage fully read; block maxima visible
    float mb[G];
    int keepmask = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mb[h] = fmaxf(fmaxf(redm[h], redm[G + h]), fmaxf(redm[2 * G + h], redm[3 * G + h]));
      const bool skip = (i > 0) && thresholding && (mb[h] - m[h] < p.log2_lambda);
      if (!skip) keepmask |= 1 << h;
    }
    if (*abort_flag) {
      ok = false;
      break;
    }
    if (t == 0) {
      if (keepmask) load_tile(&tmV, sb + C::OFF_V, key0, bar(C::NK));
      if (i + C::NK < nblk) load_tile(&tmK, sb + C::OFF_K + stage * C::KV_BYTES, key0 + C::NK * BC, bar(stage));
      st_vis += G;
      st_skip += G - __popc(keepmask);
      st_vload += keepmask ? 1 : 0;
      st_flops += 2ull * G * BC * D + 2ull * __popc(keepmask) * BC * D;
    }
    if (p.mask && t < G) {
      const int hq = hk * G + t;
      p.mask[(static_cast<size_t>(b) * p.Hq + hq) * p.nKt + key0 / BC] = ((keepmask >> t) & 1) ? 0 : 1;
    }
    if (!keepmask) continue;  // skipped by every head: no V bytes, no P.V

    // ---- online softmax for the heads that keep the block -------------------
    float alpha[G];
    float* reds = red + 8 * G;  // second reduction area (sums)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const bool kh = (keepmask >> h) & 1;
      const float m_new = kh ? fmaxf(m[h], mb[h]) : m[h];
      alpha[h] = (kh && m[h] != m_new) ? ptx::ex2(m[h] - m_new) : 1.0f;
      const float pv = kh ? ptx::ex2(s[h] - m_new) : 0.0f;
      if (t < BC) ps[h * BC + t] = pv;
      float v = pv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) reds[warp * G + h] = v;
      m[h] = m_new;
    }
    bool vw = true;
    if (lane == 0) vw = ptx::mbar_wait(bar(C::NK), vphase & 1, abort_flag, p.timeout_ns);
    vw = __shfl_sync(0xffffffffu, vw ? 1 : 0, 0) != 0;
    ++vphase;
    if (!vw) *abort_flag = 1;
    __syncthreads();  // P weights and partial sums visible, V landed
#pragma unroll
    for (int h = 0; h < G; ++h) {
      l[h] = l[h] * alpha[h] + (reds[h] + reds[G + h] + reds[2 * G + h] + reds[3 * G + h]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] *= alpha[h];
    }
    // ---- O += P V: rows kg, kg+KG, ... ; dims [8c, 8c+8) -----------------
    {
      const uint8_t* vst = smem + C::OFF_V;
      const int bx = (c * 8) / 64;
      const int chk = c & 7;
#pragma unroll 4
      for (int r = 0; r < C::RPT; ++r) {
        const int j = kg + r * C::KG;
        const uint4 raw = *reinterpret_cast<const uint4*>(vst + bx * C::KV_BOX + j * 128 + ((chk ^ (j & 7)) << 4));
        const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
        float vf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          vf[2 * e] = __uint_as_float(wds[e] << 16);
          vf[2 * e + 1] = __uint_as_float(wds[e] & 0xffff0000u);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pw = ps[h * BC + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(pw, vf[e], acc[h][e]);
        }
      }
    }
    __syncthreads();  // V stage and weights free for the next block
  }

  // ---- reduce the KG partial accumulators, write the split's partials -----
  __syncthreads();
  float* oacc = reinterpret_cast<float*>(smem + C::OFF_K);  // K/V ring is idle now
  if (ok && !*abort_flag) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) oacc[(kg * G + h) * D + c * 8 + e] = acc[h][e];
  }
  __syncthreads();
  if (ok && !*abort_flag) {
    for (int i = t; i < G * D; i += C::NT) {
      const int h = i / D, x = i % D;
      float v = 0.0f;
      for (int k = 0; k < C::KG; ++k) v += oacc[(k * G + h) * D + x];
      const int hq = hk * G + h;
      const size_t prow = (static_cast<size_t>(b) * p.Hq + hq) * p.S + split;
      const bool has = l[h] > 0.0f;
      p.o_parts[prow * D + x] = has ? v / l[h] : 0.0f;
      if (x == 0) p.lse_parts[prow] = has ? (m[h] + log2f(l[h])) * 0.6931471805599453f : -INFINITY;
    }
    if (t == 0 && p.stats) {
      const unsigned long long kvb = static_cast<unsigned long long>(BC) * D * 2ull;
      atomicAdd(&p.stats->tiles_visited, st_vis);
      atomicAdd(&p.stats->tiles_skipped, st_skip);
      atomicAdd(&p.stats->v_blocks_loaded, st_vload);
      atomicAdd(&p.stats->mma_flops, st_flops);
      atomicAdd(&p.stats->bytes_loaded, kvb * (nblk + st_vload));
    }
  } else if (t == 0) {
    if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
  }
}

// o = sum_s w_s o_s / sum_s w_s, lse = M + ln(sum_s w_s), w_s = exp(lse_s - M).
// One CTA per row; thread x handles output dims x, x + blockDim, ...
template <typename OutT>
__global__ void blasst_lse_merge_kernel(const float* __restrict__ o_parts,
                                        const float* __restrict__ lse_parts, OutT* __restrict__ o,
                                        float* __restrict__ lse, int d, int S) {
  const int row = blockIdx.x;
  const float* lp = lse_parts + static_cast<size_t>(row) * S;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, lp[s]);
  float wsum = 0.0f;
  for (int s = 0; s < S; ++s) wsum += (lp[s] == -INFINITY) ? 0.0f : expf(lp[s] - M);
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  for (int x = threadIdx.x; x < d; x += blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < S; ++s) {
      const float ls = lp[s];
      if (ls == -INFINITY) continue;
      acc = fmaf(expf(ls - M), o_parts[(static_cast<size_t>(row) * S + s) * d + x], acc);
    }
    const float v = acc * inv;
    if constexpr (sizeof(OutT) == 2) o[static_cast<size_t>(row) * d + x] = __float2bfloat16_rn(v);
    else o[static_cast<size_t>(row) * d + x] = v;
  }
  if (threadIdx.x == 0) lse[row] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
}

}  // namespace blasst
