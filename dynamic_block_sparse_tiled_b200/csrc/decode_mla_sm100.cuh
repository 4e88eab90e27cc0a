// decode_mla_sm100.cuh - split-KV decode with softmax thresholding for
// multi-head latent attention (MLA) shaped caches.
//
// The Telegram post ("BLASST: Dynamic BLocked Attention Sparsity via Softmax
// Thresholding", seeallochnaya 3655, paragraph 9 after the headline) says the
// method is compatible with DeepSeek MLA and nothing more. The MLA decode step
// in its absorbed form: every query head h has a 576-wide query (512 latent +
// 64 rotary dims), every cached token one 576-wide row c_j shared by all heads
// (the latent c_kv in dims 0-511, the rotary key in 512-575), scores
// s = scale * q_h . c_j, and the output o_h = sum_j p_hj c_j[0:512]: softmax
// attention with one KV head, K = c and V = the first 512 dims of c. The skip
// rule is the one of the other kernels, per (head, KV block): a block is
// dropped for head h when exp(m_blk - m_run) < lambda, the first block of every
// split computed, dropped blocks add nothing. V is part of the K rows already
// loaded, so a skip saves no bytes here; it saves the P V product of a group
// of 16 heads when all of them drop the block.
//
// One CTA (256 threads) per (sequence, split, group of 16 heads); KV blocks of
// 64 keys through a 2-stage TMA ring (72 KB each, 128-byte swizzle, nine
// 64-column boxes). Per block, on mma.sync m16n8k16 tiles (M = the 16 heads):
//   S = Q C^T       warp w scores keys [8w, 8w + 8), 36 k-steps;
//   block max per head (quad shuffles, then across warps in shared memory),
//   the vote and the running statistics (threads 0-15, one head each);
//   P (bf16, 128-byte swizzled rows in shared memory), row sums;
//   O += P C[:, 0:512]  warp w owns output columns [64w, 64w + 64).
// At the end of the split the normalised O and lse of each head go to the
// workspace and blasst_lse_merge_kernel combines the splits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/blasst.h"
#include "ptx_sm100.cuh"

namespace blasst {

struct MlaParams {
  float* o_parts;    // [B, H, S, 512]
  float* lse_parts;  // [B, H, S]
  uint8_t* mask;     // [B, H, nKt] or null: 0 computed, 1 skipped
  blasst_stats* stats;
  int* err;
  int B, H, L, S, Ls, nKt;
  float scale_log2, log2_lambda;
  uint64_t timeout_ns;
};

struct MlaCfg {
  static constexpr int DQK = 576, DV = 512, BC = 64, HG = 16;
  static constexpr int NTHREADS = 256;
  static constexpr int NBOX = DQK / 64;          // 9 column boxes
  static constexpr int KV_BOX = BC * 128;        // [64 keys][64 dims] bf16, 8 KB
  static constexpr int KV_BYTES = NBOX * KV_BOX; // 72 KB
  static constexpr int Q_BOX = HG * 128;         // [16 heads][64 dims], 2 KB
  static constexpr int Q_BYTES = NBOX * Q_BOX;   // 18 KB
  static constexpr int OFF_K = 0;
  static constexpr int OFF_Q = OFF_K + 2 * KV_BYTES;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;  // [16][64] bf16, swizzled rows
  static constexpr int OFF_RED = OFF_P + HG * 128;  // [2][8 warps][16] floats
  static constexpr int OFF_ST = OFF_RED + 2 * 8 * HG * 4;  // m, l, alpha [16] floats, keep [16] ints
  static constexpr int OFF_BAR = OFF_ST + 4 * HG * 4;      // Q, KF[2]
  static constexpr int OFF_MISC = OFF_BAR + 3 * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

namespace mla {
// D += A * B, m16n8k16, bf16 in, fp32 accumulation, all 16 rows.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Byte offset of the 16-byte chunk holding dims [8 chunk, 8 chunk + 8) of row
// `row` in a 128-byte-swizzled tile of 64-column boxes of `box_bytes`.
__device__ __forceinline__ uint32_t swz(int row, int chunk, int box_bytes) {
  return static_cast<uint32_t>((chunk >> 3) * box_bytes + row * 128 +
                               (((chunk & 7) ^ (row & 7)) << 4));
}
}  // namespace mla

__global__ void __launch_bounds__(256, 1)
    blasst_decode_mla_kernel(const __grid_constant__ CUtensorMap tmQ,
                             const __grid_constant__ CUtensorMap tmC, const MlaParams p) {
  using C = MlaCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);  // [8 warps][16 heads]
  float* red_sum = red_max + 8 * C::HG;
  float* st_m = reinterpret_cast<float*>(smem + C::OFF_ST);      // running max (log2 units)
  float* st_l = st_m + C::HG;                                    // running sum
  float* st_a = st_m + 2 * C::HG;                                // rescale factor of the block
  int* st_keep = reinterpret_cast<int*>(st_m + 3 * C::HG);       // head keeps the block
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);  // [0] abort, [1] 0
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };  // 0: Q, 1-2: stages

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c4 = lane & 3;  // accumulator rows r, r + 8; columns 2 c4 + {0, 1}
  // (sequence, split, head group), head groups innermost: the CTAs of one
  // split read the same cache rows from L2
  const int NG = p.H / C::HG;
  const int hg = static_cast<int>(blockIdx.x) % NG;
  const int bs = static_cast<int>(blockIdx.x) / NG;
  const int s = bs % p.S, b = bs / p.S;
  const int key_lo = s * p.Ls;
  const int key_hi = min(key_lo + p.Ls, p.L);
  const int nblk = key_hi > key_lo ? (key_hi - key_lo + C::BC - 1) / C::BC : 0;
  const size_t head0 = static_cast<size_t>(b) * p.H + hg * C::HG;

  if (nblk == 0) {  // an empty split: nothing kept, lse = -inf
    for (int e = tid; e < C::HG * C::DV; e += C::NTHREADS)
      p.o_parts[((head0 + e / C::DV) * p.S + s) * C::DV + e % C::DV] = 0.0f;
    if (tid < C::HG) p.lse_parts[(head0 + tid) * p.S + s] = -INFINITY;
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) ptx::mbar_init(bar(i), 1);
    misc[0] = 0;
    misc[1] = 0;
    ptx::fence_mbar_init();
  }
  if (tid < C::HG) {
    st_m[tid] = -INFINITY;
    st_l[tid] = 0.0f;
  }
  __syncthreads();
  auto load_block = [&](int n) {
    const int st = n & 1;
    ptx::mbar_arrive_expect_tx(bar(1 + st), C::KV_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx)
      ptx::tma_load_3d(sb + C::OFF_K + st * C::KV_BYTES + bx * C::KV_BOX, &tmC, bx * 64,
                       key_lo + n * C::BC, b, bar(1 + st));
  };
  int issued = 0;  // thread 0: blocks whose loads were issued
  if (tid == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmC);
    ptx::mbar_arrive_expect_tx(bar(0), C::Q_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx)
      ptx::tma_load_3d(sb + C::OFF_Q + bx * C::Q_BOX, &tmQ, bx * 64, hg * C::HG, b, bar(0));
    for (; issued < 2 && issued < nblk; ++issued) load_block(issued);
  }
  bool ok = __syncthreads_and(ptx::mbar_wait(bar(0), 0, misc, p.timeout_ns) ? 1 : 0) != 0;

  float oa[8][4];
#pragma unroll
  for (int nn = 0; nn < 8; ++nn) oa[nn][0] = oa[nn][1] = oa[nn][2] = oa[nn][3] = 0.0f;
  unsigned long long n_skip = 0, flops = 0;
  const uint32_t qsm = sb + C::OFF_Q;
  const uint32_t psm = sb + C::OFF_P;
  int n = 0;
  for (; ok && n < nblk; ++n) {
    const int st = n & 1;
    ok = __syncthreads_and(ptx::mbar_wait(bar(1 + st), (n >> 1) & 1, misc, p.timeout_ns) ? 1 : 0) != 0;
    if (!ok) break;
    const uint32_t kst = sb + C::OFF_K + st * C::KV_BYTES;
    // ---- S = Q C^T for keys [8 warp, 8 warp + 8) of the block
    float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int key = 8 * warp + (lane & 7);
#pragma unroll 6
    for (int kk = 0; kk < C::DQK / 16; kk += 2) {
      uint32_t a0, a1, a2, a3, e0, e1, e2, e3, b0, b1, b2, b3;
      mla::ldsm_x4(qsm + mla::swz(lane & 15, 2 * kk + (lane >> 4), C::Q_BOX), a0, a1, a2, a3);
      mla::ldsm_x4(qsm + mla::swz(lane & 15, 2 * kk + 2 + (lane >> 4), C::Q_BOX), e0, e1, e2, e3);
      mla::ldsm_x4(kst + mla::swz(key, 2 * kk + (lane >> 3), C::KV_BOX), b0, b1, b2, b3);
      mla::mma16816(sc, a0, a1, a2, a3, b0, b1);
      mla::mma16816(sc, e0, e1, e2, e3, b2, b3);
    }
    // scale to log2 units, mask keys past the split, per-head block max
    const int kcol = key_lo + n * C::BC + 8 * warp + 2 * c4;
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] = (kcol + (e & 1) < key_hi) ? sc[e] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(sc[0], sc[1]), mx1 = fmaxf(sc[2], sc[3]);
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if (c4 == 0) {
      red_max[warp * C::HG + r] = mx0;
      red_max[warp * C::HG + r + 8] = mx1;
    }
    __syncthreads();
    // ---- the vote and the running max, one head per thread
    if (tid < C::HG) {
      float mb = -INFINITY;
#pragma unroll
      for (int w = 0; w < 8; ++w) mb = fmaxf(mb, red_max[w * C::HG + tid]);
      const float mo = st_m[tid];
      const bool skip = n > 0 && p.log2_lambda > -INFINITY && (mb - mo < p.log2_lambda);
      if (!skip) {
        const float mn = fmaxf(mo, mb);
        st_a[tid] = (mo == -INFINITY) ? 0.0f : ptx::ex2(mo - mn);
        st_m[tid] = mn;
        st_keep[tid] = 1;
      } else {
        st_a[tid] = 1.0f;
        st_keep[tid] = 0;
      }
      if (p.mask)
        p.mask[(head0 + tid) * p.nKt + (key_lo / C::BC + n)] = skip ? 1 : 0;
    }
    __syncthreads();
    int gk = 0;
#pragma unroll
    for (int h = 0; h < C::HG; ++h) gk |= st_keep[h];
    if (tid == 0) {
      for (int h = 0; h < C::HG; ++h) n_skip += st_keep[h] ? 0 : 1;
      flops += 2ull * C::HG * C::BC * C::DQK + (gk ? 2ull * C::HG * C::BC * C::DV : 0ull);
    }
    if (gk) {
      // ---- P (bf16, swizzled rows) and its row sums
      const int kr0 = st_keep[r], kr1 = st_keep[r + 8];
      const float mr0 = st_m[r], mr1 = st_m[r + 8];
      const float p0 = kr0 ? ptx::ex2(sc[0] - mr0) : 0.0f;
      const float p1 = kr0 ? ptx::ex2(sc[1] - mr0) : 0.0f;
      const float p2 = kr1 ? ptx::ex2(sc[2] - mr1) : 0.0f;
      const float p3 = kr1 ? ptx::ex2(sc[3] - mr1) : 0.0f;
      float s0 = p0 + p1, s1 = p2 + p3;
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (c4 == 0) {
        red_sum[warp * C::HG + r] = s0;
        red_sum[warp * C::HG + r + 8] = s1;
      }
      const uint32_t pch = static_cast<uint32_t>((warp ^ (r & 7)) << 4) + 4 * c4;
      *reinterpret_cast<uint32_t*>(smem + C::OFF_P + r * 128 + pch) = ptx::pack_bf16x2(p0, p1);
      *reinterpret_cast<uint32_t*>(smem + C::OFF_P + (r + 8) * 128 + pch) = ptx::pack_bf16x2(p2, p3);
      __syncthreads();
      if (tid < C::HG) {
        float ssum = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) ssum += red_sum[w * C::HG + tid];
        st_l[tid] = st_a[tid] * st_l[tid] + ssum;
      }
      const float al0 = st_a[r], al1 = st_a[r + 8];
#pragma unroll
      for (int nn = 0; nn < 8; ++nn) {
        oa[nn][0] *= al0;
        oa[nn][1] *= al0;
        oa[nn][2] *= al1;
        oa[nn][3] *= al1;
      }
      // ---- O[:, 64 warp + (0..63)] += P V, V = cache dims 0-511 of the block
#pragma unroll
      for (int kk = 0; kk < C::BC / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        const int prow = lane & 15;
        mla::ldsm_x4(psm + prow * 128 + (((2 * kk + (lane >> 4)) ^ (prow & 7)) << 4), a0, a1, a2, a3);
        const int vkey = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nn = 0; nn < 8; nn += 2) {
          uint32_t b0, b1, b2, b3;
          mla::ldsm_x4_t(kst + mla::swz(vkey, 8 * warp + nn + (lane >> 4), C::KV_BOX), b0, b1, b2, b3);
          mla::mma16816(oa[nn], a0, a1, a2, a3, b0, b1);
          mla::mma16816(oa[nn + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();  // the stage, P and the reductions are free again
    if (tid == 0 && issued < nblk) {
      load_block(issued);
      ++issued;
    }
  }
  if (!ok) {
    if (tid == 0) {
      misc[0] = 1;
      if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
      // let the copies still in flight land before the CTA exits
      for (int k = n; k < issued; ++k)
        ptx::mbar_wait(bar(1 + (k & 1)), (k >> 1) & 1, &misc[1], p.timeout_ns);
    }
    return;
  }
  __syncthreads();
  // ---- this split's normalised O and lse
  const float l0 = st_l[r], l1 = st_l[r + 8];
  const float inv0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, inv1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
  float* op0 = p.o_parts + ((head0 + r) * p.S + s) * C::DV + 64 * warp + 2 * c4;
  float* op1 = p.o_parts + ((head0 + r + 8) * p.S + s) * C::DV + 64 * warp + 2 * c4;
#pragma unroll
  for (int nn = 0; nn < 8; ++nn) {
    *reinterpret_cast<float2*>(op0 + 8 * nn) = make_float2(oa[nn][0] * inv0, oa[nn][1] * inv0);
    *reinterpret_cast<float2*>(op1 + 8 * nn) = make_float2(oa[nn][2] * inv1, oa[nn][3] * inv1);
  }
  if (tid < C::HG)
    p.lse_parts[(head0 + tid) * p.S + s] =
        st_l[tid] > 0.0f ? (st_m[tid] + log2f(st_l[tid])) * 0.6931471805599453f : -INFINITY;
  if (tid == 0 && p.stats) {
    atomicAdd(&p.stats->tiles_visited, static_cast<unsigned long long>(nblk) * C::HG);
    atomicAdd(&p.stats->tiles_skipped, n_skip);
    atomicAdd(&p.stats->v_blocks_loaded, static_cast<unsigned long long>(nblk));
    atomicAdd(&p.stats->mma_flops, flops);
    atomicAdd(&p.stats->bytes_loaded,
              static_cast<unsigned long long>(nblk) * C::KV_BYTES + C::Q_BYTES);
  }
}

}  // namespace blasst
