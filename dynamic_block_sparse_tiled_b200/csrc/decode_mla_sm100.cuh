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
  const __nv_bfloat16* q;  // [B, H, 576]
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

// ---------------------------------------------------------------------------
// Tensor-core version for 128 heads per latent KV head (M = 128): tcgen05.mma
// with the scores and the output in TMEM. The 128 x 512 fp32 output needs all
// 512 TMEM columns, so two CTAs share a (sequence, split): both compute the
// same scores and decisions, each accumulates one half of the 512 output
// columns.
//   warps 0-3  one head per thread (TMEM lane): the block's scores, the vote,
//              lazy rescaling (the reference max moves only when it has grown
//              by more than 8 in log2 units; then the O half in TMEM is scaled
//              after the previous P V has completed), P (bf16) over S;
//   warp 4     TMA: query dims 256-575 once, 64-key blocks of the cache
//              through a 2-stage ring;
//   warp 6     tcgen05 issuer of S = Q C^T (M 128, N 64, K 576) into one of
//              two S buffers (once the block is loaded and the buffer's P has
//              been read by its P V); query dims 0-255 are a TMEM operand
//              (written by warps 0-3 at start), dims 256-575 come from shared
//              memory, which leaves room for two 72 KB cache stages;
//   warp 5     tcgen05 issuer of O_half += P V_half (M 128, N 256, K 64, P
//              from TMEM, V MN-major from the stage), skipped when no head of
//              the 128 keeps the block; owns the TMEM allocation. Two issuers
//              so that a P V never waits behind a score product that waits
//              for its block's load.
namespace mla {
struct TcCfg {
  static constexpr int DQK = 576, DV = 512, BC = 64, HM = 128;
  static constexpr int NTHREADS = 224;
  static constexpr int NBOX = DQK / 64;             // 9
  static constexpr int QT_BOX = 4;                  // dims 0-255 of Q live in TMEM (TS operand)
  static constexpr int Q_BOX = HM * 128;            // 16 KB
  static constexpr int Q_SM_BYTES = (NBOX - QT_BOX) * Q_BOX;  // dims 256-575 in shared memory, 80 KB
  static constexpr int KV_BOX = BC * 128;           // 8 KB
  static constexpr int KV_BYTES = NBOX * KV_BOX;    // 72 KB
  static constexpr int NST = 2;                     // cache stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_SM_BYTES;
  static constexpr int OFF_BAR = OFF_K + NST * KV_BYTES;
  static constexpr int NSB = 2;                     // S buffers
  static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + NST, B_SF = B_KE + NST;
  static constexpr int B_PR = B_SF + NSB, B_PVD = B_PR + NSB, B_DRAIN = B_PVD + NSB;
  static constexpr int B_SFREE = B_DRAIN + 1;   // [NSB] P of the S buffer read by its P V
  static constexpr int B_DRAIN_S = B_SFREE + NSB; // the S issuer's drain
  static constexpr int B_QT = B_DRAIN_S + 1;    // Q dims 0-255 written to TMEM (4 warps)
  static constexpr int B_KES = B_QT + 1;        // [NST] the stage's score-only boxes free (S done)
  static constexpr int NBAR = B_KES + NST;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc words: [0] tmem base, [1] abort, [2] always 0, [4..5] block kept by some head (per S buffer)
  static constexpr int MISC_BYTES = 64;
  static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
  static constexpr int S_COL = 0;    // S buffer b at 64 b (P: first 32 columns)
  static constexpr int QT_COL = 128;  // Q dims 0-255, packed bf16 pairs: 128 columns
  static constexpr int O_COL = 256;  // this CTA's 256 output columns
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32acc(128, BC, false, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32acc(128, 256, false, true);
  static constexpr float TAU = 8.0f;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(NSB * BC <= QT_COL && QT_COL + 128 <= O_COL, "TMEM columns");
};
}  // namespace mla

__global__ void __launch_bounds__(224, 1)
    blasst_decode_mla_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                const __grid_constant__ CUtensorMap tmC, const MlaParams p) {
  using C = mla::TcCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort_flag = misc + 1;
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // (sequence, split, head group of 128, half of the output columns)
  const int NG = p.H / C::HM;
  const int half = static_cast<int>(blockIdx.x) & 1;
  const int rest = static_cast<int>(blockIdx.x) >> 1;
  const int hgrp = rest % NG;
  const int bs = rest / NG;
  const int s = bs % p.S, b = bs / p.S;
  const int key_lo = s * p.Ls;
  const int key_hi = min(key_lo + p.Ls, p.L);
  const int nblk = key_hi > key_lo ? (key_hi - key_lo + C::BC - 1) / C::BC : 0;
  const size_t head0 = static_cast<size_t>(b) * p.H + hgrp * C::HM;

  if (nblk == 0) {  // an empty split: nothing kept, lse = -inf
    for (int e = tid; e < C::HM * 256; e += C::NTHREADS)
      p.o_parts[((head0 + e / 256) * p.S + s) * C::DV + 256 * half + e % 256] = 0.0f;
    if (half == 0 && tid < C::HM) p.lse_parts[(head0 + tid) * p.S + s] = -INFINITY;
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      ptx::mbar_init(bar(i), ((i >= C::B_PR && i < C::B_PR + C::NSB) || i == C::B_QT) ? 4 : 1);
    for (int i = 1; i < C::MISC_BYTES / 4; ++i) misc[i] = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  if (warp == 4) {
    // ======================= TMA producer ================================
    if (lane == 0) {
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmC);
      ptx::mbar_arrive_expect_tx(bar(C::B_Q), C::Q_SM_BYTES);
#pragma unroll
      for (int bx = C::QT_BOX; bx < C::NBOX; ++bx)
        ptx::tma_load_3d(sb + C::OFF_Q + (bx - C::QT_BOX) * C::Q_BOX, &tmQ, bx * 64, hgrp * C::HM, b,
                         bar(C::B_Q));
      bool ok = true;
      int n = 0;
      for (; n < nblk && ok; ++n) {
        const int st = n % C::NST;
        // the boxes this CTA reads only for the scores reload once the block's
        // score product is done; its V boxes (dims [256 half, 256 half + 256))
        // once its P V is done. One full barrier counts all nine boxes.
        auto load_box = [&](int bx) {
          ptx::tma_load_3d(sb + C::OFF_K + st * C::KV_BYTES + bx * C::KV_BOX, &tmC, bx * 64,
                           key_lo + n * C::BC, b, bar(C::B_KF + st));
        };
        const bool reuse = n >= C::NST;
        if (reuse)
          ok = ptx::mbar_wait(bar(C::B_KES + st), ((n / C::NST) - 1) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(bar(C::B_KF + st), C::KV_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          if (bx < 4 * half || bx >= 4 * half + 4) load_box(bx);
        if (reuse)
          ok = ptx::mbar_wait(bar(C::B_KE + st), ((n / C::NST) - 1) & 1, abort_flag, p.timeout_ns);
        // the V boxes go out even when that wait gave up, so that the stage's
        // byte count completes and the drain below can wait for it
#pragma unroll
        for (int bx = 4 * half; bx < 4 * half + 4; ++bx) load_box(bx);
        if (!ok) {
          ++n;  // block n's loads are in flight too
          break;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
        // let the copies in flight land before the CTA exits
        ptx::mbar_wait(bar(C::B_Q), 0, &misc[2], p.timeout_ns);
        for (int k = n - C::NST < 0 ? 0 : n - C::NST; k < n; ++k)
          ptx::mbar_wait(bar(C::B_KF + k % C::NST), (k / C::NST) & 1, &misc[2], p.timeout_ns);
      }
    }
  } else if (warp == 5 || warp == 6) {
    // ======================= tcgen05 issuers =============================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(bar(C::B_Q), 0, abort_flag, p.timeout_ns);
      ptx::tc_fence_after();
      if (warp == 6) {
        // S(n) = Q C_n^T into S buffer n % 2: dims 0-255 with Q from TMEM,
        // dims 256-575 with Q from shared memory
        if (ok) ok = ptx::mbar_wait(bar(C::B_QT), 0, abort_flag, p.timeout_ns);
        ptx::tc_fence_after();
        const uint64_t q_desc = ptx::sw128_desc(sb + C::OFF_Q, 16, 1024);
        const uint64_t k_desc = ptx::sw128_desc(sb + C::OFF_K, 16, 1024);
        for (int n = 0; n < nblk && ok; ++n) {
          const int sbuf = n % C::NSB, st = n % C::NST;
          ok = ptx::mbar_wait(bar(C::B_KF + st), (n / C::NST) & 1, abort_flag, p.timeout_ns);
          if (ok && n >= C::NSB)
            ok = ptx::mbar_wait(bar(C::B_SFREE + sbuf), ((n / C::NSB) - 1) & 1, abort_flag,
                                p.timeout_ns);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t d_tm = tmem + C::S_COL + sbuf * C::BC;
          const uint64_t kd = k_desc + static_cast<uint64_t>((st * C::KV_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4 * C::QT_BOX; ++kk) {
            const uint64_t bd = kd + static_cast<uint64_t>(((kk >> 2) * C::KV_BOX + (kk & 3) * 32) >> 4);
            ptx::mma_ts(d_tm, tmem + C::QT_COL + kk * 8, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 4 * C::QT_BOX; kk < C::DQK / 16; ++kk) {
            const uint64_t a =
                q_desc + static_cast<uint64_t>((((kk >> 2) - C::QT_BOX) * C::Q_BOX + (kk & 3) * 32) >> 4);
            const uint64_t bd = kd + static_cast<uint64_t>(((kk >> 2) * C::KV_BOX + (kk & 3) * 32) >> 4);
            ptx::mma_ss(d_tm, a, bd, C::IDESC_S, 1u);
          }
          ptx::mma_commit(bar(C::B_SF + sbuf));
          ptx::mma_commit(bar(C::B_KES + st));  // the stage's score-only boxes may be reloaded
        }
      } else {
        // O_half += P(n) V_half(n); the commits free the stage, the S buffer
        // and mark O as holding every P V up to block n
        const uint64_t v_desc = ptx::sw128_desc(sb + C::OFF_K + 4 * half * C::KV_BOX, C::KV_BOX, 1024);
        bool any_pv = false;
        for (int n = 0; n < nblk && ok; ++n) {
          const int sbuf = n % C::NSB, stg = n % C::NST;
          ok = ptx::mbar_wait(bar(C::B_PR + sbuf), (n / C::NSB) & 1, abort_flag, p.timeout_ns);
          if (!ok) break;
          ptx::tc_fence_after();
          if (misc[4 + sbuf] != 0) {
            const uint32_t p_tm = tmem + C::S_COL + sbuf * C::BC;
            const uint64_t vd = v_desc + static_cast<uint64_t>((stg * C::KV_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < C::BC / 16; ++kk)
              ptx::mma_ts(tmem + C::O_COL, p_tm + kk * 8, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                          C::IDESC_PV, (any_pv || kk > 0) ? 1u : 0u);
            any_pv = true;
          }
          ptx::mma_commit(bar(C::B_KE + stg));
          ptx::mma_commit(bar(C::B_SFREE + sbuf));
          ptx::mma_commit(bar(C::B_PVD + sbuf));
        }
      }
      if (!ok) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      const uint32_t drain = warp == 5 ? bar(C::B_DRAIN) : bar(C::B_DRAIN_S);
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, &misc[2], p.timeout_ns);
    }
  } else {
    // ======================= softmax: one head per thread ===================
    // Every exit from the loop and every optional wait is agreed by the four
    // warps through barrier reductions, so no warp is left at a named barrier.
    const int h = tid;  // TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m = -INFINITY, mref = -INFINITY, l = 0.0f;
    bool ok = true;
    unsigned long long n_skip = 0, n_pv = 0;
    {
      // this head's query dims 0-255 into TMEM (the score product's TS operand)
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (head0 + h) * C::DQK);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = qrow[8 * c + u];
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        ptx::tmem_st32(tmem + lane_base + C::QT_COL + 32 * c, w);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_QT));
    }
    for (int n = 0; n < nblk; ++n) {
      const int st = n % C::NSB;  // S buffer
      ok = ptx::named_bar_and(2, 128, ptx::mbar_wait(bar(C::B_SF + st), (n / C::NSB) & 1, abort_flag,
                                                      p.timeout_ns));
      if (!ok) break;
      ptx::tc_fence_after();
      const int kbase = key_lo + n * C::BC;
      float sv[C::BC];
      float mb = -INFINITY;
#pragma unroll
      for (int hc = 0; hc < C::BC / 32; ++hc) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_base + C::S_COL + st * C::BC + 32 * hc, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int cc = 32 * hc + c;
          sv[cc] = (kbase + cc < key_hi) ? __uint_as_float(r[c]) * p.scale_log2 : -INFINITY;
          mb = fmaxf(mb, sv[cc]);
        }
      }
      const bool skip = n > 0 && p.log2_lambda > -INFINITY && (mb - m < p.log2_lambda);
      const float m_new = skip ? m : fmaxf(m, mb);
      const bool move_ref = !skip && (mref == -INFINITY || m_new - mref > C::TAU);
      const bool scale_o = move_ref && n > 0;  // O holds P V of earlier blocks
      // some head must scale O: wait (all threads) for the previous P V
      if (!ptx::named_bar_and(3, 128, !scale_o)) {
        ok = ptx::named_bar_and(4, 128, ptx::mbar_wait(bar(C::B_PVD + ((n - 1) % C::NSB)),
                                                        ((n - 1) / C::NSB) & 1, abort_flag,
                                                        p.timeout_ns));
        if (!ok) break;
        ptx::tc_fence_after();
      }
      // O rescale, warp-uniform: tcgen05.ld/st are warp-wide instructions, so
      // every lane takes part when any head of the warp moves its reference
      // (factor 1 for the others)
      const float f_move = (mref == -INFINITY) ? 0.0f : ptx::ex2(mref - m_new);
      if (__any_sync(0xffffffffu, scale_o)) {
        const float fo = scale_o ? f_move : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          ptx::tmem_ld32(tmem + lane_base + C::O_COL + 32 * c, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * fo);
          ptx::tmem_st32(tmem + lane_base + C::O_COL + 32 * c, o);
        }
      }
      uint32_t pk[C::BC / 2];
      if (!skip) {
        m = m_new;
        if (move_ref) {
          l *= f_move;
          mref = m;
        }
        float ps = 0.0f;
#pragma unroll
        for (int c = 0; c < C::BC / 2; ++c) {
          const float p0 = ptx::ex2(sv[2 * c] - mref), p1 = ptx::ex2(sv[2 * c + 1] - mref);
          ps += p0 + p1;
          pk[c] = ptx::pack_bf16x2(p0, p1);
        }
        l += ps;
      } else {
        ++n_skip;
#pragma unroll
        for (int c = 0; c < C::BC / 2; ++c) pk[c] = 0u;
      }
      static_assert(C::BC == 64, "P is stored as one 32-column row");
      ptx::tmem_st32(tmem + lane_base + C::S_COL + st * C::BC, pk);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      // does any of the 128 heads keep the block? (P V is skipped otherwise)
      const bool none = ptx::named_bar_and(1, 128, skip);
      if (tid == 0) {
        misc[4 + st] = none ? 0 : 1;
        n_pv += none ? 0 : 1;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_PR + st));
      if (half == 0 && p.mask) p.mask[(head0 + h) * p.nKt + (key_lo / C::BC + n)] = skip ? 1 : 0;
    }
    if (ok) {
      // the last P V, then this split's O half and lse
      ok = ptx::named_bar_and(2, 128, ptx::mbar_wait(bar(C::B_PVD + ((nblk - 1) % C::NSB)),
                                                      ((nblk - 1) / C::NSB) & 1, abort_flag,
                                                      p.timeout_ns));
    }
    if (!ok) {
      *abort_flag = 1;
      if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
    } else {
      ptx::tc_fence_after();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
      float* op = p.o_parts + ((head0 + h) * p.S + s) * C::DV + 256 * half;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + 32 * c, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          reinterpret_cast<float4*>(op + 32 * c)[u] =
              make_float4(__uint_as_float(o[4 * u]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                          __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
      }
      if (half == 0)
        p.lse_parts[(head0 + h) * p.S + s] =
            l > 0.0f ? (mref + log2f(l)) * 0.6931471805599453f : -INFINITY;
      if (p.stats) {
        if (half == 0) atomicAdd(&p.stats->tiles_skipped, n_skip);
        if (h == 0) {
          const unsigned long long s_fl = 2ull * C::HM * C::BC * C::DQK;
          const unsigned long long pv_fl = 2ull * C::HM * C::BC * 256;
          atomicAdd(&p.stats->mma_flops, static_cast<unsigned long long>(nblk) * s_fl + n_pv * pv_fl);
          atomicAdd(&p.stats->bytes_loaded,
                    static_cast<unsigned long long>(nblk) * C::KV_BYTES + C::Q_SM_BYTES + C::HM * 512);
          if (half == 0) {
            atomicAdd(&p.stats->tiles_visited, static_cast<unsigned long long>(nblk) * C::HM);
            atomicAdd(&p.stats->v_blocks_loaded, static_cast<unsigned long long>(nblk));
          }
        }
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace blasst
