// prefill_f32_sm100.cuh - fp32 prefill (d = 64, Bc = 64, Br in {64, 128}) for
// blocked attention with softmax thresholding, on tcgen05 kind::tf32.
//
// Same method and readings as prefill_sm100.cuh ("BLASST: Dynamic BLocked
// Attention Sparsity via Softmax Thresholding", Telegram channel
// seeallochnaya, post 3655, paragraphs 2-6 after the headline; "BLASST wins
// Best Paper at MLSys 2026 ...", digg.com/ai/al6mgdew): blocks left to right,
// skip when exp(m_blk - m_run) < lambda on every row of the query tile, block
// 0 always computed, a skipped block's V is not loaded and adds nothing.
//
// Precision: tf32 keeps 10 mantissa bits, too few for scores whose
// threshold margin is compared to 1e-3. Scores therefore use the
// error-compensated three-product split S = Qh Kh + Qh Kl + Ql Kh, where
// xh = x with its 13 low mantissa bits cleared (exact in tf32) and
// xl = x - xh (exact in fp32); the neglected Ql Kl term and the tf32
// rounding of xl leave a relative error near 2^-20. P.V uses the same split
// (P in TMEM as Ph and Pl, V in shared memory as Vh and Vl), so the output
// carries fp32-level error rather than tf32's 2^-11.
//
// This is the small fp32 workload's kernel, so it is written for clarity: one
// CTA of 128 threads per 128 query rows, one block at a time, every step
// waiting for the previous one; thread 0 issues TMA and tcgen05, all threads
// split operands and run the softmax (thread t owns row t).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/blasst.h"
#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"

namespace blasst {

template <int BR>
struct PrefillF32Cfg {
  static constexpr int D = 64, BC = 64, BM = 128;
  static constexpr int NG = BM / BR;
  static constexpr int WPG = BR / 32;
  static constexpr int Q_BOX = BM * 128;        // 32 fp32 columns x 128 rows
  static constexpr int KV_BOX = BC * 128;       // 32 fp32 columns x 64 rows
  static constexpr int Q_BYTES = 2 * Q_BOX;     // 64 columns
  static constexpr int KV_BYTES = 2 * KV_BOX;
  static constexpr int OFF_QH = 0;
  static constexpr int OFF_QL = OFF_QH + Q_BYTES;
  static constexpr int OFF_KH = OFF_QL + Q_BYTES;
  static constexpr int OFF_KL = OFF_KH + KV_BYTES;
  static constexpr int OFF_V = OFF_KL + KV_BYTES;    // V as loaded: rows = keys
  static constexpr int OFF_VTH = OFF_V + KV_BYTES;   // Vh^T: rows = d, 32-key boxes
  static constexpr int OFF_VTL = OFF_VTH + KV_BYTES; // Vl^T
  static constexpr int OFF_BAR = OFF_VTL + KV_BYTES; // [0] Q, [1] K, [2] V, [3] MMA
  static constexpr int OFF_MISC = OFF_BAR + 4 * 8;   // tmem base, abort, votes[4]
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static constexpr int S_COL = 0, P_COL = 64, PL_COL = 128, O_COL = 192, TMEM_COLS = 256;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t IDESC_QK = ptx::idesc_f32acc(2, 128, BC, false);
  // V enters P V K-major (transposed in shared memory): an N-major 32-bit
  // operand would need the 32-byte-atom 128B swizzle, not the TMA's
  static constexpr uint32_t IDESC_PV = ptx::idesc_f32acc(2, 128, D, false);
};

__device__ __forceinline__ float tf32_trunc(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

template <int BR>
__global__ void __launch_bounds__(128, 1)
    blasst_prefill_f32_kernel(const __grid_constant__ CUtensorMap tmQ,
                              const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillF32Cfg<BR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* votes = misc + 4;  // [4] per-warp "all rows skip" bits (+2 on abort)
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

  // work item: (b, hq, 128-row block), longest causal rows first
  const int BH = p.B * p.Hq;
  const int qblk = p.nQblk - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int hq = bh % p.Hq, b = bh / p.Hq;
  const int bhk = b * p.Hkv + hq / p.g;
  const int r0 = qblk * C::BM;
  int kt_last[C::NG];
  int nblk = 0;
#pragma unroll
  for (int gg = 0; gg < C::NG; ++gg) {
    const int gr0 = r0 + gg * BR;
    if (gr0 >= p.Lq) {
      kt_last[gg] = -1;
    } else {
      const int gr1 = min(gr0 + BR, p.Lq);
      int kl = p.nKt - 1;
      if (p.causal) kl = min(kl, (gr1 - 1 + p.off) / C::BC);
      kt_last[gg] = kl;
    }
    nblk = max(nblk, kt_last[gg] + 1);
  }

  if (t == 0) {
    for (int i = 0; i < 4; ++i) ptx::mbar_init(bar(i), 1);
    for (int i = 1; i < 16; ++i) misc[i] = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  // every thread waits on the barrier; a wait that gives up marks the thread
  // and tells the others (their waits then return at once); the CTA leaves
  // the block loop together at the next __syncthreads_or
  bool bad = false;
  auto wait_all = [&](int i, int parity) {
    if (!ptx::mbar_wait(bar(i), parity, &misc[1], p.timeout_ns)) {
      bad = true;
      misc[1] = 1;
    }
  };
  // split a tile of fp32 in place into its tf32 head and a separate tail
  auto split = [&](uint32_t off_h, uint32_t off_l, int bytes) {
    float* h = reinterpret_cast<float*>(smem + off_h);
    float* l = reinterpret_cast<float*>(smem + off_l);
    for (int i = t; i < bytes / 4; i += 128) {
      const float x = h[i];
      const float xh = tf32_trunc(x);
      h[i] = xh;
      l[i] = x - xh;
    }
    ptx::fence_proxy_async_smem();  // generic writes -> visible to tcgen05
  };

  // ---- Q --------------------------------------------------------------------
  if (t == 0) {
    ptx::mbar_arrive_expect_tx(bar(0), C::Q_BYTES);
    ptx::tma_load_3d(sb + C::OFF_QH, &tmQ, 0, r0, bh, bar(0));
    ptx::tma_load_3d(sb + C::OFF_QH + C::Q_BOX, &tmQ, 32, r0, bh, bar(0));
  }
  wait_all(0, 0);
  split(C::OFF_QH, C::OFF_QL, C::Q_BYTES);

  const int row = r0 + t;
  const bool row_exists = row < p.Lq;
  const int gi = t / BR;
  const int last_col = p.causal ? min(row + p.off, p.Lkv - 1) : p.Lkv - 1;
  const float sl2 = p.scale_log2;
  const bool thresholding = p.log2_lambda > -INFINITY;
  float m = -INFINITY, l = 0.0f;
  int ncomp = 0, mma_phase = 0, v_phase = 0, kload = 0;
  int nvis[C::NG] = {};  // blocks visited so far per row group (first-block rule)
  unsigned long long st_vis = 0, st_skip = 0, st_vload = 0, st_flops = 0;

  for (int j = 0; j < nblk; ++j) {
    // row groups that visit block j (causal range, optional static mask)
    uint32_t gvis = 0;
#pragma unroll
    for (int gg = 0; gg < C::NG; ++gg)
      if (j <= kt_last[gg] &&
          (!p.smask ||
           p.smask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + j] == 0))
        gvis |= 1u << gg;
    if (!gvis) {  // excluded before anything is computed
      if (t == 0 && p.mask) {
#pragma unroll
        for (int gg = 0; gg < C::NG; ++gg)
          if (kt_last[gg] >= 0)
            p.mask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + j] = 2;
      }
      continue;
    }
    // ---- K_j, split, S = Qh Kh + Qh Kl + Ql Kh ------------------------------
    __syncthreads();  // previous block's K/V tiles and MMAs are done with
    if (t == 0) {
      ptx::mbar_arrive_expect_tx(bar(1), C::KV_BYTES);
      ptx::tma_load_3d(sb + C::OFF_KH, &tmK, 0, j * C::BC, bhk, bar(1));
      ptx::tma_load_3d(sb + C::OFF_KH + C::KV_BOX, &tmK, 32, j * C::BC, bhk, bar(1));
    }
    wait_all(1, kload & 1);
    ++kload;
    split(C::OFF_KH, C::OFF_KL, C::KV_BYTES);
    ptx::tc_fence_before();
    if (__syncthreads_or(bad ? 1 : 0)) break;
    if (t == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::D / 8; ++kk) {
        const uint32_t qo = (kk >> 2) * C::Q_BOX + (kk & 3) * 32;
        const uint32_t ko = (kk >> 2) * C::KV_BOX + (kk & 3) * 32;
        const uint64_t qh = ptx::sw128_desc(sb + C::OFF_QH + qo, 16, 1024);
        const uint64_t ql = ptx::sw128_desc(sb + C::OFF_QL + qo, 16, 1024);
        const uint64_t kh = ptx::sw128_desc(sb + C::OFF_KH + ko, 16, 1024);
        const uint64_t kl = ptx::sw128_desc(sb + C::OFF_KL + ko, 16, 1024);
        ptx::mma_ss_tf32(tmem + C::S_COL, qh, kh, C::IDESC_QK, kk > 0 ? 1u : 0u);
        ptx::mma_ss_tf32(tmem + C::S_COL, qh, kl, C::IDESC_QK, 1u);
        ptx::mma_ss_tf32(tmem + C::S_COL, ql, kh, C::IDESC_QK, 1u);
      }
      ptx::mma_commit(bar(3));
    }
    wait_all(3, mma_phase & 1);
    ++mma_phase;
    ptx::tc_fence_after();

    // ---- row max, vote -----------------------------------------------------
    float s[C::BC];
    {
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < C::BC / 32; ++c) {
        ptx::tmem_ld32(tmem + lane_base + C::S_COL + 32 * c, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[i]);
      }
    }
    const int col0 = j * C::BC;
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < C::BC; ++c) {
      if (col0 + c > last_col) s[c] = -INFINITY;
      mx = fmaxf(mx, s[c]);
    }
    const float mb = mx * sl2;
    const bool visited = (gvis >> gi) & 1;
    bool rowskip;
    if (!row_exists || !visited) rowskip = true;
    else if (nvis[gi] == 0 || !thresholding) rowskip = false;  // first visited block
    else if (mb == -INFINITY) rowskip = true;                    // no visible key here
    else rowskip = (mb - m) < p.log2_lambda;
#pragma unroll
    for (int gg = 0; gg < C::NG; ++gg) nvis[gg] += (gvis >> gg) & 1;
    const unsigned all = __all_sync(0xffffffffu, rowskip) ? 1u : 0u;
    if (lane == 0) votes[warp] = static_cast<int>(all);
    __syncthreads();
    int keepmask = 0;
#pragma unroll
    for (int gg = 0; gg < C::NG; ++gg) {
      bool gskip = true;
#pragma unroll
      for (int w = 0; w < C::WPG; ++w) gskip = gskip && votes[gg * C::WPG + w] != 0;
      if (((gvis >> gg) & 1) && !gskip) keepmask |= 1 << gg;
    }
    if (t == 0) {
      const unsigned long long tile_flops = 2ull * 128ull * C::BC * C::D;
      st_flops += 3ull * tile_flops + (keepmask ? 3ull * tile_flops : 0ull);
      st_vload += keepmask ? 1ull : 0ull;
#pragma unroll
      for (int gg = 0; gg < C::NG; ++gg) {
        if (kt_last[gg] < 0) continue;
        uint8_t code = 2;
        if ((gvis >> gg) & 1) {
          ++st_vis;
          code = ((keepmask >> gg) & 1) ? 0 : 1;
          if (code == 1) ++st_skip;
        }
        if (p.mask) p.mask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + j] = code;
      }
    }
    if (!keepmask) continue;

    // ---- V_j, online softmax (eager rescale), P, O += P V -------------------
    if (t == 0) {
      ptx::mbar_arrive_expect_tx(bar(2), C::KV_BYTES);
      ptx::tma_load_3d(sb + C::OFF_V, &tmV, 0, j * C::BC, bhk, bar(2));
      ptx::tma_load_3d(sb + C::OFF_V + C::KV_BOX, &tmV, 32, j * C::BC, bhk, bar(2));
    }
    const bool my_keep = (keepmask >> gi) & 1;
    const float m_new = my_keep ? fmaxf(m, mb) : m;
    const float alpha = (my_keep && ncomp > 0 && m_new != m) ? ptx::ex2(m - m_new) : 1.0f;
    if (ncomp > 0) {  // the previous P.V finished (mma barrier above); rescale O
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < C::D / 32; ++c) {
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + 32 * c, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        ptx::tmem_st32(tmem + lane_base + C::O_COL + 32 * c, r);
      }
    }
    l *= alpha;
    m = m_new;
    {
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < C::BC / 32; ++c) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float pv = (my_keep && m > -INFINITY) ? ptx::ex2(fmaf(s[32 * c + i], sl2, -m)) : 0.0f;
          l += pv;
          s[32 * c + i] = pv;
          r[i] = __float_as_uint(tf32_trunc(pv));
        }
        ptx::tmem_st32(tmem + lane_base + C::P_COL + 32 * c, r);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          r[i] = __float_as_uint(s[32 * c + i] - tf32_trunc(s[32 * c + i]));
        ptx::tmem_st32(tmem + lane_base + C::PL_COL + 32 * c, r);
      }
    }
    ptx::tmem_wait_st();
    wait_all(2, v_phase & 1);
    ++v_phase;
    {
      // split V and transpose it into two K-major tiles (rows = d, 128-byte
      // rows of 32 keys, 16-byte chunks swizzled by row % 8, as TMA lays out
      // the tiles it loads)
      const uint8_t* src = smem + C::OFF_V;
      for (int i = t; i < C::BC * C::D; i += 128) {
        const int key = i & (C::BC - 1), dc = i / C::BC;
        const float x = *reinterpret_cast<const float*>(
            src + (dc >> 5) * C::KV_BOX + key * 128 + ((((dc & 31) >> 2) ^ (key & 7)) << 4) +
            (dc & 3) * 4);
        const int dst = (key >> 5) * (C::D * 128) + dc * 128 +
                        ((((key & 31) >> 2) ^ (dc & 7)) << 4) + (key & 3) * 4;
        const float xh = tf32_trunc(x);
        *reinterpret_cast<float*>(smem + C::OFF_VTH + dst) = xh;
        *reinterpret_cast<float*>(smem + C::OFF_VTL + dst) = x - xh;
      }
      ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (t == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::BC / 8; ++kk) {
        const uint32_t vo = (kk >> 2) * (C::D * 128) + (kk & 3) * 32;
        const uint64_t vh = ptx::sw128_desc(sb + C::OFF_VTH + vo, 16, 1024);
        const uint64_t vl = ptx::sw128_desc(sb + C::OFF_VTL + vo, 16, 1024);
        ptx::mma_ts_tf32(tmem + C::O_COL, tmem + C::P_COL + kk * 8, vh, C::IDESC_PV,
                         (ncomp > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_ts_tf32(tmem + C::O_COL, tmem + C::P_COL + kk * 8, vl, C::IDESC_PV, 1u);
        ptx::mma_ts_tf32(tmem + C::O_COL, tmem + C::PL_COL + kk * 8, vh, C::IDESC_PV, 1u);
      }
      ptx::mma_commit(bar(3));
    }
    wait_all(3, mma_phase & 1);
    ++mma_phase;
    ptx::tc_fence_after();
    ++ncomp;
  }

  if (!__syncthreads_or(bad ? 1 : 0)) {
    // ---- epilogue: O / l -> fp32, lse, masks of unvisited blocks ----------
    const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
    float* orow = reinterpret_cast<float*>(p.o) + (static_cast<size_t>(bh) * p.Lq + row) * C::D;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < C::D / 32; ++c) {
      ptx::tmem_ld32(tmem + lane_base + C::O_COL + 32 * c, r);
      ptx::tmem_wait_ld();
      if (row_exists) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(orow + 32 * c + i) =
              make_float4(__uint_as_float(r[i]) * inv_l, __uint_as_float(r[i + 1]) * inv_l,
                          __uint_as_float(r[i + 2]) * inv_l, __uint_as_float(r[i + 3]) * inv_l);
      }
    }
    if (row_exists) p.lse[static_cast<size_t>(bh) * p.Lq + row] = (m + log2f(l)) * 0.6931471805599453f;
    if (p.mask) {
#pragma unroll
      for (int gg = 0; gg < C::NG; ++gg) {
        if (kt_last[gg] < 0) continue;
        uint8_t* mrow = p.mask + (static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt;
        for (int jj = nblk + t; jj < p.nKt; jj += 128) mrow[jj] = 2;
      }
    }
    if (t == 0 && p.stats) {
      const unsigned long long kvb = static_cast<unsigned long long>(C::BC) * C::D * 4ull;
      atomicAdd(&p.stats->tiles_visited, st_vis);
      atomicAdd(&p.stats->tiles_skipped, st_skip);
      atomicAdd(&p.stats->v_blocks_loaded, st_vload);
      atomicAdd(&p.stats->mma_flops, st_flops);
      atomicAdd(&p.stats->bytes_loaded, static_cast<unsigned long long>(C::Q_BYTES) +
                                            kvb * (kload + st_vload));
    }
  } else if (t == 0) {
    record_error(p.err, BLASST_ETIMEOUT);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace blasst
