// prefill_sm100.cuh - forward prefill kernel for blocked attention with
// softmax thresholding on sm_100a (tcgen05 + TMEM + TMA).
//
// Method ("BLASST: Dynamic BLocked Attention Sparsity via Softmax
// Thresholding", Telegram channel seeallochnaya, post 3655, paragraphs 2-6
// after the headline; "BLASST wins Best Paper at MLSys 2026 ...",
// digg.com/ai/al6mgdew, the authors' announcement): KV blocks are walked
// left to right with an online softmax; a block is dropped when
// exp(m_blk - m_run) < lambda on every row of the query tile, in which case
// its V is never loaded and no P.V product is formed; block 0 is always kept.
// The lazy rescaling of FlashAttention 4 (paragraph 4) is used for the
// output accumulator; the skip test always uses the exact running max.
//
// One CTA owns 128 query rows of one (batch, query head) and walks the KV
// blocks of its KV head. Warp roles (384 threads):
//   warps 0-7  softmax: warps w and w+4 share the 32 rows of TMEM lanes
//              32*(w%4).. and split the block's columns in halves; each takes
//              its half-row max, the half-row skip test, exp2, its half of P
//              (into TMEM), its half of the lazy O rescale and of the
//              epilogue. The row skip test is exact on halves:
//              max(a, b) - m < t  <=>  a - m < t  and  b - m < t;
//   warp 8     TMA producer for Q and K (K runs ahead through a 3-stage ring,
//              independent of the votes);
//   warp 9     TMA producer for V: loads V of block j only after the vote on
//              block j says some row group keeps it;
//   warp 10    tcgen05 issuer for S = Q K^T into one of two TMEM S buffers,
//              two blocks ahead, as soon as the softmax has read the buffer;
//              it also owns the TMEM allocation;
//   warp 11    tcgen05 issuer for O += P V, P read from one of two TMEM P
//              buffers, as soon as P and V are there.
// The two issuers are separate threads because issuing eight MMAs blocks
// the issuing thread while the tensor pipe's queue is full: with one
// thread, P V of block j waited behind the look-ahead Q K^T and vice versa.
// P has TMEM of its own, so no issuer waits for an MMA to finish; they wait
// only for the softmax (S read, P ready), for K and for V.
// With Br = 64 the 128 rows form two independent vote groups that share the
// MMAs: a group that skips contributes zero rows of P and leaves its running
// statistics untouched.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/blasst.h"
#include "ptx_sm100.cuh"

namespace blasst {

struct PrefillParams {
  void* o;
  float* lse;
  uint8_t* mask;
  blasst_stats* stats;
  int* err;
  int B, Hq, Hkv, Lq, Lkv;
  int g;      // Hq / Hkv
  int nQt;    // ceil(Lq / Br)  (mask rows per head)
  int nKt;    // ceil(Lkv / Bc)
  int nQblk;  // ceil(Lq / 128) (CTAs per head)
  int causal;
  int off;    // Lkv - Lq
  float scale_log2;   // scale * log2(e)
  float log2_lambda;  // log2(lambda); -inf when lambda == 0
  uint64_t timeout_ns;
};

constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int D, int BC, int BR>
struct PrefillCfg {
  static constexpr int BM = 128;
  static constexpr int NTHREADS = 384;
  static constexpr int NSOFT = 256;      // softmax threads (warps 0-7)
  static constexpr int WARP_K = 8, WARP_V = 9, WARP_MMA = 10, WARP_PV = 11;
  static constexpr int NG = BM / BR;     // vote groups
  static constexpr int WPG = BR / 32;    // TMEM lane quarters per vote group
  static constexpr int HALF = BC / 2;    // S columns per softmax warp
  static constexpr int DHALF = D / 2;    // O columns per softmax warp
  static constexpr int NK = 3;
  static constexpr int NV = 2;
  static constexpr int NS = 2;   // S buffers (fp32, BC columns each)
  static constexpr int NP = 2;   // P buffers (bf16 pairs, BC/2 columns each)
  static constexpr int NSLOT = 4;
  static constexpr int DBOX = D / 64;
  static constexpr int Q_BOX = BM * 128;
  static constexpr int KV_BOX = BC * 128;
  static constexpr int Q_BYTES = Q_BOX * DBOX;
  static constexpr int KV_BYTES = KV_BOX * DBOX;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;
  static constexpr int B_KE = B_KF + NK;
  static constexpr int B_VF = B_KE + NK;
  static constexpr int B_VE = B_VF + NV;
  static constexpr int B_SF = B_VE + NV;   // S written (tcgen05 commit)
  static constexpr int B_SC = B_SF + NS;   // S read by all softmax warps (buffer reusable)
  static constexpr int B_PV = B_SC + NS;   // P.V done, one barrier per P buffer
  static constexpr int B_DEC = B_PV + NP;
  static constexpr int B_P = B_DEC + NSLOT;
  static constexpr int B_DRAIN = B_P + NSLOT;  // [2]: QK issuer, PV issuer
  static constexpr int NBAR = B_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc words: [0] tmem base, [1] abort, [3] always 0 (for waits only a timeout ends),
  // [4..7] decisions, [8..23] votes (2 x 8 warps),
  // [24..25] softmax-only abort words (by block parity)
  static constexpr int MISC_BYTES = 128;
  static constexpr int OFF_PMAX = OFF_MISC + MISC_BYTES;  // [2][2 halves][128 rows] floats
  static constexpr int OFF_LSUM = OFF_PMAX + 2 * 2 * 128 * 4;  // [2 halves][128 rows] floats
  static constexpr int SMEM_BYTES = OFF_LSUM + 2 * 128 * 4 + 1024;  // + alignment slack
  static constexpr int S_COL = 0;                   // S buffer b at column b * BC
  static constexpr int P_COL = NS * BC;             // P buffer b at P_COL + b * BC / 2
  static constexpr int O_COL = P_COL + NP * BC / 2; // O accumulator
  static constexpr int TMEM_COLS = pow2_at_least(O_COL + D);
  static constexpr uint32_t IDESC_QK = ptx::idesc_f32acc(1, 128, BC, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc_f32acc(1, 128, D, true);
  static constexpr float TAU = 8.0f;  // lazy-rescale slack, log2 units
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BC == 64 || BC == 128, "KV block");
  static_assert(BR == 64 || BR == 128, "query tile");
  static_assert(TMEM_COLS <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

template <int D, int BC, int BR>
__global__ void __launch_bounds__(384, 1)
    blasst_prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                               const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D, BC, BR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort_flag = misc + 1;
  volatile int* dec_val = misc + 4;
  volatile int* votes = misc + 8;
  volatile int* sm_abort = misc + 24;
  volatile float* pmax = reinterpret_cast<volatile float*>(smem + C::OFF_PMAX);
  volatile float* lsum = reinterpret_cast<volatile float*>(smem + C::OFF_LSUM);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item ----------------------------------------------------------
  // KV-head major: the CTAs in flight share one KV head's K/V in L2; within
  // a KV head, the longest causal rows go first and the g query heads of the
  // group are adjacent.
  const int per_kv = p.nQblk * p.g;
  const int bhk = static_cast<int>(blockIdx.x) / per_kv;
  const int rem = static_cast<int>(blockIdx.x) % per_kv;
  const int qblk = p.nQblk - 1 - rem / p.g;
  const int b = bhk / p.Hkv;
  const int hq = (bhk % p.Hkv) * p.g + rem % p.g;
  const int bh = b * p.Hq + hq;
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
      if (p.causal) kl = min(kl, (gr1 - 1 + p.off) / BC);
      kt_last[gg] = kl;
    }
    nblk = max(nblk, kt_last[gg] + 1);
  }

  // ---- set-up -------------------------------------------------------------
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_Q), 1);
    for (int i = 0; i < C::NK; ++i) {
      ptx::mbar_init(bar(C::B_KF + i), 1);
      ptx::mbar_init(bar(C::B_KE + i), 1);
    }
    for (int i = 0; i < C::NV; ++i) {
      ptx::mbar_init(bar(C::B_VF + i), 1);
      ptx::mbar_init(bar(C::B_VE + i), 1);
    }
    for (int i = 0; i < C::NS; ++i) {
      ptx::mbar_init(bar(C::B_SF + i), 1);
      ptx::mbar_init(bar(C::B_SC + i), 8);
    }
    for (int i = 0; i < C::NP; ++i) ptx::mbar_init(bar(C::B_PV + i), 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      ptx::mbar_init(bar(C::B_DEC + i), 1);
      ptx::mbar_init(bar(C::B_P + i), 8);
    }
    ptx::mbar_init(bar(C::B_DRAIN), 1);
    ptx::mbar_init(bar(C::B_DRAIN + 1), 1);
    for (int i = 1; i < C::MISC_BYTES / 4; ++i) misc[i] = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  auto load_kv = [&](const CUtensorMap* tm, uint32_t dst, int blk, uint32_t fb) {
    ptx::mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::DBOX; ++bx)
      ptx::tma_load_3d(dst + bx * C::KV_BOX, tm, bx * 64, blk * BC, bhk, fb);
  };

  if (warp == C::WARP_K) {
    // ======================= TMA producer: Q and K ========================
    if (lane == 0) {
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmK);
      bool ok = true;
      ptx::mbar_arrive_expect_tx(bar(C::B_Q), C::Q_BYTES);
#pragma unroll
      for (int bx = 0; bx < C::DBOX; ++bx)
        ptx::tma_load_3d(sb + C::OFF_Q + bx * C::Q_BOX, &tmQ, bx * 64, r0, bh, bar(C::B_Q));
      for (int j = 0; j < nblk && ok; ++j) {
        const int ks = j % C::NK;
        if (j >= C::NK)
          ok = ptx::mbar_wait(bar(C::B_KE + ks), ((j / C::NK) - 1) & 1, abort_flag,
                              p.timeout_ns);
        if (!ok) break;
        load_kv(&tmK, sb + C::OFF_K + ks * C::KV_BYTES, j, bar(C::B_KF + ks));
      }
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
        // Let the copies already in flight land before the CTA exits.
        ptx::mbar_wait(bar(C::B_Q), 0, abort_flag, p.timeout_ns);
      }
    }
  } else if (warp == C::WARP_V) {
    // ======================= TMA producer: V (after the vote) ==============
    if (lane == 0) {
      ptx::prefetch_tmap(&tmV);
      bool ok = true;
      int vcount = 0;
      unsigned long long st_vis = 0, st_skip = 0, st_flops = 0;
      for (int j = 0; j < nblk && ok; ++j) {
        const int slot = j % C::NSLOT;
        ok = ptx::mbar_wait(bar(C::B_DEC + slot), (j / C::NSLOT) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        const int keepmask = dec_val[slot];
        // skip-mask entries and counters for block j (off the softmax path)
        const unsigned long long tile_flops = 2ull * 128ull * BC * D;
        st_flops += tile_flops + (keepmask ? tile_flops : 0ull);
#pragma unroll
        for (int gg = 0; gg < C::NG; ++gg) {
          if (kt_last[gg] < 0) continue;
          uint8_t code = 2;
          if (j <= kt_last[gg]) {
            ++st_vis;
            code = ((keepmask >> gg) & 1) ? 0 : 1;
            if (code == 1) ++st_skip;
          }
          if (p.mask)
            p.mask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + j] = code;
        }
        if (keepmask != 0) {
          const int vs = vcount % C::NV;
          if (vcount >= C::NV)
            ok = ptx::mbar_wait(bar(C::B_VE + vs), ((vcount / C::NV) - 1) & 1, abort_flag,
                                p.timeout_ns);
          if (!ok) break;
          load_kv(&tmV, sb + C::OFF_V + vs * C::KV_BYTES, j, bar(C::B_VF + vs));
          ++vcount;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
      } else if (p.stats) {
        const unsigned long long qbytes = 128ull * D * 2ull;
        const unsigned long long kvb = static_cast<unsigned long long>(BC) * D * 2ull;
        atomicAdd(&p.stats->tiles_visited, st_vis);
        atomicAdd(&p.stats->tiles_skipped, st_skip);
        atomicAdd(&p.stats->v_blocks_loaded, static_cast<unsigned long long>(vcount));
        atomicAdd(&p.stats->mma_flops, st_flops);
        atomicAdd(&p.stats->bytes_loaded, qbytes + kvb * (nblk + vcount));
      }
    }
  } else if (warp == C::WARP_MMA) {
    // ======================= tcgen05 issuer: S = Q K^T =====================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(bar(C::B_Q), 0, abort_flag, p.timeout_ns);
      ptx::tc_fence_after();
      // The few instructions between two tcgen05.mma of one thread are on the
      // critical path: the descriptors are built once and each k-step adds a
      // compile-time offset (16-byte units) to the start-address field, which
      // cannot carry (shared addresses < 256 KB).
      const uint64_t q_desc = ptx::sw128_desc(sb + C::OFF_Q, 16, 1024);
      const uint64_t k_desc = ptx::sw128_desc(sb + C::OFF_K, 16, 1024);
      auto issue_qk = [&](int j) -> bool {
        const int ks = j % C::NK;
        if (!ptx::mbar_wait(bar(C::B_KF + ks), (j / C::NK) & 1, abort_flag, p.timeout_ns))
          return false;
        ptx::tc_fence_after();
        const uint32_t d_tm = tmem + C::S_COL + (j % C::NS) * BC;
        const uint64_t kd = k_desc + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a =
              q_desc + static_cast<uint64_t>(((kk >> 2) * C::Q_BOX + (kk & 3) * 32) >> 4);
          const uint64_t bd =
              kd + static_cast<uint64_t>(((kk >> 2) * C::KV_BOX + (kk & 3) * 32) >> 4);
          ptx::mma_ss(d_tm, a, bd, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(C::B_KE + ks));
        ptx::mma_commit(bar(C::B_SF + (j % C::NS)));
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nblk > 1) ok = issue_qk(1);
      // S = Q K^T of block j+2 goes into the S buffer of block j as soon as
      // every softmax warp has read S_j (well before block j's exponentials
      // are done), keeping the tensor pipe busy while V_j lands.
      for (int j = 0; j + 2 < nblk && ok; ++j) {
        ok = ptx::mbar_wait(bar(C::B_SC + (j % C::NS)), (j / C::NS) & 1, abort_flag,
                            p.timeout_ns);
        if (ok) ok = issue_qk(j + 2);
      }
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
      }
      // Drain: every MMA issued above has completed before TMEM is freed
      // (bounded, but not cut short by the abort flag).
      ptx::mma_commit(bar(C::B_DRAIN));
      ptx::mbar_wait(bar(C::B_DRAIN), 0, &misc[3], p.timeout_ns);
    }
  } else if (warp == C::WARP_PV) {
    // ======================= tcgen05 issuer: O += P V ======================
    if (lane == 0) {
      bool ok = true;
      const uint64_t v_desc = ptx::sw128_desc(sb + C::OFF_V, C::KV_BOX, 1024);
      int pv_count = 0;
      for (int j = 0; j < nblk && ok; ++j) {
        const int slot = j % C::NSLOT;
        ok = ptx::mbar_wait(bar(C::B_P + slot), (j / C::NSLOT) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        ptx::tc_fence_after();
        if (dec_val[slot] != 0) {
          const int vs = pv_count % C::NV;
          ok = ptx::mbar_wait(bar(C::B_VF + vs), (pv_count / C::NV) & 1, abort_flag,
                              p.timeout_ns);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t p_tm = tmem + C::P_COL + (j % C::NP) * (BC / 2);
          const uint64_t vd = v_desc + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
          ptx::mma_ts(tmem + C::O_COL, p_tm, vd, C::IDESC_PV, pv_count > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < BC / 16; ++kk)
            ptx::mma_ts(tmem + C::O_COL, p_tm + kk * 8,
                        vd + static_cast<uint64_t>(kk * (2048 >> 4)), C::IDESC_PV, 1u);
          ptx::mma_commit(bar(C::B_VE + vs));
          ptx::mma_commit(bar(C::B_PV + (j % C::NP)));
          ++pv_count;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
      }
      ptx::mma_commit(bar(C::B_DRAIN + 1));
      ptx::mbar_wait(bar(C::B_DRAIN + 1), 0, &misc[3], p.timeout_ns);
    }
  } else {
    // ======================= softmax warps 0-7 ===========================
    const int quad = warp & 3;        // TMEM lane quarter
    const int half = warp >> 2;       // column half
    const int t = quad * 32 + lane;   // row within the CTA tile
    const int row = r0 + t;
    const bool row_exists = row < p.Lq;
    const int gi = t / BR;
    const int my_kt_last = kt_last[gi];
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int last_col = p.causal ? min(row + p.off, p.Lkv - 1) : p.Lkv - 1;
    const float sl2 = p.scale_log2;
    const bool thresholding = p.log2_lambda > -INFINITY;
    const bool leader = threadIdx.x == 0;

    float m = -INFINITY, mref = -INFINITY, l = 0.0f;  // l: this half's partial sum
    int pvn0 = 0, pvn1 = 0;  // P.V products issued on P buffer 0 / 1
    int last_buf = -1, ncomp = 0;
    bool aborted = false;

    for (int j = 0; j < nblk; ++j) {
      const int sbuf = j % C::NS;
      const int pbuf = j % C::NP;
      bool ok = true;
      if (lane == 0)
        ok = ptx::mbar_wait(bar(C::B_SF + sbuf), (j / C::NS) & 1, abort_flag, p.timeout_ns);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ptx::tc_fence_after();

      float s[C::HALF];
      float mbh = -INFINITY;  // this half-row's max (log2 units)
      bool rowskip = true;
      const int col0 = j * BC + half * C::HALF;
      if (ok) {
        uint32_t sr[C::HALF];
#pragma unroll
        for (int c = 0; c < C::HALF / 32; ++c)
          ptx::tmem_ld32p(tmem + lane_base + C::S_COL + sbuf * BC + half * C::HALF + 32 * c,
                          sr + 32 * c);
        ptx::tmem_wait_ld();
        // S_j is in registers: its TMEM buffer may take block j+2's scores.
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_SC + sbuf));
#pragma unroll
        for (int c = 0; c < C::HALF; ++c) s[c] = __uint_as_float(sr[c]);
        const bool need_mask =
            (j * BC + BC > p.Lkv) || (p.causal && j * BC + BC - 1 > r0 + p.off);
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < C::HALF; ++c)
            if (col0 + c > last_col) s[c] = -INFINITY;
        }
        // half-row max: 8 independent chains of three-input max, then a tree
        float mc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          constexpr int W = C::HALF / 8;
          float a = s[i * W];
#pragma unroll
          for (int c = 1; c + 1 < W; c += 2) a = ptx::fmax3(a, s[i * W + c], s[i * W + c + 1]);
          if ((W - 1) % 2) a = fmaxf(a, s[i * W + W - 1]);
          mc[i] = a;
        }
        mbh = ptx::fmax3(ptx::fmax3(mc[0], mc[1], mc[2]), ptx::fmax3(mc[3], mc[4], mc[5]),
                         fmaxf(mc[6], mc[7])) * sl2;
        const bool visited = j <= my_kt_last;
        if (!row_exists || !visited) rowskip = true;
        else if (j == 0 || !thresholding) rowskip = false;
        else rowskip = (mbh - m) < p.log2_lambda;
      }
      pmax[((j & 1) * 2 + half) * 128 + t] = mbh;
      int keepmask = 0;
      bool any_abort = false;
      if constexpr (C::NG == 1) {
        // One vote group: the barrier itself ANDs the half-row tests of all
        // 256 softmax threads. A warp whose wait gave up marks the
        // softmax-private abort word of this block parity before the barrier.
        if (!ok && lane == 0) sm_abort[j & 1] = 1;
        const bool all_skip = ptx::named_bar_and(1, C::NSOFT, rowskip);
        any_abort = sm_abort[j & 1] != 0;
        if (j <= kt_last[0] && !all_skip) keepmask = 1;
      } else {
        const unsigned all_skip = __all_sync(0xffffffffu, rowskip) ? 1u : 0u;
        if (lane == 0) votes[(j & 1) * 8 + warp] = ok ? static_cast<int>(all_skip) : 2;
        ptx::named_bar_sync(1, C::NSOFT);
#pragma unroll
        for (int gg = 0; gg < C::NG; ++gg) {
          bool gskip = true;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int w = 0; w < C::WPG; ++w) {
              const int v = votes[(j & 1) * 8 + hh * 4 + gg * C::WPG + w];
              if (v == 2) any_abort = true;
              gskip = gskip && (v != 0);
            }
          if (j <= kt_last[gg] && !gskip) keepmask |= 1 << gg;
        }
      }
      const float mb = fmaxf(mbh, pmax[((j & 1) * 2 + (half ^ 1)) * 128 + t]);
      if (any_abort) {
        aborted = true;
        break;
      }
      if (leader) {
        dec_val[j % C::NSLOT] = keepmask;
        ptx::mbar_arrive(bar(C::B_DEC + (j % C::NSLOT)));
      }
      if (keepmask) {
        const bool my_keep = (keepmask >> gi) & 1;
        const float m_new = my_keep ? fmaxf(m, mb) : m;
        const bool need = my_keep && (m_new > mref + C::TAU);
        if (__any_sync(0xffffffffu, need)) {
          const float mref_new = need ? m_new : mref;
          if (ncomp > 0) {
            // O must be quiescent: wait for the last issued P.V.
            bool ok2 = true;
            if (lane == 0)
              ok2 = ptx::mbar_wait(bar(C::B_PV + last_buf),
                                   ((last_buf ? pvn1 : pvn0) - 1) & 1, abort_flag, p.timeout_ns);
            ok2 = __shfl_sync(0xffffffffu, ok2 ? 1 : 0, 0) != 0;
            if (!ok2) {
              *abort_flag = 1;
              record_error(p.err, BLASST_ETIMEOUT);
            }
            ptx::tc_fence_after();
            const float alpha = need ? ptx::ex2(mref - mref_new) : 1.0f;
            l *= alpha;
#pragma unroll
            for (int c = 0; c < C::DHALF / 32; ++c) {
              uint32_t r[32];
              const uint32_t ta = tmem + lane_base + C::O_COL + half * C::DHALF + 32 * c;
              ptx::tmem_ld32(ta, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              ptx::tmem_st32(ta, r);
            }
            ptx::tmem_wait_st();
          }
          mref = mref_new;
        }
        if (my_keep) m = m_new;

        uint32_t pk[C::HALF / 2];
        if (my_keep) {
          const float neg = -mref;
          float rs[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) rs[i] = 0.0f;
#pragma unroll
          for (int c = 0; c < C::HALF; c += 2) {
            float x0, x1, p0, p1;
            ptx::fma2(x0, x1, s[c], s[c + 1], sl2, sl2, neg, neg);
            // every eighth pair of columns takes the FMA-pipe exp2
            if (((c >> 1) & 7) == 7) {
              ptx::exp2_poly2(p0, p1, x0, x1);
            } else {
              p0 = ptx::ex2(x0);
              p1 = ptx::ex2(x1);
            }
            const int a = ((c >> 1) & 3) * 2;
            ptx::add2(rs[a], rs[a + 1], rs[a], rs[a + 1], p0, p1);
            pk[c / 2] = ptx::pack_bf16x2(p0, p1);
          }
          l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        } else {
#pragma unroll
          for (int c = 0; c < C::HALF / 2; ++c) pk[c] = 0u;
        }
        // P buffer pbuf was last read by the P.V of block j-2 (if computed).
        const int pv_here = pbuf ? pvn1 : pvn0;
        if (pv_here > 0) {
          bool ok3 = true;
          if (lane == 0)
            ok3 = ptx::mbar_wait(bar(C::B_PV + pbuf), (pv_here - 1) & 1, abort_flag,
                                 p.timeout_ns);
          ok3 = __shfl_sync(0xffffffffu, ok3 ? 1 : 0, 0) != 0;
          if (!ok3) {
            *abort_flag = 1;
            record_error(p.err, BLASST_ETIMEOUT);
          }
          ptx::tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < C::HALF / 32; ++c)
          ptx::tmem_st16(tmem + lane_base + C::P_COL + pbuf * (BC / 2) + half * (C::HALF / 2) +
                             16 * c,
                         pk + 16 * c);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ++ncomp;
        last_buf = pbuf;
        if (pbuf) ++pvn1;
        else ++pvn0;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_P + (j % C::NSLOT)));
    }

    if (aborted) {
      if (leader) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
      }
    } else {
      // ---- epilogue: O / l -> bf16, lse, masks of unvisited blocks ------
      bool ok = true;
      if (ncomp > 0 && lane == 0)
        ok = ptx::mbar_wait(bar(C::B_PV + last_buf), ((last_buf ? pvn1 : pvn0) - 1) & 1,
                            abort_flag, p.timeout_ns);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ptx::tc_fence_after();
      lsum[half * 128 + t] = l;
      ptx::named_bar_sync(1, C::NSOFT);
      const float ltot = l + lsum[(half ^ 1) * 128 + t];
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
      } else {
        const float inv_l = (ltot > 0.0f) ? 1.0f / ltot : 0.0f;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                              (static_cast<size_t>(bh) * p.Lq + row) * D + half * C::DHALF;
#pragma unroll
        for (int c = 0; c < C::DHALF / 32; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(tmem + lane_base + C::O_COL + half * C::DHALF + 32 * c, r);
          ptx::tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = ptx::pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                                    __uint_as_float(r[2 * i + 1]) * inv_l);
          if (row_exists) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
        if (row_exists && half == 0)
          p.lse[static_cast<size_t>(bh) * p.Lq + row] = (mref + log2f(ltot)) * 0.6931471805599453f;
        if (p.mask) {
#pragma unroll
          for (int gg = 0; gg < C::NG; ++gg) {
            if (kt_last[gg] < 0) continue;
            const int qt = r0 / BR + gg;
            uint8_t* mrow = p.mask + (static_cast<size_t>(bh) * p.nQt + qt) * p.nKt;
            for (int jj = nblk + static_cast<int>(threadIdx.x); jj < p.nKt; jj += C::NSOFT)
              mrow[jj] = 2;
          }
        }
      }
    }
  }

  __syncwarp();  // role warps reconverge (only their lane 0 worked)
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace blasst
