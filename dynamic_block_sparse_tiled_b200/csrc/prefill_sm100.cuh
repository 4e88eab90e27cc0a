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
// blocks of its KV head. TMEM holds two S buffers (fp32, one per softmax
// set), two P buffers (bf16, one per set) and O. Warp roles (384 threads):
//   warps 0-3  softmax of the even blocks, warps 4-7 softmax of the odd
//              blocks; thread t of a set owns row t (TMEM lane t) over all
//              Bc columns of its blocks and holds the whole S row in
//              registers after the max pass, so the S buffer is free again at
//              once. The two sets alternate, so on each SM sub-partition one
//              warp runs the exponentials of block j while the other reads S,
//              takes the row max and votes on block j+1. The running max after
//              block j is the prefix max of the visited blocks' maxima whatever
//              the votes (a skipped block lies below it on every row), so each
//              set hands the running statistics to the other right after its
//              row max, before its own vote;
//   warp 8     TMA producer for Q and K (3-stage ring, ahead of the votes);
//   warp 9     TMA producer for V: loads V of block j only after the vote on
//              block j says some row group keeps it; writes the skip mask;
//   warp 10    tcgen05 issuer for S = Q K^T: one wait and one commit per
//              block (the K-full barrier also counts the set that freed the S
//              buffer and the P V issuer and V producer past block j-3);
//              owns the TMEM allocation;
//   warp 11    tcgen05 issuer for O += P V, P from its set's TMEM P buffer.
// With Br = 64 the 128 rows form two independent vote groups that share the
// MMAs: a group that skips contributes zero rows of P and leaves its running
// statistics untouched.
// An optional static block mask (block-sparse input) excludes (query tile,
// KV block) pairs before anything is computed: the CTA then walks a list of
// the blocks some row group still visits, built in shared memory at start;
// every role iterates over list positions (pipeline slots and parities) and
// reads the block index from the list. The first-block rule applies to the
// first listed block.
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
  const uint8_t* smask;  // optional static block mask [B, Hq, nQt, nKt], nonzero = excluded
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
  static constexpr int NSOFT = 256;  // softmax threads (warps 0-7), two sets of 128
  static constexpr int WARP_K = 8, WARP_V = 9, WARP_MMA = 10, WARP_PV = 11;
  static constexpr int NG = BM / BR;   // vote groups
  static constexpr int WPG = BR / 32;  // TMEM lane quarters (warps of a set) per vote group
  static constexpr int NCH = BC / 32;  // 32-column chunks of a block row
  static constexpr int NK = 3;
  static constexpr int NV = 2;
  static constexpr int NS = 2;     // S buffers (fp32, BC columns), one per softmax set
  static constexpr int NPV = 4;    // "every P V up to block j done" barriers (j % 4)
  static constexpr int NSLOT = 4;  // decision slots
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
  // B_KF + s completes for block j (j % NK == s) when K_j has landed and S
  // buffer j % NS may take S_j: the K producer's arrival (with the bytes), the
  // four warps of the softmax set of block j-2 once S_{j-2} is in registers,
  // and the PV issuer and the V producer once each has read decision j-3 (so
  // the decision slots, P and DEC barriers never run more than three blocks
  // ahead of their readers). The S issuer waits once per block. The first
  // phases get the arrivals of the blocks before 0 at set-up.
  static constexpr int B_KF = 1;
  static constexpr int KF_COUNT = 7;
  // B_KE + s: K stage s free again (the four warps of the set that read S_j)
  static constexpr int B_KE = B_KF + NK;
  static constexpr int B_VF = B_KE + NK;
  static constexpr int B_VE = B_VF + NV;
  static constexpr int B_SF = B_VE + NV;      // [NS] S written (tcgen05 commit)
  static constexpr int B_PV = B_SF + NS;   // [NPV] every P V up to the block done
  static constexpr int B_DEC = B_PV + NPV;    // [NSLOT] decision (V producer)
  static constexpr int B_P = B_DEC + NSLOT;   // [NSLOT] P ready or block skipped (PV issuer)
  static constexpr int B_HS = B_P + NSLOT;  // [2] running statistics handed to set s
  static constexpr int B_DRAIN = B_HS + 2;      // [2] QK issuer, PV issuer
  static constexpr int NBAR = B_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc words: [0] tmem base, [1] abort, [3] always 0 (for waits only a timeout
  // ends), [4..7] decisions, [8..15] votes [set][warp of set] (Br = 64),
  // [16..17] softmax abort word per set, [24..27] the CTA's start (clock64,
  // %globaltimer) for the telemetry
  static constexpr int MISC_BYTES = 128;
  static constexpr int OFF_ST = OFF_MISC + MISC_BYTES;  // [2 sets][2: m, mref][128 rows] floats
  static constexpr int OFF_LSUM = OFF_ST + 2 * 2 * 128 * 4;  // [2 sets][128 rows] floats
  static constexpr int MAX_LIST = 4096;  // listed blocks with a static mask (Lkv <= 4096 Bc)
  static constexpr int OFF_LIST = OFF_LSUM + 2 * 128 * 4;     // [MAX_LIST] kt | groups << 16
  static constexpr int OFF_SCAN = OFF_LIST + MAX_LIST * 4;    // [NTHREADS] counts
  static constexpr int SMEM_BYTES = OFF_LIST + 1024;                   // + alignment slack
  static constexpr int SMEM_BYTES_LISTED = OFF_SCAN + NTHREADS * 4 + 1024;
  static constexpr int S_COL = 0;          // S buffer b (set b) at column b * BC
  static constexpr int P_COL = NS * BC;    // P buffer b (bf16 pairs, BC/2 columns) after them
  static constexpr int O_COL = P_COL + NS * (BC / 2);  // O accumulator
  static constexpr int TMEM_COLS = pow2_at_least(O_COL + D);
  static constexpr uint32_t IDESC_QK = ptx::idesc_f32acc(1, 128, BC, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc_f32acc(1, 128, D, true);
  static constexpr float TAU = 8.0f;  // lazy-rescale slack, log2 units
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BC == 64 || BC == 128, "KV block");
  static_assert(BR == 64 || BR == 128, "query tile");
  static_assert(TMEM_COLS <= 512, "TMEM budget");
  static_assert(NK == 3 && NS == 2, "the K-full barrier counts the readers of block j - NK");
  static_assert(NSLOT > NK, "decision slots must outlive the readers' lag");
  static_assert(SMEM_BYTES_LISTED <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// LISTED: compiled for a static block mask (p.smask != null) or without one;
// the version without keeps no list and none of its bookkeeping.
template <int D, int BC, int BR, bool LISTED>
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
  volatile int* sm_abort = misc + 16;
  volatile float* st_rows = reinterpret_cast<volatile float*>(smem + C::OFF_ST);
  volatile float* lsum = reinterpret_cast<volatile float*>(smem + C::OFF_LSUM);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // A CTA that starts while the device error word holds an error (a bounded
  // wait of this launch, or of an earlier one not yet read by blasst_check,
  // gave up) does nothing: the launch then ends within one wave of waits
  // instead of every CTA waiting out its own bounds.
  // (misc[0] holds the TMEM base only once it is allocated, below)
  if (threadIdx.x == 0)
    misc[0] = (p.err != nullptr && *reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
  __syncthreads();
  if (misc[0] != 0) return;

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

  // ---- static block mask: list of the blocks some row group visits --------
  constexpr bool listed = LISTED;
  uint32_t* vlist = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
  if constexpr (LISTED) {
    // every thread takes a contiguous strip of blocks; counts, an exclusive
    // scan over the CTA, then the strips are written in order
    int* scan = reinterpret_cast<int*>(smem + C::OFF_SCAN);
    const int strip = (nblk + C::NTHREADS - 1) / C::NTHREADS;
    const int k0 = static_cast<int>(threadIdx.x) * strip;
    const int k1 = min(k0 + strip, nblk);
    auto groups_of = [&](int kt) -> uint32_t {
      uint32_t gm = 0;
#pragma unroll
      for (int gg = 0; gg < C::NG; ++gg)
        if (kt <= kt_last[gg] &&
            p.smask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + kt] == 0)
          gm |= 1u << gg;
      return gm;
    };
    int cnt = 0;
    for (int kt = k0; kt < k1; ++kt) cnt += groups_of(kt) ? 1 : 0;
    scan[threadIdx.x] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0;
      for (int i = 0; i < C::NTHREADS; ++i) {
        const int c = scan[i];
        scan[i] = acc;
        acc += c;
      }
      misc[2] = acc;
    }
    __syncthreads();
    int pos = scan[threadIdx.x];
    for (int kt = k0; kt < k1; ++kt) {
      const uint32_t gm = groups_of(kt);
      if (gm) vlist[pos++] = static_cast<uint32_t>(kt) | (gm << 16);
    }
    // every (tile, block) pair starts as "not visited"; the V warp writes the
    // visited ones after the barrier below
    if (p.mask) {
#pragma unroll
      for (int gg = 0; gg < C::NG; ++gg) {
        if (kt_last[gg] < 0) continue;
        uint8_t* mrow = p.mask + (static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt;
        for (int kt = static_cast<int>(threadIdx.x); kt < p.nKt; kt += C::NTHREADS) mrow[kt] = 2;
      }
    }
    __syncthreads();
    nblk = misc[2];  // from here on: number of listed blocks
  }
  // block index and visiting row groups of list position j
  auto kt_of = [&](int j) -> int {
    if constexpr (LISTED) return static_cast<int>(vlist[j] & 0xFFFFu);
    else return j;
  };
  auto groups_at = [&](int j) -> uint32_t {
    if constexpr (LISTED) return vlist[j] >> 16;
    uint32_t gm = 0;
#pragma unroll
    for (int gg = 0; gg < C::NG; ++gg)
      if (j <= kt_last[gg]) gm |= 1u << gg;
    return gm;
  };

  // ---- set-up -------------------------------------------------------------
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_Q), 1);
    for (int i = 0; i < C::NK; ++i) {
      ptx::mbar_init(bar(C::B_KF + i), C::KF_COUNT);
      ptx::mbar_init(bar(C::B_KE + i), 4);
    }
    for (int i = 0; i < C::NV; ++i) {
      ptx::mbar_init(bar(C::B_VF + i), 1);
      ptx::mbar_init(bar(C::B_VE + i), 1);
    }
    for (int i = 0; i < C::NS; ++i) {
      ptx::mbar_init(bar(C::B_SF + i), 1);
    }
    for (int i = 0; i < C::NPV; ++i) ptx::mbar_init(bar(C::B_PV + i), 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      ptx::mbar_init(bar(C::B_DEC + i), 1);
      ptx::mbar_init(bar(C::B_P + i), 4);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(C::B_HS + i), 4);
      ptx::mbar_init(bar(C::B_DRAIN + i), 1);
    }
    for (int i = 1; i < C::MISC_BYTES / 4; ++i)
      if (i != 2) misc[i] = 0;
    // (in shared memory: no register stays live across the kernel for it)
    reinterpret_cast<volatile unsigned long long*>(misc + 24)[0] =
        static_cast<unsigned long long>(clock64());
    reinterpret_cast<volatile unsigned long long*>(misc + 24)[1] = ptx::globaltimer_ns();
    // blocks 0 .. NS-1 have no S_{j-2} reader and blocks 0 .. NK-1 no
    // decision j-3: those arrivals are made here
    for (int i = 0; i < C::NK; ++i)
      for (int a = 0; a < (i < C::NS ? 4 : 0) + 2; ++a) ptx::mbar_arrive(bar(C::B_KF + i));
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
        load_kv(&tmK, sb + C::OFF_K + ks * C::KV_BYTES, kt_of(j), bar(C::B_KF + ks));
      }
      if (!ok) {
        *abort_flag = 1;
        record_error(p.err, BLASST_ETIMEOUT);
        // Let the copies already in flight land before the CTA exits.
        ptx::mbar_wait(bar(C::B_Q), 0, &misc[3], p.timeout_ns);
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
        ptx::mbar_arrive(bar(C::B_KF + (j % C::NK)));  // decision j read (block j + NK)
        // skip-mask entries and counters for block j (off the softmax path)
        const unsigned long long tile_flops = 2ull * 128ull * BC * D;
        st_flops += tile_flops + (keepmask ? tile_flops : 0ull);
        const int kt = kt_of(j);
        const uint32_t gvis = groups_at(j);
#pragma unroll
        for (int gg = 0; gg < C::NG; ++gg) {
          if (kt_last[gg] < 0) continue;
          uint8_t code = 2;
          if ((gvis >> gg) & 1) {
            ++st_vis;
            code = ((keepmask >> gg) & 1) ? 0 : 1;
            if (code == 1) ++st_skip;
          }
          if (p.mask)
            p.mask[(static_cast<size_t>(bh) * p.nQt + (r0 / BR + gg)) * p.nKt + kt] = code;
        }
        if (keepmask != 0) {
          const int vs = vcount % C::NV;
          if (vcount >= C::NV)
            ok = ptx::mbar_wait(bar(C::B_VE + vs), ((vcount / C::NV) - 1) & 1, abort_flag,
                                p.timeout_ns);
          if (!ok) break;
          load_kv(&tmV, sb + C::OFF_V + vs * C::KV_BYTES, kt, bar(C::B_VF + vs));
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
        ptx::mma_commit(bar(C::B_SF + (j % C::NS)));
        return true;
      };
      // S_j goes into the buffer of its softmax set (j % 2) once that set has
      // read S_{j-2} into registers (right after its row max: neither its
      // exponentials nor P V hold the buffer) and the PV issuer and the V
      // producer are past block j-3, all in one wait (B_KF). That also keeps
      // the Q K^T products from running far ahead of the P V ones, which
      // helps the dense step.
      for (int j = 0; j < nblk && ok; ++j) ok = issue_qk(j);
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
        const bool keep = dec_val[slot] != 0;
        ptx::mbar_arrive(bar(C::B_KF + (j % C::NK)));  // decision j read (block j + NK)
        if (keep) {
          const int vs = pv_count % C::NV;
          ok = ptx::mbar_wait(bar(C::B_VF + vs), (pv_count / C::NV) & 1, abort_flag,
                              p.timeout_ns);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t p_tm = tmem + C::P_COL + (j % C::NS) * (BC / 2);
          const uint64_t vd = v_desc + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
          ptx::mma_ts(tmem + C::O_COL, p_tm, vd, C::IDESC_PV, pv_count > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < BC / 16; ++kk)
            ptx::mma_ts(tmem + C::O_COL, p_tm + kk * 8,
                        vd + static_cast<uint64_t>(kk * (2048 >> 4)), C::IDESC_PV, 1u);
          ptx::mma_commit(bar(C::B_VE + vs));
          ++pv_count;
        }
        // every P V up to block j done (P buffer reuse, lazy rescale, epilogue)
        ptx::mma_commit(bar(C::B_PV + j % C::NPV));
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
    const int set = warp >> 2;        // 0: even blocks, 1: odd blocks
    const int quad = warp & 3;        // TMEM lane quarter
    const int t = quad * 32 + lane;   // row within the CTA tile
    const int row = r0 + t;
    const bool row_exists = row < p.Lq;
    const int gi = t / BR;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int last_col = p.causal ? min(row + p.off, p.Lkv - 1) : p.Lkv - 1;
    const float sl2 = p.scale_log2;
    const bool thresholding = p.log2_lambda > -INFINITY;
    const bool leader = lane == 0 && quad == 0;  // one per set
    volatile float* st_out = st_rows + (1 - set) * 256;  // handed to the other set
    volatile float* st_in = st_rows + set * 256;

    // l: this set's partial row sum, relative to the reference lref
    float l = 0.0f, lref = -INFINITY;
    bool aborted = false;

    auto lane0_wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
      bool ok = true;
      if (lane == 0) ok = ptx::mbar_wait(bar_addr, parity, abort_flag, p.timeout_ns);
      return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };

    for (int j = set; j < nblk; j += 2) {
      const int sbuf = j % C::NS;  // == set
      const uint32_t s_tm = tmem + lane_base + C::S_COL + sbuf * BC;
      const uint32_t p_tm = tmem + lane_base + C::P_COL + sbuf * (BC / 2);
      bool ok = lane0_wait(bar(C::B_SF + sbuf), (j / C::NS) & 1);
      ptx::tc_fence_after();

      // ---- row max of block j (masked); the row's S stays in registers ----
      uint32_t sk[C::NCH * 32];
      float mbh = -INFINITY;
      const int kt = kt_of(j);
      const uint32_t gvis = groups_at(j);
      const int col0 = kt * BC;
      const bool need_mask = (col0 + BC > p.Lkv) || (p.causal && col0 + BC - 1 > r0 + p.off);
      if (ok) {
        float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          uint32_t* sr = sk + 32 * c;
          ptx::tmem_ld32p(s_tm + 32 * c, sr);
          ptx::tmem_wait_ld();
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + 32 * c + i > last_col) sr[i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            mc[0] = ptx::fmax3(mc[0], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
            mc[1] = ptx::fmax3(mc[1], __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
            mc[2] = ptx::fmax3(mc[2], __uint_as_float(sr[i + 4]), __uint_as_float(sr[i + 5]));
            mc[3] = ptx::fmax3(mc[3], __uint_as_float(sr[i + 6]), __uint_as_float(sr[i + 7]));
          }
        }
        mbh = fmaxf(ptx::fmax3(mc[0], mc[1], mc[2]), mc[3]) * sl2;
      }
      // S_j is in registers: its buffer may take S_{j+2}, and K_j's stage
      // (read by the finished Q K_j^T) may take K_{j+NK}
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(bar(C::B_KF + (j + 2) % C::NK));
        ptx::mbar_arrive(bar(C::B_KE + j % C::NK));
      }

      // ---- running statistics after block j-1 (from the other set) -------
      float m = -INFINITY, mref = -INFINITY;
      if (j > 0) {
        const bool ok2 = lane0_wait(bar(C::B_HS + set), ((j - 1) >> 1) & 1);
        ok = ok && ok2;
        m = st_in[t];
        mref = st_in[128 + t];
      }

      const float m_new = ((gvis >> gi) & 1) ? fmaxf(m, mbh) : m;
      const bool need = m_new > mref + C::TAU;
      const float mref_new = need ? m_new : mref;
      st_out[t] = m_new;
      st_out[128 + t] = mref_new;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_HS + (1 - set)));

      // ---- the vote: every row of the tile (group) must find block j
      //      negligible; a block beyond a row's causal range votes skip -----
      bool rowskip = true;
      if (ok) {
        const bool visited = (gvis >> gi) & 1;
        if (!row_exists || !visited) rowskip = true;
        else if (j == 0 || !thresholding) rowskip = false;
        else if (LISTED && mbh == -INFINITY) rowskip = true;  // no visible key here
        else rowskip = (mbh - m) < p.log2_lambda;
      }
      int keepmask = 0;
      bool any_abort = false;
      if constexpr (C::NG == 1) {
        if (!ok && lane == 0) sm_abort[set] = 1;
        const bool all_skip = ptx::named_bar_and(1 + set, 128, rowskip);
        any_abort = sm_abort[set] != 0;
        if ((gvis & 1u) && !all_skip) keepmask = 1;
      } else {
        const unsigned all_skip = __all_sync(0xffffffffu, rowskip) ? 1u : 0u;
        volatile int* vw = votes + set * 4;  // one word per warp of the set
        if (lane == 0) vw[quad] = ok ? static_cast<int>(all_skip) : 2;
        ptx::named_bar_sync(1 + set, 128);
#pragma unroll
        for (int gg = 0; gg < C::NG; ++gg) {
          bool gskip = true;
#pragma unroll
          for (int w = 0; w < C::WPG; ++w) {
            const int v = vw[gg * C::WPG + w];
            if (v == 2) any_abort = true;
            gskip = gskip && (v != 0);
          }
          if (((gvis >> gg) & 1) && !gskip) keepmask |= 1 << gg;
        }
        if (sm_abort[set] != 0) any_abort = true;
        // the words are rewritten only after this set's next barrier below
        ptx::named_bar_sync(1 + set, 128);
      }
      if (any_abort) {
        aborted = true;
        break;
      }

      // ---- new running statistics, handed to the other set ---------------
      const bool my_keep = (keepmask >> gi) & 1;
      if (leader) {
        dec_val[j % C::NSLOT] = keepmask;
        ptx::mbar_arrive(bar(C::B_DEC + (j % C::NSLOT)));
      }

      // A skipped block has no P to write: it goes to the P V issuer at once.
      if (!keepmask) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_P + (j % C::NSLOT)));
      }

      // This set's P buffer was last read by the P V of block j-2. The wait is
      // taken at every block (kept or not), so each set awaits its "P V done"
      // phases in order. It stays exact after a skipped block was handed on:
      // the P V issuer can then pass block j+1 but not j+2 (this set's next),
      // and the phase of j-2 + NPV (NPV = 4) needs it past j+2.
      if (j >= 2) {
        const bool okp = lane0_wait(bar(C::B_PV + (j - 2) % C::NPV), ((j - 2) / C::NPV) & 1);
        if (!okp) {
          *abort_flag = 1;
          if (lane == 0) sm_abort[set] = 1;
          record_error(p.err, BLASST_ETIMEOUT);
        }
      }

      if (keepmask) {
        // l and O follow the reference mref_new
        if (mref_new != lref) {
          l = (lref == -INFINITY) ? 0.0f : l * ptx::ex2(lref - mref_new);
          lref = mref_new;
        }
        if (__any_sync(0xffffffffu, need) && j > 0) {
          // O must be quiescent: every P V up to block j-1 has completed (the
          // first block is always kept, so O holds its P V by then).
          const bool ok3 = lane0_wait(bar(C::B_PV + (j - 1) % C::NPV), ((j - 1) / C::NPV) & 1);
          if (!ok3) {
            *abort_flag = 1;
            if (lane == 0) sm_abort[set] = 1;
            record_error(p.err, BLASST_ETIMEOUT);
          }
          ptx::tc_fence_after();
          const float alpha = need ? ptx::ex2(mref - mref_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            const uint32_t ta = tmem + lane_base + C::O_COL + 32 * c;
            ptx::tmem_ld32(ta, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            ptx::tmem_st32(ta, r);
          }
          ptx::tmem_wait_st();
        }

        // ---- P = exp2(s * scale*log2e - mref) as bf16 into the P buffer ----
        const float neg = -mref_new;
        float rs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rs[i] = 0.0f;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint32_t* sr = sk + 32 * c;
          uint32_t pk[16];
          // (with a static mask a row may have no key yet: it adds nothing)
          if (my_keep && (!LISTED || mref_new > -INFINITY)) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float x0, x1, p0, p1;
              ptx::fma2(x0, x1, __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]), sl2, sl2,
                        neg, neg);
              // every eighth pair of columns takes the FMA-pipe exp2
              if (((i >> 1) & 7) == 7) {
                ptx::exp2_poly2(p0, p1, x0, x1);
              } else {
                p0 = ptx::ex2(x0);
                p1 = ptx::ex2(x1);
              }
              const int a = ((i >> 1) & 3) * 2;
              ptx::add2(rs[a], rs[a + 1], rs[a], rs[a + 1], p0, p1);
              pk[i / 2] = ptx::pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
          ptx::tmem_st16(p_tm + 16 * c, pk);
        }
        l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_P + (j % C::NSLOT)));
      }
    }

    // ---- epilogue ----------------------------------------------------------
    if (aborted && leader) {
      *abort_flag = 1;
      record_error(p.err, BLASST_ETIMEOUT);
    }
    ptx::named_bar_sync(3, C::NSOFT);
    // final statistics: the state after block nblk-1, handed to set nblk & 1
    const int fin = nblk & 1;
    // (a static mask can leave no block at all: then O = 0, lse = -inf)
    const float mref_fin = nblk > 0 ? st_rows[fin * 256 + 128 + t] : -INFINITY;
    const float l_mine =
        (lref == -INFINITY || mref_fin == -INFINITY) ? 0.0f : l * ptx::ex2(lref - mref_fin);
    lsum[set * 128 + t] = l_mine;
    bool ok = __shfl_sync(0xffffffffu, (lane == 0 && *abort_flag == 0) ? 1 : 0, 0) != 0;
    if (ok && nblk > 0)  // every P V has completed
      ok = lane0_wait(bar(C::B_PV + (nblk - 1) % C::NPV), ((nblk - 1) / C::NPV) & 1);
    ptx::tc_fence_after();
    ptx::named_bar_sync(3, C::NSOFT);
    const float ltot = lsum[t] + lsum[128 + t];
    if (!ok || *abort_flag) {
      if (lane == 0) *abort_flag = 1;
      record_error(p.err, BLASST_ETIMEOUT);
    } else {
      // warp w writes columns [half*D/2, (half+1)*D/2) of its quarter's rows
      const int half = set;
      const float inv_l = (ltot > 0.0f) ? 1.0f / ltot : 0.0f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                            (static_cast<size_t>(bh) * p.Lq + row) * D + half * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + half * (D / 2) + 32 * c, r);
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
        p.lse[static_cast<size_t>(bh) * p.Lq + row] = (mref_fin + log2f(ltot)) * 0.6931471805599453f;
      if (p.mask && !listed) {  // with a static mask every entry was preset
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

  __syncwarp();  // role warps reconverge (only their lane 0 worked)
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && p.stats) {
    const volatile unsigned long long* t0 =
        reinterpret_cast<const volatile unsigned long long*>(misc + 24);
    atomicAdd(&p.stats->sm_cycles, static_cast<unsigned long long>(clock64()) - t0[0]);
    atomicAdd(&p.stats->sm_ns, static_cast<unsigned long long>(ptx::globaltimer_ns()) - t0[1]);
  }
  if (warp == C::WARP_MMA) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace blasst
