// bwd_sm100.cuh - backward pass of blocked attention with softmax
// thresholding on sm_100a (tcgen05 + TMEM + TMA), with the forward's
// decisions held fixed.
//
// What is differentiated ("BLASST: Dynamic BLocked Attention Sparsity via
// Softmax Thresholding", Telegram channel seeallochnaya, post 3655,
// paragraphs 2-6 after the headline): the forward's output is softmax
// attention over the keys it kept; a dropped (query tile, KV block) pair adds
// nothing, its V is never used. The skip decisions are a step function of the
// scores, so with them held fixed the gradient is the gradient of attention
// restricted to the kept pairs:
//   P  = exp(scale q.k - lse)   on kept (row, key) pairs, 0 elsewhere,
//   Dr = rowsum(dO * O),
//   dS = P * (dO.v - Dr),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO,
// summed over the query heads of a GQA group for dK and dV. The pages give
// no backward pass; this is the plain reading that the forward's definition
// fixes.
//
// Layout of the work: one CTA per (batch, KV head, 128-key block j). K_j and
// V_j stay in shared memory; the CTA walks the 64-row query tiles of the g
// query heads whose pair with block j the forward kept, in order. Per pair
// (all products on the tensor cores, 128 x 64 or 128 x 128 tiles):
//   S^T  = K Q^T          (TMEM, lanes = keys)       bf16 SS
//   dP^T = V dO^T         (TMEM, lanes = keys)       bf16 SS
//   P^T, dS^T by the compute warps, one key row per thread;
//   P^T (bf16) overwrites S^T in TMEM, dS^T (bf16) goes to shared memory;
//   dV  += P^T dO         (TMEM accumulator)         bf16 TS
//   dK  += dS^T Q         (TMEM accumulator)         bf16 SS
//   dQ^T = K^T dS^T       (TMEM, lanes = head dims)  bf16 SS, then staged in
//                          shared memory as four [64 rows][32 dims] fp32
//                          tiles and added to the fp32 dQ in global memory by
//                          four TMA reduce-adds (the add happens in L2).
// Computing the transposed S and dP puts the keys on TMEM lanes, so P^T can
// feed dV straight from TMEM and every product keeps M = 128; dQ^T keeps the
// head dims on lanes, so a warp's store of one staged dQ row covers 32
// consecutive dims (128 contiguous bytes, no bank conflicts). The staging
// tile reuses the pair's Q and dO stage: both are dead once dQ^T is done
// (every product that reads them was issued before it and the tensor core
// completes them in order).
//
// Warp roles (352 threads):
//   warps 0-3, 4-7  two compute sets on alternating pairs (set = pair % 2 =
//              the S^T, dP^T and dS^T buffer): P^T and dS^T, one key row per
//              thread, then the set drains its pair's dQ^T (warp q: head dims
//              [32 q, 32 q + 32)), stages it and issues the reduce-adds; at
//              the end set 0 writes dV and set 1 writes dK;
//   warp 8     producer: K and V once, then per pair Q, dO (TMA, 4-stage
//              ring) and the pair's row statistics (bulk copies); builds the
//              pair list by scanning the forward's decisions;
//   warp 9     tcgen05 issuer of dV, dK and dQ^T; owns the TMEM allocation;
//   warp 10    tcgen05 issuer of S^T and dP^T.
// TMEM (512 columns): S^T/P^T x2 [0,128), dP^T/dQ^T x2 [128,256),
// dV [256,384), dK [384,512).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/blasst.h"
#include "ptx_sm100.cuh"

namespace blasst {

struct BwdParams {
  float* dq;                // [B, Hq, Lq, 128] fp32, zeroed by the row pass, accumulated here
  float* dk;                // [B, Hkv, Lkv, 128] fp32
  float* dv;                // [B, Hkv, Lkv, 128] fp32
  const float* nl2;         // [B*Hq, LqP]: -lse * log2(e), -inf for rows without keys / padding
  const float* drow;        // [B*Hq, LqP]: rowsum(dO * O), 0 on padding
  const uint8_t* fmask;     // forward decisions [B, Hq, nQf, nKf], 0 = computed; null = all
  int* err;
  int B, Hq, Hkv, Lq, Lkv, g;
  int LqP;    // Lq rounded up to 64
  int nT;     // ceil(Lq / 64) query tiles of the backward
  int nKb;    // ceil(Lkv / 128) key blocks of the backward
  int Brf, Bcf;  // the forward's tile sizes (decisions are per Brf x Bcf pair)
  int nQf, nKf;  // ceil(Lq / Brf), ceil(Lkv / Bcf)
  int causal;
  int off;       // Lkv - Lq
  float scale;       // score scale
  float scale_log2;  // scale * log2(e)
  uint64_t timeout_ns;
};

struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int BK = 128;  // keys per CTA
  static constexpr int BQ = 64;   // query rows per pair
  static constexpr int NTHREADS = 352;
  static constexpr int WARP_LOAD = 8, WARP_MMA = 9, WARP_SP = 10;
  static constexpr int NST = 4;  // Q / dO stages
  static constexpr int KV_BOX = BK * 128;      // [128 keys][64 dims] bf16, 16 KB
  static constexpr int KV_BYTES = 2 * KV_BOX;  // 32 KB
  static constexpr int Q_BOX = BQ * 128;       // [64 rows][64 dims] bf16, 8 KB
  static constexpr int Q_BYTES = 2 * Q_BOX;    // 16 KB
  static constexpr int DS_BYTES = BK * 128;    // [128 keys][64 q] bf16, 16 KB
  static constexpr int DQS_BYTES = BQ * 32 * 4;  // one warp's staged [64 rows][32 dims] fp32, 8 KB
  static constexpr int ROWST_BYTES = 2 * BQ * 4;  // nl2[64], drow[64]
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + NST * Q_BYTES;
  static constexpr int OFF_DS = OFF_DO + NST * Q_BYTES;
  static constexpr int OFF_RS = OFF_DS + 2 * DS_BYTES;
  static constexpr int OFF_REC = OFF_RS + NST * ROWST_BYTES;  // [NST] {hq, t, keep bits, end}
  static constexpr int OFF_BAR = OFF_REC + NST * 16;
  // barriers
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;               // [NST] stage loaded (+ record)
  static constexpr int B_QE = B_QF + NST;      // [NST] stage free (QE_COUNT)
  static constexpr int B_SF = B_QE + NST;      // [2] S^T ready
  static constexpr int B_PR = B_SF + 2;        // [2] P^T in TMEM (4 warps of a compute set)
  static constexpr int B_DPF = B_PR + 2;       // [2] dP^T ready
  static constexpr int B_DSR = B_DPF + 2;      // [2] dS^T in shared memory (4 warps of a set)
  static constexpr int B_DQF = B_DSR + 2;      // [2] dQ^T ready (the set then knows dK and
                                               // dQ^T of the pair have read its dS^T buffer)
  static constexpr int B_ZERO = B_DQF + 2;     // dV, dK accumulators cleared (8 compute warps)
  static constexpr int B_ACC = B_ZERO + 1;     // dV, dK final
  static constexpr int B_DRAIN = B_ACC + 1;    // [2] the two issuers' drains
  static constexpr int NBAR = B_DRAIN + 2;
  // stage free: the 4 warps of the pair's set once their dQ adds have read
  // the staged tiles (after dQ^T was ready, so every product that read the
  // stage's Q and dO is done: the tensor core completes in order)
  static constexpr int QE_COUNT = 4;
  // stage loaded for pair i, and the buffers of pair i-2 free for pair i: the
  // producer's arrival (with the bytes), the dV issuer's commit after dV of
  // pair i-2 (its P^T read) and the 4 warps of that pair's set once they have
  // drained its dQ^T (the dP^T / dQ^T buffer). The S^T / dP^T issuer waits
  // once per pair. Pairs 0 and 1 get the pair-before arrivals at set-up.
  static constexpr int QF_COUNT = 1 + 1 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc words: [0] tmem base, [1] abort, [3] always 0 (waits only a timeout ends)
  static constexpr int MISC_BYTES = 64;
  // no alignment slack: the kernel checks that the dynamic shared memory
  // base is 1024-byte aligned (it is when the kernel has no static shared
  // memory) and reports BLASST_EUNSUPPORTED otherwise
  static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES;
  static constexpr int S_COL = 0;      // S^T buffer b at b * 64 (P^T: first 32 columns)
  static constexpr int DP_COL = 128;   // dP^T / dQ^T buffer b at 128 + b * 64
  static constexpr int DV_COL = 256;
  static constexpr int DK_COL = 384;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32acc(128, BQ, false, false);
  static constexpr uint32_t IDESC_DV = ptx::idesc_bf16_f32acc(128, D, false, true);
  static constexpr uint32_t IDESC_DK = ptx::idesc_bf16_f32acc(128, D, false, true);
  static constexpr uint32_t IDESC_DQ = ptx::idesc_bf16_f32acc(128, BQ, true, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_DS % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_DO % 1024 == 0, "1 KB aligned tiles");
};

// Row pass before the pair kernel, one warp per (batch, query head, row) of
// the 64-padded query range: drow = rowsum(dO * O) (fp32 accumulation of the
// bf16 operands), nl2 = -lse * log2(e) (-inf where the forward kept no key,
// so that P = 0 there, and on padding rows), and the fp32 dQ row cleared for
// the pair kernel's additions.
__global__ void __launch_bounds__(256)
    blasst_bwd_rows_kernel(const __nv_bfloat16* __restrict__ o,
                           const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                           float* __restrict__ nl2, float* __restrict__ drow,
                           float* __restrict__ dq, long long n_rows, int Lq, int LqP) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  const long long bh = r / LqP;
  const int q = static_cast<int>(r % LqP);
  if (q >= Lq) {
    if (lane == 0) {
      nl2[r] = -INFINITY;
      drow[r] = 0.0f;
    }
    return;
  }
  const size_t row = static_cast<size_t>(bh) * Lq + q;
  const uint2 ov = reinterpret_cast<const uint2*>(o + row * 128)[lane];
  const uint2 dv = reinterpret_cast<const uint2*>(dout + row * 128)[lane];
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
  const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 a = __bfloat1622float2(o2[i]);
    const float2 c = __bfloat1622float2(d2[i]);
    acc = fmaf(a.x, c.x, acc);
    acc = fmaf(a.y, c.y, acc);
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  reinterpret_cast<float4*>(dq + row * 128)[lane] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (lane == 0) {
    const float l = lse[row];
    nl2[r] = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
    drow[r] = acc;
  }
}

__device__ __forceinline__ void bwd_record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Which 64-key halves of the CTA's key block j the forward kept for query
// tile t (64 rows) of head bh: bit h set = keys [128 j + 64 h, +64) kept.
__device__ __forceinline__ uint32_t bwd_keep_bits(const BwdParams& p, int bh, int t, int j) {
  if (p.causal && j * BwdCfg::BK > t * BwdCfg::BQ + (BwdCfg::BQ - 1) + p.off) return 0u;
  if (!p.fmask) return 3u;
  const int qf = (t * BwdCfg::BQ) / p.Brf;
  const uint8_t* row = p.fmask + (static_cast<size_t>(bh) * p.nQf + qf) * p.nKf;
  if (p.Bcf == BwdCfg::BK) return row[j] == 0 ? 3u : 0u;
  uint32_t r = row[2 * j] == 0 ? 1u : 0u;
  if (2 * j + 1 < p.nKf && row[2 * j + 1] == 0) r |= 2u;
  return r;
}


__global__ void __launch_bounds__(352, 1)
    blasst_bwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmDO,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = ptx::smem_u32(smem);
  if ((sb & 1023u) != 0u) {  // uniform over the CTA; nothing set up yet
    if (threadIdx.x == 0) bwd_record_error(p.err, BLASST_EUNSUPPORTED);
    return;
  }
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort_flag = misc + 1;
  volatile int* recw = reinterpret_cast<volatile int*>(smem + C::OFF_REC);
  auto put_rec = [&](int s, int hq, int t, int keep, int end) {
    recw[4 * s] = hq;
    recw[4 * s + 1] = t;
    recw[4 * s + 2] = keep;
    recw[4 * s + 3] = end;
  };
  auto get_rec = [&](int s) -> int4 {
    return make_int4(recw[4 * s], recw[4 * s + 1], recw[4 * s + 2], recw[4 * s + 3]);
  };
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: key block j of KV head (b, hk), KV-head major: the CTAs
  // in flight work on one KV head, so the query rows they read (Q, dO) and
  // add into (dQ) are those of one GQA group. Under a causal mask block 0
  // meets the most query tiles, so ascending j runs the longest CTAs first.
  const int j = static_cast<int>(blockIdx.x) % p.nKb;
  const int bhk = static_cast<int>(blockIdx.x) / p.nKb;
  const int b = bhk / p.Hkv;
  const int hk = bhk % p.Hkv;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_KV), 1);
    for (int i = 0; i < C::NST; ++i) {
      ptx::mbar_init(bar(C::B_QF + i), C::QF_COUNT);
      ptx::mbar_init(bar(C::B_QE + i), C::QE_COUNT);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(C::B_SF + i), 1);
      ptx::mbar_init(bar(C::B_PR + i), 4);
      ptx::mbar_init(bar(C::B_DPF + i), 1);
      ptx::mbar_init(bar(C::B_DSR + i), 4);
      ptx::mbar_init(bar(C::B_DQF + i), 1);
    }
    ptx::mbar_init(bar(C::B_ZERO), 8);
    ptx::mbar_init(bar(C::B_ACC), 1);
    for (int i = 0; i < 2; ++i) ptx::mbar_init(bar(C::B_DRAIN + i), 1);
    for (int i = 1; i < C::MISC_BYTES / 4; ++i) misc[i] = 0;
    for (int i = 0; i < 2; ++i)
      for (int a = 1; a < C::QF_COUNT; ++a) ptx::mbar_arrive(bar(C::B_QF + i));
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

  // every lane of the warp waits (the data behind the barrier is read by all)
  auto warp_wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    const bool ok = ptx::mbar_wait(bar_addr, parity, abort_flag, p.timeout_ns);
    return __all_sync(0xffffffffu, ok) != 0;
  };
  auto fail = [&]() {
    *abort_flag = 1;
    bwd_record_error(p.err, BLASST_ETIMEOUT);
  };

  if (warp == C::WARP_LOAD) {
    // ======================= producer ====================================
    bool ok = true;
    if (lane == 0) {
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmDO);
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
      ptx::mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KV_BYTES);
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        ptx::tma_load_3d(sb + C::OFF_K + bx * C::KV_BOX, &tmK, bx * 64, j * C::BK, bhk, bar(C::B_KV));
        ptx::tma_load_3d(sb + C::OFF_V + bx * C::KV_BOX, &tmV, bx * 64, j * C::BK, bhk, bar(C::B_KV));
      }
    }
    // first query tile that can see block j
    int t_lo = 0;
    if (p.causal) {
      const int num = j * C::BK - p.off - (C::BQ - 1);
      t_lo = num <= 0 ? 0 : (num + C::BQ - 1) / C::BQ;
    }
    // Query tiles from the last one down, 32 at a time, the group's heads
    // interleaved within each 32-tile chunk: the CTAs of a KV head start on
    // the same last rows and move down together, so the Q, dO and dQ rows
    // they touch at any time stay few and in L2. (The gradients are sums
    // over pairs: their order only changes the fp32 rounding order.)
    int i = 0;  // pairs issued
    for (int tc = p.nT - 1; tc >= t_lo && ok; tc -= 32) {
      for (int hh = 0; hh < p.g && ok; ++hh) {
        const int hq = hk * p.g + hh;
        const int bh = b * p.Hq + hq;
        const int t = tc - lane;  // lane 0: the highest tile of the chunk
        const uint32_t km = t >= t_lo ? bwd_keep_bits(p, bh, t, j) : 0u;
        uint32_t bal = __ballot_sync(0xffffffffu, km != 0u);
        while (bal != 0u) {
          const int l = __ffs(bal) - 1;
          bal &= bal - 1u;
          const int tt = tc - l;
          const uint32_t kmv = __shfl_sync(0xffffffffu, km, l);
          bool okl = true;
          if (lane == 0) {
            const int s = i % C::NST;
            if (i >= C::NST)
              okl = ptx::mbar_wait(bar(C::B_QE + s), ((i / C::NST) - 1) & 1, abort_flag,
                                   p.timeout_ns);
            if (okl) {
              put_rec(s, hq, tt, static_cast<int>(kmv), 0);
              const uint32_t fb = bar(C::B_QF + s);
              ptx::mbar_arrive_expect_tx(fb, 2 * C::Q_BYTES + C::ROWST_BYTES);
#pragma unroll
              for (int bx = 0; bx < 2; ++bx) {
                ptx::tma_load_3d(sb + C::OFF_Q + s * C::Q_BYTES + bx * C::Q_BOX, &tmQ, bx * 64,
                                 tt * C::BQ, bh, fb);
                ptx::tma_load_3d(sb + C::OFF_DO + s * C::Q_BYTES + bx * C::Q_BOX, &tmDO, bx * 64,
                                 tt * C::BQ, bh, fb);
              }
              const size_t ro = static_cast<size_t>(bh) * p.LqP + static_cast<size_t>(tt) * C::BQ;
              const uint32_t rs = sb + C::OFF_RS + s * C::ROWST_BYTES;
              ptx::bulk_load(rs, p.nl2 + ro, C::BQ * 4, fb);
              ptx::bulk_load(rs + C::BQ * 4, p.drow + ro, C::BQ * 4, fb);
            }
          }
          ok = __shfl_sync(0xffffffffu, okl ? 1 : 0, 0) != 0;
          if (!ok) break;
          ++i;
        }
      }
    }
    if (lane == 0) {
      // two end records (pair indices i and i + 1): the issuers stop at the
      // first, each compute set at the first of its parity
      for (int e = 0; e < 2 && ok; ++e) {
        const int ie = i + e;
        const int s = ie % C::NST;
        if (ie >= C::NST)
          ok = ptx::mbar_wait(bar(C::B_QE + s), ((ie / C::NST) - 1) & 1, abort_flag, p.timeout_ns);
        if (ok) {
          put_rec(s, -1, 0, 0, 1);
          ptx::mbar_arrive(bar(C::B_QF + s));
        }
      }
      if (!ok) {
        fail();
        // let the copies already in flight land before the CTA exits
        // (a stage's phase also counts the other roles' arrivals for the pair
        // two back, which an abort may leave out: 1 ms each is ample for the
        // copies themselves)
        const uint64_t drain_ns = p.timeout_ns < 1000000ull ? p.timeout_ns : 1000000ull;
        for (int k = i - C::NST < 0 ? 0 : i - C::NST; k < i; ++k)
          ptx::mbar_wait(bar(C::B_QF + k % C::NST), (k / C::NST) & 1, &misc[3], drain_ns);
        ptx::mbar_wait(bar(C::B_KV), 0, &misc[3], p.timeout_ns);
      }
    }
  } else if (warp == C::WARP_SP || warp == C::WARP_MMA) {
    // ======================= tcgen05 issuers =============================
    // Two threads issue MMAs, each in its own order; what one reads of the
    // other's results is ordered through the compute sets' barriers or an
    // explicit commit:
    //   warp 10: S^T(i) (into S buffer i%2 once dV(i-2) has read P^T(i-2))
    //            and dP^T(i) (into dP buffer i%2 once dQ^T(i-2) is drained);
    //   warp 9:  dV(i) (after P^T(i)), dK(i) and dQ^T(i) (after dS^T(i)).
    //            S^T(i) and dP^T(i) are complete by then (the compute set has
    //            read them), so the commit after dQ^T(i) also frees the stage.
    if (lane == 0) {
      bool ok = ptx::mbar_wait(bar(C::B_KV), 0, abort_flag, p.timeout_ns);
      if (warp == C::WARP_MMA && ok) ok = ptx::mbar_wait(bar(C::B_ZERO), 0, abort_flag, p.timeout_ns);
      ptx::tc_fence_after();
      // descriptors (k-steps add 16-byte units to the start-address field)
      const uint64_t dK_kmaj = ptx::sw128_desc(sb + C::OFF_K, 16, 1024);
      const uint64_t dV_kmaj = ptx::sw128_desc(sb + C::OFF_V, 16, 1024);
      const uint64_t dK_mn = ptx::sw128_desc(sb + C::OFF_K, C::KV_BOX, 1024);
      const uint64_t dQ_kmaj = ptx::sw128_desc(sb + C::OFF_Q, 16, 1024);
      const uint64_t dDO_kmaj = ptx::sw128_desc(sb + C::OFF_DO, 16, 1024);
      const uint64_t dQ_mn = ptx::sw128_desc(sb + C::OFF_Q, C::Q_BOX, 1024);
      const uint64_t dDO_mn = ptx::sw128_desc(sb + C::OFF_DO, C::Q_BOX, 1024);
      const uint64_t dDS_kmaj = ptx::sw128_desc(sb + C::OFF_DS, 16, 1024);
      const uint64_t dDS_mn = ptx::sw128_desc(sb + C::OFF_DS, C::DS_BYTES, 1024);
      constexpr uint64_t QST = C::Q_BYTES >> 4;   // stage stride, 16-byte units
      constexpr uint64_t DSB = C::DS_BYTES >> 4;  // dS buffer stride
      // 1: pair ready, 0: end record, -1: the wait gave up. Neither issuer
      // can fall a full stage cycle behind: a stage is reloaded only after
      // warp 9's commit for its pair.
      auto stage_ready = [&](int i) -> int {
        const int s = i % C::NST;
        if (!ptx::mbar_wait(bar(C::B_QF + s), (i / C::NST) & 1, abort_flag, p.timeout_ns))
          return -1;
        return recw[4 * s + 3] != 0 ? 0 : 1;
      };
      for (int i = 0; ok; ++i) {
        const int r = stage_ready(i);
        if (r < 0) {
          ok = false;
          break;
        }
        if (r == 0) break;
        const int bs = i & 1;
        const uint64_t st = static_cast<uint64_t>(i % C::NST) * QST;
        if (warp == C::WARP_SP) {
          // S^T = K Q^T and dP^T = V dO^T: M = 128 keys, N = 64 rows, K = 128 dims
          // (the buffers of pair i-2 are free: counted by the stage's barrier)
          ptx::tc_fence_after();
          const uint32_t s_tm = tmem + C::S_COL + bs * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = dK_kmaj + static_cast<uint64_t>(((kk >> 2) * C::KV_BOX + (kk & 3) * 32) >> 4);
            const uint64_t bq = dQ_kmaj + st + static_cast<uint64_t>(((kk >> 2) * C::Q_BOX + (kk & 3) * 32) >> 4);
            ptx::mma_ss(s_tm, a, bq, C::IDESC_S, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(bar(C::B_SF + bs));
          const uint32_t dp_tm = tmem + C::DP_COL + bs * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = dV_kmaj + static_cast<uint64_t>(((kk >> 2) * C::KV_BOX + (kk & 3) * 32) >> 4);
            const uint64_t bo = dDO_kmaj + st + static_cast<uint64_t>(((kk >> 2) * C::Q_BOX + (kk & 3) * 32) >> 4);
            ptx::mma_ss(dp_tm, a, bo, C::IDESC_S, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(bar(C::B_DPF + bs));
        } else {
          // dV += P^T dO: M = 128 keys, N = 128 dims, K = 64 rows (P^T from TMEM)
          if (!ptx::mbar_wait(bar(C::B_PR + bs), (i >> 1) & 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t p_tm = tmem + C::S_COL + bs * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_ts(tmem + C::DV_COL, p_tm + kk * 8,
                        dDO_mn + st + static_cast<uint64_t>((kk * 2048) >> 4), C::IDESC_DV, 1u);
          // P^T of pair i read: its S^T buffer may take pair i+2
          ptx::mma_commit(bar(C::B_QF + (i + 2) % C::NST));
          // dK += dS^T Q (M = 128 keys, N = 128 dims, K = 64 rows) and
          // dQ^T = K^T dS^T (M = 128 dims, N = 64 rows, K = 128 keys)
          if (!ptx::mbar_wait(bar(C::B_DSR + bs), (i >> 1) & 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t dsk = dDS_kmaj + static_cast<uint64_t>(bs) * DSB;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_ss(tmem + C::DK_COL, dsk + static_cast<uint64_t>((kk * 32) >> 4),
                        dQ_mn + st + static_cast<uint64_t>((kk * 2048) >> 4), C::IDESC_DK, 1u);
          const uint64_t dsm = dDS_mn + static_cast<uint64_t>(bs) * DSB;
          const uint32_t dq_tm = tmem + C::DP_COL + bs * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::mma_ss(dq_tm, dK_mn + static_cast<uint64_t>((kk * 2048) >> 4),
                        dsm + static_cast<uint64_t>((kk * 2048) >> 4), C::IDESC_DQ,
                        kk > 0 ? 1u : 0u);
          ptx::mma_commit(bar(C::B_DQF + bs));
        }
      }
      if (warp == C::WARP_MMA) ptx::mma_commit(bar(C::B_ACC));
      if (!ok) fail();
      // drain: every MMA this thread issued has completed before TMEM is
      // freed (bounded, not cut short by the abort flag)
      const int dr = warp == C::WARP_MMA ? 0 : 1;
      ptx::mma_commit(bar(C::B_DRAIN + dr));
      ptx::mbar_wait(bar(C::B_DRAIN + dr), 0, &misc[3], p.timeout_ns);
    }
  } else {
    // ======================= compute sets: P^T, dS^T, dQ ==================
    // set 0 takes the even pairs, set 1 the odd ones (S^T, dP^T, P^T and dS^T
    // buffer = set), so one set's exponentials overlap the other set's TMEM
    // reads and waits on the same SM sub-partition. After dS^T a set drains
    // its pair's dQ^T: TMEM lanes are head dims there, warp quad takes dims
    // [32 quad, 32 quad + 32), stages them as a [64 rows][32 dims] fp32 tile
    // in the pair's Q / dO stage (dead once dQ^T is done: every product that
    // reads the stage was issued before it and the tensor core completes them
    // in order) and adds the tile to global dQ with one TMA reduce-add.
    const int set = warp >> 2;
    const int quad = warp & 3;
    const int kl = quad * 32 + lane;  // key row of the block (TMEM lane)
    const int kg = j * C::BK + kl;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const bool key_ok = kg < p.Lkv;
    const float sl2 = p.scale_log2;
    const uint32_t acc_col = set == 0 ? C::DV_COL : C::DK_COL;
    {
      // clear this set's accumulator rows (set 0: dV, set 1: dK); every dV and
      // dK product then accumulates
      uint32_t z[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) z[u] = 0u;
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_st32(tmem + lane_base + acc_col + 32 * c, z);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_ZERO));
    }
    bool ok = true;
    const int bs = set;
    int pend_stage = -1;  // stage whose dQ add this warp has issued but not yet released
    for (int i = set;; i += 2) {
      const int s = i % C::NST;
      ok = warp_wait(bar(C::B_QF + s), (i / C::NST) & 1);
      if (!ok) break;
      const int4 rc = get_rec(s);
      if (rc.w != 0) break;
      ok = warp_wait(bar(C::B_SF + bs), (i >> 1) & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      // column c (query row 64 t + c) is kept for this key iff c >= lim
      int lim;
      if (!key_ok || ((static_cast<uint32_t>(rc.z) >> (kl >> 6)) & 1u) == 0u) lim = C::BQ;
      else if (p.causal) lim = kg - p.off - rc.y * C::BQ;
      else lim = 0;
      const float* rs = reinterpret_cast<const float*>(smem + C::OFF_RS + s * C::ROWST_BYTES);
      float pv[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_base + C::S_COL + bs * 64 + 32 * h, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 nl = reinterpret_cast<const float4*>(rs)[8 * h + c4];
          const float nla[4] = {nl.x, nl.y, nl.z, nl.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = 32 * h + 4 * c4 + u;
            const float x = fmaf(__uint_as_float(r[4 * c4 + u]), sl2, nla[u]);
            pv[c] = (c >= lim) ? ptx::ex2(x) : 0.0f;
          }
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = ptx::pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
        ptx::tmem_st32(tmem + lane_base + C::S_COL + bs * 64, pk);
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(bar(C::B_PR + bs));
        if (pend_stage >= 0) {
          // the previous pair's dQ add has long been issued: once it has read
          // its staged tile, that pair's stage may be reloaded
          ptx::bulk_wait_group_read0();
          ptx::mbar_arrive(bar(C::B_QE + pend_stage));
        }
      }
      pend_stage = -1;

      ok = warp_wait(bar(C::B_DPF + bs), (i >> 1) & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      // (dS^T of pair i-2 has been read: this set waited for that pair's dQ^T,
      // committed after its dK and dQ^T products)
      uint8_t* dsrow = smem + C::OFF_DS + bs * C::DS_BYTES + kl * 128;
      const float* dr = rs + C::BQ;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_base + C::DP_COL + bs * 64 + 32 * h, r);
        ptx::tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 dd = reinterpret_cast<const float4*>(dr)[8 * h + c4];
          const int c = 32 * h + 4 * c4;
          const float d0 = pv[c] * (__uint_as_float(r[4 * c4]) - dd.x);
          const float d1 = pv[c + 1] * (__uint_as_float(r[4 * c4 + 1]) - dd.y);
          const float d2 = pv[c + 2] * (__uint_as_float(r[4 * c4 + 2]) - dd.z);
          const float d3 = pv[c + 3] * (__uint_as_float(r[4 * c4 + 3]) - dd.w);
          w[2 * c4] = ptx::pack_bf16x2(d0, d1);
          w[2 * c4 + 1] = ptx::pack_bf16x2(d2, d3);
        }
        // row kl of the 128-byte-swizzled tile: 16-byte chunk c8 at c8 ^ (kl % 8)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int c8 = 4 * h + ch;
          *reinterpret_cast<uint4*>(dsrow + ((c8 ^ (kl & 7)) << 4)) =
              make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_DSR + bs));

      ok = warp_wait(bar(C::B_DQF + bs), (i >> 1) & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      {
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(tmem + lane_base + C::DP_COL + bs * 64, r0);
        ptx::tmem_ld32(tmem + lane_base + C::DP_COL + bs * 64 + 32, r1);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        // dQ^T drained: the dP^T / dQ^T buffer may take pair i+2
        if (lane == 0) ptx::mbar_arrive(bar(C::B_QF + (i + 2) % C::NST));
        const int slot = (quad < 2 ? C::OFF_Q + quad * C::DQS_BYTES
                                   : C::OFF_DO + (quad - 2) * C::DQS_BYTES) + s * C::Q_BYTES;
        float* tile = reinterpret_cast<float*>(smem + slot);
        const float scale = p.scale;
#pragma unroll
        for (int c = 0; c < 32; ++c) tile[c * 32 + lane] = __uint_as_float(r0[c]) * scale;
#pragma unroll
        for (int c = 0; c < 32; ++c) tile[(32 + c) * 32 + lane] = __uint_as_float(r1[c]) * scale;
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_reduce_add_3d(&tmDQ, sb + slot, 32 * quad, rc.y * C::BQ, b * p.Hq + rc.x);
          ptx::bulk_commit_group();
        }
        pend_stage = s;  // released once the add has read it (after the next P^T)
      }
    }
    if (lane == 0) {
      ptx::bulk_wait_group0();  // every dQ add of this warp has completed
      if (pend_stage >= 0) ptx::mbar_arrive(bar(C::B_QE + pend_stage));
    }
    if (!ok) fail();
    // ---- epilogue: set 0 writes dV, set 1 writes dK (scaled); row kl = TMEM lane
    if (ok) ok = warp_wait(bar(C::B_ACC), 0);
    ptx::tc_fence_after();
    if (ok && *abort_flag == 0) {
      const float f = set == 0 ? 1.0f : p.scale;
      float* dst = (set == 0 ? p.dv : p.dk) +
                   (static_cast<size_t>(bhk) * p.Lkv + (key_ok ? kg : 0)) * C::D;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_base + acc_col + 32 * c, r);
        ptx::tmem_wait_ld();
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<float4*>(dst + 32 * c)[u] =
                make_float4(__uint_as_float(r[4 * u]) * f, __uint_as_float(r[4 * u + 1]) * f,
                            __uint_as_float(r[4 * u + 2]) * f, __uint_as_float(r[4 * u + 3]) * f);
        }
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace blasst
