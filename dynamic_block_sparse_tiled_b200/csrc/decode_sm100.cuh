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
// The kernel is bound by HBM bytes (K always, V of kept blocks), so it is
// built to keep loads in flight and the per-block arithmetic off one chain:
//   - persistent CTAs, one per SM, each streaming a fixed sequence of tasks
//     (a task = one KV block of one split of one (sequence, KV head)), so the
//     K prefetch runs across split boundaries without pipeline drains;
//   - warp 8 streams K through a TMA ring (128-byte swizzled tiles: a thread
//     reading one key row is bank-conflict free); warp 9 loads V when a vote
//     keeps the block and writes the skip mask and the counters;
//   - warps 0-3 score and vote: q K^T, the per-head block max, the vote
//     against the running max, P = exp2(s - m) and the running sums; a task
//     record (P fragments, rescale factors, keep flags) goes to shared memory;
//   - warps 4-7 accumulate O += P V from those records, up to NP tasks
//     behind, and write each split's normalised output. The two groups run
//     concurrently (one warp of each per SM sub-partition), so the vote chain
//     of one block overlaps the P V of an earlier one.
// Both contractions run as warp-level bf16 mma.sync tiles with the G =
// Hq/Hkv rows padded to 16: far too thin for tcgen05, but one tile
// instruction replaces hundreds of dependent FMAs and shared-memory loads.
// Warp w of each group owns keys [w*Bc/4, (w+1)*Bc/4) of every block; P stays
// in the accumulator layout of q K^T, which is the operand layout of P V.
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
  static constexpr int NC = 128;        // vote threads (warps 0-3); P V threads are warps 4-7
  static constexpr int NT = 320;        // + P V warps 4-7, K producer 8, V producer 9
  static constexpr int DBOX = D / 64;
  static constexpr int KV_BOX = BC * 128;
  static constexpr int KV_BYTES = KV_BOX * DBOX;
  static constexpr int NK = 3;          // K ring stages
  static constexpr int NV = 3;          // V ring stages
  static constexpr int NP = 4;          // task records (P fragments, alpha, keep)
  static constexpr int NFIN = 8;        // split finals ring (> NP + 1 open splits)
  static constexpr int NDEC = 8;        // decision ring between the vote warps and the V warp
  static constexpr int KW = BC / 4;     // keys per warp
  static constexpr int NTQ = KW / 8;    // q K^T n-tiles (8 keys) per warp
  static constexpr int KSP = KW / 16;   // P V k-steps (16 keys) per warp
  static constexpr int NTO = D / 8;     // P V n-tiles (8 dims)
  static constexpr int PREGS = KSP * 2; // bf16x2 P registers per thread per task
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_PF = OFF_V + NV * KV_BYTES;              // NP x NC x PREGS words
  static constexpr int OFF_TASK = OFF_PF + NP * NC * PREGS * 4;      // NP x (G alpha, G keep)
  static constexpr int OFF_RED = OFF_TASK + NP * 2 * G * 4;          // 4 warps x G max, x G sums
  static constexpr int OFF_FIN = OFF_RED + 2 * 4 * G * 4;            // NFIN x (G m, G l)
  static constexpr int OFF_DEC = OFF_FIN + NFIN * 2 * G * 4;         // NDEC keep masks
  static constexpr int OFF_FLAG = OFF_DEC + NDEC * 4;                // abort words
  static constexpr int OFF_OACC = (OFF_FLAG + 64 + 15) & ~15;        // 4 warps x G x D fp32
  static constexpr int OFF_BAR = (OFF_OACC + 4 * G * D * 4 + 7) & ~7;
  // K full/empty, V full/empty, decision written/read, task record ready/free
  static constexpr int NBAR = 2 * NK + 2 * NV + 2 * NDEC + 2 * NP;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  static_assert(G <= 8, "rows of the padded tile");
  static_assert(KW % 16 == 0 && (D / 16) % 2 == 0 && NTO % 2 == 0, "tile shapes");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Position in the task sequence of one persistent CTA: splits cta,
// cta + nctas, ... in order, each contributing its blocks.
struct TaskCursor {
  int split_id;  // flat (b, hk, split) index; >= nsplits: sequence finished
  int blk;       // block within the split
  int nblk;      // blocks in this split
};

namespace dmma {
// D = A * B + C, m16n8k16, bf16 inputs, fp32 accumulation (rows 8-15 unused
// here: a1 = a3 = 0 and c2/c3 discarded).
#pragma nv_diag_suppress 550  // d2, d3: outputs of rows 8-15, never read
__device__ __forceinline__ void mma16816(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1, float c0, float c1) {
  float d2, d3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(0.0f),
        "f"(0.0f));
}
#pragma nv_diag_default 550
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
// Byte offset of the 16-byte chunk holding dims [8*chunk, 8*chunk+8) of row
// `row` in a 128B-swizzled tile made of 64-column boxes of `box_bytes`.
__device__ __forceinline__ uint32_t sw_chunk(int row, int chunk, int box_bytes) {
  return static_cast<uint32_t>((chunk >> 3) * box_bytes + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}
}  // namespace dmma

template <int D, int BC, int G>
// 320 threads: at most 3 warps on one SM sub-partition, so up to 168
// registers per thread.
__global__ void __launch_bounds__(320, 1)
    blasst_decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecodeCfg<D, BC, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  uint32_t* pfrag = reinterpret_cast<uint32_t*>(smem + C::OFF_PF);          // [NP][NC][PREGS]
  float* task_alpha = reinterpret_cast<float*>(smem + C::OFF_TASK);         // [NP][G]
  int* task_keep = reinterpret_cast<int*>(smem + C::OFF_TASK) + C::NP * G;  // [NP][G]
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);                 // [2][4][G]
  float* split_fin = reinterpret_cast<float*>(smem + C::OFF_FIN);           // [NFIN][2][G]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  volatile int* abort_seen = abort_flag + 2;  // [2], decided by thread 0 per task parity
  float* oacc = reinterpret_cast<float*>(smem + C::OFF_OACC);               // [4][G][D]
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  volatile int* dec_ring = reinterpret_cast<volatile int*>(smem + C::OFF_DEC);  // [NDEC]
  const int B_KF = 0, B_KE = C::NK, B_VF = 2 * C::NK, B_VE = B_VF + C::NV;
  const int B_DEC = B_VE + C::NV, B_DR = B_DEC + C::NDEC;
  const int B_TR = B_DR + C::NDEC, B_TF = B_TR + C::NP;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, c4 = lane & 3;  // mma fragment row (head) and column pair
  const int nsplits = p.B * p.Hkv * p.S;
  const bool thresholding = p.log2_lambda > -INFINITY;

  auto split_blocks = [&](int sid) -> int {
    const int sp = sid % p.S;
    const int k0 = sp * p.Ls;
    const int k1 = min(k0 + p.Ls, p.Lkv);
    return k1 > k0 ? (k1 - k0 + BC - 1) / BC : 0;
  };
  // First split from `sid` on (stepping by the grid) with at least one
  // block; the compute side writes the partials of the empty ones it passes
  // (o = 0, lse = -inf).
  auto advance_split = [&](int sid, bool write_empty) -> TaskCursor {
    for (; sid < nsplits; sid += gridDim.x) {
      const int nb = split_blocks(sid);
      if (nb > 0) return TaskCursor{sid, 0, nb};
      if (write_empty) {
        const int sp = sid % p.S, bhk = sid / p.S;
        const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
        for (int i = t; i < G * D; i += C::NC) {
          const int h = i / D, x = i % D;
          const size_t prow = (static_cast<size_t>(b) * p.Hq + hk * G + h) * p.S + sp;
          p.o_parts[prow * D + x] = 0.0f;
          if (x == 0) p.lse_parts[prow] = -INFINITY;
        }
      }
    }
    return TaskCursor{nsplits, 0, 0};
  };
  auto next_task = [&](TaskCursor c, bool write_empty) -> TaskCursor {
    if (c.blk + 1 < c.nblk) return TaskCursor{c.split_id, c.blk + 1, c.nblk};
    return advance_split(c.split_id + static_cast<int>(gridDim.x), write_empty);
  };
  auto task_key0 = [&](const TaskCursor& c) -> int {
    return (c.split_id % p.S) * p.Ls + c.blk * BC;
  };

  if (t == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      ptx::mbar_init(bar(i), ((i >= B_VE && i < B_VE + C::NV) || (i >= B_TF && i < B_TF + C::NP))
                                 ? 4 : 1);
    abort_flag[0] = 0;
    abort_seen[0] = 0;
    abort_seen[1] = 0;
    abort_flag[4] = 0;  // never set: for waits that only a timeout ends
    ptx::fence_mbar_init();
  }
  __syncthreads();

  auto load_tile = [&](const CUtensorMap* tm, uint32_t dst, int key0, int bhk, uint32_t fb) {
    ptx::mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::DBOX; ++bx)
      ptx::tma_load_3d(dst + bx * C::KV_BOX, tm, bx * 64, key0, bhk, fb);
  };

  if (warp == 8) {
    // ======================= K producer ====================================
    if (lane == 0) {
      ptx::prefetch_tmap(&tmK);
      TaskCursor c = advance_split(blockIdx.x, false);
      int n = 0;
      for (; c.split_id < nsplits; ++n) {
        const int ks = n % C::NK;
        if (n >= C::NK &&
            !ptx::mbar_wait(bar(B_KE + ks), ((n / C::NK) - 1) & 1, abort_flag, p.timeout_ns)) {
          *abort_flag = 1;
          break;
        }
        load_tile(&tmK, sb + C::OFF_K + ks * C::KV_BYTES, task_key0(c), c.split_id / p.S,
                  bar(B_KF + ks));
        c = next_task(c, false);
      }
      // Let the last copies land before this warp leaves (they normally have).
      for (int m = (n > C::NK ? n - C::NK : 0); m < n; ++m)
        ptx::mbar_wait(bar(B_KF + m % C::NK), (m / C::NK) & 1, abort_flag, p.timeout_ns);
    }
    return;  // the producer warp takes no part in the compute barriers
  }
  if (warp == 9) {
    // ======================= V producer, skip mask, counters =============
    if (lane == 0) {
      ptx::prefetch_tmap(&tmV);
      TaskCursor c = advance_split(blockIdx.x, false);
      unsigned long long st_vis = 0, st_skip = 0, st_flops = 0, st_bytes = 0;
      int n = 0, vcount = 0;
      bool ok = true;
      for (; c.split_id < nsplits; ++n) {
        const int ds = n % C::NDEC;
        ok = ptx::mbar_wait(bar(B_DEC + ds), (n / C::NDEC) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        const int keepmask = dec_ring[ds];
        ptx::mbar_arrive(bar(B_DR + ds));
        const int bhk = c.split_id / p.S;
        const int key0 = task_key0(c);
        if (keepmask) {
          const int vs = vcount % C::NV;
          if (vcount >= C::NV) {
            ok = ptx::mbar_wait(bar(B_VE + vs), ((vcount / C::NV) - 1) & 1, abort_flag,
                                p.timeout_ns);
            if (!ok) break;
          }
          load_tile(&tmV, sb + C::OFF_V + vs * C::KV_BYTES, key0, bhk, bar(B_VF + vs));
          ++vcount;
        }
        if (p.mask) {
          const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
          for (int h = 0; h < G; ++h) {
            const size_t hq = static_cast<size_t>(b) * p.Hq + hk * G + h;
            p.mask[hq * p.nKt + key0 / BC] = ((keepmask >> h) & 1) ? 0 : 1;
          }
        }
        st_vis += G;
        st_skip += G - __popc(keepmask);
        st_flops += 2ull * G * BC * D + 2ull * __popc(keepmask) * BC * D;
        st_bytes += static_cast<unsigned long long>(BC) * D * 2ull * (keepmask ? 2ull : 1ull);
        c = next_task(c, false);
      }
      if (!ok) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
      } else if (p.stats) {
        atomicAdd(&p.stats->tiles_visited, st_vis);
        atomicAdd(&p.stats->tiles_skipped, st_skip);
        atomicAdd(&p.stats->v_blocks_loaded, static_cast<unsigned long long>(vcount));
        atomicAdd(&p.stats->mma_flops, st_flops);
        atomicAdd(&p.stats->bytes_loaded, st_bytes);
      }
      // V copies in flight land before this warp leaves (they normally have).
      for (int v = (vcount > C::NV ? vcount - C::NV : 0); v < vcount; ++v)
        ptx::mbar_wait(bar(B_VF + v % C::NV), (v / C::NV) & 1, &abort_flag[4], p.timeout_ns);
    }
    return;
  }

  if (warp >= 4) {
    // ======================= P V warps 4-7 =================================
    // Warp pw owns keys [pw*KW, pw*KW + KW) of every block; thread (g, c4)
    // accumulates, for head g < G, dims 8nn + 2c4, 8nn + 2c4 + 1 of each
    // n-tile nn. Tasks come in the order of the vote side's records.
    const int pw = warp - 4;
    float oa[C::NTO][2];
#pragma unroll
    for (int i = 0; i < C::NTO; ++i) oa[i][0] = oa[i][1] = 0.0f;
    int vconsumed = 0;  // V tiles consumed
    int pv_seq = 0;     // splits finished
    bool failed = false;
    auto pv_barrier = [&]() { ptx::named_bar_sync(2, 128); };
    TaskCursor c = advance_split(blockIdx.x, false);
    for (int n = 0; c.split_id < nsplits; ++n) {
      const int slot = n % C::NP;
      bool w = true;
      if (lane == 0) w = ptx::mbar_wait(bar(B_TR + slot), (n / C::NP) & 1, abort_flag, p.timeout_ns);
      w = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
      if (!w) failed = true;  // keep going (waits now return at once) so the
                              // four warps take the same barriers
      const int* keep = task_keep + slot * G;
      int any = 0;
#pragma unroll
      for (int h = 0; h < G; ++h) any |= keep[h];
      if (c.blk == 0) {
#pragma unroll
        for (int i = 0; i < C::NTO; ++i) oa[i][0] = oa[i][1] = 0.0f;
      }
      if (any) {
        const int vs = vconsumed % C::NV;
        bool wv = true;
        if (lane == 0)
          wv = ptx::mbar_wait(bar(B_VF + vs), (vconsumed / C::NV) & 1, abort_flag, p.timeout_ns);
        wv = __shfl_sync(0xffffffffu, wv ? 1 : 0, 0) != 0;
        if (!wv) failed = true;
        ++vconsumed;
        const float alpha = g < G ? task_alpha[slot * G + g] : 1.0f;
#pragma unroll
        for (int i = 0; i < C::NTO; ++i) {
          oa[i][0] *= alpha;
          oa[i][1] *= alpha;
        }
        uint32_t pr[C::PREGS];
#pragma unroll
        for (int i = 0; i < C::PREGS; ++i)
          pr[i] = pfrag[(slot * C::NC + pw * 32 + lane) * C::PREGS + i];
        const uint32_t vst = sb + C::OFF_V + vs * C::KV_BYTES;
#pragma unroll
        for (int k2 = 0; k2 < C::KSP; ++k2) {
          // keys of this k-step: pw*KW + 16*k2 + [0, 16)
          const int key = pw * C::KW + 16 * k2 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int nn = 0; nn < C::NTO; nn += 2) {
            uint32_t b0, b1, b2, b3;
            dmma::ldsm_x4_t(vst + dmma::sw_chunk(key, nn + (lane >> 4), C::KV_BOX), b0, b1, b2, b3);
            dmma::mma16816(oa[nn][0], oa[nn][1], pr[2 * k2], pr[2 * k2 + 1], b0, b1, oa[nn][0],
                           oa[nn][1]);
            dmma::mma16816(oa[nn + 1][0], oa[nn + 1][1], pr[2 * k2], pr[2 * k2 + 1], b2, b3,
                           oa[nn + 1][0], oa[nn + 1][1]);
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_VE + vs));  // this warp is done reading V
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_TF + slot));  // task record read
      if (c.blk + 1 == c.nblk) {
        // split epilogue: sum the four warps' partial outputs, normalise, write
        if (g < G) {
#pragma unroll
          for (int i = 0; i < C::NTO; ++i) {
            oacc[(pw * G + g) * D + 8 * i + 2 * c4] = oa[i][0];
            oacc[(pw * G + g) * D + 8 * i + 2 * c4 + 1] = oa[i][1];
          }
        }
        pv_barrier();
        const float* fin = split_fin + (pv_seq % C::NFIN) * 2 * G;  // [m[G], l[G]]
        const int sp = c.split_id % p.S, bhk = c.split_id / p.S;
        const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
        for (int i = t - 128; i < G * D; i += 128) {
          const int h = i / D, x = i % D;
          const float v = (oacc[(0 * G + h) * D + x] + oacc[(1 * G + h) * D + x]) +
                          (oacc[(2 * G + h) * D + x] + oacc[(3 * G + h) * D + x]);
          const float lf = fin[G + h];
          const size_t prow = (static_cast<size_t>(b) * p.Hq + hk * G + h) * p.S + sp;
          p.o_parts[prow * D + x] = lf > 0.0f ? v / lf : 0.0f;
          if (x == 0)
            p.lse_parts[prow] = lf > 0.0f ? (fin[h] + log2f(lf)) * 0.6931471805599453f : -INFINITY;
        }
        pv_barrier();  // oacc free again
        ++pv_seq;
      }
      c = next_task(c, false);
    }
    if (failed && t == 128) {
      *abort_flag = 1;
      if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
    }
    return;
  }

  // ======================= vote warps 0-3 ===================================
  // Warp w owns keys [w*KW, w*KW + KW) of every block; thread (g, c4) holds,
  // for head g < G, the scores of keys 8j + 2c4, 8j + 2c4 + 1 of each n-tile j.
  uint32_t qa[D / 16][2];  // q fragments (bf16 pairs) of head g for each k-step
  float m[G], l[G];        // running statistics of the split being voted
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.0f;
  }
  bool aborted = false;
  int q_split = -1;  // split whose q rows are in qa
  int vote_seq = 0;  // splits finished on the vote side

  auto compute_barrier = [&]() { ptx::named_bar_sync(1, C::NC); };

  TaskCursor cur = advance_split(blockIdx.x, true);
  int n = 0;
  while (cur.split_id < nsplits) {
    {
      // ---- score and vote task n -------------------------------------------
      const int bhk = cur.split_id / p.S;
      const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
      if (cur.split_id != q_split) {
        // q fragments of head g (rows g >= G of the padded tile are zero)
        const __nv_bfloat16* qrow = p.q + (static_cast<size_t>(b) * p.Hq + hk * G + g) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * c4) : 0u;
          qa[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * c4) : 0u;
        }
        q_split = cur.split_id;
      }
      if (cur.blk == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m[h] = -INFINITY;
          l[h] = 0.0f;
        }
      }
      const int ks = n % C::NK;
      bool w = true;
      if (lane == 0) w = ptx::mbar_wait(bar(B_KF + ks), (n / C::NK) & 1, abort_flag, p.timeout_ns);
      w = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
      if (!w) *abort_flag = 1;
      const int key0 = task_key0(cur);
      const int k1 = min((cur.split_id % p.S) * p.Ls + p.Ls, p.Lkv);
      // S = q K^T for this warp's keys: n-tile j covers keys warp*KW + 8j + [0, 8)
      float sc[C::NTQ][2];
      const uint32_t kst = sb + C::OFF_K + ks * C::KV_BYTES;
#pragma unroll
      for (int j = 0; j < C::NTQ; ++j) {
        sc[j][0] = sc[j][1] = 0.0f;
        const int key = warp * C::KW + 8 * j + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          uint32_t b0, b1, b2, b3;
          dmma::ldsm_x4(kst + dmma::sw_chunk(key, 2 * kk + (lane >> 3), C::KV_BOX), b0, b1, b2, b3);
          dmma::mma16816(sc[j][0], sc[j][1], qa[kk][0], qa[kk][1], b0, b1, sc[j][0], sc[j][1]);
          dmma::mma16816(sc[j][0], sc[j][1], qa[kk + 1][0], qa[kk + 1][1], b2, b3, sc[j][0],
                         sc[j][1]);
        }
      }
      // scale to log2 units, mask keys outside the split, row max of head g
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < C::NTQ; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kk = key0 + warp * C::KW + 8 * j + 2 * c4 + e;
          sc[j][e] = (kk < k1 && g < G) ? sc[j][e] * p.scale_log2 : -INFINITY;
          mx = fmaxf(mx, sc[j][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (c4 == 0 && g < G) red[warp * G + g] = mx;
      if (t == 0) abort_seen[n & 1] = *abort_flag;  // one reading, shared by all below
      compute_barrier();  // K stage read; maxima visible
      if (abort_seen[n & 1]) {
        aborted = true;
        break;
      }
      if (t == 0) ptx::mbar_arrive(bar(B_KE + ks));
      const int slot = n % C::NP;
      float mb[G];
      int keepmask = 0;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mb[h] = fmaxf(fmaxf(red[h], red[G + h]), fmaxf(red[2 * G + h], red[3 * G + h]));
        const bool skip = (cur.blk > 0) && thresholding && (mb[h] - m[h] < p.log2_lambda);
        if (!skip) keepmask |= 1 << h;
      }
      if (t == 0) {
        // hand the decision to the V warp; its slot was read NDEC tasks ago
        const int ds = n % C::NDEC;
        if (n >= C::NDEC &&
            !ptx::mbar_wait(bar(B_DR + ds), ((n / C::NDEC) - 1) & 1, abort_flag, p.timeout_ns))
          *abort_flag = 1;
        dec_ring[ds] = keepmask;
        ptx::mbar_arrive(bar(B_DEC + ds));
      }
      // the task record slot was last read by the P V warps NP tasks ago
      if (n >= C::NP) {
        bool wf = true;
        if (lane == 0)
          wf = ptx::mbar_wait(bar(B_TF + slot), ((n / C::NP) - 1) & 1, abort_flag, p.timeout_ns);
        wf = __shfl_sync(0xffffffffu, wf ? 1 : 0, 0) != 0;
        if (!wf) *abort_flag = 1;  // seen by every warp at the next task's check
      }
      // online softmax on the vote side; P of head g into bf16 fragments
      float alpha[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const bool kh = (keepmask >> h) & 1;
        const float m_new = kh ? fmaxf(m[h], mb[h]) : m[h];
        alpha[h] = (kh && m[h] != m_new) ? ptx::ex2(m[h] - m_new) : 1.0f;
        if (t == 0) {
          task_alpha[slot * G + h] = alpha[h];
          task_keep[slot * G + h] = kh ? 1 : 0;
        }
        m[h] = m_new;
      }
      const bool gk = g < G && ((keepmask >> g) & 1);
      const float mg = g < G ? m[g] : 0.0f;
      float sum = 0.0f;
      uint32_t pr[C::PREGS];
#pragma unroll
      for (int j = 0; j < C::NTQ; ++j) {
        const float p0 = gk ? ptx::ex2(sc[j][0] - mg) : 0.0f;
        const float p1 = gk ? ptx::ex2(sc[j][1] - mg) : 0.0f;
        sum += p0 + p1;
        pr[j] = ptx::pack_bf16x2(p0, p1);  // n-tile j = (k-step j/2, half j%2)
      }
#pragma unroll
      for (int i = 0; i < C::PREGS; ++i) pfrag[(slot * C::NC + t) * C::PREGS + i] = pr[i];
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      float* reds = red + 4 * G;
      if (c4 == 0 && g < G) reds[warp * G + g] = sum;
      compute_barrier();  // sums and the task record visible
#pragma unroll
      for (int h = 0; h < G; ++h)
        l[h] = l[h] * alpha[h] + ((reds[h] + reds[G + h]) + (reds[2 * G + h] + reds[3 * G + h]));
      if (cur.blk + 1 == cur.nblk) {
        if (t == 0) {
          float* fin = split_fin + (vote_seq % C::NFIN) * 2 * G;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            fin[h] = m[h];
            fin[G + h] = l[h];
          }
        }
        ++vote_seq;
      }
      if (t == 0) ptx::mbar_arrive(bar(B_TR + slot));  // record (and finals) published
      cur = next_task(cur, true);
      ++n;
    }
  }

  if (aborted && t == 0) {
    *abort_flag = 1;
    if (p.err) atomicCAS(p.err, 0, BLASST_ETIMEOUT);
  }
}

// o = sum_s w_s o_s / sum_s w_s, lse = M + ln(sum_s w_s), w_s = exp(lse_s - M).
// One CTA per row; thread x handles output dims x, x + blockDim, ...
// `err` (nullable): the device error word. If it is set when the kernel
// starts (a bounded wait of the split kernel gave up, so some partials were
// never written), the row gets NaN outputs and lse = -inf instead.
template <typename OutT>
__global__ void blasst_lse_merge_kernel(const float* __restrict__ o_parts,
                                        const float* __restrict__ lse_parts, OutT* __restrict__ o,
                                        float* __restrict__ lse, int d, int S,
                                        const int* __restrict__ err) {
  const int row = blockIdx.x;
  if (err != nullptr && *reinterpret_cast<const volatile int*>(err) != 0) {
    for (int x = threadIdx.x; x < d; x += blockDim.x) {
      if constexpr (sizeof(OutT) == 2) o[static_cast<size_t>(row) * d + x] = __float2bfloat16_rn(NAN);
      else o[static_cast<size_t>(row) * d + x] = NAN;
    }
    if (threadIdx.x == 0) lse[row] = -INFINITY;
    return;
  }
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
