/*
 * blasst.h - C ABI of the B200 (sm_100a) library for blocked attention with
 * softmax thresholding.
 *
 * The method: a FlashAttention-style forward pass walks the KV blocks of each
 * query tile left to right with an online softmax (running row max m, running
 * sum l, rescaled output accumulator). A KV block is skipped when its local
 * score max is negligible against the running max, i.e. when
 *     exp(m_blk - m_run) < lambda      for every row of the query tile;
 * a skipped block's P.V product and V loads never happen, and the first block
 * is always processed. Sources:
 *   - "BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding"
 *     (Telegram channel seeallochnaya, post 3655), paragraphs 2-6 counted
 *     after the headline: blocked left-to-right FlashAttention, online
 *     softmax, FlashAttention-4 lazy rescaling, the skip rule (V of a dropped
 *     block is not used), the first block always processed;
 *   - "BLASST wins Best Paper at MLSys 2026 ..." (digg.com/ai/al6mgdew), the
 *     authors' announcement: one scalar threshold on the online-softmax
 *     statistics;
 *   - "В тени длинного контекста ..." (denisavetisyan.com, LongCA-bench
 *     review), section on masking strategies (causal and full masks) and the
 *     closing section on the KV cache (the decode input).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them. Work is enqueued on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream) and the call
 *     returns without synchronising.
 *   - Layouts are dense row-major: q, o [B, Hq, Lq, d]; k, v [B, Hkv, Lkv, d];
 *     lse [B, Hq, Lq] fp32 (natural log). Every tensor pointer must be 16-byte
 *     aligned.
 *   - GQA: query head hq reads KV head hq / (Hq / Hkv).
 *   - Causal masks are bottom-right aligned: key j is visible from query row
 *     i when j <= i + (Lkv - Lq).
 *   - Scores are scale * q.k with scale = 1/sqrt(d) unless stated otherwise.
 *   - A negative return value is an error from host-side validation or from
 *     the launch; nothing is enqueued after a validation error. Errors raised
 *     inside a kernel (a bounded wait that gave up) are recorded in a device
 *     error word that blasst_check() reads and clears.
 */
#ifndef BLASST_H
#define BLASST_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BLASST_API __attribute__((visibility("default")))
#else
#define BLASST_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BLASST_OK = 0,
  BLASST_EINVAL = -1,        /* bad argument (shape, pointer, lambda, alignment) */
  BLASST_EUNSUPPORTED = -2,  /* valid request this build does not implement */
  BLASST_ECUDA = -3,         /* a CUDA runtime/driver call failed */
  BLASST_ETIMEOUT = -4,      /* a device-side bounded wait gave up */
  BLASST_EWORKSPACE = -5     /* workspace missing or too small */
} blasst_status;

typedef enum { BLASST_BF16 = 0, BLASST_FP32 = 1 } blasst_dtype;

/* Telemetry counters, accumulated (atomically added) into a caller-owned
 * DEVICE struct when one is passed; the library never clears it. */
typedef struct blasst_stats {
  unsigned long long tiles_visited;   /* (query tile, KV block) pairs whose scores were formed */
  unsigned long long tiles_skipped;   /* of those, pairs dropped by the threshold */
  unsigned long long v_blocks_loaded; /* KV blocks whose V was fetched */
  unsigned long long mma_flops;       /* tensor-core / FMA flops actually executed (2 per MAC) */
  unsigned long long bytes_loaded;    /* Q, K, V bytes requested from global memory */
  /* bf16 prefill only (other calls leave them as they are): summed over the
   * launch's CTAs, the SM clock cycles (clock64) and the nanoseconds
   * (%globaltimer) from each CTA's start to its end. Their ratio is the mean
   * SM clock while the kernel ran, which a sampler outside the GPU can miss
   * on short calls. */
  unsigned long long sm_cycles;
  unsigned long long sm_ns;
} blasst_stats;

/* Forward prefill pass, bf16 in / bf16 out, fp32 lse, on the legacy default
 * stream, scale 1/sqrt(d).
 *   q, k, v, o  device pointers, layouts above. o may not alias q, k or v.
 *   lse         [B, Hq, Lq] fp32, natural-log row log-sum-exp of the kept keys.
 *   causal      1: bottom-right causal mask (requires Lq <= Lkv); 0: full.
 *   lambda      threshold in [0, 1); 0 never skips (exact attention).
 *   Br, Bc      query-tile rows and KV-block keys, each 64 or 128; the skip
 *               decision is taken per (Br-row tile, Bc-key block).
 *   d           head dimension, 64 or 128.
 *   skip_mask_out  nullable device pointer to uint8 [B, Hq, ceil(Lq/Br),
 *               ceil(Lkv/Bc)], fully written: 0 computed, 1 skipped,
 *               2 not visited (causally invisible).
 * Returns BLASST_OK or a negative blasst_status. */
BLASST_API int blasst_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Lq, int Lkv, int d, int causal, float lambda, int Br, int Bc,
               uint8_t* skip_mask_out);

/* Extended form of blasst_fwd: same operation and arguments plus
 *   dtype      BLASST_BF16 (q, k, v, o bf16) or BLASST_FP32 (fp32; d = 64, Bc = 64 only;
 *              both products use an error-compensated three-product tf32 split);
 *   scale      score scale; <= 0 selects 1/sqrt(d);
 *   stream     cudaStream_t to enqueue on (NULL = legacy default stream);
 *   stats_out  nullable DEVICE pointer; counters are added to it;
 *   block_mask_in  nullable DEVICE pointer, uint8 [B, Hq, ceil(Lq/Br), ceil(Lkv/Bc)]:
 *              a static block-sparse mask. A nonzero entry excludes that
 *              (query tile, KV block) pair before anything is computed: no
 *              scores, no vote, nothing added, reported as 2 (not visited) in
 *              skip_mask_out. The threshold skip then runs over the blocks
 *              left, and the first of them is always computed (the
 *              first-block rule of "BLASST: Dynamic BLocked Attention
 *              Sparsity via Softmax Thresholding", the post's figure, read
 *              for the blocks the mask leaves). Rows left with no key get
 *              O = 0 and lse = -inf. This is the block-sparse input that a
 *              pre-pass selector feeds; the pages describe such selectors
 *              (CRISP, FlashPrefill) but give no interface for it. Requires
 *              ceil(Lkv/Bc) <= 4096, else BLASST_EUNSUPPORTED. */
typedef struct blasst_fwd_args {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  float lambda;
  int Br, Bc;
  uint8_t* skip_mask_out;
  int dtype;
  float scale;
  void* stream;
  blasst_stats* stats_out;
  const uint8_t* block_mask_in;
} blasst_fwd_args;
BLASST_API int blasst_fwd_ex(const blasst_fwd_args* args);

/* Backward pass of the prefill with the forward's skip decisions held fixed.
 * The decisions are a step function of the scores, so the gradient is that
 * of softmax attention restricted to the (row, key) pairs the forward kept
 * (a dropped block adds nothing to O: "BLASST: Dynamic BLocked Attention
 * Sparsity via Softmax Thresholding", paragraph 5 after the headline, the
 * skip rule). With P = exp(scale q.k - lse) on kept pairs (0 elsewhere),
 * Dr = rowsum(dO * O) and dS = P * (dO.v - Dr):
 *     dq = scale dS K,   dk = scale dS^T Q,   dv = P^T dO,
 * dk and dv summed over the query heads of each GQA group. The pages give no
 * backward pass; this is the reading the forward's definition fixes.
 *   q, o, dout [B, Hq, Lq, d] bf16; k, v [B, Hkv, Lkv, d] bf16; lse [B, Hq, Lq]
 *              fp32 (natural log), the forward's outputs for these inputs.
 *   dq         [B, Hq, Lq, d] fp32, overwritten.
 *   dk, dv     [B, Hkv, Lkv, d] fp32, overwritten.
 *   causal     as in the forward (bottom-right aligned; Lq <= Lkv).
 *   Br, Bc     the forward's tile sizes (64 or 128): skip_mask is read per
 *              (Br-row tile, Bc-key block).
 *   skip_mask  the forward's skip_mask_out, uint8 [B, Hq, ceil(Lq/Br),
 *              ceil(Lkv/Bc)]: only pairs with entry 0 take part. NULL: every
 *              causally visible pair does (a forward with lambda = 0 and no
 *              static mask).
 *   scale      score scale; <= 0 selects 1/sqrt(d).
 *   workspace  device buffer of at least blasst_bwd_workspace_bytes(B, Hq, Lq)
 *              bytes, 16-byte aligned (per-row statistics).
 * d must be 128 (else BLASST_EUNSUPPORTED). Rows whose lse is -inf (no key
 * kept) get dq = 0 and add nothing to dk, dv. */
typedef struct blasst_bwd_args {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  float* dq;
  float* dk;
  float* dv;
  int B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  int Br, Bc;
  const uint8_t* skip_mask;
  float scale;
  void* workspace;
  size_t workspace_bytes;
  void* stream;
} blasst_bwd_args;
BLASST_API int blasst_bwd(const blasst_bwd_args* args);

/* Bytes of workspace blasst_bwd needs: two fp32 [B, Hq, ceil(Lq/64)*64]. */
BLASST_API size_t blasst_bwd_workspace_bytes(int B, int Hq, int Lq);

/* Pre-pass block selector producing a static block mask for blasst_fwd_ex
 * (block_mask_in), after the CRISP review (rit.work, blog/crisp-sparse-
 * attention-long-prefill, section "What was done", paragraphs 3-5). The page
 * gives no formulas; the readings:
 *   - map: per query head, qb_t = mean of the rows of query tile t, kb_j =
 *     mean of the keys of KV block j, A[t][j] = softmax over the blocks
 *     visible from tile t (causal: bottom-right) of scale * qb_t . kb_j;
 *   - C_struct = mean over tiles of A[t][0] + A[t][last(t)], last(t) the
 *     tile's last visible block; the head is "structured" when C_struct >= tau;
 *   - structured: keep block 0, block last(t), and the blocks in between
 *     whose A is strictly above the mean A of those in-between blocks;
 *   - otherwise: keep the largest-A blocks until they cover gamma of the row,
 *     plus every block tied with the last one taken.
 *   q [B, Hq, Lq, d], k [B, Hkv, Lkv, d] bf16 (device).
 *   Br, Bc     tile sizes of the forward that will read the mask (64 or 128).
 *   mask_out   uint8 [B, Hq, ceil(Lq/Br), ceil(Lkv/Bc)], fully written:
 *              0 = selected, 1 = not selected (invisible blocks are 1).
 *   cstruct_out nullable fp32 [B, Hq].
 *   tau, gamma route threshold and pooled-path coverage (0 < gamma <= 1).
 *   scale      <= 0 selects 1/sqrt(d).
 *   workspace  >= blasst_select_workspace_bytes(...) bytes, 16-byte aligned.
 * d in {64, 128}; ceil(Lkv/Bc) <= 2048 (else BLASST_EUNSUPPORTED). */
typedef struct blasst_select_args {
  const void* q;
  const void* k;
  int B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  int Br, Bc;
  float scale;
  float tau;
  float gamma;
  uint8_t* mask_out;
  float* cstruct_out;
  void* workspace;
  size_t workspace_bytes;
  void* stream;
} blasst_select_args;
BLASST_API int blasst_select_blocks(const blasst_select_args* args);

/* Workspace bytes of blasst_select_blocks: the pooled rows (fp32
 * [B*Hq, nQt, d] and [B*Hkv, nKt, d]), three fp32 row statistics per query
 * tile and the fp32 block scores [B*Hq, nQt, nKt]. */
BLASST_API size_t blasst_select_workspace_bytes(int B, int Hq, int Hkv, int Lq, int Lkv, int d,
                                                int Br, int Bc);

/* Bytes of caller workspace that blasst_decode needs: fp32 partial outputs
 * [B, Hq, num_splits, d] plus fp32 partial lse [B, Hq, num_splits]. */
BLASST_API size_t blasst_decode_workspace_bytes(int B, int Hq, int d, int num_splits);

/* Split-KV decode: one new query row per sequence and head against a
 * contiguous KV cache, then a log-sum-exp merge of the splits.
 *   q          [B, Hq, 1, d] bf16;  k_cache, v_cache [B, Hkv, Lkv, d] bf16.
 *   o          [B, Hq, 1, d] bf16;  lse [B, Hq] fp32 (natural log).
 *   Bc         KV block size (64 or 128); the skip decision is per (head, block).
 *   num_splits S: keys are cut into S chunks of ceil(ceil(Lkv/S)/Bc)*Bc keys;
 *              each chunk runs its own pass (its first block always
 *              computed, running statistics restart), then chunks are merged.
 *   workspace  device buffer of at least blasst_decode_workspace_bytes().
 *   skip_mask_out nullable uint8 [B, Hq, ceil(Lkv/Bc)] (0 computed, 1 skipped).
 *   stats_out  nullable device blasst_stats.
 * A KV block's V rows are read only if at least one query head of its GQA
 * group keeps the block; heads that skip it add nothing.
 * If a bounded wait of the split kernel gives up (blasst_check then returns
 * BLASST_ETIMEOUT), the merge writes NaN to o and -inf to lse rather than
 * merging partials that were never written; the same holds for any decode
 * call made while the device error word still holds an earlier error. */
BLASST_API int blasst_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                  int B, int Hq, int Hkv, int Lkv, int d, float lambda, int Bc, int num_splits,
                  void* workspace, size_t workspace_bytes, uint8_t* skip_mask_out,
                  blasst_stats* stats_out, void* stream);

/* Allocation-free form of blasst_decode. The pages have no counterpart: this
 * is for callers that cannot allocate device memory where they run decode
 * (a plugin inside a framework that owns all device allocations, a serving
 * loop whose memory was planned once at start-up, a host thread for which a
 * cudaMalloc would be too costly or would synchronise the device).
 * Same operation and arguments as blasst_decode, minus the workspace: the
 * split partials live in a fixed device array inside the library, of
 * blasst_decode_noalloc_max_bytes() bytes (32 MiB), which every GPU that loads
 * the library holds until the process exits. The call allocates nothing and
 * frees nothing.
 *   - Requests whose partials, blasst_decode_workspace_bytes(B, Hq, d,
 *     num_splits), exceed that size are rejected with BLASST_EWORKSPACE.
 *   - The first call on a device looks up the array's device address (one
 *     cudaGetSymbolAddress with that device current); make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     every partial a call merges is written earlier in the same call, so
 *     nothing needs clearing between calls. If a bounded wait of the split
 *     kernel gives up (blasst_check then returns BLASST_ETIMEOUT), some
 *     partials of that call are never written: its merge sees the device
 *     error word and writes NaN to o and -inf to lse instead (so does any
 *     decode call made while the word still holds an error).
 *     Calls that may run concurrently on the GPU (different streams, or
 *     different host threads on the same device) race on the array: order
 *     them on one stream. */
BLASST_API int blasst_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     void* o, float* lse, int B, int Hq, int Hkv, int Lkv, int d,
                                     float lambda, int Bc, int num_splits, uint8_t* skip_mask_out,
                                     blasst_stats* stats_out, void* stream);

/* Size in bytes of the fixed array blasst_decode_noalloc uses. */
BLASST_API size_t blasst_decode_noalloc_max_bytes(void);

/* Split-KV decode with softmax thresholding for multi-head latent attention
 * (MLA) caches, in the absorbed form: every query head has a 576-wide query
 * (512 latent + 64 rotary dims); every cached token one 576-wide row c shared
 * by all heads (latent in dims 0-511, rotary key in 512-575); scores
 * scale * q_h . c_j; the output o_h = sum_j p_hj c_j[0:512]. That is softmax
 * attention with one KV head, K = c, V = c[:, 0:512]. The post ("BLASST:
 * Dynamic BLocked Attention Sparsity via Softmax Thresholding", paragraph 9
 * after the headline) says only that the method is compatible with MLA; the
 * skip rule here is the decode one, per (head, Bc-key block), the first
 * block of each split always computed, then the log-sum-exp merge of
 * blasst_decode. V is part of the cached rows already read for the scores, so
 * a skip saves no bytes; a block's P V is skipped for a group of heads (128
 * when H is a multiple of 128: the tensor-core kernel; else 16: the mma.sync
 * kernel) when every head of the group drops it.
 *   q          [B, H, 576] bf16;  cache [B, L, 576] bf16.
 *   o          [B, H, 512] bf16;  lse [B, H] fp32 (natural log).
 *   H          a multiple of 16.
 *   Bc         decision block: 64 (others: BLASST_EUNSUPPORTED).
 *   num_splits splits of ceil(ceil(L/S)/Bc)*Bc keys each.
 *   scale      score scale; <= 0 selects 1/sqrt(576).
 *   workspace  >= blasst_decode_mla_workspace_bytes(B, H, num_splits).
 *   skip_mask_out nullable uint8 [B, H, ceil(L/Bc)] (0 computed, 1 skipped).
 *   stats_out  nullable device blasst_stats. */
BLASST_API int blasst_decode_mla(const void* q, const void* cache, void* o, float* lse, int B, int H,
                                 int L, float lambda, int Bc, int num_splits, float scale,
                                 void* workspace,
                                 size_t workspace_bytes, uint8_t* skip_mask_out,
                                 blasst_stats* stats_out, void* stream);

/* Workspace bytes of blasst_decode_mla: fp32 [B, H, S, 512] + [B, H, S]. */
BLASST_API size_t blasst_decode_mla_workspace_bytes(int B, int H, int num_splits);

/* A split count for blasst_decode_mla (64-key blocks) that fills whole waves
 * of the GPU: every CTA of the decode kernel occupies one SM (the tensor-core
 * kernel launches 2 B H/128 CTAs per split, the mma.sync kernel B H/16), so
 * the launch takes about ceil(CTAs / num_sms) x (blocks per split) block
 * times. Returns the smallest S within 3 % of the best such estimate over
 * S = 1 .. min(ceil(L / 64), 1024) (fewer splits: less partial traffic for
 * the merge). Host only, no device work.
 *   num_sms  SMs to fill; <= 0 queries the current device.
 * Returns S >= 1, or BLASST_EINVAL for B, H, L <= 0 or H not a multiple of
 * 16, BLASST_ECUDA if the device query fails. Decisions depend on the split
 * boundaries (each split restarts the running statistics), so the oracle
 * must be run with the same S. */
BLASST_API int blasst_decode_mla_splits(int B, int H, int L, int num_sms);

/* Log-sum-exp merge of split partials (the second half of blasst_decode):
 *   o_parts [n_rows, num_splits, d] fp32, normalised per split;
 *   lse_parts [n_rows, num_splits] fp32, -inf marks an empty split;
 *   o [n_rows, d] in `out_dtype` (BLASST_BF16 or BLASST_FP32); lse [n_rows].
 * o = sum_s w_s o_s / sum_s w_s, lse = M + ln sum_s w_s, w_s = exp(lse_s - M),
 * M = max_s lse_s. */
BLASST_API int blasst_lse_merge(const float* o_parts, const float* lse_parts, void* o, float* lse, int n_rows,
                     int d, int num_splits, int out_dtype, void* stream);

/* Synchronises `stream`, then returns (and clears) the device error word:
 * BLASST_OK, BLASST_ETIMEOUT if a kernel's bounded wait gave up, or
 * BLASST_ECUDA if the stream reported a CUDA error. While the word holds an
 * error, prefill CTAs that start return without computing (so a failing
 * launch ends within one wave of bounded waits) and decode merges write NaN:
 * outputs of calls made after an error and before this check are undefined. */
BLASST_API int blasst_check(void* stream);

/* Self-test of the two exponentials the prefill kernel uses, so that a test
 * can check them against float64: y_mufu[i] = 2^x[i] from the hardware
 * approximation (ex2.approx), y_poly[i] = 2^x[i] from the FMA-pipe
 * polynomial that takes part of the softmax exponentials (relative
 * error <= 1.1e-4 for x in [-125, 64]). x, y_mufu, y_poly: device fp32 [n]. */
BLASST_API int blasst_selftest_exp2(const float* x, float* y_mufu, float* y_poly, int n,
                                    void* stream);

/* Self-test of the failure path every kernel's waits share: launches one warp
 * that waits on an mbarrier nothing arrives on, with a bound of limit_ns
 * (1 ns to 10 s); the wait gives up, the kernel records BLASST_ETIMEOUT in
 * the device error word (which blasst_check then returns and clears) and
 * exits normally, leaving the context usable. Nothing is faulted or trapped.
 * Returns the launch status. */
BLASST_API int blasst_selftest_timeout(unsigned long long limit_ns, void* stream);

/* Text of the last CUDA error this library saw on the calling host thread
 * (the reason behind the latest BLASST_ECUDA), or "no error". */
BLASST_API const char* blasst_last_cuda_error(void);

/* Human-readable name of a blasst_status value (static storage). */
BLASST_API const char* blasst_status_string(int status);

/* Library ABI version (major * 100 + minor). */
BLASST_API int blasst_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BLASST_H */
