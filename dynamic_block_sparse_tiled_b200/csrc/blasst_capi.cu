// blasst_capi.cu - the exported C ABI (include/blasst.h): argument checks,
// TMA tensor maps, kernel selection and launch, the device error word.
//
// Single translation unit: the kernels are included here so that the error
// word and every template instantiation live in one module.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/blasst.h"
#include "bwd_sm100.cuh"
#include "decode_mla_sm100.cuh"
#include "decode_sm100.cuh"
#include "prefill_f32_sm100.cuh"
#include "prefill_sm100.cuh"
#include "select_sm100.cuh"

namespace {

// Device error word: set (first error wins) by kernels whose bounded waits
// gave up; read and cleared by blasst_check().
__device__ int g_blasst_error = 0;

constexpr int kMaxDevices = 64;
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per bounded wait

std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {nullptr};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Address of the error word on the current device (looked up once per device).
int* error_word() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_blasst_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_err_ptr[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Text of the last failing CUDA call made by this library on this host thread.
thread_local const char* g_last_cuda_error = "no error";

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BLASST_OK;
  g_last_cuda_error = cudaGetErrorString(e);
  return BLASST_ECUDA;
}

// 3-D map over a dense [heads, L, d] tensor: dims (d, L, heads), box
// (64 columns, rows, 1), 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
              int d, int L, int heads, int box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(d) * elem_bytes * L};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes),
                       static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over a dense fp32 [heads, L, d] tensor without swizzle, box
// (32 columns, rows, 1): the target of TMA reduce-adds.
bool make_map_f32_plain(CUtensorMap* map, void* base, int d, int L, int heads, int box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(d) * 4 * L};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) g_last_cuda_error = cudaGetErrorString(e);
  return e;
}

template <int D, int BC, int BR>
int launch_prefill_bf16(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const blasst::PrefillParams& p, cudaStream_t stream) {
  using C = blasst::PrefillCfg<D, BC, BR>;
  const bool listed = p.smask != nullptr;
  auto kernel = listed ? blasst::blasst_prefill_bf16_kernel<D, BC, BR, true>
                       : blasst::blasst_prefill_bf16_kernel<D, BC, BR, false>;
  const int smem = listed ? C::SMEM_BYTES_LISTED : C::SMEM_BYTES;
  if (set_smem(kernel, smem) != cudaSuccess) return BLASST_ECUDA;
  const dim3 grid(static_cast<unsigned>(p.nQblk) * p.B * p.Hq);
  kernel<<<grid, C::NTHREADS, smem, stream>>>(mq, mk, mv, p);
  return cuda_status(cudaGetLastError());
}

template <int BR>
int launch_prefill_f32(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const blasst::PrefillParams& p, cudaStream_t stream) {
  using C = blasst::PrefillF32Cfg<BR>;
  auto kernel = blasst::blasst_prefill_f32_kernel<BR>;
  if (set_smem(kernel, C::SMEM_BYTES) != cudaSuccess) return BLASST_ECUDA;
  const dim3 grid(static_cast<unsigned>(p.nQblk) * p.B * p.Hq);
  kernel<<<grid, 128, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  return cuda_status(cudaGetLastError());
}

int dispatch_prefill_bf16(int d, int Bc, int Br, const CUtensorMap& mq, const CUtensorMap& mk,
                          const CUtensorMap& mv, const blasst::PrefillParams& p,
                          cudaStream_t s) {
#define BLASST_PF(D_, BC_, BR_) \
  if (d == D_ && Bc == BC_ && Br == BR_) return launch_prefill_bf16<D_, BC_, BR_>(mq, mk, mv, p, s);
  BLASST_PF(128, 128, 128)
  BLASST_PF(128, 128, 64)
  BLASST_PF(128, 64, 128)
  BLASST_PF(128, 64, 64)
  BLASST_PF(64, 128, 128)
  BLASST_PF(64, 128, 64)
  BLASST_PF(64, 64, 128)
  BLASST_PF(64, 64, 64)
#undef BLASST_PF
  return BLASST_EUNSUPPORTED;
}

template <int D, int BC, int G>
int launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const blasst::DecodeParams& p,
                  cudaStream_t stream) {
  using C = blasst::DecodeCfg<D, BC, G>;
  auto kernel = blasst::blasst_decode_split_kernel<D, BC, G>;
  if (set_smem(kernel, C::SMEM_BYTES) != cudaSuccess) return BLASST_ECUDA;
  // persistent: one CTA per SM, each streaming its share of the splits
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long nsplits = static_cast<long long>(p.B) * p.Hkv * p.S;
  const unsigned grid = static_cast<unsigned>(nsplits < sms ? nsplits : sms);
  kernel<<<grid, C::NT, C::SMEM_BYTES, stream>>>(mk, mv, p);
  return cuda_status(cudaGetLastError());
}

int dispatch_decode(int d, int Bc, int g, const CUtensorMap& mk, const CUtensorMap& mv,
                    const blasst::DecodeParams& p, cudaStream_t s) {
#define BLASST_DC(D_, BC_, G_) \
  if (d == D_ && Bc == BC_ && g == G_) return launch_decode<D_, BC_, G_>(mk, mv, p, s);
  BLASST_DC(128, 128, 1)
  BLASST_DC(128, 128, 2)
  BLASST_DC(128, 128, 4)
  BLASST_DC(128, 128, 8)
  BLASST_DC(128, 64, 1)
  BLASST_DC(128, 64, 2)
  BLASST_DC(128, 64, 4)
  BLASST_DC(128, 64, 8)
  BLASST_DC(64, 128, 1)
  BLASST_DC(64, 128, 2)
  BLASST_DC(64, 128, 4)
  BLASST_DC(64, 128, 8)
  BLASST_DC(64, 64, 1)
  BLASST_DC(64, 64, 2)
  BLASST_DC(64, 64, 4)
  BLASST_DC(64, 64, 8)
#undef BLASST_DC
  return BLASST_EUNSUPPORTED;
}

__global__ void selftest_exp2_kernel(const float* x, float* y_mufu, float* y_poly, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    y_mufu[i] = blasst::ptx::ex2(x[i]);
    float y1;
    blasst::ptx::exp2_poly2(y_poly[i], y1, x[i], -x[i]);  // the two-wide form the kernel uses
  }
}

// Bounded-wait self test: one warp waits on an mbarrier that nothing ever
// arrives on; the wait gives up after limit_ns and the kernel records
// BLASST_ETIMEOUT in the error word, the path every kernel's waits take.
__global__ void selftest_timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long mbar;
  __shared__ int never;
  const uint32_t b = blasst::ptx::smem_u32(&mbar);
  if (threadIdx.x == 0) {
    blasst::ptx::mbar_init(b, 1);
    never = 0;
    blasst::ptx::fence_mbar_init();
  }
  __syncwarp();
  const bool ok = blasst::ptx::mbar_wait(b, 0, &never, limit_ns);
  if (__all_sync(0xffffffffu, !ok) && threadIdx.x == 0 && err) atomicCAS(err, 0, BLASST_ETIMEOUT);
}

float log2_lambda_of(float lambda) {
  return lambda > 0.0f ? static_cast<float>(std::log2(static_cast<double>(lambda)))
                       : -INFINITY;
}

}  // namespace

extern "C" {

int blasst_version(void) { return 100; }

const char* blasst_last_cuda_error(void) { return g_last_cuda_error; }

const char* blasst_status_string(int status) {
  switch (status) {
    case BLASST_OK: return "BLASST_OK";
    case BLASST_EINVAL: return "BLASST_EINVAL: invalid argument";
    case BLASST_EUNSUPPORTED: return "BLASST_EUNSUPPORTED: configuration not implemented";
    case BLASST_ECUDA: return "BLASST_ECUDA: CUDA call failed";
    case BLASST_ETIMEOUT: return "BLASST_ETIMEOUT: a device-side bounded wait gave up";
    case BLASST_EWORKSPACE: return "BLASST_EWORKSPACE: workspace missing or too small";
    default: return "BLASST: unknown status";
  }
}

int blasst_fwd_ex(const blasst_fwd_args* a) {
  if (!a) return BLASST_EINVAL;
  if (!a->q || !a->k || !a->v || !a->o || !a->lse) return BLASST_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o) ||
      !aligned16(a->lse))
    return BLASST_EINVAL;
  if (a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Lq <= 0 || a->Lkv <= 0) return BLASST_EINVAL;
  if (a->Hq % a->Hkv != 0) return BLASST_EINVAL;
  if (!(a->lambda >= 0.0f && a->lambda < 1.0f)) return BLASST_EINVAL;
  if (a->d != 64 && a->d != 128) return BLASST_EUNSUPPORTED;
  if ((a->Br != 64 && a->Br != 128) || (a->Bc != 64 && a->Bc != 128)) return BLASST_EUNSUPPORTED;
  if (a->causal && a->Lq > a->Lkv) return BLASST_EUNSUPPORTED;
  if (a->dtype != BLASST_BF16 && a->dtype != BLASST_FP32) return BLASST_EUNSUPPORTED;
  if (a->dtype == BLASST_FP32 && (a->d != 64 || a->Bc != 64)) return BLASST_EUNSUPPORTED;
  if (a->block_mask_in && (a->Lkv + a->Bc - 1) / a->Bc > 4096) return BLASST_EUNSUPPORTED;
  if (static_cast<long long>(a->B) * a->Hq > (1ll << 24) ||
      static_cast<long long>(a->B) * a->Hq * ((a->Lq + 127) / 128) > 0x7fffffffll)
    return BLASST_EINVAL;

  int* err = error_word();
  if (!err) return BLASST_ECUDA;

  blasst::PrefillParams p{};
  p.o = a->o;
  p.lse = a->lse;
  p.mask = a->skip_mask_out;
  p.smask = a->block_mask_in;
  p.stats = a->stats_out;
  p.err = err;
  p.B = a->B;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.Lq = a->Lq;
  p.Lkv = a->Lkv;
  p.g = a->Hq / a->Hkv;
  p.nQt = (a->Lq + a->Br - 1) / a->Br;
  p.nKt = (a->Lkv + a->Bc - 1) / a->Bc;
  p.nQblk = (a->Lq + 127) / 128;
  p.causal = a->causal ? 1 : 0;
  p.off = a->Lkv - a->Lq;
  const double scale = a->scale > 0.0f ? static_cast<double>(a->scale)
                                       : 1.0 / std::sqrt(static_cast<double>(a->d));
  p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  p.log2_lambda = log2_lambda_of(a->lambda);
  p.timeout_ns = kTimeoutNs;

  CUtensorMap mq, mk, mv;
  if (a->dtype == BLASST_FP32) {
    const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!make_map(&mq, a->q, dt, 4, a->d, a->Lq, a->B * a->Hq, 128) ||
        !make_map(&mk, a->k, dt, 4, a->d, a->Lkv, a->B * a->Hkv, a->Bc) ||
        !make_map(&mv, a->v, dt, 4, a->d, a->Lkv, a->B * a->Hkv, a->Bc))
      return BLASST_ECUDA;
    const cudaStream_t s = static_cast<cudaStream_t>(a->stream);
    return a->Br == 64 ? launch_prefill_f32<64>(mq, mk, mv, p, s)
                       : launch_prefill_f32<128>(mq, mk, mv, p, s);
  }
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&mq, a->q, dt, 2, a->d, a->Lq, a->B * a->Hq, 128) ||
      !make_map(&mk, a->k, dt, 2, a->d, a->Lkv, a->B * a->Hkv, a->Bc) ||
      !make_map(&mv, a->v, dt, 2, a->d, a->Lkv, a->B * a->Hkv, a->Bc))
    return BLASST_ECUDA;
  return dispatch_prefill_bf16(a->d, a->Bc, a->Br, mq, mk, mv, p,
                               static_cast<cudaStream_t>(a->stream));
}

int blasst_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Lq, int Lkv, int d, int causal, float lambda, int Br, int Bc,
               uint8_t* skip_mask_out) {
  blasst_fwd_args a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lq = Lq;
  a.Lkv = Lkv;
  a.d = d;
  a.causal = causal;
  a.lambda = lambda;
  a.Br = Br;
  a.Bc = Bc;
  a.skip_mask_out = skip_mask_out;
  a.dtype = BLASST_BF16;
  a.scale = 0.0f;
  a.stream = nullptr;
  a.stats_out = nullptr;
  a.block_mask_in = nullptr;
  return blasst_fwd_ex(&a);
}

size_t blasst_bwd_workspace_bytes(int B, int Hq, int Lq) {
  if (B <= 0 || Hq <= 0 || Lq <= 0) return 0;
  const size_t lqp = (static_cast<size_t>(Lq) + 63) / 64 * 64;
  return 2 * static_cast<size_t>(B) * Hq * lqp * sizeof(float);
}

int blasst_bwd(const blasst_bwd_args* a) {
  if (!a) return BLASST_EINVAL;
  if (!a->q || !a->k || !a->v || !a->o || !a->dout || !a->lse || !a->dq || !a->dk || !a->dv)
    return BLASST_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o) ||
      !aligned16(a->dout) || !aligned16(a->lse) || !aligned16(a->dq) || !aligned16(a->dk) ||
      !aligned16(a->dv))
    return BLASST_EINVAL;
  if (a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Lq <= 0 || a->Lkv <= 0) return BLASST_EINVAL;
  if (a->Hq % a->Hkv != 0) return BLASST_EINVAL;
  if (a->d != 128) return BLASST_EUNSUPPORTED;
  if ((a->Br != 64 && a->Br != 128) || (a->Bc != 64 && a->Bc != 128)) return BLASST_EUNSUPPORTED;
  if (a->causal && a->Lq > a->Lkv) return BLASST_EUNSUPPORTED;
  if (static_cast<long long>(a->B) * a->Hq > (1ll << 24) ||
      static_cast<long long>(a->B) * a->Hkv * ((a->Lkv + 127) / 128) > 0x7fffffffll ||
      static_cast<long long>(a->B) * a->Hq * (((a->Lq + 63) / 64) * 64) / 8 > 0x7fffffffll)
    return BLASST_EINVAL;
  const size_t need = blasst_bwd_workspace_bytes(a->B, a->Hq, a->Lq);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return BLASST_EWORKSPACE;

  int* err = error_word();
  if (!err) return BLASST_ECUDA;

  const int LqP = (a->Lq + 63) / 64 * 64;
  const long long n_rows = static_cast<long long>(a->B) * a->Hq * LqP;
  blasst::BwdParams p{};
  p.dq = a->dq;
  p.dk = a->dk;
  p.dv = a->dv;
  p.nl2 = static_cast<const float*>(a->workspace);
  p.drow = static_cast<const float*>(a->workspace) + n_rows;
  p.fmask = a->skip_mask;
  p.err = err;
  p.B = a->B;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.Lq = a->Lq;
  p.Lkv = a->Lkv;
  p.g = a->Hq / a->Hkv;
  p.LqP = LqP;
  p.nT = LqP / 64;
  p.nKb = (a->Lkv + 127) / 128;
  p.Brf = a->Br;
  p.Bcf = a->Bc;
  p.nQf = (a->Lq + a->Br - 1) / a->Br;
  p.nKf = (a->Lkv + a->Bc - 1) / a->Bc;
  p.causal = a->causal ? 1 : 0;
  p.off = a->Lkv - a->Lq;
  const double scale = a->scale > 0.0f ? static_cast<double>(a->scale)
                                       : 1.0 / std::sqrt(static_cast<double>(a->d));
  p.scale = static_cast<float>(scale);
  p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  p.timeout_ns = kTimeoutNs;

  CUtensorMap mq, mdo, mk, mv, mdq;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map_f32_plain(&mdq, a->dq, a->d, a->Lq, a->B * a->Hq, 64) ||
      !make_map(&mq, a->q, dt, 2, a->d, a->Lq, a->B * a->Hq, 64) ||
      !make_map(&mdo, a->dout, dt, 2, a->d, a->Lq, a->B * a->Hq, 64) ||
      !make_map(&mk, a->k, dt, 2, a->d, a->Lkv, a->B * a->Hkv, 128) ||
      !make_map(&mv, a->v, dt, 2, a->d, a->Lkv, a->B * a->Hkv, 128))
    return BLASST_ECUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(a->stream);
  blasst::blasst_bwd_rows_kernel<<<static_cast<unsigned>((n_rows + 7) / 8), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(a->o), static_cast<const __nv_bfloat16*>(a->dout), a->lse,
      const_cast<float*>(p.nl2), const_cast<float*>(p.drow), a->dq, n_rows, a->Lq, LqP);
  int rc = cuda_status(cudaGetLastError());
  if (rc != BLASST_OK) return rc;
  using C = blasst::BwdCfg;
  if (set_smem(blasst::blasst_bwd_kernel, C::SMEM_BYTES) != cudaSuccess) return BLASST_ECUDA;
  const dim3 grid(static_cast<unsigned>(p.nKb) * p.B * p.Hkv);
  blasst::blasst_bwd_kernel<<<grid, C::NTHREADS, C::SMEM_BYTES, s>>>(mq, mdo, mk, mv, mdq, p);
  return cuda_status(cudaGetLastError());
}

size_t blasst_select_workspace_bytes(int B, int Hq, int Hkv, int Lq, int Lkv, int d, int Br,
                                     int Bc) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lkv <= 0 || d <= 0 || Br <= 0 || Bc <= 0)
    return 0;
  const size_t nQt = (static_cast<size_t>(Lq) + Br - 1) / Br;
  const size_t nKt = (static_cast<size_t>(Lkv) + Bc - 1) / Bc;
  return (static_cast<size_t>(B) * Hq * nQt * d + static_cast<size_t>(B) * Hkv * nKt * d +
          static_cast<size_t>(B) * Hq * nQt * 3 + static_cast<size_t>(B) * Hq * nQt * nKt) *
         sizeof(float);
}

int blasst_select_blocks(const blasst_select_args* a) {
  if (!a) return BLASST_EINVAL;
  if (!a->q || !a->k || !a->mask_out) return BLASST_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->k)) return BLASST_EINVAL;
  if (a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Lq <= 0 || a->Lkv <= 0) return BLASST_EINVAL;
  if (a->Hq % a->Hkv != 0) return BLASST_EINVAL;
  if (!(a->gamma > 0.0f && a->gamma <= 1.0f) || !std::isfinite(a->tau)) return BLASST_EINVAL;
  if (a->d != 64 && a->d != 128) return BLASST_EUNSUPPORTED;
  if ((a->Br != 64 && a->Br != 128) || (a->Bc != 64 && a->Bc != 128)) return BLASST_EUNSUPPORTED;
  if (a->causal && a->Lq > a->Lkv) return BLASST_EUNSUPPORTED;
  const int nQt = (a->Lq + a->Br - 1) / a->Br, nKt = (a->Lkv + a->Bc - 1) / a->Bc;
  if (nKt > 32 * blasst::SEL_MAXJ) return BLASST_EUNSUPPORTED;
  const long long rows = static_cast<long long>(a->B) * a->Hq * nQt;
  if (rows + static_cast<long long>(a->B) * a->Hkv * nKt > 0x7fffffffll) return BLASST_EINVAL;
  const size_t need = blasst_select_workspace_bytes(a->B, a->Hq, a->Hkv, a->Lq, a->Lkv, a->d,
                                                    a->Br, a->Bc);
  if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace))
    return BLASST_EWORKSPACE;
  blasst::SelectParams p{};
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.k = static_cast<const __nv_bfloat16*>(a->k);
  p.qbar = static_cast<float*>(a->workspace);
  p.kbar = p.qbar + static_cast<size_t>(rows) * a->d;
  p.rowst = p.kbar + static_cast<size_t>(a->B) * a->Hkv * nKt * a->d;
  p.scores = p.rowst + static_cast<size_t>(rows) * 3;
  p.mask = a->mask_out;
  p.cstruct = a->cstruct_out;
  p.B = a->B;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.Lq = a->Lq;
  p.Lkv = a->Lkv;
  p.d = a->d;
  p.g = a->Hq / a->Hkv;
  p.Br = a->Br;
  p.Bc = a->Bc;
  p.nQt = nQt;
  p.nKt = nKt;
  p.causal = a->causal ? 1 : 0;
  p.off = a->Lkv - a->Lq;
  p.scale = a->scale > 0.0f ? a->scale
                            : static_cast<float>(1.0 / std::sqrt(static_cast<double>(a->d)));
  p.tau = a->tau;
  p.gamma = a->gamma;
  const cudaStream_t s = static_cast<cudaStream_t>(a->stream);
  const unsigned npool = static_cast<unsigned>(rows + static_cast<long long>(a->B) * a->Hkv * nKt);
  blasst::blasst_select_pool_kernel<<<npool, 128, 0, s>>>(p);
  int rc = cuda_status(cudaGetLastError());
  if (rc != BLASST_OK) return rc;
  const unsigned nrow_blocks = static_cast<unsigned>((rows + 7) / 8);
  const unsigned ntile_blocks = static_cast<unsigned>(static_cast<long long>(a->B) * a->Hq *
                                                      ((nQt + 7) / 8));
  blasst::blasst_select_rows_kernel<<<ntile_blocks, 256, 0, s>>>(p);
  rc = cuda_status(cudaGetLastError());
  if (rc != BLASST_OK) return rc;
  blasst::blasst_select_mask_kernel<<<nrow_blocks, 256, 0, s>>>(p);
  return cuda_status(cudaGetLastError());
}

size_t blasst_decode_workspace_bytes(int B, int Hq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || d <= 0 || num_splits <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * Hq * num_splits;
  const size_t o_bytes = rows * d * sizeof(float);
  return o_bytes + rows * sizeof(float);
}

}  // extern "C"

namespace {

// The merge kernel launch. `err` (nullable) is the device error word: when it
// holds an error on entry (a bounded wait of the split kernel before it gave
// up), the kernel writes NaN outputs and -inf lse instead of merging partials
// that may not have been written.
int launch_lse_merge(const float* o_parts, const float* lse_parts, void* o, float* lse,
                     int n_rows, int d, int num_splits, int out_dtype, const int* err,
                     cudaStream_t s) {
  const int threads = d >= 128 ? 128 : ((d + 31) / 32) * 32;
  if (out_dtype == BLASST_BF16) {
    blasst::blasst_lse_merge_kernel<__nv_bfloat16><<<n_rows, threads, 0, s>>>(
        o_parts, lse_parts, static_cast<__nv_bfloat16*>(o), lse, d, num_splits, err);
  } else if (out_dtype == BLASST_FP32) {
    blasst::blasst_lse_merge_kernel<float><<<n_rows, threads, 0, s>>>(
        o_parts, lse_parts, static_cast<float*>(o), lse, d, num_splits, err);
  } else {
    return BLASST_EINVAL;
  }
  return cuda_status(cudaGetLastError());
}

// Argument checks of blasst_decode that need no workspace (shared with the
// allocation-free entry point, which checks them before the size of its
// fixed array).
int decode_args_status(const void* q, const void* k_cache, const void* v_cache, const void* o,
                       const float* lse, int B, int Hq, int Hkv, int Lkv, int d, float lambda,
                       int Bc, int num_splits) {
  if (!q || !k_cache || !v_cache || !o || !lse) return BLASST_EINVAL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(lse))
    return BLASST_EINVAL;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lkv <= 0 || num_splits <= 0) return BLASST_EINVAL;
  if (Hq % Hkv != 0) return BLASST_EINVAL;
  if (!(lambda >= 0.0f && lambda < 1.0f)) return BLASST_EINVAL;
  if (d != 64 && d != 128) return BLASST_EUNSUPPORTED;
  if (Bc != 64 && Bc != 128) return BLASST_EUNSUPPORTED;
  const int g = Hq / Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return BLASST_EUNSUPPORTED;
  if (num_splits > 65535 || B > 65535 || Hkv > 65535) return BLASST_EINVAL;
  return BLASST_OK;
}

}  // namespace

extern "C" {

int blasst_lse_merge(const float* o_parts, const float* lse_parts, void* o, float* lse, int n_rows,
                     int d, int num_splits, int out_dtype, void* stream) {
  if (!o_parts || !lse_parts || !o || !lse || n_rows <= 0 || d <= 0 || num_splits <= 0)
    return BLASST_EINVAL;
  return launch_lse_merge(o_parts, lse_parts, o, lse, n_rows, d, num_splits, out_dtype, nullptr,
                          static_cast<cudaStream_t>(stream));
}

int blasst_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                  int B, int Hq, int Hkv, int Lkv, int d, float lambda, int Bc, int num_splits,
                  void* workspace, size_t workspace_bytes, uint8_t* skip_mask_out,
                  blasst_stats* stats_out, void* stream) {
  const int arc = decode_args_status(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d, lambda, Bc,
                                     num_splits);
  if (arc != BLASST_OK) return arc;
  const int g = Hq / Hkv;
  const size_t need = blasst_decode_workspace_bytes(B, Hq, d, num_splits);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return BLASST_EWORKSPACE;

  int* err = error_word();
  if (!err) return BLASST_ECUDA;

  const size_t rows = static_cast<size_t>(B) * Hq * num_splits;
  blasst::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o_parts = static_cast<float*>(workspace);
  p.lse_parts = static_cast<float*>(workspace) + rows * d;
  p.mask = skip_mask_out;
  p.stats = stats_out;
  p.err = err;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lkv = Lkv;
  p.S = num_splits;
  {
    const long long per = (static_cast<long long>(Lkv) + num_splits - 1) / num_splits;
    p.Ls = static_cast<int>(((per + Bc - 1) / Bc) * Bc);
  }
  p.nKt = (Lkv + Bc - 1) / Bc;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  p.log2_lambda = log2_lambda_of(lambda);
  p.timeout_ns = kTimeoutNs;

  CUtensorMap mk, mv;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&mk, k_cache, dt, 2, d, Lkv, B * Hkv, Bc) ||
      !make_map(&mv, v_cache, dt, 2, d, Lkv, B * Hkv, Bc))
    return BLASST_ECUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = dispatch_decode(d, Bc, g, mk, mv, p, s);
  if (rc != BLASST_OK) return rc;
  return launch_lse_merge(p.o_parts, p.lse_parts, o, lse, B * Hq, d, num_splits, BLASST_BF16, err,
                          s);
}

size_t blasst_decode_mla_workspace_bytes(int B, int H, int num_splits) {
  if (B <= 0 || H <= 0 || num_splits <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * H * num_splits;
  return rows * (blasst::MlaCfg::DV + 1) * sizeof(float);
}

int blasst_decode_mla_splits(int B, int H, int L, int num_sms) {
  using C = blasst::MlaCfg;
  using T = blasst::mla::TcCfg;
  if (B <= 0 || H <= 0 || L <= 0 || H % C::HG != 0) return BLASST_EINVAL;
  if (num_sms <= 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        num_sms <= 0)
      return BLASST_ECUDA;
  }
  const long long per_split =
      H % T::HM == 0 ? 2ll * B * (H / T::HM) : static_cast<long long>(B) * (H / C::HG);
  const long long nb = (static_cast<long long>(L) + C::BC - 1) / C::BC;
  const int s_max = static_cast<int>(nb < 1024 ? nb : 1024);
  auto cost = [&](int S) {
    const long long per = (static_cast<long long>(L) + S - 1) / S;
    const long long blocks = (per + C::BC - 1) / C::BC;
    const long long waves = (per_split * S + num_sms - 1) / num_sms;
    return waves * blocks;
  };
  long long best = cost(1);
  for (int S = 2; S <= s_max; ++S) best = std::min(best, cost(S));
  for (int S = 1; S <= s_max; ++S)
    if (static_cast<double>(cost(S)) <= 1.03 * static_cast<double>(best)) return S;
  return 1;
}

int blasst_decode_mla(const void* q, const void* cache, void* o, float* lse, int B, int H, int L,
                      float lambda, int Bc, int num_splits, float scale, void* workspace,
                      size_t workspace_bytes, uint8_t* skip_mask_out, blasst_stats* stats_out,
                      void* stream) {
  using C = blasst::MlaCfg;
  using T = blasst::mla::TcCfg;
  if (!q || !cache || !o || !lse) return BLASST_EINVAL;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(o) || !aligned16(lse)) return BLASST_EINVAL;
  if (B <= 0 || H <= 0 || L <= 0 || num_splits <= 0) return BLASST_EINVAL;
  if (!(lambda >= 0.0f && lambda < 1.0f)) return BLASST_EINVAL;
  static_assert(T::BC == C::BC, "both MLA kernels decide per 64-key block");
  if (Bc != C::BC) return BLASST_EUNSUPPORTED;
  if (H % C::HG != 0) return BLASST_EUNSUPPORTED;
  const bool tc = H % T::HM == 0;  // tcgen05 kernel for groups of 128 heads, else mma.sync
  if (num_splits > 65535 || B > 65535 || static_cast<long long>(B) * num_splits * (H / C::HG) >
                                            0x7fffffffll)
    return BLASST_EINVAL;
  const size_t need = blasst_decode_mla_workspace_bytes(B, H, num_splits);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return BLASST_EWORKSPACE;
  int* err = error_word();
  if (!err) return BLASST_ECUDA;
  const size_t rows = static_cast<size_t>(B) * H * num_splits;
  blasst::MlaParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o_parts = static_cast<float*>(workspace);
  p.lse_parts = static_cast<float*>(workspace) + rows * C::DV;
  p.mask = skip_mask_out;
  p.stats = stats_out;
  p.err = err;
  p.B = B;
  p.H = H;
  p.L = L;
  p.S = num_splits;
  {
    const long long per = (static_cast<long long>(L) + num_splits - 1) / num_splits;
    p.Ls = static_cast<int>(((per + Bc - 1) / Bc) * Bc);
  }
  p.nKt = (L + Bc - 1) / Bc;
  const double sc = scale > 0.0f ? static_cast<double>(scale)
                                 : 1.0 / std::sqrt(static_cast<double>(C::DQK));
  p.scale_log2 = static_cast<float>(sc * 1.4426950408889634);
  p.log2_lambda = log2_lambda_of(lambda);
  p.timeout_ns = kTimeoutNs;
  CUtensorMap mq, mc;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&mq, q, dt, 2, C::DQK, H, B, tc ? T::HM : C::HG) ||
      !make_map(&mc, cache, dt, 2, C::DQK, L, B, Bc))
    return BLASST_ECUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tc) {
    if (set_smem(blasst::blasst_decode_mla_tc_kernel, T::SMEM_BYTES) != cudaSuccess) return BLASST_ECUDA;
    const unsigned grid =
        static_cast<unsigned>(static_cast<long long>(B) * num_splits * (H / T::HM) * 2);
    blasst::blasst_decode_mla_tc_kernel<<<grid, T::NTHREADS, T::SMEM_BYTES, s>>>(mq, mc, p);
  } else {
    if (set_smem(blasst::blasst_decode_mla_kernel, C::SMEM_BYTES) != cudaSuccess) return BLASST_ECUDA;
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(B) * num_splits * (H / C::HG));
    blasst::blasst_decode_mla_kernel<<<grid, C::NTHREADS, C::SMEM_BYTES, s>>>(mq, mc, p);
  }
  int rc = cuda_status(cudaGetLastError());
  if (rc != BLASST_OK) return rc;
  return launch_lse_merge(p.o_parts, p.lse_parts, o, lse, B * H, C::DV, num_splits, BLASST_BF16,
                          err, s);
}

int blasst_selftest_exp2(const float* x, float* y_mufu, float* y_poly, int n, void* stream) {
  if (!x || !y_mufu || !y_poly || n <= 0) return BLASST_EINVAL;
  selftest_exp2_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_mufu,
                                                                                     y_poly, n);
  return cuda_status(cudaGetLastError());
}

int blasst_selftest_timeout(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return BLASST_EINVAL;
  int* err = error_word();
  if (!err) return BLASST_ECUDA;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
  return cuda_status(cudaGetLastError());
}

int blasst_check(void* stream) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BLASST_ECUDA;
  int* err = error_word();
  if (!err) return BLASST_ECUDA;
  int host = 0;
  if (cudaMemcpy(&host, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return BLASST_ECUDA;
  if (host != 0) {
    const int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return BLASST_ECUDA;
  }
  return host;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode.
//
// Some callers cannot allocate device memory at the point where they run
// decode: a plugin inside a framework that owns every device allocation
// through its own pool, a serving loop that has planned its memory once at
// start-up and must not touch the allocator afterwards, or a host thread for
// which cudaMalloc would be too costly or would synchronise the device. For
// them blasst_decode_noalloc keeps the split partials in the fixed array
// below, which every GPU that loads this library holds (32 MiB) until the
// process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

// Split partials of blasst_decode_noalloc. Host code must not use the
// symbol's host-side shadow as a device address: the device address comes
// from cudaGetSymbolAddress, looked up once per device below.
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device, looked up (and
// cached) on the first call made with that device current.
void* decode_scratch() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t blasst_decode_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

int blasst_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                          float* lse, int B, int Hq, int Hkv, int Lkv, int d, float lambda, int Bc,
                          int num_splits, uint8_t* skip_mask_out, blasst_stats* stats_out,
                          void* stream) {
  // The shape and pointer checks of blasst_decode come first, so an
  // unsupported shape is reported as such rather than as a size problem.
  const int arc = decode_args_status(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d, lambda, Bc,
                                     num_splits);
  if (arc != BLASST_OK) return arc;
  const size_t need = blasst_decode_workspace_bytes(B, Hq, d, num_splits);
  if (need == 0 || need > kNoAllocScratchBytes) return BLASST_EWORKSPACE;
  void* scratch = decode_scratch();
  if (!scratch) return BLASST_ECUDA;
  // Every partial the merge reads is written by the split kernel of the same
  // call (empty splits included), so nothing in the array needs clearing. If
  // a bounded wait of that kernel gives up, the merge sees the device error
  // word and writes NaN / -inf instead of reading partials it did not write.
  return blasst_decode(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d, lambda, Bc, num_splits,
                       scratch, kNoAllocScratchBytes, skip_mask_out, stats_out, stream);
}

}  // extern "C"
