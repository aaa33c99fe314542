// C ABI of libfa (declared in include/fa.h): host-side argument checks,
// TMA tensor-map encoding and kernel launches. Everything runs in the
// caller's stream; nothing here allocates device memory.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fa.h"
#include "bwd_kernels.cuh"
#include "fwd_kernel.cuh"

namespace fa {

__device__ int g_selftest_zero = 0;  // never written: the flag nothing sets

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, N, H, d] 16-bit tensor viewed as 4-D (d, H, N, B), read in boxes of
// 64 elements x 1 head x 128 rows with 128-byte swizzle. Rows past N (and
// boxes past d) read as zeros.
bool make_bnhd_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int N, int H, int d, float scale, fa_dtype dtype) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  const int64_t elems = (int64_t)B * N * H * d;
  if (elems >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

template <typename Kernel>
cudaError_t set_smem(Kernel k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, bool CAUSAL, bool BF16>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdArgs& a,
                       cudaStream_t stream) {
  using C = FwdCfg<D>;
  const unsigned units = static_cast<unsigned>(a.n_mblocks * a.B * a.H);
  if constexpr (!CAUSAL) {
    if (a.split == 2) {
      // Two CTAs per row block, launched as 2-CTA clusters so they are
      // resident together and can merge through distributed shared memory.
      auto kern2 = fa_fwd_kernel<D, false, BF16, true>;
      cudaError_t e = set_smem(kern2, C::kSmemBytes);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * units);
      cfg.blockDim = dim3(C::kThreads);
      cfg.dynamicSmemBytes = C::kSmemBytes;
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, kern2, mq, mk, mv, a) == cudaSuccess) return cudaSuccess;
      (void)cudaGetLastError();  // no cluster fits: run unsplit
    }
  }
  auto kern = fa_fwd_kernel<D, CAUSAL, BF16, false>;
  cudaError_t e = set_smem(kern, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  FwdArgs one = a;
  one.split = 1;
  kern<<<dim3(units), C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, one);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_fwd(bool causal, bool bf16, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const FwdArgs& a, cudaStream_t s) {
  if (causal) return bf16 ? launch_fwd<D, true, true>(mq, mk, mv, a, s) : launch_fwd<D, true, false>(mq, mk, mv, a, s);
  return bf16 ? launch_fwd<D, false, true>(mq, mk, mv, a, s) : launch_fwd<D, false, false>(mq, mk, mv, a, s);
}

// Failure-detection self-test: one warp waits, with a short limit, for an
// mbarrier phase that nothing completes (which == 1) or for a global counter
// that nothing advances (which == 2), exactly as the real kernels wait. The
// wait gives up, records FA_ERR_DEVICE_TIMEOUT and the kernel returns.
__global__ void fa_selftest_kernel(int which, unsigned long long limit_ns, const int* never) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (which == 1) {
    mbar_wait(&bar, 0, &abort_flag, true, limit_ns);
  } else {
    const uint64_t t0 = globaltimer();
    while (*reinterpret_cast<const volatile int*>(never) != 1) {
      if (globaltimer() - t0 > limit_ns) {
        record_timeout(2);
        break;
      }
      __nanosleep(1000);
    }
  }
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Forward work split. A row block's key tiles go to one CTA, or are halved
// between the two CTAs of a cluster when that makes the whole launch shorter.
// With W CTAs resident at a time, U row blocks of n key tiles take about
// ceil(U / W) * (n + F) tile-times unsplit and ceil(2U / W) * (ceil(n / 2) + F)
// + 1 split, where F is a CTA's fixed cost (start, first loads, epilogue) in
// tile-times and the + 1 is the merge. F = 8 matches a B200 at d = 64: there,
// 2 x 2048 x 12 heads split (384 CTAs in 3 waves instead of 192 in 2) ran 8%
// slower. So only launches that leave SMs idle unsplit gain. Causal launches
// keep one CTA per row block (their longest-first order already fills the
// machine). FA_FWD_SPLIT=1 or 2 in the environment forces the choice (2 only
// where a split is possible).
int fwd_split(int B, int N, int H, bool causal, int n_mblocks) {
  const int n_kv = (N + 127) / 128;
  if (causal || n_kv < 2) return 1;
  if (const char* env = std::getenv("FA_FWD_SPLIT")) {
    if (env[0] == '1') return 1;
    if (env[0] == '2') return 2;
  }
  constexpr long long kFixed = 8;
  const long long w = num_sms() > 0 ? num_sms() : 148;
  const long long units = static_cast<long long>(B) * H * n_mblocks;
  const long long t1 = (units + w - 1) / w * (n_kv + kFixed);
  const long long t2 = (2 * units + w - 1) / w * ((n_kv + 1) / 2 + kFixed) + 1;
  return t2 < t1 ? 2 : 1;
}

template <int D>
cudaError_t dispatch_bwd(bool causal, bool bf16, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, const BwdArgs& a, int sms,
                         cudaStream_t s) {
  if (causal)
    return bf16 ? launch_bwd_t<D, true, true>(mq, mk, mv, mdo, a, sms, s)
                : launch_bwd_t<D, true, false>(mq, mk, mv, mdo, a, sms, s);
  return bf16 ? launch_bwd_t<D, false, true>(mq, mk, mv, mdo, a, sms, s)
              : launch_bwd_t<D, false, false>(mq, mk, mv, mdo, a, sms, s);
}

cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, uint8_t* ws, const BwdLayout& L, int B,
                       int N, int H, int d, float scale, bool causal, bool bf16, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mdo;
  if (!make_bnhd_map(&mq, q, B, N, H, d) || !make_bnhd_map(&mk, k, B, N, H, d) ||
      !make_bnhd_map(&mv, v, B, N, H, d) || !make_bnhd_map(&mdo, dout, B, N, H, d))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  if (sms <= 0) return cudaErrorInvalidDevice;
  BwdArgs a;
  a.o = static_cast<const uint16_t*>(o);
  a.dout = static_cast<const uint16_t*>(dout);
  a.lse = lse;
  a.dq = static_cast<uint16_t*>(dq);
  a.dk = static_cast<uint16_t*>(dk);
  a.dv = static_cast<uint16_t*>(dv);
  a.lse2 = reinterpret_cast<float*>(ws + L.off_lse2);
  a.dd = reinterpret_cast<float*>(ws + L.off_dd);
  a.dqacc = reinterpret_cast<float*>(ws + L.off_dqacc);
  a.cnt = reinterpret_cast<int*>(ws + L.off_cnt);
  a.sched = reinterpret_cast<int*>(ws + L.off_sched);
  a.B = B;
  a.N = N;
  a.H = H;
  a.npad = L.npad;
  a.ntiles = L.ntiles;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  return d == 64 ? dispatch_bwd<64>(causal, bf16, mq, mk, mv, mdo, a, sms, s)
                 : dispatch_bwd<128>(causal, bf16, mq, mk, mv, mdo, a, sms, s);
}

// ---------------------------------------------------------------------------
// Built-in scratch for fa_bwd_noalloc.
//
// A file-scope device array: every GPU that loads this library holds it until
// the process exits. In host code `g_bwd_scratch` is only a host-side stand-in
// for the symbol, never a device address; the device address is looked up
// with cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_bwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_bwd_scratch on the current device (set up on the first
// call for that device). Returns nullptr and sets *err on failure.
uint8_t* noalloc_scratch(cudaError_t* err) {
  static std::mutex mu;
  static uint8_t* addr[kMaxDevices] = {};
  int dev = -1;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  return addr[dev];
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  fa_status st = check_common(B, N, H, d, softmax_scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  CUtensorMap mq, mk, mv;
  if (!make_bnhd_map(&mq, q, B, N, H, d) || !make_bnhd_map(&mk, k, B, N, H, d) || !make_bnhd_map(&mv, v, B, N, H, d))
    return FA_ERR_CUDA;
  FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.N = N;
  a.H = H;
  a.n_mblocks = (N + 255) / 256;
  a.split = fwd_split(B, N, H, causal != 0, a.n_mblocks);
  a.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
  const bool bf16 = dtype == FA_BF16;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = d == 64 ? dispatch_fwd<64>(causal, bf16, mq, mk, mv, a, s) : dispatch_fwd<128>(causal, bf16, mq, mk, mv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int N, int H, int d, int causal) {
  (void)causal;
  if (B < 1 || N < 1 || H < 1 || (d != 64 && d != 128)) return 0;
  return BwdLayout::make(B, N, H, d).total_bytes;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  fa_status st = check_common(B, N, H, d, softmax_scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  const BwdLayout L = BwdLayout::make(B, N, H, d);
  if (!aligned16(workspace) || workspace_bytes < L.total_bytes) return FA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, static_cast<uint8_t*>(workspace), L, B, N, H, d,
                             softmax_scale, causal != 0, dtype == FA_BF16, s);
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                         float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  fa_status st = check_common(B, N, H, d, softmax_scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  const BwdLayout L = BwdLayout::make(B, N, H, d);
  if (L.total_bytes > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;  // shape needs more than the built-in scratch
  cudaError_t e = cudaSuccess;
  uint8_t* scratch = noalloc_scratch(&e);
  if (scratch == nullptr) return FA_ERR_CUDA;
  // The preprocessing launch rewrites D and LSE*log2(e), zeroes the ordering
  // counters and the work counter; the first key tile stores (not adds) each
  // dQ tile. Nothing left in the scratch by an earlier call is read.
  e = launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, scratch, L, B, N, H, d, softmax_scale, causal != 0,
                 dtype == FA_BF16, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_check_device_status(fa_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  int host = 0;
  if (cudaMemcpyFromSymbol(&host, g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return host == 0 ? FA_OK : static_cast<fa_status>(host);
}

fa_status fa_selftest_bounded_wait(int which, int limit_ms, fa_stream_t stream) {
  if ((which != 1 && which != 2) || limit_ms < 1 || limit_ms > 1000) return FA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The counter that never advances is a zero-initialised device symbol of
  // this library that nothing writes.
  int* never = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&never), g_selftest_zero) != cudaSuccess) return FA_ERR_CUDA;
  fa_selftest_kernel<<<1, 32, 0, s>>>(which, (unsigned long long)limit_ms * 1000000ull, never);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
  }
  return "FA_ERR_UNKNOWN";
}

}  // extern "C"
