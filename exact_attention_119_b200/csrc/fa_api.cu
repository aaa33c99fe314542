// C ABI of libfa (declared in include/fa.h): host-side argument checks,
// TMA tensor-map encoding and kernel launches. Everything runs in the
// caller's stream; nothing here allocates device memory.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fa.h"
#include "bwd_kernels.cuh"
#include "decode_kernels.cuh"
#include "fwd_kernel.cuh"

namespace fa {

__device__ int g_selftest_zero = 0;  // never written: the flag nothing sets

namespace {

// What the last failing call of this host thread ran into (fa_last_error_detail).
thread_local char t_detail[256] = "";

void clear_detail() { t_detail[0] = '\0'; }

void set_detail_cuda(const char* step, cudaError_t e) {
  std::snprintf(t_detail, sizeof(t_detail), "%s: %s (%d)", step, cudaGetErrorName(e), static_cast<int>(e));
}

void set_detail_text(const char* text) { std::snprintf(t_detail, sizeof(t_detail), "%s", text); }

// Events the next launches of fa_bwd_dkdv in this thread are bracketed with
// (fa_profile_bwd_events); null = none.
thread_local cudaEvent_t t_prof_begin = nullptr;
thread_local cudaEvent_t t_prof_end = nullptr;

// One kernel launch whose own return code decides success. (A launch with
// <<<...>>> has no return code, and cudaGetLastError would also report an
// error that some earlier, unrelated runtime call left pending in this host
// thread.) `cluster` > 1 launches clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch(const char* name, void (*kern)(KArgs...), dim3 grid, unsigned block, size_t smem,
                   cudaStream_t stream, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (cluster > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) set_detail_cuda(name, e);
  return e;
}

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

// ------------------------------------------------------------------ problem

// Element strides of a [B, N, H, d] view (head size contiguous).
struct Strides {
  long long sb, sn, sh;
};

// One attention call, checked and normalised: dense defaults filled in, the
// kernel's head-size tile D chosen.
struct Problem {
  int B, N, H, d, D;
  bool causal, bf16;
  float scale;
  const int* cu;  // variable length: row offsets [B + 1] (device), else nullptr
  int total;      // variable length: rows of the packed tensors
  Strides q, k, v, o, dout, dq, dk, dv;
  long long lse_sb, lse_sh;
  bool dropout;
  Dropout drop;
  int rows() const { return cu ? total : N; }
};

fa_status bad_arg(const char* what) {
  set_detail_text(what);
  return FA_ERR_INVALID_ARG;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Dense strides of the caller's tensors when all three are zero; otherwise
// check them: positive (the batch stride may be 0 when it is never used),
// multiples of 8 elements (16 bytes, for TMA and vector stores), < 2^36.
fa_status fill_strides(Strides* st, const char* name, const Problem& p) {
  if (st->sb == 0 && st->sn == 0 && st->sh == 0) {
    st->sh = p.d;
    st->sn = (long long)p.H * p.d;
    st->sb = p.cu ? 0 : (long long)p.N * p.H * p.d;
    return FA_OK;
  }
  const bool batch_used = p.cu == nullptr && p.B > 1;
  const long long lim = 1LL << 36;
  auto ok = [&](long long x, bool used) { return used ? (x > 0 && x < lim && x % 8 == 0) : (x >= 0 && x < lim); };
  if (!ok(st->sn, true) || !ok(st->sh, true) || !ok(st->sb, batch_used) || st->sb % 8 != 0) {
    std::snprintf(t_detail, sizeof(t_detail),
                  "%s strides (batch %lld, row %lld, head %lld): each must be a positive multiple of 8 elements "
                  "below 2^36 (the batch stride may be 0 only when unused)",
                  name, st->sb, st->sn, st->sh);
    return FA_ERR_INVALID_ARG;
  }
  return FA_OK;
}

fa_status make_problem(const fa_desc* desc, Problem* p, bool backward) {
  if (desc == nullptr) return bad_arg("desc is NULL");
  p->B = desc->B;
  p->N = desc->N;
  p->H = desc->H;
  p->d = desc->d;
  p->scale = desc->softmax_scale;
  p->cu = desc->cu_seqlens;
  p->total = desc->total;
  if (p->B < 1 || p->N < 1 || p->H < 1 || p->d < 1) return bad_arg("B, N, H and d must be >= 1");
  if (!(std::isfinite(p->scale) && p->scale > 0.f)) return bad_arg("softmax_scale must be finite and > 0");
  if (desc->dtype != FA_FP16 && desc->dtype != FA_BF16) return bad_arg("dtype must be FA_FP16 or FA_BF16");
  if (desc->causal != 0 && desc->causal != 1) return bad_arg("causal must be 0 or 1");
  if (p->d > 128 || p->d % 8 != 0) {
    set_detail_text("head_dim d must be a multiple of 8 between 8 and 128");
    return FA_ERR_UNSUPPORTED;
  }
  if (p->cu != nullptr) {
    if (reinterpret_cast<uintptr_t>(p->cu) & 3u) return bad_arg("cu_seqlens must be 4-byte aligned");
    if (p->total < 1) return bad_arg("total (rows of the packed tensors) must be >= 1 with cu_seqlens");
  }
  if ((long long)p->B * p->H > 65535) {
    set_detail_text("B * H must be at most 65535");
    return FA_ERR_UNSUPPORTED;
  }
  const long long rows = p->cu ? (long long)p->total : (long long)p->B * p->N;
  if (rows * p->H * p->d >= (1LL << 31)) {
    set_detail_text("the number of elements of a tensor must be < 2^31");
    return FA_ERR_UNSUPPORTED;
  }
  p->D = p->d <= 64 ? 64 : 128;
  p->causal = desc->causal != 0;
  p->bf16 = desc->dtype == FA_BF16;
  p->q = {desc->stride_q.batch, desc->stride_q.row, desc->stride_q.head};
  p->k = {desc->stride_k.batch, desc->stride_k.row, desc->stride_k.head};
  p->v = {desc->stride_v.batch, desc->stride_v.row, desc->stride_v.head};
  p->o = {desc->stride_o.batch, desc->stride_o.row, desc->stride_o.head};
  p->dout = {desc->stride_do.batch, desc->stride_do.row, desc->stride_do.head};
  p->dq = {desc->stride_dq.batch, desc->stride_dq.row, desc->stride_dq.head};
  p->dk = {desc->stride_dk.batch, desc->stride_dk.row, desc->stride_dk.head};
  p->dv = {desc->stride_dv.batch, desc->stride_dv.row, desc->stride_dv.head};
  fa_status st;
  if ((st = fill_strides(&p->q, "q", *p)) != FA_OK || (st = fill_strides(&p->k, "k", *p)) != FA_OK ||
      (st = fill_strides(&p->v, "v", *p)) != FA_OK || (st = fill_strides(&p->o, "o", *p)) != FA_OK)
    return st;
  if (backward && ((st = fill_strides(&p->dout, "dout", *p)) != FA_OK ||
                   (st = fill_strides(&p->dq, "dq", *p)) != FA_OK || (st = fill_strides(&p->dk, "dk", *p)) != FA_OK ||
                   (st = fill_strides(&p->dv, "dv", *p)) != FA_OK))
    return st;
  if (!(desc->dropout_p >= 0.f && desc->dropout_p < 1.f)) return bad_arg("dropout_p must be in [0, 1)");
  p->dropout = desc->dropout_p > 0.f;
  p->drop.thr = static_cast<uint32_t>(std::min(static_cast<double>(desc->dropout_p) * 4294967296.0, 4294967295.0));
  p->drop.seed_lo = static_cast<uint32_t>(desc->seed & 0xFFFFFFFFull);
  p->drop.seed_hi = static_cast<uint32_t>(desc->seed >> 32);
  p->drop.offset = desc->offset;
  p->drop.rkeep = static_cast<float>(1.0 / (1.0 - static_cast<double>(desc->dropout_p)));
  // LSE: [B, H, N] fp32, or [H, total] when variable-length.
  p->lse_sb = p->cu ? 0 : (long long)p->H * p->N;
  p->lse_sh = p->cu ? p->total : p->N;
  return FA_OK;
}

// TMA view of one input tensor: dims (d, H, rows, B), or (d, rows, H, B) when
// its head stride exceeds its row stride (head-major storage), read in boxes
// of 64 head-size columns x 128 rows with 128-byte swizzle. Rows past the end
// (and columns past d) read as zeros.
fa_status make_map_rows(CUtensorMap* map, bool* head_major, const void* ptr, const Strides& st, int d, int H,
                        int rows_i, int nb_i, int box_rows, const char* name);

fa_status make_map(CUtensorMap* map, bool* head_major, const void* ptr, const Strides& st, const Problem& p,
                   const char* name) {
  return make_map_rows(map, head_major, ptr, st, p.d, p.H, p.rows(), p.cu ? 1 : p.B, 128, name);
}

// The same view for any row count and box height.
fa_status make_map_rows(CUtensorMap* map, bool* head_major, const void* ptr, const Strides& st, int d, int H,
                        int rows_i, int nb_i, int box_rows, const char* name) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    set_detail_text("cuTensorMapEncodeTiled: driver entry point not found");
    return FA_ERR_CUDA;
  }
  const bool hm = st.sh > st.sn;
  const cuuint64_t rows = static_cast<cuuint64_t>(rows_i);
  const cuuint64_t nb = static_cast<cuuint64_t>(nb_i);
  // A batch dimension of one is never stepped; give it a valid stride.
  const long long sb = nb > 1 ? st.sb : std::max(st.sn, st.sh) * static_cast<long long>(std::max(rows, (cuuint64_t)H));
  const cuuint64_t dims[4] = {(cuuint64_t)d, hm ? rows : (cuuint64_t)H, hm ? (cuuint64_t)H : rows, nb};
  const cuuint64_t strides[3] = {(cuuint64_t)(hm ? st.sn : st.sh) * 2, (cuuint64_t)(hm ? st.sh : st.sn) * 2,
                                 (cuuint64_t)sb * 2};
  const cuuint32_t br = static_cast<cuuint32_t>(box_rows);
  const cuuint32_t box[4] = {64, hm ? br : 1u, hm ? 1u : br, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled rejected the view of %s: CUresult %d", name,
                  static_cast<int>(r));
    return FA_ERR_INVALID_ARG;
  }
  *head_major = hm;
  return FA_OK;
}

// Make the current device's primary context current in this host thread.
// A thread that has made no CUDA runtime call needing a context yet (e.g. the
// autograd engine's backward worker, whose tensors came from the allocator's
// cache) has none, and cuTensorMapEncodeTiled, a driver call, then fails with
// CUDA_ERROR_INVALID_CONTEXT. cudaSetDevice on the current device binds it.
fa_status bind_context() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaSetDevice(dev);
  if (e != cudaSuccess) {
    set_detail_cuda("binding the current device's context", e);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

template <typename Kernel>
cudaError_t set_smem(Kernel k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
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
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaDeviceGetAttribute(MultiProcessorCount)", e);
    return 0;
  }
  return n;
}

// ------------------------------------------------------------------ forward

template <int D, bool CAUSAL, bool BF16, bool VARLEN, bool DROPOUT>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                       const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D>;
  const unsigned units = static_cast<unsigned>(a.n_mblocks * a.B * a.H);
  if constexpr (!CAUSAL && !VARLEN && !DROPOUT) {
    if (a.split == 2) {
      // Two CTAs per row block, launched as 2-CTA clusters so they are
      // resident together and can merge through distributed shared memory.
      auto kern2 = fa_fwd_kernel<D, false, BF16, true, false, false>;
      cudaError_t e = set_smem(kern2, C::kSmemBytes);
      if (e != cudaSuccess) {
        set_detail_cuda("cudaFuncSetAttribute(fa_fwd_kernel split)", e);
        return e;
      }
      if (launch("fa_fwd_kernel split", kern2, 2 * units, C::kThreads, C::kSmemBytes, stream, 2, mq, mk, mv, mo, a) ==
          cudaSuccess)
        return cudaSuccess;
      // No 2-CTA cluster fits: run unsplit. The failed launch's error is this
      // call's own, the most recent in this thread; clear it.
      (void)cudaGetLastError();
      clear_detail();
    }
  }
  auto kern = fa_fwd_kernel<D, CAUSAL, BF16, false, VARLEN, DROPOUT>;
  cudaError_t e = set_smem(kern, C::kSmemBytes);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaFuncSetAttribute(fa_fwd_kernel)", e);
    return e;
  }
  FwdArgs one = a;
  one.split = 1;
  // d = 128: persistent, one CTA per SM (or fewer), each walking its items.
  // d = 64: one CTA per item (the same kernel walks a single item); measured
  // on a B200 the persistent launch was 7% slower there (B2 N2048 H12) and
  // 1-3% faster at d = 128.
  const int sms = num_sms();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = D == 128 ? std::min(units, static_cast<unsigned>(sms)) : units;
  return launch("fa_fwd_kernel", kern, grid, C::kThreads, C::kSmemBytes, stream, 1, mq, mk, mv, mo, one);
}

template <int D, bool VARLEN, bool DROPOUT>
cudaError_t dispatch_fwd(bool causal, bool bf16, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mo, const FwdArgs& a, cudaStream_t s) {
  if (causal)
    return bf16 ? launch_fwd<D, true, true, VARLEN, DROPOUT>(mq, mk, mv, mo, a, s)
                : launch_fwd<D, true, false, VARLEN, DROPOUT>(mq, mk, mv, mo, a, s);
  return bf16 ? launch_fwd<D, false, true, VARLEN, DROPOUT>(mq, mk, mv, mo, a, s)
              : launch_fwd<D, false, false, VARLEN, DROPOUT>(mq, mk, mv, mo, a, s);
}

template <int D>
cudaError_t dispatch_fwd_all(const Problem& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const CUtensorMap& mo, const FwdArgs& a, cudaStream_t s) {
  if (p.cu)
    return p.dropout ? dispatch_fwd<D, true, true>(p.causal, p.bf16, mq, mk, mv, mo, a, s)
                     : dispatch_fwd<D, true, false>(p.causal, p.bf16, mq, mk, mv, mo, a, s);
  return p.dropout ? dispatch_fwd<D, false, true>(p.causal, p.bf16, mq, mk, mv, mo, a, s)
                   : dispatch_fwd<D, false, false>(p.causal, p.bf16, mq, mk, mv, mo, a, s);
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

fa_status run_fwd(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                  cudaStream_t s) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return bad_arg("a pointer is null or not 16-byte aligned");
  fa_status st = bind_context();
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv, mo;
  bool hq = false, hk = false, hv = false, ho = false;
  if ((st = make_map(&mq, &hq, q, p.q, p, "q")) != FA_OK || (st = make_map(&mk, &hk, k, p.k, p, "k")) != FA_OK ||
      (st = make_map(&mv, &hv, v, p.v, p, "v")) != FA_OK || (st = make_map(&mo, &ho, o, p.o, p, "o")) != FA_OK)
    return st;
  FwdArgs a;
  a.o = static_cast<uint16_t*>(o);
  a.o_sb = p.o.sb;
  a.o_sn = p.o.sn;
  a.o_sh = p.o.sh;
  a.lse = lse;
  a.lse_sb = p.lse_sb;
  a.lse_sh = p.lse_sh;
  a.cu = p.cu;
  a.total = p.total;
  a.B = p.B;
  a.N = p.N;
  a.H = p.H;
  a.d = p.d;
  a.hm = (hq ? kHmQ : 0u) | (hk ? kHmK : 0u) | (hv ? kHmV : 0u) | (ho ? kHmO : 0u);
  a.n_mblocks = (p.N + 255) / 256;
  a.split = (p.cu || p.dropout) ? 1 : fwd_split(p.B, p.N, p.H, p.causal, a.n_mblocks);
  a.drop = p.drop;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  const cudaError_t e =
      p.D == 64 ? dispatch_fwd_all<64>(p, mq, mk, mv, mo, a, s) : dispatch_fwd_all<128>(p, mq, mk, mv, mo, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ----------------------------------------------------------------- backward

// The two backward launches on one stream: preprocessing, and the
// persistent dK/dV kernel (which also sums, scales and casts dQ).
// Tensor maps of the backward: inputs q, k, v, dout and outputs dk, dv.
struct BwdMaps {
  CUtensorMap q, k, v, dout, dk, dv;
};

template <int D, bool CAUSAL, bool BF16, bool DROPOUT>
cudaError_t launch_bwd_t(const BwdMaps& m, const BwdArgs& a, int sms, cudaStream_t s) {
  using C = BwdCfg<D>;
  constexpr int kPrepRows = 256 / (D / 8);
  cudaError_t e = launch("fa_bwd_prep", fa_bwd_prep<D, BF16>,
                         dim3((a.npad + kPrepRows - 1) / kPrepRows, a.B * a.H), 256, 0, s, 1, a);
  if (e != cudaSuccess) return e;
  auto kern = fa_bwd_dkdv<D, CAUSAL, BF16, DROPOUT>;
  e = set_smem(kern, C::kSmem);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaFuncSetAttribute(fa_bwd_dkdv)", e);
    return e;
  }
  const int items = a.B * a.H * a.ntiles;
  const int grid = std::min(items, sms);
  if (t_prof_begin != nullptr && (e = cudaEventRecord(t_prof_begin, s)) != cudaSuccess) {
    set_detail_cuda("cudaEventRecord(profile begin)", e);
    return e;
  }
  e = launch("fa_bwd_dkdv", kern, grid, C::kThreads, C::kSmem, s, 1, m.q, m.k, m.v, m.dout, m.dk, m.dv, a);
  if (e != cudaSuccess) return e;
  if (t_prof_end != nullptr && (e = cudaEventRecord(t_prof_end, s)) != cudaSuccess) {
    set_detail_cuda("cudaEventRecord(profile end)", e);
    return e;
  }
  return cudaSuccess;
}

template <int D, bool DROPOUT>
cudaError_t dispatch_bwd(bool causal, bool bf16, const BwdMaps& m, const BwdArgs& a, int sms, cudaStream_t s) {
  if (causal)
    return bf16 ? launch_bwd_t<D, true, true, DROPOUT>(m, a, sms, s) : launch_bwd_t<D, true, false, DROPOUT>(m, a, sms, s);
  return bf16 ? launch_bwd_t<D, false, true, DROPOUT>(m, a, sms, s) : launch_bwd_t<D, false, false, DROPOUT>(m, a, sms, s);
}

BwdLayout bwd_layout(const Problem& p) { return BwdLayout::make(p.B, p.N, p.H, p.D); }

fa_status check_bwd_pointers(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return bad_arg("a pointer is null or not 16-byte aligned");
  return FA_OK;
}

fa_status run_bwd(const Problem& p, const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, uint8_t* ws, cudaStream_t s) {
  fa_status st = bind_context();
  if (st != FA_OK) return st;
  BwdMaps m;
  bool hq = false, hk = false, hv = false, hd = false, hdk = false, hdv = false;
  if ((st = make_map(&m.q, &hq, q, p.q, p, "q")) != FA_OK || (st = make_map(&m.k, &hk, k, p.k, p, "k")) != FA_OK ||
      (st = make_map(&m.v, &hv, v, p.v, p, "v")) != FA_OK ||
      (st = make_map(&m.dout, &hd, dout, p.dout, p, "dout")) != FA_OK ||
      (st = make_map(&m.dk, &hdk, dk, p.dk, p, "dk")) != FA_OK || (st = make_map(&m.dv, &hdv, dv, p.dv, p, "dv")) != FA_OK)
    return st;
  const int sms = num_sms();
  if (sms <= 0) return FA_ERR_CUDA;
  const BwdLayout L = bwd_layout(p);
  BwdArgs a;
  a.o = static_cast<const uint16_t*>(o);
  a.o_sb = p.o.sb, a.o_sn = p.o.sn, a.o_sh = p.o.sh;
  a.dout = static_cast<const uint16_t*>(dout);
  a.do_sb = p.dout.sb, a.do_sn = p.dout.sn, a.do_sh = p.dout.sh;
  a.lse = lse;
  a.lse_sb = p.lse_sb, a.lse_sh = p.lse_sh;
  a.dq = static_cast<uint16_t*>(dq);
  a.dq_sb = p.dq.sb, a.dq_sn = p.dq.sn, a.dq_sh = p.dq.sh;
  a.dk = static_cast<uint16_t*>(dk);
  a.dk_sb = p.dk.sb, a.dk_sn = p.dk.sn, a.dk_sh = p.dk.sh;
  a.dv = static_cast<uint16_t*>(dv);
  a.dv_sb = p.dv.sb, a.dv_sn = p.dv.sn, a.dv_sh = p.dv.sh;
  a.cu = p.cu;
  a.total = p.total;
  a.lse2 = reinterpret_cast<float*>(ws + L.off_lse2);
  a.dd = reinterpret_cast<float*>(ws + L.off_dd);
  a.dqacc = reinterpret_cast<float*>(ws + L.off_dqacc);
  a.cnt = reinterpret_cast<int*>(ws + L.off_cnt);
  a.sched = reinterpret_cast<int*>(ws + L.off_sched);
  a.B = p.B;
  a.N = p.N;
  a.H = p.H;
  a.d = p.d;
  a.npad = L.npad;
  a.ntiles = L.ntiles;
  // Causal items interleave over groups of heads whose Q, dO and two fp32 dQ
  // sums (12 bytes per row and column) take at most 48 MiB of L2. Measured on
  // a B200: +2.5% (B4 N4096 H8 d128, groups of 8) and +3% (B2 N4096 H16 d64,
  // 16), but 1-9% slower at 128 key tiles per head (N16384 H16, 2), so only
  // launches of at most 32 key tiles per head interleave.
  {
    const long long per_head = 12LL * L.npad * p.D;
    a.hgroup = p.causal && L.ntiles <= 32 ? (int)std::max(1LL, std::min(16LL, (48LL << 20) / per_head)) : 1;
  }
  a.hm = (hq ? kHmQ : 0u) | (hk ? kHmK : 0u) | (hv ? kHmV : 0u) | (hd ? kHmDO : 0u) | (hdk ? kHmDK : 0u) |
         (hdv ? kHmDV : 0u);
  a.scale = p.scale;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.drop = p.drop;
  cudaError_t e;
  if (p.dropout)
    e = p.D == 64 ? dispatch_bwd<64, true>(p.causal, p.bf16, m, a, sms, s)
                  : dispatch_bwd<128, true>(p.causal, p.bf16, m, a, sms, s);
  else
    e = p.D == 64 ? dispatch_bwd<64, false>(p.causal, p.bf16, m, a, sms, s)
                  : dispatch_bwd<128, false>(p.causal, p.bf16, m, a, sms, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ------------------------------------------------------------------- decode

struct DecPlan {
  int D, tiles_per_unit, units;
  size_t off_ml, total_bytes;
};

// Units of the cache's key axis: about eight CTAs per SM over the whole
// launch (two or three waves, with two or three resident per SM), at least
// two 64-key tiles each.
DecPlan dec_plan(int B, int Nq, int H, int d, int Nmax, int sms) {
  DecPlan pl;
  pl.D = d <= 64 ? 64 : 128;
  const long long ntiles = (Nmax + kDecKeys - 1) / kDecKeys;
  const long long target = 8LL * (sms > 0 ? sms : 148);
  long long tpu = (static_cast<long long>(B) * H * ntiles + target - 1) / target;
  tpu = std::max(2LL, std::min(tpu, ntiles));
  pl.tiles_per_unit = static_cast<int>(tpu);
  pl.units = static_cast<int>((ntiles + tpu - 1) / tpu);
  const size_t rows = static_cast<size_t>(B) * H * pl.units * Nq;
  pl.off_ml = (rows * pl.D * 4 + 255) & ~size_t(255);
  pl.total_bytes = pl.off_ml + ((rows * 2 * 4 + 255) & ~size_t(255));
  return pl;
}

fa_status dec_check(int B, int Nq, int H, int d, int Nmax, float scale, int causal, fa_dtype dtype) {
  if (B < 1 || H < 1 || Nq < 1 || Nmax < 1 || d < 1) return bad_arg("B, Nq, H, Nmax and d must be >= 1");
  if (Nq > kDecMaxNq) {
    set_detail_text("decode takes at most 8 query rows per sequence; use fa_fwd_ex for more");
    return FA_ERR_UNSUPPORTED;
  }
  if (!(std::isfinite(scale) && scale > 0.f)) return bad_arg("softmax_scale must be finite and > 0");
  if (dtype != FA_FP16 && dtype != FA_BF16) return bad_arg("dtype must be FA_FP16 or FA_BF16");
  if (causal != 0 && causal != 1) return bad_arg("causal must be 0 or 1");
  if (d > 128 || d % 8 != 0) {
    set_detail_text("head_dim d must be a multiple of 8 between 8 and 128");
    return FA_ERR_UNSUPPORTED;
  }
  if ((long long)B * Nmax * H * d >= (1LL << 31)) {
    set_detail_text("the number of elements of a cache must be < 2^31");
    return FA_ERR_UNSUPPORTED;
  }
  return FA_OK;
}

template <int D, bool BF16, int NQ>
cudaError_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const DecArgs& a, cudaStream_t s) {
  using C = DecCfg<D, NQ>;
  auto kern = fa_decode_split<D, BF16, NQ>;
  cudaError_t e = set_smem(kern, C::kSmem);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaFuncSetAttribute(fa_decode_split)", e);
    return e;
  }
  e = launch("fa_decode_split", kern, static_cast<unsigned>(a.B * a.H * a.units), C::kThreads, C::kSmem, s, 1, mk,
             mv, a);
  if (e != cudaSuccess) return e;
  const unsigned rows = static_cast<unsigned>(a.B * a.H * a.Nq);
  return launch("fa_decode_combine", fa_decode_combine<D, BF16>, (rows + 3) / 4, 128, 0, s, 1, a);
}

template <int NQ>
cudaError_t launch_decode_nq(int D, bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const DecArgs& a,
                             cudaStream_t s) {
  if (D == 64) return bf16 ? launch_decode<64, true, NQ>(mk, mv, a, s) : launch_decode<64, false, NQ>(mk, mv, a, s);
  return bf16 ? launch_decode<128, true, NQ>(mk, mv, a, s) : launch_decode<128, false, NQ>(mk, mv, a, s);
}

// ---------------------------------------------------------------------------
// Built-in scratch for fa_bwd_noalloc.
//
// A file-scope device array: every GPU that loads this library holds it until
// the process exits. In host code `g_bwd_scratch` is only a host-side stand-in
// for the symbol, never a device address; the device address comes from
// cudaGetSymbolAddress with the device current.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_bwd_scratch[kNoAllocScratchBytes];

// Device address of g_bwd_scratch in the current device's context, looked
// up on every call: the lookup allocates nothing and is cheap, and a cached
// address would go stale if the caller tore the context down and made a new
// one (cudaDeviceReset). The first lookup on a device also loads this
// library's device code there. Returns nullptr and sets *err on failure.
uint8_t* noalloc_scratch(cudaError_t* err) {
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_bwd_scratch);
  if (*err != cudaSuccess) {
    set_detail_cuda("cudaGetSymbolAddress(built-in scratch)", *err);
    return nullptr;
  }
  return static_cast<uint8_t*>(p);
}

// The plain [B, N, H, d] call as a descriptor (dense strides).
fa_desc dense_desc(int B, int N, int H, int d, float scale, int causal, fa_dtype dtype) {
  fa_desc x;
  std::memset(&x, 0, sizeof(x));
  x.B = B;
  x.N = N;
  x.H = H;
  x.d = d;
  x.softmax_scale = scale;
  x.causal = causal;
  x.dtype = dtype;
  return x;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

fa_status fa_fwd_ex(const fa_desc* desc, const void* q, const void* k, const void* v, void* o, float* lse,
                    fa_stream_t stream) {
  clear_detail();
  Problem p;
  const fa_status st = make_problem(desc, &p, false);
  if (st != FA_OK) return st;
  return run_fwd(p, q, k, v, o, lse, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  const fa_desc x = dense_desc(B, N, H, d, softmax_scale, causal, dtype);
  return fa_fwd_ex(&x, q, k, v, o, lse, stream);
}

size_t fa_bwd_ex_workspace_size(const fa_desc* desc) {
  Problem p;
  if (make_problem(desc, &p, true) != FA_OK) return 0;
  return bwd_layout(p).total_bytes;
}

size_t fa_bwd_workspace_size(int B, int N, int H, int d, int causal) {
  const fa_desc x = dense_desc(B, N, H, d, 1.0f, causal != 0, FA_FP16);
  return fa_bwd_ex_workspace_size(&x);
}

fa_status fa_bwd_ex(const fa_desc* desc, const void* q, const void* k, const void* v, const void* o,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, fa_stream_t stream) {
  clear_detail();
  Problem p;
  fa_status st = make_problem(desc, &p, true);
  if (st != FA_OK) return st;
  if ((st = check_bwd_pointers(q, k, v, o, dout, lse, dq, dk, dv)) != FA_OK) return st;
  if (!aligned16(workspace) || workspace_bytes < bwd_layout(p).total_bytes) {
    set_detail_text("workspace is null, misaligned or smaller than the workspace size of this call");
    return FA_ERR_WORKSPACE;
  }
  return run_bwd(p, q, k, v, o, dout, lse, dq, dk, dv, static_cast<uint8_t*>(workspace),
                 reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  const fa_desc x = dense_desc(B, N, H, d, softmax_scale, causal, dtype);
  return fa_bwd_ex(&x, q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                         float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  clear_detail();
  const fa_desc x = dense_desc(B, N, H, d, softmax_scale, causal, dtype);
  Problem p;
  fa_status st = make_problem(&x, &p, true);
  if (st != FA_OK) return st;
  if ((st = check_bwd_pointers(q, k, v, o, dout, lse, dq, dk, dv)) != FA_OK) return st;
  if (bwd_layout(p).total_bytes > kNoAllocScratchBytes) {
    set_detail_text("this shape needs more scratch than the built-in 32 MiB; use fa_bwd with a workspace");
    return FA_ERR_WORKSPACE;
  }
  cudaError_t e = cudaSuccess;
  uint8_t* scratch = noalloc_scratch(&e);
  if (scratch == nullptr) return FA_ERR_CUDA;
  // The preprocessing launch rewrites D and -LSE*log2(e), zeroes the ordering
  // counters and both work counters; the first contributor of each dQ sum
  // stores (not adds). Nothing left in the scratch by an earlier call is read.
  return run_bwd(p, q, k, v, o, dout, lse, dq, dk, dv, scratch, reinterpret_cast<cudaStream_t>(stream));
}

size_t fa_decode_workspace_size(int B, int Nq, int H, int d, int Nmax) {
  if (dec_check(B, Nq, H, d, Nmax, 1.0f, 0, FA_FP16) != FA_OK) return 0;
  return dec_plan(B, Nq, H, d, Nmax, num_sms()).total_bytes;
}

fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens, void* o,
                    float* lse, void* workspace, size_t workspace_bytes, int B, int Nq, int H, int d, int Nmax,
                    float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  clear_detail();
  fa_status st = dec_check(B, Nq, H, d, Nmax, softmax_scale, causal, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(lse))
    return bad_arg("a pointer is null or not 16-byte aligned");
  if (cache_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u))
    return bad_arg("cache_seqlens must be a 4-byte aligned device pointer");
  if ((st = bind_context()) != FA_OK) return st;
  const int sms = num_sms();
  if (sms <= 0) return FA_ERR_CUDA;
  const DecPlan pl = dec_plan(B, Nq, H, d, Nmax, sms);
  if (!aligned16(workspace) || workspace_bytes < pl.total_bytes) {
    set_detail_text("workspace is null, misaligned or smaller than fa_decode_workspace_size()");
    return FA_ERR_WORKSPACE;
  }
  const Strides cache = {(long long)Nmax * H * d, (long long)H * d, d};
  CUtensorMap mk, mv;
  bool hk = false, hv = false;
  if ((st = make_map_rows(&mk, &hk, k_cache, cache, d, H, Nmax, B, kDecKeys, "k_cache")) != FA_OK ||
      (st = make_map_rows(&mv, &hv, v_cache, cache, d, H, Nmax, B, kDecKeys, "v_cache")) != FA_OK)
    return st;
  DecArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.q_sb = (long long)Nq * H * d, a.q_sn = (long long)H * d, a.q_sh = d;
  a.o = static_cast<uint16_t*>(o);
  a.o_sb = a.q_sb, a.o_sn = a.q_sn, a.o_sh = a.q_sh;
  a.lse = lse;
  a.cache_seqlens = cache_seqlens;
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.off_ml);
  a.B = B, a.H = H, a.Nq = Nq, a.Nmax = Nmax, a.d = d;
  a.units = pl.units;
  a.tiles_per_unit = pl.tiles_per_unit;
  a.causal = causal;
  a.hm = (hk ? kHmK : 0u) | (hv ? kHmV : 0u);
  a.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FA_BF16;
  cudaError_t e;
  e = Nq == 1 ? launch_decode_nq<1>(pl.D, bf16, mk, mv, a, s)
    : Nq == 2 ? launch_decode_nq<2>(pl.D, bf16, mk, mv, a, s)
    : Nq <= 4 ? launch_decode_nq<4>(pl.D, bf16, mk, mv, a, s)
              : launch_decode_nq<8>(pl.D, bf16, mk, mv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_check_device_status(fa_stream_t stream) {
  clear_detail();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaStreamSynchronize", e);
    return FA_ERR_CUDA;
  }
  int host = 0;
  if ((e = cudaMemcpyFromSymbol(&host, g_status, sizeof(int))) != cudaSuccess) {
    set_detail_cuda("reading the device status word", e);
    return FA_ERR_CUDA;
  }
  const int zero = 0;
  if ((e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int))) != cudaSuccess) {
    set_detail_cuda("clearing the device status word", e);
    return FA_ERR_CUDA;
  }
  if (host != 0) set_detail_text("a bounded device-side wait gave up (status word)");
  return host == 0 ? FA_OK : static_cast<fa_status>(host);
}

fa_status fa_selftest_bounded_wait(int which, int limit_ms, fa_stream_t stream) {
  clear_detail();
  if ((which != 1 && which != 2) || limit_ms < 1 || limit_ms > 1000)
    return bad_arg("which must be 1 or 2 and limit_ms in 1..1000");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The counter that never advances is a zero-initialised device symbol of
  // this library that nothing writes.
  int* never = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&never), g_selftest_zero);
  if (e != cudaSuccess) {
    set_detail_cuda("cudaGetSymbolAddress(self-test flag)", e);
    return FA_ERR_CUDA;
  }
  e = launch("fa_selftest_kernel", fa_selftest_kernel, 1, 32, 0, s, 1, which,
             (unsigned long long)limit_ms * 1000000ull, static_cast<const int*>(never));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_profile_bwd_events(void* begin_event, void* end_event) {
  clear_detail();
  if ((begin_event == nullptr) != (end_event == nullptr)) return bad_arg("give both events or neither");
  t_prof_begin = static_cast<cudaEvent_t>(begin_event);
  t_prof_end = static_cast<cudaEvent_t>(end_event);
  return FA_OK;
}

const char* fa_last_error_detail(void) { return t_detail; }

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
