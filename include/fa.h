/*
 * fa.h - C ABI of libfa: exact scaled-dot-product attention on NVIDIA B200
 * (sm_100a), forward and backward, computed I/O-aware so that the N x N score
 * matrix S and probability matrix P never reach device memory.
 *
 * What is computed (one (batch, head) at a time; all heads independent):
 *
 *     S = softmax_scale * Q K^T            (N x N, on chip only)
 *     causal: S_ij = -inf for key j > query i
 *     P = softmax(S) along the key axis    (on chip only)
 *     O = P V,   LSE_i = ln sum_j exp(S_ij)
 *
 * Sources: the three-step definition and the tiling / online-softmax /
 * recomputation method are those of the lab write-up
 * "从Attention矩阵到显存读写：FlashAttention真正解决的痛点" (dpshk.com, §2.1,
 * §3.1-§3.3); the [batch, seqlen, heads, head_dim] layout, fp16/bf16-only
 * inputs, softmax_scale (default 1/sqrt(head_dim)) and the causal flag are its
 * §4.2 description of flash_attn_func; the einsum restatement and the idea of
 * fusing QK^T, softmax and PV into one kernel are from "使用FlashAttention优化
 * PyTorch模型注意力计算" (tiemojia.cn). The pages give no backward formulas;
 * fa_bwd implements the chain rule through softmax with P recomputed from LSE.
 *
 * Conventions shared by every entry point:
 *   - Layout: q, k, v, o, dout, dq, dk, dv are dense, contiguous
 *     [B, N, H, d] arrays of 16-bit floats (row stride H*d elements, head
 *     stride d). lse is a dense [B, H, N] fp32 array.
 *   - Supported: d in {64, 128}; N >= 1 of any value; B, H >= 1;
 *     B*N*H*d < 2^31. Other head sizes return FA_ERR_UNSUPPORTED.
 *   - All pointers are DEVICE pointers on the current CUDA device, 16-byte
 *     aligned. The caller owns every buffer; the library allocates no device
 *     memory and keeps no per-call state.
 *   - softmax_scale must be finite and > 0 (callers wanting the default pass
 *     1/sqrt(d)).
 *   - Calls are asynchronous on `stream` and never synchronise. Arguments are
 *     checked on the host before any launch; on an error nothing is launched
 *     and no output is touched. A launch failure returns FA_ERR_CUDA.
 *   - Device-side waits are bounded; a wait that gives up records
 *     FA_ERR_DEVICE_TIMEOUT in a device status word that
 *     fa_check_device_status() reports.
 *   - Results are bitwise deterministic for fixed inputs and arguments.
 */
#ifndef FA_B200_FA_H
#define FA_B200_FA_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                       /* cudaStream_t == struct CUstream_st* */
typedef struct CUstream_st* fa_stream_t;  /* NULL = the legacy default stream */

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size or scale   */
  FA_ERR_UNSUPPORTED = 2,     /* valid request this build does not implement */
  FA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed           */
  FA_ERR_DEVICE_TIMEOUT = 4,  /* a bounded device-side wait gave up          */
  FA_ERR_WORKSPACE = 5        /* workspace pointer null or too small         */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

/*
 * Forward pass. Lab write-up §2.1 (definition), §3.1 (tiling), §3.2 (online
 * softmax with running max m and exp-sum l, rescaling of the O accumulator,
 * final O / l).
 *   q, k, v  in:  [B, N, H, d], dtype `dtype`
 *   o        out: [B, N, H, d], dtype `dtype` (round to nearest even)
 *   lse      out: [B, H, N] fp32, natural-log logsumexp of the scaled
 *                 (and masked) logits of each query row; fa_bwd needs it.
 *   causal   0 = full attention; 1 = query i attends keys 0..i.
 * Work split: where it shortens the launch (few row blocks per SM), a
 * non-causal call halves each row block's key tiles between the two CTAs of
 * a 2-CTA cluster, and one merges the two online-softmax states (rescale by
 * the larger running max, add O and l) before O and lse are written. The
 * choice follows the shape and the device's SM count; FA_FWD_SPLIT=1 or 2 in
 * the environment forces it. The two paths round differently, each
 * deterministically.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs for this shape (0 on invalid sizes).
 * It holds D = rowsum(dO o O) [B, H, N] fp32, an fp32 dQ accumulator and the
 * per-tile ordering counters that make the dQ sum deterministic.
 */
FA_API size_t fa_bwd_workspace_size(int B, int N, int H, int d, int causal);

/*
 * Backward pass: gradients of a loss L through O = attention(Q, K, V), given
 * dout = dL/dO. Lab write-up §3.3 (recompute S and P instead of storing them);
 * the gradient formulas are the chain rule through softmax:
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_j dO_ij O_ij,  dS = P o (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q,
 * with P recomputed on chip as exp(S - LSE).
 *   q, k, v, o, dout in:  [B, N, H, d] (o and lse from fa_fwd with the same
 *                         arguments)
 *   lse              in:  [B, H, N] fp32
 *   dq, dk, dv       out: [B, N, H, d], dtype `dtype`
 *   workspace        scratch of at least fa_bwd_workspace_size() bytes,
 *                    16-byte aligned; overwritten; need not be zeroed.
 * dQ is accumulated in fp32 in a fixed key-tile order, so the result does not
 * depend on scheduling.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int N, int H, int d,
                 float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * fa_bwd without a workspace argument, for callers that cannot allocate
 * device memory. The pages have no counterpart to this entry point.
 *
 * Some callers cannot call cudaMalloc: a plug-in or runtime whose host process
 * owns all device memory through its own pool and allows no other allocations,
 * code running near the device's memory capacity where a new allocation would
 * fail, or a latency-critical loop that must not pay for the allocator. They
 * still pass every input and output buffer; only the scratch is built in.
 *
 * The scratch is one file-scope device array of 32 MiB (33554432 bytes),
 * which every GPU that loads this library holds until the process exits. No call allocates or frees device memory. A shape whose
 * fa_bwd_workspace_size() exceeds that maximum returns FA_ERR_WORKSPACE and
 * launches nothing.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture. All calls on a device share the one
 * array and it keeps the last call's contents: each call re-initialises what it
 * needs (nothing has to start at zero), but calls whose work overlaps on the
 * GPU (different streams, or host threads, without ordering between them)
 * race on the scratch and their results are undefined. Serialise them.
 *
 * Arguments, layout, results and errors are otherwise those of fa_bwd.
 */
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                                float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device. Returns FA_ERR_DEVICE_TIMEOUT if any kernel of this library
 * gave up a bounded wait since the last call, FA_ERR_CUDA if the stream
 * reports an error, FA_OK otherwise.
 */
FA_API fa_status fa_check_device_status(fa_stream_t stream);

/*
 * Failure-detection self-test (not part of the attention computation).
 * Launches one small kernel on `stream` whose bounded wait can never be
 * satisfied: which = 1 waits on a shared-memory mbarrier phase that nothing
 * completes, which = 2 polls a device counter that nothing advances (the wait
 * fa_bwd uses to order dQ additions). After limit_ms (1..1000) the wait gives
 * up, records FA_ERR_DEVICE_TIMEOUT in the status word and the kernel returns;
 * nothing hangs or faults and the context stays usable. A following
 * fa_check_device_status() reports and clears it. Returns FA_ERR_INVALID_ARG
 * for other arguments, FA_ERR_CUDA if the launch fails.
 */
FA_API fa_status fa_selftest_bounded_wait(int which, int limit_ms, fa_stream_t stream);

/* Human-readable name of a status code (static storage; never NULL). */
FA_API const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
