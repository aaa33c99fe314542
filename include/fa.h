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
 *   - Supported: head size d a multiple of 8 from 8 to 128; N >= 1 of any
 *     value; B, H >= 1; fewer than 2^31 elements per tensor. Other head
 *     sizes return FA_ERR_UNSUPPORTED.
 *   - All pointers are DEVICE pointers on the current CUDA device, 16-byte
 *     aligned. The caller owns every buffer; the library allocates no device
 *     memory and keeps no per-call state.
 *   - softmax_scale must be finite and > 0 (callers wanting the default pass
 *     1/sqrt(d)).
 *   - Calls are asynchronous on `stream` and never synchronise. Arguments are
 *     checked on the host before any launch; on an error nothing is launched
 *     and no output is touched. A launch whose own return code is an error
 *     returns FA_ERR_CUDA (an error some earlier, unrelated CUDA call left
 *     pending in the calling thread is neither reported nor cleared).
 *     fa_last_error_detail() says which step failed and why.
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
 * Element strides of a [B, N, H, d] view of a 16-bit tensor: element
 * (b, n, h, c) is at base[b*batch + n*row + h*head + c] (the head-size axis is
 * contiguous). All three zero means dense [B, N, H, d]. Otherwise each must be
 * a positive multiple of 8 elements (16 bytes) below 2^36; the batch stride
 * may be 0 where it is never used (B = 1, or variable length). Any order of
 * the three is accepted: e.g. a packed QKV tensor [B, N, 3, H, d] gives q, k
 * and v the strides {N*3*H*d, 3*H*d, d} at offsets 0, H*d and 2*H*d, and
 * PyTorch's [B, H, N, d] layout gives {H*N*d, d, N*d}.
 */
typedef struct {
  long long batch, row, head;
} fa_strides;

/*
 * One attention call's shape, options and tensor layout, for fa_fwd_ex /
 * fa_bwd_ex. Zero-initialise it and set what is needed.
 *   B, N, H, d       batch, sequence length, heads, head size. With
 *                    cu_seqlens: N is the longest sequence (max_seqlen).
 *   softmax_scale, causal, dtype   as for fa_fwd.
 *   stride_q .. stride_dv   layout of q, k, v, o, dout, dq, dk, dv (the
 *                    backward tensors are read only by fa_bwd_ex).
 *   cu_seqlens       NULL: every batch entry has N rows. Otherwise a
 *                    variable-length batch packed without padding: a device
 *                    array of B + 1 int32 row offsets (0 = cu[0] <= cu[1] <=
 *                    ... <= cu[B] = total), sequence b owning rows
 *                    cu[b] .. cu[b+1]-1 of every tensor, each tensor viewed
 *                    as [total, H, d] (batch strides unused) and lse as
 *                    [H, total] fp32. Each sequence attends only to itself
 *                    (causal: to its own earlier rows). The kernels clamp the
 *                    offsets to [0, total] and lengths to N, so a malformed
 *                    array gives wrong results, never an access outside the
 *                    tensors.
 *   total            rows of the packed tensors (with cu_seqlens).
 *   dropout_p, seed, offset
 *                    dropout on the attention probabilities (the
 *                    dropout_p of flash_attn_func in the lab write-up §4.2
 *                    and the README's usage line), 0 <= dropout_p < 1, 0 =
 *                    none: O = (P o Z) V with Z = keep / (1 - dropout_p),
 *                    the LSE that of the undropped softmax. Element (query i,
 *                    key j) of head h of batch (or sequence) b, i and j
 *                    counted from the sequence's first row, is dropped when
 *                    word j mod 4 of Philox4x32-10 (Salmon et al., SC 2011)
 *                    with counter (j / 4, i, b*H + h, offset) and key
 *                    (seed mod 2^32, seed / 2^32) is below
 *                    floor(dropout_p * 2^32). fa_bwd_ex regenerates the same
 *                    mask from the same desc; nothing is stored.
 */
typedef struct {
  int B, N, H, d;
  float softmax_scale;
  int causal;
  fa_dtype dtype;
  fa_strides stride_q, stride_k, stride_v, stride_o;
  fa_strides stride_do, stride_dq, stride_dk, stride_dv;
  const int* cu_seqlens;
  int total;
  float dropout_p;
  unsigned long long seed;
  unsigned int offset;
} fa_desc;

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
 * Forward pass on any layout fa_desc describes: strided views (e.g. the q, k
 * and v of one packed [B, N, 3, H, d] tensor, as flash_attn_qkvpacked_func
 * takes it in "使用FlashAttention优化PyTorch模型注意力计算", or the
 * [B, H, N, d] layout the lab write-up §4.2 warns about), head sizes that
 * are multiples of 8 up to 128, and variable-length batches packed without
 * padding (the lab write-up §4.2, third pitfall: flash_attn_varlen_func).
 * lse is dense [B, H, N] fp32, or [H, total] with cu_seqlens. Otherwise as
 * fa_fwd.
 */
FA_API fa_status fa_fwd_ex(const fa_desc* desc, const void* q, const void* k, const void* v, void* o, float* lse,
                           fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs for this shape (0 on invalid sizes).
 * It holds D = rowsum(dO o O) [B, H, N] fp32, an fp32 dQ accumulator and the
 * per-tile ordering counters that make the dQ sum deterministic.
 * Layout after a call (for inspection; N_pad = 128 * ceil(N / 128),
 * up256(x) = x rounded up to a multiple of 256):
 *   byte 0:                           -LSE * log2(e), [B*H, N_pad] fp32
 *   byte up256(4 * B*H*N_pad):        D,             [B*H, N_pad] fp32
 *   then the dQ sums and counters (internal).
 * Rows N .. N_pad-1 of each head hold -inf (-LSE * log2(e)) and 0 (D).
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

/* Workspace bytes fa_bwd_ex needs for `desc` (0 if desc is invalid). */
FA_API size_t fa_bwd_ex_workspace_size(const fa_desc* desc);

/*
 * Backward pass on any layout fa_desc describes (see fa_fwd_ex): q, k, v, o,
 * dout, dq, dk, dv each with its own strides (dq, dk, dv may be the three
 * slices of one packed [B, N, 3, H, d] gradient), variable-length batches,
 * head sizes that are multiples of 8 up to 128. o and lse as fa_fwd_ex wrote
 * them. Otherwise as fa_bwd.
 */
FA_API fa_status fa_bwd_ex(const fa_desc* desc, const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                           size_t workspace_bytes, fa_stream_t stream);

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
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress; it allocates nothing, and no address is cached, so a
 * context torn down and made again by cudaDeviceReset is handled). The first
 * call on a device also loads this library's device code there: make that
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
 * Decode step against a key/value cache (the lab write-up §6.1: inference
 * reads a KV cache that grows one position at a time; there the work is
 * streaming the cache, bound by memory bandwidth, not by the tensor cores).
 *   q              in:  [B, Nq, H, d], the Nq newest positions of each
 *                       sequence (1 <= Nq <= 8), dtype `dtype`
 *   k_cache,
 *   v_cache        in:  [B, Nmax, H, d]; batch b holds L_b valid rows
 *   cache_seqlens  in:  device int32 [B], L_b (clamped to [0, Nmax]);
 *                       rows L_b .. Nmax-1 are never read into the result
 *                       (they may hold anything)
 *   o              out: [B, Nq, H, d], dtype `dtype`
 *   lse            out: [B, H, Nq] fp32
 *   workspace      at least fa_decode_workspace_size() bytes, 16-byte
 *                  aligned; holds each split's partial (m, l, O)
 * Query t of batch b sits at position L_b - Nq + t; it attends keys
 * 0 .. L_b - 1, or with causal = 1 keys 0 .. L_b - Nq + t. A row with no key
 * to attend gets O = 0 and LSE = -inf. The cache's key axis is split across
 * CTAs and the partial online-softmax states are merged by rescaling with
 * the larger running max (a second launch on the same stream). All tensors
 * dense; head size a multiple of 8 up to 128. Errors as fa_fwd; Nq > 8
 * returns FA_ERR_UNSUPPORTED.
 */
FA_API size_t fa_decode_workspace_size(int B, int Nq, int H, int d, int Nmax);
FA_API fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens,
                           void* o, float* lse, void* workspace, size_t workspace_bytes, int B, int Nq, int H,
                           int d, int Nmax, float softmax_scale, int causal, fa_dtype dtype, fa_stream_t stream);

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

/*
 * Profiling hook (not part of the attention computation): after this call,
 * every fa_bwd / fa_bwd_noalloc made from the calling host thread records
 * `begin_event` on its stream right before the launch of its dK/dV kernel
 * (fa_bwd_dkdv, the backward's dominant kernel) and `end_event` right after
 * it, so cudaEventElapsedTime gives that kernel's device time. Both are
 * cudaEvent_t handles owned by the caller; pass NULL, NULL to stop. One
 * argument NULL and the other not returns FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_profile_bwd_events(void* begin_event, void* end_event);

/*
 * What the most recent call of this library from the calling host thread
 * failed on: the step (argument check, tensor-map encoding, which launch) and,
 * for CUDA failures, the CUDA error's name and number. Empty when that call
 * succeeded. Thread-local storage, valid until the thread's next call.
 */
FA_API const char* fa_last_error_detail(void);

/* Human-readable name of a status code (static storage; never NULL). */
FA_API const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
