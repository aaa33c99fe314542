// Decode against a key/value cache: O = softmax(scale q K^T [+causal]) V for a
// few new query rows per sequence over a cache of L_b keys.
//
// The lab write-up "从Attention矩阵到显存读写：FlashAttention真正解决的痛点"
// (§6.1) notes that inference runs step by step against a KV cache that grows
// one position at a time, and that blocking over a fixed Q tile wastes work
// there. Here the query side is tiny (Nq rows) and the work is reading the
// cache: each (batch, head) streams L_b * d * 2 * 2 bytes of K and V once, so
// the bound is HBM bandwidth, not the tensor cores. The cache's key axis is
// split into units of up to kTilesPerUnit tiles of 64 keys; each CTA runs one
// unit with the online softmax (running max m, exp-sum l, rescaled O) of the
// forward kernel, and writes its partial state. A second launch merges the
// units of each query row: with M = max m_u, w_u = 2^(m_u - M),
// O = sum w_u O_u / sum w_u l_u, LSE = (M + log2 sum w_u l_u) ln 2.
//
// Query row t of batch b sits at position L_b - Nq + t; it attends keys
// 0 .. L_b - 1, or with `causal` keys 0 .. L_b - Nq + t. A row with no key
// gets O = 0 and LSE = -inf.
//
// Roles (128 threads): thread 0 also issues the TMA loads of the K and V
// tiles into a 2-stage ring (64 keys x up to 128 columns each, 128-byte
// swizzle); all threads then compute, two threads per key for the scores
// (one per half of the head size), one warp per query row for the softmax
// update, and one thread per (column pair, part of the keys) for P V.
#pragma once

#include "sm100.cuh"

namespace fa {

struct DecArgs {
  const uint16_t* q;           // [B, Nq, H, d]: element (b, t, h, c) at q[b*q_sb + t*q_sn + h*q_sh + c]
  long long q_sb, q_sn, q_sh;
  uint16_t* o;                 // same layout as q
  long long o_sb, o_sn, o_sh;
  float* lse;                  // [B, H, Nq] fp32
  const int* cache_seqlens;    // [B] valid rows of each cache (clamped to [0, Nmax])
  float* part_o;               // [B*H, U, Nq, D] fp32: unnormalised O of each unit
  float* part_ml;              // [B*H, U, Nq, 2] fp32: m (log2 units), l of each unit
  int B, H, Nq, Nmax, d;
  int units;                   // U: units per (batch, head)
  int tiles_per_unit;
  int causal;
  uint32_t hm;                 // head-major K / V maps (kHmK | kHmV)
  float scale_log2;            // softmax_scale * log2(e)
};

constexpr int kDecMaxNq = 8;   // query rows per sequence and call
constexpr int kDecKeys = 64;   // keys per tile

// NQ: the launch's bound on query rows (1, 2, 4 or 8). Shared memory is sized
// for NQ rows and the ring has two stages, so that three CTAs share an SM at
// d = 128 up to NQ = 4 (more loads in flight, and one CTA's barriers overlap
// the others' streaming). Measured on a B200 at NQ = 1: 3758 GB/s with two
// stages and three CTAs against 2887 with three stages and two CTAs.
template <int D, int NQ>
struct DecCfg {
  static constexpr int kStages = 2;
  static constexpr int kBoxBytes = kDecKeys * 128;           // 64 rows x 64 columns x 2 B
  static constexpr int kTileBytes = kDecKeys * D * 2;        // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;         // K then V
  static constexpr int kQ = 0;                               // [NQ][D] fp32
  static constexpr int kS = kQ + NQ * D * 4;                 // [NQ][64] fp32: scores, then P
  static constexpr int kAlpha = kS + NQ * kDecKeys * 4;      // [NQ] rescale factors (16-byte padded)
  static constexpr int kThreads = 128;
  static constexpr int kWarps = kThreads / 32;
  // Scores: kSplit threads per key, each over D / kSplit columns.
  static constexpr int kSplit = kThreads / kDecKeys;
  // P V: thread = (column pair, part of the tile's keys)
  static constexpr int kPairs = D / 2;
  static constexpr int kParts = kThreads / kPairs;
  static constexpr int kKeysPerPart = kDecKeys / kParts;
  static constexpr int kRed = kAlpha + ((NQ * 4 + 15) / 16) * 16;  // [kParts][NQ][D] fp32: parts' sums
  static constexpr int kBar = kRed + kParts * NQ * D * 4;
  static constexpr int kRing = (kBar + 64 + 1023) / 1024 * 1024;
  static constexpr int kSmem = kRing + kStages * kStageBytes + 1024;  // + alignment slack
};

// The 16-byte chunk `c` (8 columns) of key row j of a [64 rows][64 columns]
// 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz_off(int j, int c) { return j * 128 + ((c ^ (j & 7)) << 4); }

// NQ: the query rows' compile-time bound (1, 2, 4 or 8; Nq <= NQ), so the
// per-key loops do no work for rows that do not exist.
template <int D, bool BF16, int NQ>
__global__ void __launch_bounds__(DecCfg<D, NQ>::kThreads)
    fa_decode_split(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecArgs a) {
  using C = DecCfg<D, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sQ = reinterpret_cast<float*>(smem + C::kQ);
  float* sS = reinterpret_cast<float*>(smem + C::kS);
  float* sAlpha = reinterpret_cast<float*>(smem + C::kAlpha);
  float* sRed = reinterpret_cast<float*>(smem + C::kRed);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBar);
  int* abort_flag = reinterpret_cast<int*>(smem + C::kBar + 8 * C::kStages);
  uint8_t* ring = smem + C::kRing;

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid & 31;
  const int unit = blockIdx.x % a.units;
  const int bh = blockIdx.x / a.units;
  const int b = bh / a.H, h = bh % a.H;
  const int Nq = a.Nq;
  int L = __ldg(a.cache_seqlens + b);
  L = L < 0 ? 0 : (L > a.Nmax ? a.Nmax : L);
  // Keys any query row of this batch may attend: [0, L) (causal rows end earlier).
  const int key0 = unit * a.tiles_per_unit * kDecKeys;
  const int key1 = min(L, key0 + a.tiles_per_unit * kDecKeys);
  const int ntiles = key1 > key0 ? (key1 - key0 + kDecKeys - 1) / kDecKeys : 0;

  float* pml = a.part_ml + ((size_t)bh * a.units + unit) * Nq * 2;
  float* po = a.part_o + ((size_t)bh * a.units + unit) * Nq * D;
  if (ntiles == 0) {  // nothing cached here: an empty partial state
    for (int i = tid; i < Nq * D; i += C::kThreads) po[i] = 0.f;
    for (int t = tid; t < Nq; t += C::kThreads) {
      pml[2 * t] = -INFINITY;
      pml[2 * t + 1] = 0.f;
    }
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // q rows in fp32 (columns past d are zero), pre-scaled by scale * log2(e).
  for (int i = tid; i < Nq * D; i += C::kThreads) {
    const int t = i / D, c = i % D;
    float x = 0.f;
    if (c < a.d) {
      const uint16_t raw = a.q[b * a.q_sb + t * a.q_sn + h * a.q_sh + c];
      x = BF16 ? __uint_as_float((uint32_t)raw << 16) : __half2float(__ushort_as_half(raw));
    }
    sQ[i] = x * a.scale_log2;
  }
  __syncthreads();

  auto issue = [&](int i) {  // tile i of this unit into stage i % C::kStages
    const int st = i % C::kStages;
    uint8_t* dst = ring + st * C::kStageBytes;
    mbar_arrive_expect_tx(&full[st], C::kStageBytes);
    const int row = key0 + i * kDecKeys;
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_load_rows(&tm_k, a.hm & kHmK, dst + kb * C::kBoxBytes, &full[st], kb * 64, h, row, b);
      tma_load_rows(&tm_v, a.hm & kHmV, dst + C::kTileBytes + kb * C::kBoxBytes, &full[st], kb * 64, h, row, b);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    for (int i = 0; i < C::kStages - 1 && i < ntiles; ++i) issue(i);
  }

  // Softmax state of query row t lives in warp t % kWarps (all lanes hold it).
  constexpr int kRowsPerWarp = (NQ + C::kWarps - 1) / C::kWarps;
  float m_run[kRowsPerWarp], l_run[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
  }
  // P V accumulators: column pair cp (columns 2cp, 2cp+1), keys of part kh of
  // each tile, every query row.
  const int cp = tid % C::kPairs, kh = tid / C::kPairs;
  // Two sets by key parity (even, odd) keep the FMA chains short; added at the end.
  float acc[NQ][2], acc2[NQ][2];
#pragma unroll
  for (int t = 0; t < NQ; ++t) acc[t][0] = acc[t][1] = acc2[t][0] = acc2[t][1] = 0.f;

  bool ok = true;
  int issued = min(C::kStages - 1, ntiles);
  for (int i = 0; i < ntiles; ++i) {
    const int st = i % C::kStages;
    // The stage refilled here was released by the barrier at the end of the
    // previous tile.
    if (tid == 0 && issued < ntiles) issue(issued++);
    const bool got = mbar_wait(&full[st], (i / C::kStages) & 1, abort_flag);
    ok = __syncthreads_and(got) != 0;
    if (!ok) break;
    const uint8_t* kt = ring + st * C::kStageBytes;
    const uint8_t* vt = kt + C::kTileBytes;
    const int kbase = key0 + i * kDecKeys;

    // ---- scores: key j = tid / kSplit, columns of part hf = tid % kSplit
    {
      const int j = tid / C::kSplit, hf = tid % C::kSplit;
      const int key = kbase + j;
      // Four partial sums per row (columns 0-3 and 4-7 of each chunk, even
      // and odd chunks) keep the FMA chains short.
      float dot[NQ][4];
#pragma unroll
      for (int t = 0; t < NQ; ++t) dot[t][0] = dot[t][1] = dot[t][2] = dot[t][3] = 0.f;
      constexpr int kChunks = D / (8 * C::kSplit);  // 16-byte chunks per part
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        const int col = hf * (D / C::kSplit) + cc * 8;  // first column of this chunk
        const uint8_t* box = kt + (col / 64) * C::kBoxBytes;
        const uint4 w = *reinterpret_cast<const uint4*>(box + swz_off(j, (col % 64) / 8));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<BF16>(ws[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (t < Nq) {
            const float4 q0 = *reinterpret_cast<const float4*>(sQ + t * D + col);
            const float4 q1 = *reinterpret_cast<const float4*>(sQ + t * D + col + 4);
            float x = dot[t][2 * (cc & 1)], y = dot[t][2 * (cc & 1) + 1];
            x = fmaf(q0.x, kf[0], x);
            y = fmaf(q1.x, kf[4], y);
            x = fmaf(q0.y, kf[1], x);
            y = fmaf(q1.y, kf[5], y);
            x = fmaf(q0.z, kf[2], x);
            y = fmaf(q1.z, kf[6], y);
            x = fmaf(q0.w, kf[3], x);
            y = fmaf(q1.w, kf[7], y);
            dot[t][2 * (cc & 1)] = x;
            dot[t][2 * (cc & 1) + 1] = y;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NQ; ++t) {
        if (t < Nq) {
          float s = (dot[t][0] + dot[t][1]) + (dot[t][2] + dot[t][3]);
#pragma unroll
          for (int off = 1; off < C::kSplit; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
          const int last = a.causal ? L - Nq + t : L - 1;  // last key row t attends
          if (hf == 0) sS[t * kDecKeys + j] = key <= last ? s : -INFINITY;
        }
      }
    }
    __syncthreads();

    // ---- online softmax: warp w updates rows t = w, w + kWarps, ...
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int t = warp + C::kWarps * r;
      if (t < Nq) {
        const float s0 = sS[t * kDecKeys + lane], s1 = sS[t * kDecKeys + 32 + lane];
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_run[r], mx);
        // Rows that have seen no key yet keep m = -inf; guard their factors.
        const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run[r] - m_new);
        const float base = m_new == -INFINITY ? 0.f : m_new;
        const float p0 = ex2(s0 - base), p1 = ex2(s1 - base);
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l_run[r] = l_run[r] * alpha + ps;
        m_run[r] = m_new;
        sS[t * kDecKeys + lane] = p0;
        sS[t * kDecKeys + 32 + lane] = p1;
        if (lane == 0) sAlpha[t] = alpha;
      }
    }
    __syncthreads();

    // ---- O = O * alpha + P V over this thread's 32 keys and column pair
    {
      const int col = 2 * cp;
      const uint8_t* box = vt + (col / 64) * C::kBoxBytes;
      const int chunk = (col % 64) / 8, within = (col % 8) * 2;
#pragma unroll
      for (int t = 0; t < NQ; ++t) {
        if (t < Nq) {
          const float al = sAlpha[t];
          acc[t][0] *= al;
          acc[t][1] *= al;
          acc2[t][0] *= al;
          acc2[t][1] *= al;
        }
      }
      // Only rows below the cache length: the rest may hold anything (even
      // NaN), and 0 * NaN would not vanish.
      const int kvalid = min(kDecKeys, L - kbase);
#pragma unroll 4
      for (int jj = 0; jj < C::kKeysPerPart; ++jj) {
        const int j = kh * C::kKeysPerPart + jj;
        if (j >= kvalid) break;
        const uint32_t w = *reinterpret_cast<const uint32_t*>(box + swz_off(j, chunk) + within);
        const float2 vv = unpack2<BF16>(w);
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (t < Nq) {
            const float p = sS[t * kDecKeys + j];
            if (jj & 1) {
              acc2[t][0] = fmaf(p, vv.x, acc2[t][0]);
              acc2[t][1] = fmaf(p, vv.y, acc2[t][1]);
            } else {
              acc[t][0] = fmaf(p, vv.x, acc[t][0]);
              acc[t][1] = fmaf(p, vv.y, acc[t][1]);
            }
          }
        }
      }
    }
    __syncthreads();  // stage st and sS are free again
  }

  // Never leave with copies in flight (only after an abort can any be).
  if (tid == 0)
    for (int x = max(0, issued - C::kStages); x < issued; ++x)
      mbar_wait(&full[x % C::kStages], (x / C::kStages) & 1, abort_flag, false);
  if (!ok) return;  // the status word already says why

  // ---- partial state: the key parts' O added in a fixed order, m and l of each row
#pragma unroll
  for (int t = 0; t < NQ; ++t) {
    if (t < Nq) {
      sRed[(kh * NQ + t) * D + 2 * cp] = acc[t][0] + acc2[t][0];
      sRed[(kh * NQ + t) * D + 2 * cp + 1] = acc[t][1] + acc2[t][1];
    }
  }
  __syncthreads();
  for (int i = tid; i < Nq * D; i += C::kThreads) {
    const int t = i / D, c = i % D;
    float x = 0.f;
#pragma unroll
    for (int part = 0; part < C::kParts; ++part) x += sRed[(part * NQ + t) * D + c];
    po[t * D + c] = x;
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int t = warp + C::kWarps * r;
    if (t < Nq && lane == 0) {
      pml[2 * t] = m_run[r];
      pml[2 * t + 1] = l_run[r];
    }
  }
}

// Merge of the units of each query row (b, t, h): one warp per row, the
// lanes over columns.
template <int D, bool BF16>
__global__ void __launch_bounds__(128) fa_decode_combine(const DecArgs a) {
  const int row = blockIdx.x * 4 + threadIdx.x / 32;  // (b*H + h)*Nq + t
  const int lane = threadIdx.x & 31;
  if (row >= a.B * a.H * a.Nq) return;
  const int t = row % a.Nq, bh = row / a.Nq;
  const int b = bh / a.H, h = bh % a.H;
  const float* pml = a.part_ml + (size_t)bh * a.units * a.Nq * 2;
  const float* po = a.part_o + (size_t)bh * a.units * a.Nq * D;
  float M = -INFINITY;
  for (int u = 0; u < a.units; ++u) M = fmaxf(M, pml[(u * a.Nq + t) * 2]);
  float lsum = 0.f;
  float o[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) o[c] = 0.f;
  if (M != -INFINITY) {
    for (int u = 0; u < a.units; ++u) {
      const float mu = pml[(u * a.Nq + t) * 2];
      if (mu == -INFINITY) continue;
      const float w = ex2(mu - M);
      lsum = fmaf(w, pml[(u * a.Nq + t) * 2 + 1], lsum);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) o[c] = fmaf(w, po[(size_t)(u * a.Nq + t) * D + c * 32 + lane], o[c]);
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint16_t* orow = a.o + b * a.o_sb + t * a.o_sn + h * a.o_sh;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const int col = c * 32 + lane;
    if (col < a.d) {
      const uint32_t pk = pack2<BF16>(o[c] * inv, 0.f);
      orow[col] = static_cast<uint16_t>(pk & 0xFFFFu);
    }
  }
  if (lane == 0)
    a.lse[((size_t)b * a.H + h) * a.Nq + t] = lsum > 0.f ? (M + lg2(lsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace fa
