// Backward kernels: dQ, dK, dV of O = softmax(scale Q K^T [+causal]) V.
//
// The lab write-up "从Attention矩阵到显存读写：FlashAttention真正解决的痛点"
// (§3.3) recomputes S and P in the backward pass instead of storing them; the
// pages give no gradient formulas, so these kernels implement the chain rule
// through softmax, with P rebuilt from the forward's row LSE:
//
//   P = exp(scale S - LSE),  dV = P^T dO,  dP = dO V^T,
//   D_i = rowsum(dO o O)_i,  dS = P o (dP - D),  dK = scale dS^T Q,
//   dQ = scale dS K.
//
// Two launches on the caller's stream:
//   1. fa_bwd_prep:  D and -LSE*log2(e) into padded per-head arrays; zeroes
//                    the dQ ordering counters and the two work counters.
//   2. fa_bwd_dkdv:  persistent; one CTA per SM fetches work items (b, h, key
//                    tile j) from a global counter. Per item K_j, V_j stay in
//                    shared memory and dK_j, dV_j accumulate in TMEM while
//                    (Q_i, dO_i) tiles stream through a 2-stage ring. Per
//                    step, five tcgen05 MMAs: S^T = K Q^T, dP^T = V dO^T,
//                    dV += P^T dO, dQ_part = dS K, dK += dS^T Q. dQ_part is
//                    added into two fp32 sums per query tile in a fixed
//                    key-tile order (per-tile counters say whose turn it
//                    is), so the sums are deterministic. When the items run
//                    out, each CTA's dQ warps take finished query tiles from
//                    a second counter and write dQ = scale * (sum 0 + sum 1).
//
// dQ order (BwdItem below). Query tile i's dQ is summed in fp32 over key
// tiles in a fixed descending order (two sums, added in a fixed order at the
// end), so the result does not depend on scheduling. No wait can deadlock
// (the earliest-fetched unfinished item waits for nothing, and the finishing
// of a tile waits only for items), and every wait is bounded anyway.
#pragma once

#include <algorithm>

#include "sm100.cuh"

namespace fa {

// Workspace layout (all offsets 256-byte aligned).
struct BwdLayout {
  int npad, ntiles;
  size_t off_lse2, off_dd, off_dqacc, off_cnt, off_sched;
  size_t total_bytes;
  static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
  static BwdLayout make(int B, int N, int H, int d) {
    BwdLayout L;
    L.ntiles = (N + 127) / 128;
    L.npad = L.ntiles * 128;
    const size_t bh = (size_t)B * H;
    size_t off = 0;
    L.off_lse2 = off;  off = up256(off + bh * L.npad * 4);
    L.off_dd = off;    off = up256(off + bh * L.npad * 4);
    L.off_dqacc = off; off = up256(off + 2 * bh * L.npad * (size_t)d * 4);  // sums 0, 1
    L.off_cnt = off;   off = up256(off + 2 * bh * L.ntiles * 4);            // sums 0, 1
    L.off_sched = off; off = up256(off + 16);
    L.total_bytes = off;
    return L;
  }
};

struct BwdArgs {
  // Caller tensors: element (b, n, h, c) of X at X[b*X_sb + (row0 + n)*X_sn +
  // h*X_sh + c] (row0 = 0, or the sequence's first row when variable-length).
  const uint16_t* o;
  long long o_sb, o_sn, o_sh;
  const uint16_t* dout;
  long long do_sb, do_sn, do_sh;
  const float* lse;  // at lse[b*lse_sb + h*lse_sh + row0 + n]
  long long lse_sb, lse_sh;
  uint16_t* dq;
  long long dq_sb, dq_sn, dq_sh;
  uint16_t* dk;
  long long dk_sb, dk_sn, dk_sh;
  uint16_t* dv;
  long long dv_sb, dv_sn, dv_sh;
  const int* cu;     // variable-length row offsets [B + 1], or nullptr
  int total;         // rows of the packed tensors (variable length)
  // Workspace
  float* lse2;   // [B*H, npad] -LSE * log2(e); -inf on rows past the sequence
  float* dd;     // [B*H, npad] D; 0 on rows past the sequence
  float* dqacc;  // 2 x [B*H, ntiles, d/4, 128, 4] fp32 (sum 0, sum 1)
  int* cnt;      // 2 x [B*H, ntiles] dQ ordering counters (sum 0, sum 1)
  int* sched;    // [0]: item counter, [1]: counter of query tiles to finish
  int B, N, H, npad, ntiles;  // N: sequence length (variable length: the longest)
  int hgroup;        // causal: heads whose items interleave (decode_item)
  int d;             // head size (<= D; columns d .. D-1 are zeros from TMA)
  uint32_t hm;       // head-major tensor maps (kHmQ | kHmK | kHmV | kHmDO | kHmDK | kHmDV)
  Dropout drop;      // used by the DROPOUT instantiation only
  float scale;       // softmax_scale
  float scale_log2;  // softmax_scale * log2(e)
};

// ------------------------------------------------------------------ kernel 1

template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_prep(const BwdArgs a) {
  // Block (x, bh): rows n = x * kRows + group of head bh, a group of G = D/8
  // lanes per row, 8 elements per lane. Rows of the sequence get
  // D = rowsum(dO o O) and -LSE*log2(e); rows past its end (up to npad) get 0
  // and -inf (no query: P = 0).
  constexpr int G = D / 8;
  constexpr int kRows = 256 / G;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int sub = threadIdx.x % G;
  const int n = blockIdx.x * kRows + threadIdx.x / G;
  const SeqRows seq = seq_rows(a.cu, b, a.N, a.total);
  const bool valid = n < seq.len;
  float acc = 0.f;
  if (valid && sub * 8 < a.d) {
    const long long r = seq.row0 + n;
    const uint4 ov = *reinterpret_cast<const uint4*>(a.o + b * a.o_sb + r * a.o_sn + h * a.o_sh + sub * 8);
    const uint4 dv = *reinterpret_cast<const uint4*>(a.dout + b * a.do_sb + r * a.do_sn + h * a.do_sh + sub * 8);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = unpack2<BF16>(ow[i]);
      const float2 y = unpack2<BF16>(dw[i]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, G);
  if (sub == 0 && n < a.npad) {
    const size_t row = (size_t)bh * a.npad + n;
    a.dd[row] = valid ? acc : 0.f;
    a.lse2[row] = valid ? -(a.lse[b * a.lse_sb + h * a.lse_sh + seq.row0 + n] * 1.4426950408889634f) : -INFINITY;
  }
  // This head's ordering counters (both sums), and the work counter.
  if (blockIdx.x == 0) {
    for (int t = threadIdx.x; t < a.ntiles; t += blockDim.x) {
      a.cnt[(size_t)bh * a.ntiles + t] = 0;
      a.cnt[((size_t)a.B * a.H + bh) * a.ntiles + t] = 0;
    }
    if (bh == 0 && threadIdx.x == 0) {
      a.sched[0] = 0;  // items
      a.sched[1] = 0;  // query tiles to finish
    }
  }
}

// ------------------------------------------------------------------ kernel 2

template <int D>
struct BwdCfg {
  static constexpr int kTile = 128 * D * 2;  // one 128-row tile of Q/K/V/dO
  static constexpr int kBox = 128 * 128;     // one 64-column box of a tile
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  // (Q_i, dO_i, LSE_i, D_i) ring depth: 4 stages fit at d = 64 and hide the
  // L2 latency of the next tiles; at d = 128 shared memory allows 2.
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kQ = kV + kTile;                  // kStages stages
  static constexpr int kDO = kQ + kStages * kTile;       // kStages stages
  static constexpr int kDS = kDO + kStages * kTile;      // dS^T, 128 x 128 16-bit
  static constexpr int kLSE = kDS + 128 * 128 * 2;       // kStages x 128 fp32
  static constexpr int kDD = kLSE + kStages * 512;       // kStages x 128 fp32
  static constexpr int kBar = kDD + kStages * 512;
  static constexpr int kSmem = kBar + 384;
  // TMEM columns
  static constexpr uint32_t kTdV = 0;
  static constexpr uint32_t kTdK = D;
  static constexpr uint32_t kTS = 2 * D;        // S^T, then P^T (16-bit) in place
  static constexpr uint32_t kTdP = 2 * D + 128; // dP^T
  // The dQ partial: at d = 64 two buffers of its own in the free columns, so
  // the next dP^T never waits for the dQ warps; at d = 128 TMEM is full and
  // it reuses dP^T's columns once the compute warps have read them.
  static constexpr int kDqBufs = D == 64 ? 2 : 1;
  // d = 64: the compute warps run one step ahead (P of step g+1 before dS of
  // step g) and the MMA warp issues dV(g+1), S(g+2) before dQ(g), dK(g). That
  // needs S(g+2)'s Q tile loaded before dK(g) frees a stage: kStages >= 3.
  static constexpr bool kSkew = D == 64;
  static_assert(!kSkew || kStages >= 3, "the skewed schedule needs a third Q/dO stage");
  // setmaxnreg budgets per warpgroup (one warp of each on every SM
  // sub-partition); they add up to the 4 x 128 the CTA is launched with.
  static constexpr int kRegsProd = 112;
  static constexpr int kRegsCompute = D == 64 ? 152 : 120;  // x 2 warpgroups
  static constexpr int kRegsDQ = D == 64 ? 96 : 160;
  static_assert(kRegsProd + 2 * kRegsCompute + kRegsDQ == 512, "register split must use the launch allocation");
  __host__ __device__ static constexpr uint32_t tdq(int b) { return D == 64 ? 384u + 64u * b : kTdP; }
  static constexpr int kThreads = 512;
};

struct BwdBarriers {
  uint64_t kv_full, kv_empty;
  uint64_t qdo_full[4], qdo_empty[4];
  uint64_t s_full, dp_full, p_ready, ds_ready, ds_free;
  uint64_t dq_full[2], dq_empty[2];  // per dQ-partial buffer
  uint64_t acc_full, acc_empty, drain;
  uint64_t item_full[2], item_empty[2];
  uint64_t dq_turn;            // dQ warpgroup: "our turn to add"
  uint64_t dq_added[4];        // step g's 128 rows are in (ring by g % 4)
  uint64_t dq_rel[4];          // the release warp has published step g
  int item[2];
  int dq_go;     // the ordering wait succeeded
  int dq_fail;   // some row of the step was not added (sticky)
  uint64_t fin_turn, fin_done;  // dQ warpgroup, finishing query tiles: tile chosen / tile read
  int fin_tile;  // the query tile being finished (or past the last one)
  int fin_ok;    // its sums are complete
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Invalidate one 128-byte L2 line without writing it back (its data is dead).
__device__ __forceinline__ void discard_l2(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}


// Work items and the dQ order.
//
// An item is (head bh, key tile j) and runs T steps; its s-th step visits
// query tile tile(s) = j, j+1, ..., n-1 and then (non-causal only) 0, 1, ...,
// j-1. Items are handed out head by head, in descending j within a head.
// Query tile i collects its dQ in two fp32 sums, each over key tiles in
// descending j; the contributor with pos(i) = 0 stores, the rest add, each
// after the previous one has published; dQ = scale * (sum 0 + sum 1).
//   non-causal: sum 0 (lower) from j = i, i-1, ..., 0 and sum 1 (upper) from
//     j = n-1, n-2, ..., i+1; a contributor waits for j + 1, which visited
//     the tile one step earlier.
//   causal (every key tile j <= i contributes): sum j % 2 from the key tiles
//     of that parity, j = i or i-1, then two less each time; a contributor
//     waits for j + 2, which visited the tile two steps earlier, so items
//     that start together never wait on each other's publication latency.
// The contributor a tile waits for (same head) was fetched earlier, so the
// earliest-fetched unfinished item never waits (no deadlock). (Host-callable
// too, so these properties are checked on the CPU.)
struct BwdItem {
  int bh, j, T, n;
  bool causal;
  __host__ __device__ __forceinline__ int tile(int s) const { return j + s < n ? j + s : j + s - n; }
  __host__ __device__ __forceinline__ int chain(int i) const { return causal ? (j & 1) : (i >= j ? 0 : 1); }
  __host__ __device__ __forceinline__ int pos(int i) const {
    return causal ? (i - j) >> 1 : (i >= j ? i - j : n - 1 - j);
  }
};

// Number of key tiles that add into sum c of query tile i of a head with nt
// key tiles (the finishing step waits for this many publications).
__host__ __device__ __forceinline__ int sum_contributors(int i, int nt, bool causal, int c) {
  if (causal) return c == 0 ? i / 2 + 1 : (i + 1) / 2;  // even / odd j <= i
  return c == 0 ? i + 1 : nt - 1 - i;                   // j <= i / j > i
}

// Item number p of a launch over heads of ntiles key tiles each. Non-causal
// (or group = 1): head by head, descending j within a head. Causal: groups of
// `group` heads, and within a group the k-th item (descending j) of every
// head before the (k+1)-th of any, so the group's long last items start
// earlier than head by head and the launch ends on a shorter tail. The host
// sizes the group so that its heads' Q, dO and dQ sums stay in L2.
__host__ __device__ __forceinline__ BwdItem decode_item(int p, int ntiles, bool causal, int heads, int group) {
  BwdItem it;
  if (causal && group > 1) {
    const int per_group = group * ntiles;
    const int g = p / per_group, r = p % per_group;
    const int gh = heads - g * group < group ? heads - g * group : group;
    it.bh = g * group + r % gh;
    it.j = ntiles - 1 - r / gh;
  } else {
    it.bh = p / ntiles;
    it.j = ntiles - 1 - p % ntiles;  // descending j within a head
  }
  it.n = ntiles;
  it.T = causal ? ntiles - it.j : ntiles;
  it.causal = causal;
  return it;
}

// Item number p of this launch with its sequence's rows. A variable-length
// sequence shorter than N has fewer key tiles (w.n); its items past them are
// empty (T = 0) and are skipped by the producer, never handed to the roles.
template <bool CAUSAL>
__device__ __forceinline__ BwdItem item_of(const BwdArgs& a, int p, SeqRows* seq) {
  BwdItem w = decode_item(p, a.ntiles, CAUSAL, a.B * a.H, a.hgroup);
  *seq = seq_rows(a.cu, w.bh / a.H, a.N, a.total);
  w.n = (seq->len + 127) / 128;
  w.T = w.j < w.n ? (CAUSAL ? w.n - w.j : w.n) : 0;
  return w;
}

template <int D, bool CAUSAL, bool BF16, bool DROPOUT>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_dkdv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1 KB aligned base
    if (threadIdx.x == 0) atomicCAS(&g_status, 0, 3 /*FA_ERR_CUDA*/);
    return;
  }
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::kBar);
  volatile int* abort = &bars->abort;
  const int total_items = a.B * a.H * a.ntiles;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->qdo_full[s], 1);
      mbar_init(&bars->qdo_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->item_full[s], 1);
      mbar_init(&bars->item_empty[s], 14);  // MMA + 8 compute warps + 4 dQ warps + release warp
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->ds_free, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->dq_full[b], 1);
      mbar_init(&bars->dq_empty[b], 128);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 256);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->dq_turn, 1);
    mbar_init(&bars->fin_turn, 1);
    mbar_init(&bars->fin_done, 128);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bars->dq_added[q], 128);
      mbar_init(&bars->dq_rel[q], 1);
    }
    bars->dq_fail = 0;
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // Register split per SM sub-partition (one warp of each warpgroup on each):
  // producer/MMA + 2 x compute + dQ = 512 = the 4 x 128 the CTA was launched
  // with (BwdCfg), so no setmaxnreg.inc can wait forever.
  if (warp >= 12) {
    reg_alloc_set<C::kRegsProd, 128>();
    if (warp == 12 && elect_one()) {
      // ------------------------------------------------------------ producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      int g = 0;          // Q/dO loads issued (global step counter)
      int n_item = 0;     // items taken by this CTA
      int kv_loads = 0;   // K/V loads issued
      bool ok = true;
      while (ok) {
        const int slot = n_item & 1;
        if (n_item >= 2) ok = mbar_wait(&bars->item_empty[slot], ((n_item >> 1) & 1) ^ 1, abort);
        if (!ok) break;
        int item;
        BwdItem w;
        SeqRows seq;
        do {  // the next item with work (empty ones exist only when variable-length)
          item = atomicAdd(a.sched, 1);
          if (item < total_items) w = item_of<CAUSAL>(a, item, &seq);
        } while (item < total_items && w.T == 0);
        bars->item[slot] = item < total_items ? item : -1;
        mbar_arrive(&bars->item_full[slot]);
        if (item >= total_items) break;
        const int b = seq.bcoord, h = w.bh % a.H;
        const int krow = seq.row0 + w.j * 128;
        // K_j and V_j are read from HBM once per launch; start bringing them
        // into L2 now (the previous item still has a few steps to run), so
        // their load below waits on L2, not on HBM.
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_prefetch_rows(&tm_k, a.hm & kHmK, kb * 64, h, krow, b);
          tma_prefetch_rows(&tm_v, a.hm & kHmV, kb * 64, h, krow, b);
        }
        for (int k = 0; k < w.T && ok; ++k) {
          const int st = g % C::kStages;
          const int i = w.tile(k);
          if (g >= C::kStages) ok = mbar_wait(&bars->qdo_empty[st], ((g / C::kStages) & 1) ^ 1, abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->qdo_full[st], 2 * C::kTile + 1024);
          for (int kb = 0; kb < D / 64; ++kb) {
            tma_load_rows(&tm_q, a.hm & kHmQ, smem + C::kQ + st * C::kTile + kb * C::kBox, &bars->qdo_full[st],
                          kb * 64, h, seq.row0 + i * 128, b);
            tma_load_rows(&tm_do, a.hm & kHmDO, smem + C::kDO + st * C::kTile + kb * C::kBox, &bars->qdo_full[st],
                          kb * 64, h, seq.row0 + i * 128, b);
          }
          bulk_load(smem + C::kLSE + st * 512, a.lse2 + (size_t)w.bh * a.npad + i * 128, 512, &bars->qdo_full[st]);
          bulk_load(smem + C::kDD + st * 512, a.dd + (size_t)w.bh * a.npad + i * 128, 512, &bars->qdo_full[st]);
          ++g;
          if (k == 0) {
            // K_j, V_j once the previous item released them (after this
            // item's first Q/dO load is already on its way).
            if (kv_loads >= 1) ok = mbar_wait(&bars->kv_empty, (kv_loads - 1) & 1, abort);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTile);
            for (int kb = 0; kb < D / 64; ++kb) {
              tma_load_rows(&tm_k, a.hm & kHmK, smem + C::kK + kb * C::kBox, &bars->kv_full, kb * 64, h, krow, b);
              tma_load_rows(&tm_v, a.hm & kHmV, smem + C::kV + kb * C::kBox, &bars->kv_full, kb * 64, h, krow, b);
            }
            ++kv_loads;
          }
        }
        ++n_item;
      }
      // Never leave with copies in flight: the last load of each stage, and
      // the last K/V load.
      for (int x = (g > C::kStages ? g - C::kStages : 0); x < g; ++x)
        mbar_wait(&bars->qdo_full[x % C::kStages], (x / C::kStages) & 1, abort, false);
      if (kv_loads >= 1) mbar_wait(&bars->kv_full, (kv_loads - 1) & 1, abort, false);
    } else if (warp == 13 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdSq = idesc_f16(BF16, 128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t kIdKM = idesc_f16(BF16, 128, D, false, true);     // dV (A in TMEM), dK
      constexpr uint32_t kIdQ = idesc_f16(BF16, 128, D, true, true);       // dQ part: A = dS (MN-major)
      // Descriptors of the tile bases; a K step only moves the start-address
      // field (bits 0-13, in 16-byte units), which cannot carry out of it here.
      const uint64_t dK_k = sdesc(smem_u32(smem + C::kK), 16, 1024);
      const uint64_t dV_k = sdesc(smem_u32(smem + C::kV), 16, 1024);
      const uint64_t dQ_k = sdesc(smem_u32(smem + C::kQ), 16, 1024);
      const uint64_t dDO_k = sdesc(smem_u32(smem + C::kDO), 16, 1024);
      const uint64_t dDS_k = sdesc(smem_u32(smem + C::kDS), 16, 1024);
      const uint64_t dK_mn = sdesc(smem_u32(smem + C::kK), C::kBox, 1024);
      const uint64_t dQ_mn = sdesc(smem_u32(smem + C::kQ), C::kBox, 1024);
      const uint64_t dDO_mn = sdesc(smem_u32(smem + C::kDO), C::kBox, 1024);
      const uint64_t dDS_mn = sdesc(smem_u32(smem + C::kDS), C::kBox, 1024);
      constexpr uint32_t kStage16 = C::kTile >> 4;
      auto kstep = [](int ks) { return (uint64_t)(((ks / 4) * C::kBox + (ks % 4) * 32) >> 4); };
      auto mstep = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };
      auto issue_st = [&](uint64_t a0, uint64_t b0, uint32_t dst) {  // [128 x 128] over d
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) mma_ss(tmem + dst, a0 + kstep(ks), b0 + kstep(ks), kIdSq, ks > 0);
      };
      int g = 0, n_item = 0;
      bool ok = true;
      while (ok) {
        const int slot = n_item & 1;
        ok = mbar_wait(&bars->item_full[slot], (n_item >> 1) & 1, abort);
        if (!ok) break;
        const int item = bars->item[slot];
        mbar_arrive(&bars->item_empty[slot]);
        if (item < 0) break;
        SeqRows seq;
        const BwdItem w = item_of<CAUSAL>(a, item, &seq);
        ok = mbar_wait(&bars->kv_full, n_item & 1, abort) &&
             mbar_wait(&bars->qdo_full[g % C::kStages], (g / C::kStages) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        issue_st(dK_k, dQ_k + (g % C::kStages) * kStage16, C::kTS);
        mma_commit(&bars->s_full);
        if (C::kDqBufs == 1 && g > 0) ok = mbar_wait(&bars->dq_empty[0], (g - 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        issue_st(dV_k, dDO_k + (g % C::kStages) * kStage16, C::kTdP);
        mma_commit(&bars->dp_full);
        if constexpr (C::kSkew) {
          // Order matches the compute warps, which run one step ahead:
          // P(g+1) arrives before dS(g).
          auto issue_dv = [&](int gs, bool acc) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + C::kTdV, tmem + C::kTS + kk * 8 + (kk >= 4 ? 32 : 0),
                     dDO_mn + (gs % C::kStages) * kStage16 + mstep(kk), kIdKM, (acc || kk > 0));
          };
          ok = mbar_wait(&bars->p_ready, g & 1, abort);
          if (ok && n_item > 0) ok = mbar_wait(&bars->acc_empty, (n_item - 1) & 1, abort);
          if (ok) {
            tc_fence_after();
            issue_dv(g, false);
            if (w.T > 1) {
              ok = mbar_wait(&bars->qdo_full[(g + 1) % C::kStages], ((g + 1) / C::kStages) & 1, abort);
              if (ok) {
                issue_st(dK_k, dQ_k + ((g + 1) % C::kStages) * kStage16, C::kTS);
                mma_commit(&bars->s_full);
              }
            }
          }
          for (int k = 0; k < w.T && ok; ++k, ++g) {
            const int st = g % C::kStages;
            if (k + 1 < w.T) {
              ok = mbar_wait(&bars->p_ready, (g + 1) & 1, abort);
              if (!ok) break;
              tc_fence_after();
              issue_dv(g + 1, true);
              if (k + 2 < w.T) {
                ok = mbar_wait(&bars->qdo_full[(g + 2) % C::kStages], ((g + 2) / C::kStages) & 1, abort);
                if (!ok) break;
                issue_st(dK_k, dQ_k + ((g + 2) % C::kStages) * kStage16, C::kTS);
                mma_commit(&bars->s_full);
              }
            }
            ok = mbar_wait(&bars->ds_ready, g & 1, abort);
            if (!ok) break;
            tc_fence_after();
            if (k + 1 < w.T) {
              issue_st(dV_k, dDO_k + ((g + 1) % C::kStages) * kStage16, C::kTdP);
              mma_commit(&bars->dp_full);
            }
            if (g >= 2) ok = mbar_wait(&bars->dq_empty[g & 1], ((g >> 1) & 1) ^ 1, abort);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + C::tdq(g & 1), dDS_mn + mstep(kk), dK_mn + mstep(kk), kIdQ, kk > 0);
            mma_commit(&bars->dq_full[g & 1]);
#pragma unroll
            for (int kq = 0; kq < 8; ++kq)
              mma_ss(tmem + C::kTdK, dDS_k + kstep(kq), dQ_mn + st * kStage16 + mstep(kq), kIdKM, (k > 0 || kq > 0));
            mma_commit(&bars->ds_free);
            mma_commit(&bars->qdo_empty[st]);
          }
        } else {
          for (int k = 0; k < w.T && ok; ++k, ++g) {
            const int st = g % C::kStages;
            ok = mbar_wait(&bars->p_ready, g & 1, abort);
            if (ok && k == 0 && n_item > 0) ok = mbar_wait(&bars->acc_empty, (n_item - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
            // dV += P^T dO   (A = P^T in TMEM, 16-bit packed)
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + C::kTdV, tmem + C::kTS + kk * 8 + (kk >= 4 ? 32 : 0), dDO_mn + st * kStage16 + mstep(kk),
                     kIdKM, (k > 0 || kk > 0));
            if (k + 1 < w.T) {
              ok = mbar_wait(&bars->qdo_full[(g + 1) % C::kStages], ((g + 1) / C::kStages) & 1, abort);
              if (!ok) break;
              issue_st(dK_k, dQ_k + ((g + 1) % C::kStages) * kStage16, C::kTS);
              mma_commit(&bars->s_full);
            }
            ok = mbar_wait(&bars->ds_ready, g & 1, abort);
            if (!ok) break;
            tc_fence_after();
            if (C::kDqBufs == 2 && k + 1 < w.T) {
              // dP^T(g+1) has its own columns here: issue it ahead of dQ(g) and
              // dK(g) so the compute warps' next dS phase does not queue behind them.
              issue_st(dV_k, dDO_k + ((g + 1) % C::kStages) * kStage16, C::kTdP);
              mma_commit(&bars->dp_full);
            }
            // With two dQ buffers, buffer g % 2 is free once the dQ warps have
            // read step g - 2 out of it.
            if (C::kDqBufs == 2 && g >= 2) ok = mbar_wait(&bars->dq_empty[g & 1], ((g >> 1) & 1) ^ 1, abort);
            if (!ok) break;
            tc_fence_after();
            // dQ_part = dS K   (A = dS: dS^T stored [key][query] -> MN-major)
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + C::tdq(g % C::kDqBufs), dDS_mn + mstep(kk), dK_mn + mstep(kk), kIdQ, kk > 0);
            mma_commit(&bars->dq_full[g % C::kDqBufs]);
            // dK += dS^T Q   (A = dS^T K-major)
  #pragma unroll
            for (int kq = 0; kq < 8; ++kq)
              mma_ss(tmem + C::kTdK, dDS_k + kstep(kq), dQ_mn + st * kStage16 + mstep(kq), kIdKM, (k > 0 || kq > 0));
            mma_commit(&bars->ds_free);
            mma_commit(&bars->qdo_empty[st]);
            if (C::kDqBufs == 1 && k + 1 < w.T) {
              ok = mbar_wait(&bars->dq_empty[0], g & 1, abort);
              if (!ok) break;
              tc_fence_after();
              issue_st(dV_k, dDO_k + ((g + 1) % C::kStages) * kStage16, C::kTdP);
              mma_commit(&bars->dp_full);
            }
          }
        }
        if (!ok) break;
        mma_commit(&bars->acc_full);
        mma_commit(&bars->kv_empty);
        ++n_item;
      }
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, abort, false);
    } else if (warp == 14 && lane == 0) {
      // ------------------------------------------------------- release warp
      // Publishes each step's dQ additions: waits until all 128 rows of the
      // step are in (CTA-scope acquire), then one gpu-scope release store of
      // the tile's counter lets the next contributor add.
      int g = 0, n_item = 0;
      bool ok = true;
      while (ok) {
        const int slot = n_item & 1;
        ok = mbar_wait(&bars->item_full[slot], (n_item >> 1) & 1, abort);
        if (!ok) break;
        const int item = bars->item[slot];
        mbar_arrive(&bars->item_empty[slot]);
        if (item < 0) break;
        SeqRows seq;
        const BwdItem w = item_of<CAUSAL>(a, item, &seq);
        for (int k = 0; k < w.T; ++k, ++g) {
          const int i = w.tile(k);
          if (!mbar_wait(&bars->dq_added[g & 3], (g >> 2) & 1, abort)) { ok = false; break; }
          if (bars->dq_fail) { ok = false; break; }
          st_release(a.cnt + (size_t)w.chain(i) * a.B * a.H * a.ntiles + (size_t)w.bh * a.ntiles + i, w.pos(i) + 1);
          mbar_arrive(&bars->dq_rel[g & 3]);
        }
        if (!ok) break;
        ++n_item;
      }
    }
  } else if (warp < 8) {
    reg_alloc_set<C::kRegsCompute, 128>();
    // ------------------------------------------------------- compute warps
    // Thread = key row c (TMEM lane); warpgroup wg takes query columns
    // [64 wg, 64 wg + 64) of each 128 x 128 step.
    const int wg = warp / 4;
    const int quad = warp % 4;
    const int c = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint64_t c2 = bcast2(a.scale_log2);  // (scale log2(e), scale log2(e))
    const float* sLSE = reinterpret_cast<const float*>(smem + C::kLSE);
    const float* sDD = reinterpret_cast<const float*>(smem + C::kDD);
    uint8_t* sDS = smem + C::kDS + wg * C::kBox;  // this warpgroup's 64 query columns
    int g = 0, n_item = 0;
    bool ok = true;
    while (ok) {
      const int slot = n_item & 1;
      ok = wg_all(mbar_wait_warp(&bars->item_full[slot], (n_item >> 1) & 1, abort), 1 + wg);
      if (!ok) break;
      const int item = bars->item[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->item_empty[slot]);
      if (item < 0) break;
      SeqRows seq;
      const BwdItem w = item_of<CAUSAL>(a, item, &seq);
      const int key = w.j * 128 + c;
      // A key row past the sequence's end (the next sequence's rows when
      // variable-length, TMA zeros otherwise) gets P = 0, so it adds nothing
      // to dQ, and its dK, dV rows are not stored.
      const bool key_in = key < seq.len;
      // P^T = exp2(S^T * c - LSE2) of step gs (query tile i) for this thread's
      // 64 queries, packed two per word into pk and written to TMEM over S^T
      // (columns this warpgroup has already read).
      auto p_phase = [&](int gs, int i, uint32_t* pk, uint64_t& keep) -> bool {
        const int st = gs % C::kStages;
        const bool diag = CAUSAL && i == w.j;
        if constexpr (DROPOUT) {
          // Keep bits of this thread's key for its 64 query columns. The four
          // lanes of a key group (keys 4g .. 4g+3) each draw one Philox call
          // for one query of a block of four, then trade words (a 4 x 4
          // transpose by shuffles) so that each lane holds its own key's draw
          // for all four queries.
          keep = 0;
          const uint32_t grp = static_cast<uint32_t>(key) >> 2;
          const int k4 = lane & 3;
#pragma unroll 4
          for (int blk = 0; blk < 16; ++blk) {
            const uint32_t iq0 = static_cast<uint32_t>(i * 128 + wg * 64 + 4 * blk);
            const uint4 wv = philox4x32_10(make_uint4(grp, iq0 + k4, w.bh, a.drop.offset), a.drop.seed_lo,
                                           a.drop.seed_hi);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int idx = (k4 - q) & 3;
              const uint32_t send = idx == 0 ? wv.x : idx == 1 ? wv.y : idx == 2 ? wv.z : wv.w;
              const int src = (k4 + q) & 3;
              const uint32_t got = __shfl_sync(0xffffffffu, send, (lane & ~3) | src);
              keep |= static_cast<uint64_t>(got >= a.drop.thr ? 1u : 0u) << (4 * blk + src);
            }
          }
        }
        if (!mbar_wait_warp(&bars->s_full, gs & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t sv[32];
          tmem_ld32(lane_base + C::kTS + wg * 64 + h2 * 32, sv);
          tmem_ld_wait();
          tie_regs32(sv);
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int qc = wg * 64 + h2 * 32 + 2 * x;
            // (S c - LSE2) for two queries: the smem row holds -LSE2.
            const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(sLSE + st * 128 + qc);
            float x0, x1;
            fma2(x0, x1, __uint_as_float(sv[2 * x]), __uint_as_float(sv[2 * x + 1]), c2, nl2);
            pk[h2 * 16 + x] = pack2<BF16>(ex2(x0), ex2(x1));
          }
          // The diagonal tile: keys after the query are masked, once per
          // packed pair (only this step pays for it).
          if (diag) {
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const int q0 = i * 128 + wg * 64 + h2 * 32 + 2 * x;
              pk[h2 * 16 + x] &= (key > q0 ? 0u : 0x0000FFFFu) | (key > q0 + 1 ? 0u : 0xFFFF0000u);
            }
          }
          // Past the sequence's end (only a key tile's tail): P = 0. Applied
          // once to the packed row rather than per element, which kept the
          // common path 4% faster.
          if (!key_in) {
#pragma unroll
            for (int x = 0; x < 16; ++x) pk[h2 * 16 + x] = 0u;
          }
          if constexpr (DROPOUT) {
            // dV uses the dropped P (its 1 / (1 - p) is applied to dV at the
            // end); dS below needs every P, so pk keeps them.
            uint32_t pm[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const int col = h2 * 32 + 2 * x;
              pm[x] = pk[h2 * 16 + x] & (((keep >> col) & 1u ? 0x0000FFFFu : 0u) |
                                         ((keep >> (col + 1)) & 1u ? 0xFFFF0000u : 0u));
            }
            tmem_st16(lane_base + C::kTS + wg * 64 + h2 * 16, pm);
          }
        }
        if constexpr (!DROPOUT) tmem_st32(lane_base + C::kTS + wg * 64, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
        return true;
      };
      // dS^T = P^T o (dP^T - D) of step gs -> shared memory (16-bit), from the
      // same rounded P that the dV product uses.
      auto ds_phase = [&](int gs, const uint32_t* pk, uint64_t keep) -> bool {
        const int st = gs % C::kStages;
        if (!mbar_wait_warp(&bars->dp_full, gs & 1, abort)) return false;
        if (gs > 0 && !mbar_wait_warp(&bars->ds_free, (gs - 1) & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t dp[32];
          tmem_ld32(lane_base + C::kTdP + wg * 64 + h2 * 32, dp);
          tmem_ld_wait();
          tie_regs32(dp);
          uint32_t dsk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int qc = wg * 64 + h2 * 32 + 2 * x;
            const float2 pp = unpack2<BF16>(pk[h2 * 16 + x]);
            const uint64_t dd2 = *reinterpret_cast<const uint64_t*>(sDD + st * 128 + qc);
            float dp0 = __uint_as_float(dp[2 * x]), dp1 = __uint_as_float(dp[2 * x + 1]);
            if constexpr (DROPOUT) {
              // dP = (dO V^T) o keep / (1 - p)
              const int col = h2 * 32 + 2 * x;
              dp0 = (keep >> col) & 1u ? dp0 * a.drop.rkeep : 0.f;
              dp1 = (keep >> (col + 1)) & 1u ? dp1 * a.drop.rkeep : 0.f;
            }
            float d0, d1;
            mul_sub2(d0, d1, pp.x, pp.y, dp0, dp1, dd2);
            dsk[x] = pack2<BF16>(d0, d1);
          }
          // Row c of a 128-byte-swizzled [128][64] box: 16-byte chunk x goes
          // to x ^ (c % 8).
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int chunk = h2 * 4 + x;
            uint4* dst = reinterpret_cast<uint4*>(sDS + c * 128 + ((chunk ^ (c & 7)) * 16));
            *dst = make_uint4(dsk[4 * x], dsk[4 * x + 1], dsk[4 * x + 2], dsk[4 * x + 3]);
          }
        }
        tc_fence_before();  // dP^T reads done before the next MMA may reuse these columns
        fence_proxy_async_smem();
        mbar_arrive(&bars->ds_ready);
        return true;
      };
      // Software-pipelined by one step: P of step g+1 is computed before dS
      // of step g, so dS(g) finds dP(g) finished (it was issued a whole P
      // phase earlier) and P(g+1) only waits for dV(g) and S(g+1).
      if constexpr (C::kSkew) {
        uint32_t pk_cur[32], pk_next[32];
        uint64_t keep_cur = 0, keep_next = 0;
        if (!p_phase(g, w.tile(0), pk_cur, keep_cur)) { ok = false; break; }
        for (int k = 0; k < w.T; ++k, ++g) {
          if (k + 1 < w.T && !p_phase(g + 1, w.tile(k + 1), pk_next, keep_next)) { ok = false; break; }
          if (!ds_phase(g, pk_cur, keep_cur)) { ok = false; break; }
          keep_cur = keep_next;
#pragma unroll
          for (int x = 0; x < 32; ++x) pk_cur[x] = pk_next[x];
        }
      } else {
        for (int k = 0; k < w.T; ++k, ++g) {
          uint32_t pk[32];
          uint64_t keep = 0;
          if (!p_phase(g, w.tile(k), pk, keep) || !ds_phase(g, pk, keep)) { ok = false; break; }
        }
      }
      // The warpgroup agrees on going on, so that all of it or none reaches
      // the epilogue's warpgroup barriers.
      ok = wg_all(ok, 1 + wg);
      if (!ok) break;
      // ---- epilogue: warpgroup 0 stores dV_j, warpgroup 1 stores scale * dK_j
      ok = wg_all(mbar_wait_warp(&bars->acc_full, n_item & 1, abort), 1 + wg);
      if (!ok) break;
      tc_fence_after();
      const int b = w.bh / a.H, h = w.bh % a.H;
      const float mul = wg == 0 ? (DROPOUT ? a.drop.rkeep : 1.f) : a.scale;
      const uint32_t src = lane_base + (wg == 0 ? C::kTdV : C::kTdK);
      const int tile0 = w.j * 128;
      if (a.cu == nullptr || tile0 + 128 <= seq.len) {
        // Through this warpgroup's dS box (every MMA of the item, the last
        // dS readers included, completed before acc_full) and a TMA store,
        // 64 columns at a time; rows past N are clipped by the tensor map.
        const CUtensorMap* map = wg == 0 ? &tm_dv : &tm_dk;
        const bool hm = a.hm & (wg == 0 ? kHmDV : kHmDK);
#pragma unroll 1
        for (int kb = 0; kb < D / 64; ++kb) {
          if (kb > 0) {
            if (c == 0) bulk_wait_read_all();
            named_bar_sync(1 + wg, 128);
          }
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            uint32_t v[32];
            tmem_ld32(src + (kb * 2 + q2) * 32, v);
            tmem_ld_wait();
            tie_regs32(v);
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 16; ++x)
              pk[x] = pack2<BF16>(__uint_as_float(v[2 * x]) * mul, __uint_as_float(v[2 * x + 1]) * mul);
#pragma unroll
            for (int y = 0; y < 4; ++y)
              st_shared_v4(sDS + c * 128 + (((q2 * 4 + y) ^ (c & 7)) << 4), pk[4 * y], pk[4 * y + 1], pk[4 * y + 2],
                           pk[4 * y + 3]);
          }
          fence_async_shared();
          named_bar_sync(1 + wg, 128);
          if (c == 0) {
            tma_store_rows(map, hm, sDS, kb * 64, h, seq.row0 + tile0, seq.bcoord);
            bulk_commit();
          }
        }
        // The next item's dS phase writes the box again.
        if (c == 0) bulk_wait_read_all();
        named_bar_sync(1 + wg, 128);
      } else {
        const bool valid = key_in;
        const long long r = seq.row0 + (valid ? key : 0);
        uint16_t* dst = wg == 0 ? a.dv + b * a.dv_sb + r * a.dv_sn + h * a.dv_sh
                                : a.dk + b * a.dk_sb + r * a.dk_sn + h * a.dk_sh;
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
          uint32_t v[32];
          tmem_ld32(src + q * 32, v);
          tmem_ld_wait();
          tie_regs32(v);
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x] = pack2<BF16>(__uint_as_float(v[2 * x]) * mul, __uint_as_float(v[2 * x + 1]) * mul);
          if (valid) {
            uint4* o4 = reinterpret_cast<uint4*>(dst + q * 32);
#pragma unroll
            for (int y = 0; y < 4; ++y)
              if (q * 32 + y * 8 < a.d) o4[y] = make_uint4(pk[4 * y], pk[4 * y + 1], pk[4 * y + 2], pk[4 * y + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      ++n_item;
    }
    // dK / dV stores have completed before the CTA leaves.
    if (c == 0) bulk_wait_all();
  } else {
    reg_alloc_set<C::kRegsDQ, 128>();
    // ------------------------------------------------------ dQ warps (8-11)
    // Thread = query row r of the step (TMEM lane).
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const uint32_t src0 = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    int g = 0, n_item = 0;
    bool ok = true;
    while (ok) {
      const int slot = n_item & 1;
      ok = mbar_wait_warp(&bars->item_full[slot], (n_item >> 1) & 1, abort);
      if (!ok) break;
      const int item = bars->item[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->item_empty[slot]);
      if (item < 0) break;
      SeqRows seq;
      const BwdItem w = item_of<CAUSAL>(a, item, &seq);
      for (int k = 0; k < w.T; ++k, ++g) {
        const int i = w.tile(k);
        // The warpgroup synchronises through two mbarriers (bounded waits, no
        // named barriers), so a warp that gives up cannot strand the others.
        const int buf = g % C::kDqBufs;
        const uint32_t src = src0 + C::tdq(buf);
        const bool got = mbar_wait_warp(&bars->dq_full[buf], (g / C::kDqBufs) & 1, abort);
        uint32_t v[D];
        if (got) {
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < D / 32; ++q) tmem_ld32(src + q * 32, v + q * 32);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < D / 32; ++q) tie_regs32(v + q * 32);
          tc_fence_before();
          mbar_arrive(&bars->dq_empty[buf]);
        }
        // Thread 256 waits until the previous contributor to tile i has
        // added its part (and until the release warp has published this
        // CTA's previous step), then opens the turn for the warpgroup.
        const size_t chain_off = (size_t)w.chain(i) * a.B * a.H * a.ntiles;
        const size_t tile = (size_t)w.bh * a.ntiles + i + chain_off;
        const int pos = w.pos(i);
        if (threadIdx.x == 256) {
          bool go = got;
          // Publishing step g-4 must be done before step g reuses its
          // barriers; steps g-3 .. g-1 may still be waiting for their adds
          // to complete in L2, which is the latency this ring hides.
          if (go && g >= 4) go = mbar_wait(&bars->dq_rel[g & 3], ((g - 4) >> 2) & 1, abort);
          // Every thread has passed turn g-1 (its adds are issued, not
          // necessarily complete) before turn g reuses the single turn barrier.
          if (go && g >= 1) go = mbar_wait(&bars->dq_added[(g - 1) & 3], ((g - 1) >> 2) & 1, abort);
          const int* cnt = a.cnt + tile;
          if (go && pos > 0 && ld_acquire(cnt) != pos) {
            const uint64_t t0 = globaltimer();
            for (uint32_t n = 1;; ++n) {
              if (ld_acquire(cnt) == pos) break;
              if ((n & 63u) == 0) {
                if (*abort) { go = false; break; }
                if (globaltimer() - t0 > FA_WAIT_LIMIT_NS) {
                  record_timeout(2);
                  *abort = 1;
                  go = false;
                  break;
                }
              }
              __nanosleep(32);
            }
          }
          bars->dq_go = go ? 1 : 0;
          mbar_arrive(&bars->dq_turn);
        }
        const bool turn = __all_sync(0xffffffffu, mbar_wait(&bars->dq_turn, g & 1, abort) && bars->dq_go);
        const bool step_ok = got && turn;
        if (step_ok) {
          float* acc = a.dqacc + tile * 128 * D;
#pragma unroll
          for (int q = 0; q < D / 4; ++q) {
            float* p4 = acc + ((size_t)q * 128 + r) * 4;
            if (pos == 0)
              *reinterpret_cast<float4*>(p4) = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                           __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
            else
              red_add_v4(p4, __uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                         __uint_as_float(v[4 * q + 3]));
          }
        } else {
          bars->dq_fail = 1;
        }
        // No fence here: the release warp publishes the step with one
        // gpu-scope release after all 128 rows have arrived (the arrival is a
        // CTA-scope release, so every add is ordered before that store).
        mbar_arrive(&bars->dq_added[g & 3]);
        if (!step_ok) { ok = false; break; }
      }
      if (!ok) break;
      ++n_item;
    }
    // ---- dQ of finished query tiles. Once the item queue is empty, the
    // warpgroup takes query tiles from a second counter (head by head, so
    // the tiles finished first come first), waits until each of the tile's
    // two sums has all its contributions (its counter reaches the number of
    // contributors), and writes dQ = scale * (sum 0 + sum 1), added in that
    // order. The sums are dead afterwards and their L2 lines are dropped
    // without a write-back. Every contributor was fetched before the queue
    // ran empty and waits on nothing here, so these waits end.
    const int total_tiles = a.B * a.H * a.ntiles;
    const size_t sum_stride = (size_t)a.B * a.H * a.npad * D;  // floats per sum
    for (int nf = 0; ok; ++nf) {
      if (threadIdx.x == 256) {
        const int f = atomicAdd(a.sched + 1, 1);
        bool go = true;
        if (f < total_tiles) {
          const int bh = f / a.ntiles, i = f % a.ntiles;
          const SeqRows sq = seq_rows(a.cu, bh / a.H, a.N, a.total);
          const int nt = (sq.len + 127) / 128;
          if (i < nt) {
            const int want0 = sum_contributors(i, nt, CAUSAL, 0);
            const int want1 = sum_contributors(i, nt, CAUSAL, 1);
            const int* c0 = a.cnt + (size_t)bh * a.ntiles + i;
            const int* c1 = c0 + (size_t)a.B * a.H * a.ntiles;
            if (ld_acquire(c0) != want0 || ld_acquire(c1) != want1) {
              const uint64_t t0 = globaltimer();
              for (uint32_t n = 1;; ++n) {
                if (ld_acquire(c0) == want0 && ld_acquire(c1) == want1) break;
                if ((n & 63u) == 0) {
                  if (*abort) { go = false; break; }
                  if (globaltimer() - t0 > FA_WAIT_LIMIT_NS) {
                    record_timeout(2);
                    *abort = 1;
                    go = false;
                    break;
                  }
                }
                __nanosleep(64);
              }
            }
          }
        }
        bars->fin_tile = f;
        bars->fin_ok = go ? 1 : 0;
        mbar_arrive(&bars->fin_turn);
      }
      if (!mbar_wait_warp(&bars->fin_turn, nf & 1, abort)) { ok = false; break; }
      const int f = bars->fin_tile;
      if (!bars->fin_ok) { ok = false; break; }
      if (f >= total_tiles) break;
      const int bh = f / a.ntiles, i = f % a.ntiles;
      const int b = bh / a.H, h = bh % a.H;
      const SeqRows sq = seq_rows(a.cu, b, a.N, a.total);
      const int nt = (sq.len + 127) / 128;
      const float* s0 = a.dqacc + ((size_t)bh * a.ntiles + i) * 128 * D;  // [D/4][128][4]
      const float* s1 = s0 + sum_stride;
      const bool has1 = sum_contributors(i, nt, CAUSAL, 1) > 0;
      if (i < nt) {
        const int n = i * 128 + r;
        const bool valid = n < sq.len;
        uint16_t* drow = a.dq + b * a.dq_sb + (sq.row0 + (valid ? n : 0)) * a.dq_sn + h * a.dq_sh;
#pragma unroll 1
        for (int q0 = 0; q0 < D / 4; q0 += 8) {
          float4 x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = __ldcg(reinterpret_cast<const float4*>(s0) + (q0 + k) * 128 + r);
          if (has1) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 u = __ldcg(reinterpret_cast<const float4*>(s1) + (q0 + k) * 128 + r);
              x[k].x += u.x;
              x[k].y += u.y;
              x[k].z += u.z;
              x[k].w += u.w;
            }
          }
          if (valid) {
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const int col = (q0 + k) * 4;
              if (col < a.d)
                *reinterpret_cast<uint4*>(drow + col) = make_uint4(
                    pack2<BF16>(x[k].x * a.scale, x[k].y * a.scale), pack2<BF16>(x[k].z * a.scale, x[k].w * a.scale),
                    pack2<BF16>(x[k + 1].x * a.scale, x[k + 1].y * a.scale),
                    pack2<BF16>(x[k + 1].z * a.scale, x[k + 1].w * a.scale));
            }
          }
        }
      }
      // Every row of the tile has been read: drop the sums' lines.
      mbar_arrive(&bars->fin_done);
      if (!mbar_wait_warp(&bars->fin_done, nf & 1, abort)) { ok = false; break; }
      if (i < nt) {
        for (int line = r; line < 4 * D; line += 128) {
          discard_l2(reinterpret_cast<const char*>(s0) + 128 * line);
          if (has1) discard_l2(reinterpret_cast<const char*>(s1) + 128 * line);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
