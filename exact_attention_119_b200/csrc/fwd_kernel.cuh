// Forward kernel: O = softmax(scale * Q K^T [+causal]) V and the row LSE.
//
// Method (lab write-up "从Attention矩阵到显存读写：FlashAttention真正解决的痛点",
// §3.1 tiling and §3.2 online softmax; "使用FlashAttention优化PyTorch模型注意力
// 计算", "核融合" and "分块处理"): each CTA owns 256 query rows of one (batch,
// head) as two 128-row tiles and streams the K/V tiles of that head through a
// shared-memory ring. S = Q K_j^T goes to tensor memory (TMEM) by tcgen05 MMA,
// the softmax warps turn it into P in place (16-bit, aliasing S's columns),
// and O += P V_j accumulates in TMEM. S and P never leave the SM.
//
// Roles (12 warps = 3 warpgroups):
//   warps 0-3  softmax + epilogue for Q tile 0 (thread = row = TMEM lane)
//   warps 4-7  softmax + epilogue for Q tile 1
//   warp  8    TMA producer; owns the TMEM allocation
//   warp  9    MMA issuer (one thread)
//   warps 10-11 idle (they complete the third warpgroup, which hands
//               registers to the softmax warpgroups)
// The two tiles ping-pong: while one softmax warpgroup works on its S, the
// tensor core runs the other tile's P V and next S.
//
// At d = 64 TMEM has room for P next to S (kSepP): the softmax signals "S
// consumed" as soon as S is in registers, so S of the next key tile is
// computed while the softmax is still busy with exponentials, and the
// exponential unit is not left idle waiting for the next S. At d = 128 P
// overwrites S in place and the next S follows P V.
//
// Split (SPLIT = true, non-causal launches that would leave SMs idle): the two
// CTAs of a 2-CTA cluster take the first and second half of a row block's key
// tiles, and CTA 0 merges CTA 1's online-softmax state (unnormalised O, m, l)
// through the cluster's shared-memory window before writing O and LSE.
//
// Online softmax with a lagging reference max: the running max m (log2
// units) is only moved, and O and l rescaled, when a tile's max exceeds m by
// more than kRescaleLog2 (so P <= 2^kRescaleLog2). The final O / l and
// LSE = m ln2 + ln l use that same m, so the result is exact, not approximate.
#pragma once

#include <climits>

#include "sm100.cuh"

namespace fa {

constexpr float kRescaleLog2 = 8.0f;

struct FwdArgs {
  uint16_t* o;                    // element (b, n, h, c) at o[b*o_sb + (row0 + n)*o_sn + h*o_sh + c]
  long long o_sb, o_sn, o_sh;
  float* lse;                     // row LSE at lse[b*lse_sb + h*lse_sh + row0 + n]
  long long lse_sb, lse_sh;
  const int* cu;                  // variable-length row offsets [B + 1], or nullptr
  int total;                      // rows of the packed tensors (variable length)
  int B, N, H;                    // N: sequence length (variable length: the longest)
  int d;                          // head size (<= D; columns d .. D-1 are zeros from TMA)
  uint32_t hm;                    // head-major tensor maps (kHmQ | kHmK | kHmV)
  Dropout drop;                   // used by the DROPOUT instantiation only
  int n_mblocks;                  // ceil(N / 256)
  int split;                      // 1, or 2: each row block's key tiles shared by a 2-CTA cluster
  float scale_log2;               // softmax_scale * log2(e)
};

template <int D>
struct FwdCfg {
  static constexpr int kRows = 128;                   // rows per Q tile (MMA M)
  static constexpr int kKeys = 128;                   // keys per K/V tile (MMA N of S)
  static constexpr int kBoxBytes = 128 * 128;         // one TMA box: 128 rows x 64 elems x 2 B
  static constexpr int kTileBytes = 128 * D * 2;      // one Q, K or V tile
  static constexpr int kStages = (D == 128) ? 4 : 8;  // K/V ring depth
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  static constexpr int kOStOff = kBarOff + 1024;  // O staging: one box per Q tile
  static constexpr int kSmemBytes = kOStOff + 2 * kBoxBytes + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  // A split row block's partial state (2 tiles x 128 rows x (D + 4) floats)
  // goes over Q and the K/V ring at the end.
  static_assert(2 * 128 * (D + 4) * 4 <= kBarOff, "partial rows must fit below the barriers");
  // TMEM columns: S of tile t at tmem_s(t), O at tmem_o(t), P at tmem_p(t)
  // (its own 64 columns when kSepP, else over S).
  static constexpr bool kSepP = D == 64;
  __host__ __device__ static constexpr uint32_t tmem_s(int t) { return t ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tmem_o(int t) { return t ? 256u + D : 256u; }
  __host__ __device__ static constexpr uint32_t tmem_p(int t) { return kSepP ? 384u + 64u * t : tmem_s(t); }
  static constexpr int kThreads = 384;
};

struct FwdBarriers {
  uint64_t q_full;
  uint64_t q_empty;     // the item's last S MMA has read Q: the next Q may be loaded
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t p_half[2];   // without kSepP: P of the tile's first 64 keys is in TMEM
  uint64_t o_full[2];
  uint64_t s_cons[2];   // kSepP: the softmax has S(t, j) in registers
  uint64_t pv_done[2];  // kSepP: P(t, j) V_j has completed
  uint64_t drain;
  uint64_t merge_ready;  // split: the partner's partial rows are in its shared memory
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort;
};

// One work item: 256 query rows (two 128-row tiles) of one (batch, head),
// and the key tiles this CTA visits for them.
struct FwdItem {
  int b, h, bh, q0, kv_lo, n_kv;
  SeqRows seq;
};

// Items of a launch are numbered 0 .. n_mblocks * B * H - 1. Causal: row
// blocks slowest and last-first (longest first), so the launch ends on short
// ones. Non-causal (all equal): a head's row blocks next to each other, so
// the CTAs working on one head at the same time share its K and V through L2.
template <bool CAUSAL, bool SPLIT, bool VARLEN, int KEYS>
__device__ __forceinline__ FwdItem fwd_item(const FwdArgs& args, int item, uint32_t crank) {
  const int bh_count = args.B * args.H;
  FwdItem w;
  int mblk;
  if (CAUSAL) {
    mblk = args.n_mblocks - 1 - item / bh_count;
    w.bh = item % bh_count;
  } else {
    mblk = item % args.n_mblocks;
    w.bh = item / args.n_mblocks;
  }
  w.b = w.bh / args.H;
  w.h = w.bh % args.H;
  w.q0 = mblk * 256;
  w.seq = VARLEN ? seq_rows(args.cu, w.b, args.N, args.total) : SeqRows{0, args.N, w.b};
  const int kv_end = CAUSAL ? min(w.seq.len, w.q0 + 256) : w.seq.len;
  const int n_all = (kv_end + KEYS - 1) / KEYS;
  const int half = (n_all + 1) / 2;
  w.kv_lo = SPLIT && crank == 1 ? half : 0;
  w.n_kv = !SPLIT ? n_all : (crank == 0 ? half : n_all - half);
  return w;
}

// The k-th item of this CTA. PERSISTENT: the CTAs take items in a
// back-and-forth ("snake") order over rounds of gridDim.x, which evens out
// the causal lengths. Otherwise one item per CTA (per CTA pair when split),
// known at compile time, so the item loop folds away.
template <bool SPLIT, bool PERSISTENT>
__device__ __forceinline__ int fwd_item_index(int k) {
  if (!PERSISTENT) return k == 0 ? static_cast<int>(SPLIT ? blockIdx.x / 2 : blockIdx.x) : INT_MAX;
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return k * g + ((k & 1) ? g - 1 - c : c);
}

template <int D, bool CAUSAL, bool BF16, bool SPLIT, bool VARLEN, bool DROPOUT>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdArgs args) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + C::kBarOff);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  // With split == 2 the two CTAs of a cluster take the first and the second
  // half of one row block's key tiles, and CTA 0 merges the two partial
  // results (online-softmax state and unnormalised O) at the end.
  static_assert(!(SPLIT && CAUSAL), "causal launches are not split");
  // Variable-length launches are their own instantiation: in the fixed-length
  // one the sequence bounds are kernel parameters, which the softmax warps
  // (at their register limit) need not keep in registers.
  static_assert(!(SPLIT && (VARLEN || DROPOUT)), "variable-length and dropout launches are not split");
  // Persistent at d = 128 (a grid of at most one CTA per SM); one item per
  // CTA at d = 64 and when split (the host sizes the grid to match).
  constexpr bool kPersistent = D == 128 && !SPLIT;
  const uint32_t crank = SPLIT ? cluster_ctarank() : 0u;
  const int total_items = args.n_mblocks * args.B * args.H;
  // An item with no work: a row block past the end of a shorter sequence.
  auto skip = [&](const FwdItem& w) { return w.q0 >= w.seq.len || w.n_kv <= 0; };
  if constexpr (SPLIT) {
    const FwdItem w0 = fwd_item<CAUSAL, SPLIT, VARLEN, C::kKeys>(args, fwd_item_index<SPLIT, kPersistent>(0), crank);
    if (w0.q0 >= w0.seq.len) return;  // both CTAs of the pair see the same row block
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
      mbar_init(&bars->p_half[t], 128);
      mbar_init(&bars->o_full[t], 1);
      mbar_init(&bars->s_cons[t], 128);
      mbar_init(&bars->pv_done[t], 1);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->merge_ready, 256);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (SPLIT) cluster_sync_all();  // partner's barriers initialised before any remote arrive
  const uint32_t tmem = bars->tmem_base;

  const uint32_t sQ = smem_u32(smem + C::kQOff);
  const uint32_t sKV = smem_u32(smem + C::kKVOff);

  // Barrier phases run on across the items of a CTA: `nit` items done so far
  // (q_full, q_empty, o_full complete once per item), `gs` steps done (one
  // step = one key tile for both Q tiles: s_full, p_full, s_cons complete once
  // per step; pv_done once per step but the item's last), K/V ring positions
  // (two per step) in `it`.

  // Registers: launched at 168 per thread; the producer/MMA warpgroup gives
  // back down to 104 and the two softmax warpgroups take 200 (104 + 2 x 200 =
  // 3 x 168), so the setmaxnreg.inc always finds its registers. Each role
  // sets its own count at the top of its branch.
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    reg_alloc_dec<104>();
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int it = 0, nit = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = fwd_item_index<SPLIT, kPersistent>(k);
        if (item >= total_items) break;
        const FwdItem w = fwd_item<CAUSAL, SPLIT, VARLEN, C::kKeys>(args, item, crank);
        if (skip(w)) continue;
        // Q of this item once the previous item's last S has read Q.
        if (nit > 0) ok = mbar_wait(&bars->q_empty, (nit - 1) & 1, abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->q_full, 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_rows(&tm_q, args.hm & kHmQ, smem + C::kQOff + t * C::kTileBytes + kb * C::kBoxBytes,
                          &bars->q_full, kb * 64, w.h, w.seq.row0 + w.q0 + t * 128, w.seq.bcoord);
        for (int j = 0; j < w.n_kv && ok; ++j) {
          for (int which = 0; which < 2 && ok; ++which, ++it) {
            const int st = it % C::kStages;
            if (it >= C::kStages) ok = mbar_wait(&bars->kv_empty[st], ((it / C::kStages) & 1) ^ 1, abort);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars->kv_full[st], C::kTileBytes);
            const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
            const bool hm = args.hm & (which == 0 ? kHmK : kHmV);
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_rows(map, hm, smem + C::kKVOff + st * C::kTileBytes + kb * C::kBoxBytes, &bars->kv_full[st],
                            kb * 64, w.h, w.seq.row0 + (w.kv_lo + j) * C::kKeys, w.seq.bcoord);
          }
        }
        ++nit;
      }
      // Never leave with copies in flight: wait for the last load on each
      // stage, and for the last Q load.
      const int first = it > C::kStages ? it - C::kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&bars->kv_full[i % C::kStages], (i / C::kStages) & 1, abort, false);
      if (nit > 0) mbar_wait(&bars->q_full, (nit - 1) & 1, abort, false);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    reg_alloc_dec<104>();
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_f16(BF16, 128, D, false, true);
      // Descriptors of the tile bases; a K step only moves the start-address
      // field (bits 0-13, in 16-byte units), which cannot carry out of it here.
      const uint64_t dQ0 = sdesc(sQ, 16, 1024);
      const uint64_t dKV = sdesc(sKV, 16, 1024);
      const uint64_t dKV_mn = sdesc(sKV, C::kBoxBytes, 1024);
      constexpr uint32_t kTile16 = C::kTileBytes >> 4;
      auto issue_s = [&](int t, int stage) {
        const uint64_t qa = dQ0 + (uint64_t)(t * kTile16);
        const uint64_t ka = dKV + (uint64_t)(stage * kTile16);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = (uint64_t)(((ks / 4) * C::kBoxBytes + (ks % 4) * 32) >> 4);
          mma_ss(tmem + C::tmem_s(t), qa + off, ka + off, kIdS, ks > 0);
        }
      };
      // P V over keys [16 kk0, 16 kk1) of the tile.
      auto issue_pv_keys = [&](int t, int stage, bool acc, int kk0, int kk1) {
        const uint64_t va = dKV_mn + (uint64_t)(stage * kTile16);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          mma_ts(tmem + C::tmem_o(t), tmem + C::tmem_p(t) + kk * 8, va + (uint64_t)(kk * (2048 >> 4)), kIdPV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_pv = [&](int t, int stage, bool acc) { issue_pv_keys(t, stage, acc, 0, C::kKeys / 16); };
      constexpr int kHalfK = C::kKeys / 32;  // MMAs over the first 64 keys
      auto kv_wait = [&](int pos) { return mbar_wait(&bars->kv_full[pos % C::kStages], (pos / C::kStages) & 1, abort); };

      int it0 = 0, gs = 0, pvc = 0, nit = 0;  // ring base, steps, pv_done completions, items
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = fwd_item_index<SPLIT, kPersistent>(k);
        if (item >= total_items) break;
        const FwdItem w = fwd_item<CAUSAL, SPLIT, VARLEN, C::kKeys>(args, item, crank);
        if (skip(w)) continue;
        const int n_kv = w.n_kv;
        // Ring positions of this item: K_j at it0 + 2j, V_j at it0 + 2j + 1.
        ok = mbar_wait(&bars->q_full, nit & 1, abort) && kv_wait(it0);
        if constexpr (C::kSepP) {
          // S(t, 0) overwrites S of the previous item's last step: wait until
          // the softmax has it in registers.
          for (int t = 0; t < 2 && ok && gs > 0; ++t) ok = mbar_wait(&bars->s_cons[t], (gs - 1) & 1, abort);
        }
        if (!ok) break;
        tc_fence_after();
        issue_s(0, it0 % C::kStages);
        mma_commit(&bars->s_full[0]);
        issue_s(1, it0 % C::kStages);
        mma_commit(&bars->s_full[1]);
        mma_commit(&bars->kv_empty[it0 % C::kStages]);
        if constexpr (C::kSepP) {
          // S(t, j+1) as soon as S(t, j) is in registers; P(t, j) V_j when P
          // is ready. Each half of an iteration first tests its three
          // barriers together: when this thread runs behind the softmax they
          // have all completed, and one test replaces three waits in a row.
          if (n_kv == 1) mma_commit(&bars->q_empty);
          for (int j = 0; j < n_kv && ok; ++j) {
            const int g = gs + j;
            if (j + 1 < n_kv) {
              const int pk = it0 + 2 * j + 2;
              if (mbar_ready3(&bars->kv_full[pk % C::kStages], (pk / C::kStages) & 1, &bars->s_cons[0], g & 1,
                              &bars->s_cons[1], g & 1)) {
                tc_fence_after();
                issue_s(0, pk % C::kStages);
                mma_commit(&bars->s_full[0]);
                issue_s(1, pk % C::kStages);
                mma_commit(&bars->s_full[1]);
              } else {
                ok = kv_wait(pk);
                for (int t = 0; t < 2 && ok; ++t) {
                  ok = mbar_wait(&bars->s_cons[t], g & 1, abort);
                  if (!ok) break;
                  tc_fence_after();
                  issue_s(t, pk % C::kStages);
                  mma_commit(&bars->s_full[t]);
                }
                if (!ok) break;
              }
              mma_commit(&bars->kv_empty[pk % C::kStages]);
              if (j + 2 == n_kv) mma_commit(&bars->q_empty);  // the item's last S is issued
            }
            const int pv = it0 + 2 * j + 1;
            const bool last = j + 1 == n_kv;
            if (mbar_ready3(&bars->kv_full[pv % C::kStages], (pv / C::kStages) & 1, &bars->p_full[0], g & 1,
                            &bars->p_full[1], g & 1)) {
              tc_fence_after();
              issue_pv(0, pv % C::kStages, j > 0);
              mma_commit(last ? &bars->o_full[0] : &bars->pv_done[0]);
              issue_pv(1, pv % C::kStages, j > 0);
              mma_commit(last ? &bars->o_full[1] : &bars->pv_done[1]);
            } else {
              ok = kv_wait(pv);
              for (int t = 0; t < 2 && ok; ++t) {
                ok = mbar_wait(&bars->p_full[t], g & 1, abort);
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, pv % C::kStages, j > 0);
                mma_commit(last ? &bars->o_full[t] : &bars->pv_done[t]);
              }
              if (!ok) break;
            }
            mma_commit(&bars->kv_empty[pv % C::kStages]);
          }
        } else {
          // P(t, j) V_j in two halves of the keys: the first as soon as the
          // softmax has written P of keys 0-63 (p_half), so it overlaps the
          // exponentials of keys 64-127; the second, then S(t, j+1) over the
          // same columns, once all of P is in (p_full).
          auto pv_first_half = [&](int t, int pv, bool acc, int g) {
            if (!mbar_wait(&bars->p_half[t], g & 1, abort)) return false;
            tc_fence_after();
            issue_pv_keys(t, pv % C::kStages, acc, 0, kHalfK);
            return true;
          };
          auto pv_second_half = [&](int t, int pv, int g) {
            if (!mbar_wait(&bars->p_full[t], g & 1, abort)) return false;
            tc_fence_after();
            issue_pv_keys(t, pv % C::kStages, true, kHalfK, C::kKeys / 16);
            return true;
          };
          for (int j = 1; j < n_kv && ok; ++j) {
            const int pv = it0 + 2 * j - 1, pk = it0 + 2 * j;  // ring positions of V_{j-1} and K_j
            const int g = gs + j - 1;                          // step of P(j-1)
            ok = kv_wait(pv) && pv_first_half(0, pv, j > 1, g) && kv_wait(pk) && pv_second_half(0, pv, g);
            if (!ok) break;
            issue_s(0, pk % C::kStages);
            mma_commit(&bars->s_full[0]);
            ok = pv_first_half(1, pv, j > 1, g) && pv_second_half(1, pv, g);
            if (!ok) break;
            mma_commit(&bars->kv_empty[pv % C::kStages]);
            issue_s(1, pk % C::kStages);
            mma_commit(&bars->s_full[1]);
            mma_commit(&bars->kv_empty[pk % C::kStages]);
          }
          if (ok) {
            mma_commit(&bars->q_empty);  // every S of the item is issued
            const int pv = it0 + 2 * n_kv - 1;
            const int g = gs + n_kv - 1;
            ok = kv_wait(pv) && pv_first_half(0, pv, n_kv > 1, g) && pv_second_half(0, pv, g);
            if (ok) {
              mma_commit(&bars->o_full[0]);
              ok = pv_first_half(1, pv, n_kv > 1, g) && pv_second_half(1, pv, g);
            }
            if (ok) {
              mma_commit(&bars->o_full[1]);
              mma_commit(&bars->kv_empty[pv % C::kStages]);
            }
          }
        }
        it0 += 2 * n_kv;
        gs += n_kv;
        pvc += n_kv - 1;
        ++nit;
      }
      (void)pvc;
      // Every issued MMA has finished before the CTA may release TMEM.
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, abort, false);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------ softmax warps
    reg_alloc_inc<200>();
    const int t = warp / 4;
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t tS = lane_base + C::tmem_s(t);
    const uint32_t tO = lane_base + C::tmem_o(t);
    const float c = args.scale_log2;
    // pv_done has completed gs - nit times before an item (once per step but
    // each item's last).
    int gs = 0, nit = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = fwd_item_index<SPLIT, kPersistent>(k);
      if (item >= total_items) break;
      int n_kv, rg, lim, kv_lo;
      {
        // Only what the step loop needs stays live across it; the epilogue
        // derives the rest of the item again.
        const FwdItem w = fwd_item<CAUSAL, SPLIT, VARLEN, C::kKeys>(args, item, crank);
        if (skip(w)) continue;
        n_kv = w.n_kv;
        kv_lo = w.kv_lo;
        rg = w.q0 + t * 128 + r;
        // Keys [0, lim) are kept; lim is counted from this CTA's first key tile.
        lim = (CAUSAL ? min(w.seq.len, rg + 1) : w.seq.len) - w.kv_lo * C::kKeys;
      }
      // l: sum of the exact p (for LSE); lr: sum of the 16-bit rounded p that
      // P V uses (for O / lr, so each output row's weights add up to one).
      float m = -INFINITY, l = 0.f, lr = 0.f;

      for (int j = 0; j < n_kv; ++j) {
        const int g = gs + j;
        if (!mbar_wait_warp(&bars->s_full[t], g & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, s + q * 32);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) tie_regs32(s + q * 32);
        if constexpr (C::kSepP) {
          tc_fence_before();
          mbar_arrive(&bars->s_cons[t]);  // S(t, j+1) may now be written over S(t, j)
        }

        const int kv0 = j * C::kKeys;
        if (kv0 + C::kKeys > lim) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (kv0 + i >= lim) s[i] = __float_as_uint(-INFINITY);
        }
        // Row max: eight independent chains of three-operand max, then a tree.
        float mxa[8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          float x = max3(__uint_as_float(s[kk]), __uint_as_float(s[kk + 8]), __uint_as_float(s[kk + 16]));
#pragma unroll
          for (int e = 3; e + 1 < 16; e += 2) x = max3(x, __uint_as_float(s[kk + 8 * e]), __uint_as_float(s[kk + 8 * e + 8]));
          mxa[kk] = fmaxf(x, __uint_as_float(s[kk + 120]));
        }
        const float mx = max3(max3(mxa[0], mxa[1], mxa[2]), max3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
        const float m_tile = mx * c;

        float alpha = 1.f;
        bool need = false;
        if (j == 0) {
          m = m_tile;
        } else if (m_tile > m + kRescaleLog2) {
          alpha = ex2(m - m_tile);
          m = m_tile;
          need = true;
        }
        // kSepP: P(t, j-1) V_{j-1} must be complete before O is rescaled or P is
        // rewritten (without kSepP its commit preceded s_full already).
        bool pv_waited = !C::kSepP || j == 0;
        const int pvg = gs - nit + j - 1;  // completion of pv_done for P(t, j-1) V
        if (__any_sync(0xffffffffu, need)) {
          if (!pv_waited) {
            if (!mbar_wait_warp(&bars->pv_done[t], pvg & 1, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            pv_waited = true;
          }
#pragma unroll 1
          for (int q = 0; q < D / 16; ++q) {
            uint32_t o[16];
            tmem_ld16(tO + q * 16, o);
            tmem_ld_wait();
            tie_regs16(o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tO + q * 16, o);
          }
          tmem_st_wait();
        }
        l *= alpha;
        lr *= alpha;
        const uint32_t tP = lane_base + C::tmem_p(t);
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const uint64_t c2 = bcast2(c), neg_m2 = bcast2(neg_m);
        // Four accumulators each for the exact and the rounded sums, so no add
        // waits on the one before it.
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sra[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          uint32_t p[16];
          // Dropout: keep bits of this part's 32 keys for this query row (the
          // sums above use every p; only P V sees the dropped ones as zero).
          uint32_t keep = 0xFFFFFFFFu;
          if constexpr (DROPOUT) {
            const uint32_t g0 = static_cast<uint32_t>((kv_lo + j) * C::kKeys + part * 32) >> 2;
            const uint32_t bh = static_cast<uint32_t>(CAUSAL ? item % (args.B * args.H) : item / args.n_mblocks);
            keep = 0;
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) keep |= keep4(args.drop, g0 + gg, static_cast<uint32_t>(rg), bh) << (4 * gg);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1, p0, p1;
            fma2(x0, x1, __uint_as_float(s[part * 32 + 2 * i]), __uint_as_float(s[part * 32 + 2 * i + 1]), c2, neg_m2);
            p0 = ex2(x0);
            p1 = ex2(x1);
            p[i] = pack2<BF16>(p0, p1);
            const int a = 2 * (i & 1);
            add2(sa[a], sa[a + 1], p0, p1);
            sra[a] = add_lo16<BF16>(sra[a], p[i]);
            sra[a + 1] = add_hi16<BF16>(sra[a + 1], p[i]);
            if constexpr (DROPOUT)
              p[i] &= ((keep >> (2 * i)) & 1u ? 0x0000FFFFu : 0u) | ((keep >> (2 * i + 1)) & 1u ? 0xFFFF0000u : 0u);
          }
          if constexpr (!C::kSepP) {
            if (part == 2) {
              // P of keys 0-63 is stored: let P V start on it.
              tmem_st_wait();
              tc_fence_before();
              mbar_arrive(&bars->p_half[t]);
            }
          }
          if (part == 0 && !pv_waited) {
            if (!mbar_wait_warp(&bars->pv_done[t], pvg & 1, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            pv_waited = true;
          }
          tmem_st16(tP + part * 16, p);
        }
        if (!ok) break;
        l += (sa[0] + sa[1]) + (sa[2] + sa[3]);
        lr += (sra[0] + sra[1]) + (sra[2] + sra[3]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t]);
      }
      // (A split pair runs the merge below whatever happened, so that CTA 1
      // always signals CTA 0.) Otherwise the warpgroup agrees on going on, so
      // that all of it or none reaches the epilogue's warpgroup barriers.
      if constexpr (!SPLIT) {
        ok = wg_all(ok, 1 + t);
        if (!ok) break;
      }

      // ------------------------------------------------------------ epilogue
      const FwdItem w = fwd_item<CAUSAL, SPLIT, VARLEN, C::kKeys>(args, item, crank);
      if constexpr (!SPLIT) {
        ok = wg_all(mbar_wait_warp(&bars->o_full[t], nit & 1, abort), 1 + t);
        if (!ok) break;
        tc_fence_after();
        // With dropout, the kept P's scale 1 / (1 - p) is applied here, once.
        const float inv_l = (DROPOUT ? args.drop.rkeep : 1.f) / lr;
        const bool valid = rg < w.seq.len;
        // A tile that starts inside the sequence and, with variable length,
        // ends inside it too (without, the tensor map's row extent clips rows
        // past N): TMA store. Otherwise each thread writes its own row.
        const int tile0 = w.q0 + t * 128;
        if (tile0 < w.seq.len && (!VARLEN || tile0 + 128 <= w.seq.len)) {
          uint8_t* stg = smem + C::kOStOff + t * C::kBoxBytes;
#pragma unroll 1
          for (int kb = 0; kb < D / 64; ++kb) {
            // The staging box is free once this tile's previous store has read it.
            if (r == 0) bulk_wait_read_all();
            named_bar_sync(1 + t, 128);
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
              uint32_t o[32];
              tmem_ld32(tO + (kb * 2 + q2) * 32, o);
              tmem_ld_wait();
              tie_regs32(o);
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
              // Row r of the box is 128 bytes; its 16-byte chunk c sits at c ^ (r % 8).
#pragma unroll
              for (int v = 0; v < 4; ++v)
                st_shared_v4(stg + r * 128 + (((q2 * 4 + v) ^ (r & 7)) << 4), pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                             pk[4 * v + 3]);
            }
            fence_async_shared();
            named_bar_sync(1 + t, 128);
            if (r == 0) {
              tma_store_rows(&tm_o, args.hm & kHmO, stg, kb * 64, w.h, w.seq.row0 + tile0, w.seq.bcoord);
              bulk_commit();
            }
          }
        } else {
          uint16_t* orow = args.o + w.b * args.o_sb + (w.seq.row0 + (valid ? rg : 0)) * args.o_sn + w.h * args.o_sh;
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + q * 32, o);
            tmem_ld_wait();
            tie_regs32(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                if (q * 32 + v * 8 < args.d) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        }
        if (valid)
          args.lse[w.b * args.lse_sb + w.h * args.lse_sh + w.seq.row0 + rg] = m * 0.69314718055994531f + logf(l);
        // O has been read: the next item's first P V may overwrite it (the
        // MMA issues it after this thread's next p_full arrival).
        tc_fence_before();
      } else {
        // Split row block. CTA 1 leaves its row state (unnormalised O, m, l,
        // lr) in its own shared memory, over Q and the K/V ring, which both
        // tiles' last P V products have finished reading. CTA 0 reads it
        // through the cluster's shared-memory window and merges: with
        // M = max(m0, m1) and a_i = 2^(m_i - M), O = (a0 O0 + a1 O1) / (a0 lr0 +
        // a1 lr1) and l = a0 l0 + a1 l1, the same result as one pass over all
        // key tiles with running max M. Every softmax thread of CTA 1 arrives on
        // CTA 0's barrier whatever happened before; neither CTA leaves before
        // the cluster barrier at the end, after CTA 0's last remote read.
        const bool done =
            ok && mbar_wait_warp(&bars->o_full[t], 0, abort) && mbar_wait_warp(&bars->o_full[1 - t], 0, abort);
        float* part = reinterpret_cast<float*>(smem) + static_cast<size_t>(t * 128 + r) * (D + 4);
        if (cluster_ctarank() == 1) {
          if (done) {
            tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
              uint32_t o[32];
              tmem_ld32(tO + q * 32, o);
              tmem_ld_wait();
              tie_regs32(o);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                reinterpret_cast<float4*>(part + q * 32)[v] =
                    make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]), __uint_as_float(o[4 * v + 2]),
                                __uint_as_float(o[4 * v + 3]));
            }
            *reinterpret_cast<float4*>(part + D) = make_float4(m, l, lr, 0.f);
          }
          mbar_arrive_remote(mapa_shared(smem_u32(&bars->merge_ready), 0));
        } else {
          const bool have = mbar_wait_cluster(&bars->merge_ready, 0);
          if (done && have) {
            tc_fence_after();
            const uint32_t rpart = mapa_shared(smem_u32(part), 1);
            const float4 st = ld_shared_cluster_v4(rpart + D * 4);  // m1, l1, lr1
            const float mm = fmaxf(m, st.x);
            const float a0 = ex2(m - mm), a1 = ex2(st.x - mm);
            const float l_all = a0 * l + a1 * st.y;
            const float inv = 1.f / (a0 * lr + a1 * st.z);
            const float c0 = a0 * inv, c1 = a1 * inv;
            const bool valid = rg < w.seq.len;
            uint16_t* orow = args.o + w.b * args.o_sb + (w.seq.row0 + (valid ? rg : 0)) * args.o_sn + w.h * args.o_sh;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
              uint32_t o[32];
              tmem_ld32(tO + q * 32, o);
              tmem_ld_wait();
              tie_regs32(o);
              uint32_t pk[16];
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const float4 x = ld_shared_cluster_v4(rpart + (q * 32 + 4 * v) * 4);
                pk[2 * v] = pack2<BF16>(fmaf(__uint_as_float(o[4 * v]), c0, x.x * c1),
                                        fmaf(__uint_as_float(o[4 * v + 1]), c0, x.y * c1));
                pk[2 * v + 1] = pack2<BF16>(fmaf(__uint_as_float(o[4 * v + 2]), c0, x.z * c1),
                                            fmaf(__uint_as_float(o[4 * v + 3]), c0, x.w * c1));
              }
              if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  if (q * 32 + v * 8 < args.d)
                    dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
              }
            }
            if (valid)
              args.lse[w.b * args.lse_sb + w.h * args.lse_sh + w.seq.row0 + rg] =
                  mm * 0.69314718055994531f + logf(l_all);
          }
        }
      }
      gs += n_kv;
      ++nit;
    }
    // O's last stores have completed before the CTA leaves.
    if (r == 0) bulk_wait_all();
  } else {
    reg_alloc_dec<104>();  // warps 10-11: no role
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // Every thread of both CTAs gets here after bounded waits only; no CTA of a
  // split pair leaves while the other may still touch its shared memory.
  if constexpr (SPLIT) cluster_sync_all();
}

}  // namespace fa
