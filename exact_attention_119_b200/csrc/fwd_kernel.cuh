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

#include "sm100.cuh"

namespace fa {

constexpr float kRescaleLog2 = 8.0f;

struct FwdArgs {
  void* o;       // [B, N, H, D] fp16/bf16
  float* lse;    // [B, H, N] fp32
  int B, N, H;
  int n_mblocks;       // ceil(N / 256)
  int split;           // 1, or 2: each row block's key tiles shared by a 2-CTA cluster
  float scale_log2;    // softmax_scale * log2(e)
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
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;  // + barriers + alignment slack
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
  uint64_t s_full[2];
  uint64_t p_full[2];
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

template <int D, bool CAUSAL, bool BF16, bool SPLIT>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + C::kBarOff);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  // Work item: longest-first when causal (the last row block has the most keys).
  // With split == 2 the two CTAs of a cluster take the first and the second
  // half of the row block's key tiles, and CTA 0 merges the two partial
  // results (online-softmax state and unnormalised O) at the end.
  const int bh_count = args.B * args.H;
  static_assert(!(SPLIT && CAUSAL), "causal launches are not split");
  constexpr int split = SPLIT ? 2 : 1;
  const int item = blockIdx.x / split;
  const uint32_t crank = SPLIT ? cluster_ctarank() : 0u;
  int mblk = item / bh_count;
  const int bh = item % bh_count;
  if (CAUSAL) mblk = args.n_mblocks - 1 - mblk;
  const int b = bh / args.H;
  const int h = bh % args.H;
  const int q0 = mblk * 256;
  const int kv_end = CAUSAL ? min(args.N, q0 + 256) : args.N;
  const int n_kv_all = (kv_end + C::kKeys - 1) / C::kKeys;
  const int kv_half = (n_kv_all + 1) / 2;
  const int kv_lo = crank == 0 ? 0 : kv_half;  // first key tile of this CTA
  const int n_kv = split == 1 ? n_kv_all : (crank == 0 ? kv_half : n_kv_all - kv_half);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
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
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::kTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_4d(&tm_q, smem + C::kQOff + t * C::kTileBytes + kb * C::kBoxBytes, &bars->q_full, kb * 64, h,
                      q0 + t * 128, b);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int which = 0; which < 2 && ok; ++which, ++it) {
          const int st = it % C::kStages;
          if (it >= C::kStages) ok = mbar_wait(&bars->kv_empty[st], ((it / C::kStages) & 1) ^ 1, abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->kv_full[st], C::kTileBytes);
          const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_4d(map, smem + C::kKVOff + st * C::kTileBytes + kb * C::kBoxBytes, &bars->kv_full[st],
                        kb * 64, h, (kv_lo + j) * C::kKeys, b);
        }
      }
      // Never leave with copies in flight: wait for the last load on each stage.
      const int first = it > C::kStages ? it - C::kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&bars->kv_full[i % C::kStages], (i / C::kStages) & 1, abort, false);
      mbar_wait(&bars->q_full, 0, abort, false);
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
      auto issue_pv = [&](int t, int stage, bool acc) {
        const uint64_t va = dKV_mn + (uint64_t)(stage * kTile16);
#pragma unroll
        for (int kk = 0; kk < C::kKeys / 16; ++kk)
          mma_ts(tmem + C::tmem_o(t), tmem + C::tmem_p(t) + kk * 8, va + (uint64_t)(kk * (2048 >> 4)), kIdPV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      auto kv_wait = [&](int pos) { return mbar_wait(&bars->kv_full[pos % C::kStages], (pos / C::kStages) & 1, abort); };

      bool ok = mbar_wait(&bars->q_full, 0, abort) && kv_wait(0);
      if constexpr (C::kSepP) {
        // S(t, j+1) as soon as S(t, j) is in registers; P(t, j) V_j when P is
        // ready. Ring positions: K_j at 2j, V_j at 2j + 1.
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit(&bars->s_full[0]);
          issue_s(1, 0);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->kv_empty[0]);
        }
        // Each half of an iteration first tests its three barriers together:
        // when this thread runs behind the softmax they have all completed,
        // and one test replaces three waits in a row.
        for (int j = 0; j < n_kv && ok; ++j) {
          if (j + 1 < n_kv) {
            const int pk = 2 * j + 2;
            if (mbar_ready3(&bars->kv_full[pk % C::kStages], (pk / C::kStages) & 1, &bars->s_cons[0], j & 1,
                            &bars->s_cons[1], j & 1)) {
              tc_fence_after();
              issue_s(0, pk % C::kStages);
              mma_commit(&bars->s_full[0]);
              issue_s(1, pk % C::kStages);
              mma_commit(&bars->s_full[1]);
            } else {
              ok = kv_wait(pk);
              for (int t = 0; t < 2 && ok; ++t) {
                ok = mbar_wait(&bars->s_cons[t], j & 1, abort);
                if (!ok) break;
                tc_fence_after();
                issue_s(t, pk % C::kStages);
                mma_commit(&bars->s_full[t]);
              }
              if (!ok) break;
            }
            mma_commit(&bars->kv_empty[pk % C::kStages]);
          }
          const int pv = 2 * j + 1;
          if (mbar_ready3(&bars->kv_full[pv % C::kStages], (pv / C::kStages) & 1, &bars->p_full[0], j & 1,
                          &bars->p_full[1], j & 1)) {
            tc_fence_after();
            issue_pv(0, pv % C::kStages, j > 0);
            mma_commit(j + 1 < n_kv ? &bars->pv_done[0] : &bars->o_full[0]);
            issue_pv(1, pv % C::kStages, j > 0);
            mma_commit(j + 1 < n_kv ? &bars->pv_done[1] : &bars->o_full[1]);
          } else {
            ok = kv_wait(pv);
            for (int t = 0; t < 2 && ok; ++t) {
              ok = mbar_wait(&bars->p_full[t], j & 1, abort);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, pv % C::kStages, j > 0);
              mma_commit(j + 1 < n_kv ? &bars->pv_done[t] : &bars->o_full[t]);
            }
            if (!ok) break;
          }
          mma_commit(&bars->kv_empty[pv % C::kStages]);
        }
      } else {
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit(&bars->s_full[0]);
          issue_s(1, 0);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->kv_empty[0]);
        }
        for (int j = 1; j < n_kv && ok; ++j) {
          const int pv = 2 * j - 1, pk = 2 * j;  // ring positions of V_{j-1} and K_j
          ok = kv_wait(pv) && kv_wait(pk) && mbar_wait(&bars->p_full[0], (j - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, pv % C::kStages, j > 1);
          issue_s(0, pk % C::kStages);
          mma_commit(&bars->s_full[0]);
          ok = mbar_wait(&bars->p_full[1], (j - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, pv % C::kStages, j > 1);
          mma_commit(&bars->kv_empty[pv % C::kStages]);
          issue_s(1, pk % C::kStages);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->kv_empty[pk % C::kStages]);
        }
        if (ok) {
          const int pv = 2 * n_kv - 1;
          ok = kv_wait(pv) && mbar_wait(&bars->p_full[0], (n_kv - 1) & 1, abort);
          if (ok) {
            tc_fence_after();
            issue_pv(0, pv % C::kStages, n_kv > 1);
            mma_commit(&bars->o_full[0]);
            ok = mbar_wait(&bars->p_full[1], (n_kv - 1) & 1, abort);
          }
          if (ok) {
            tc_fence_after();
            issue_pv(1, pv % C::kStages, n_kv > 1);
            mma_commit(&bars->o_full[1]);
            mma_commit(&bars->kv_empty[pv % C::kStages]);
          }
        }
      }
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
    const int rg = q0 + t * 128 + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t tS = lane_base + C::tmem_s(t);
    const uint32_t tO = lane_base + C::tmem_o(t);
    // Keys [0, lim) are kept; lim is counted from this CTA's first key tile.
    const int lim = (CAUSAL ? min(args.N, rg + 1) : args.N) - kv_lo * C::kKeys;
    const float c = args.scale_log2;
    // l: sum of the exact p (for LSE); lr: sum of the 16-bit rounded p that
    // P V uses (for O / lr, so each output row's weights add up to one).
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;

    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait_warp(&bars->s_full[t], j & 1, abort)) {
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
      for (int k = 0; k < 8; ++k) {
        float x = max3(__uint_as_float(s[k]), __uint_as_float(s[k + 8]), __uint_as_float(s[k + 16]));
#pragma unroll
        for (int e = 3; e + 1 < 16; e += 2) x = max3(x, __uint_as_float(s[k + 8 * e]), __uint_as_float(s[k + 8 * e + 8]));
        mxa[k] = fmaxf(x, __uint_as_float(s[k + 120]));
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
      if (__any_sync(0xffffffffu, need)) {
        if (!pv_waited) {
          if (!mbar_wait_warp(&bars->pv_done[t], (j - 1) & 1, abort)) {
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
      // Four accumulators each for the exact and the rounded sums, so no add
      // waits on the one before it.
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sra[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(__uint_as_float(s[part * 32 + 2 * i]), c, neg_m));
          const float p1 = ex2(fmaf(__uint_as_float(s[part * 32 + 2 * i + 1]), c, neg_m));
          p[i] = pack2<BF16>(p0, p1);
          const int a = 2 * (i & 1);
          sa[a] += p0;
          sa[a + 1] += p1;
          sra[a] = add_lo16<BF16>(sra[a], p[i]);
          sra[a + 1] = add_hi16<BF16>(sra[a + 1], p[i]);
        }
        if (part == 0 && !pv_waited) {
          if (!mbar_wait_warp(&bars->pv_done[t], (j - 1) & 1, abort)) {
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

    // -------------------------------------------------------------- epilogue
    if constexpr (!SPLIT) {
      if (ok && mbar_wait_warp(&bars->o_full[t], 0, abort)) {
        tc_fence_after();
        const float inv_l = 1.f / lr;
        const bool valid = rg < args.N;
        uint16_t* orow = reinterpret_cast<uint16_t*>(args.o) +
                         ((static_cast<size_t>(b) * args.N + (valid ? rg : 0)) * args.H + h) * D;
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
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (valid) args.lse[(static_cast<size_t>(b) * args.H + h) * args.N + rg] = m * 0.69314718055994531f + logf(l);
      }
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
      const bool done = ok && mbar_wait_warp(&bars->o_full[t], 0, abort) && mbar_wait_warp(&bars->o_full[1 - t], 0, abort);
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
          const bool valid = rg < args.N;
          uint16_t* orow = reinterpret_cast<uint16_t*>(args.o) +
                           ((static_cast<size_t>(b) * args.N + (valid ? rg : 0)) * args.H + h) * D;
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
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
          if (valid)
            args.lse[(static_cast<size_t>(b) * args.H + h) * args.N + rg] = mm * 0.69314718055994531f + logf(l_all);
        }
      }
    }
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
