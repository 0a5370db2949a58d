// Forward pass for d = 128 on CTA pairs (tcgen05 cta_group::2), two query
// tiles per CTA.
//
// Same arithmetic as the persistent forward (per-row running max, normaliser
// and output updated after every K/V block: "深度学习进阶（三十一）FlashAttention：IO
// 感知的精确注意力" §2.2), on a cluster of two CTAs that share every MMA — the
// Blackwell "2-CTA MMA" the handbook page "FlashAttention" lists for FA4 in
// its version table, and the remedy for shared-memory traffic that the
// "Flash-Attention" concept page names among FA4's observations.
//
// A cluster takes four consecutive 128-row query tiles 4i .. 4i+3 of one
// (batch, head), as two tile pairs: pair t covers tiles 4i+2t (in CTA 0) and
// 4i+2t+1 (in CTA 1).  The leader (rank 0) issues M = 256 products for each
// tile pair:
//   S_t = Q_t Kᵀ   A = each CTA's own Q tile; B = K split by keys: CTA r
//                  holds keys 64·r .. 64·r + 63 of the K tile (K-major)
//   O_t += P_t V   A = each CTA's P_t in TMEM; B = V split by columns: CTA r
//                  holds columns 64·r .. 64·r + 63 (MN-major)
// so each CTA loads and keeps half of every K/V tile, and each half feeds
// both of its query tiles: per 128-key block a CTA moves 32 KB of K/V into
// shared memory and reads 128 KB of operands out of it for its 256 query
// rows, against 64 KB and 192 KB in the single-CTA persistent kernel.
// Roles in both CTAs: warp 0 TMA producer (its Q tiles and K/V halves, their
// completion counted on the leader's barriers), warps 4-7 / 8-11 softmax of
// tile pair 0 / 1 (thread = row; P handed to the leader's barriers, which
// count both CTAs' warps).  Warp 1 of the leader issues the MMAs, the two
// tile pairs in turn, and commits to both CTAs' barriers at once.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

struct FwdPairCfg {
  static constexpr int D = 128;
  static constexpr int BM = 128;                 // query rows per tile
  static constexpr int BN = 128;                 // keys per K/V block
  static constexpr int THREADS = 384;
  static constexpr int PANEL = 128 * 128;        // 64 columns of a 128-row tile (bytes)
  static constexpr int KH_PANEL = 64 * 128;      // 64 columns of the 64-row K half
  static constexpr int Q_BYTES = BM * D * 2;     // 32 KB
  static constexpr int UNIT_BYTES = 16384;       // a K half (64 × 128) or a V half (128 × 64)
  static constexpr int NSLOT = 9;
  static constexpr int Q_OFF = 0;                // two Q tiles
  static constexpr int KV_OFF = 2 * Q_BYTES;
  // one unit of padding after the ring: the operand reads of a unit stay
  // inside the allocation whatever the split of B between the CTAs
  static constexpr int BAR_OFF = KV_OFF + (NSLOT + 1) * UNIT_BYTES;
  static constexpr int B_QFULL = 0;               // leader's copy: all four Q tiles
  static constexpr int B_KVFULL = 1;              // + slot (leader's copy counts both halves)
  static constexpr int B_KVEMPTY = 1 + NSLOT;     // + slot (both CTAs)
  static constexpr int B_SFULL = 1 + 2 * NSLOT;   // + t (both CTAs)
  static constexpr int B_PFULL = B_SFULL + 2;     // + t: P keys 0..63 (leader's copy, 8 warps)
  static constexpr int B_PFULL2 = B_PFULL + 2;    // + t: P keys 64..127
  static constexpr int B_ODONE = B_PFULL2 + 2;    // + t (both CTAs)
  static constexpr int B_DRAIN = B_ODONE + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0;    // S_t at S_COL + 128·t (P_t over its first 64 columns)
  static constexpr int O_COL = 256;  // O_t at O_COL + 128·t
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(256, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(256, D, false, true);
  // Register split (setmaxnreg), as in the persistent kernel: valid for a
  // launch allocation R with CTRL_REGS <= R <= SOFTMAX_REGS and
  // 128·CTRL_REGS + 256·SOFTMAX_REGS <= 384·R (checked on the host).
  static constexpr int CTRL_REGS = 120;
  static constexpr int SOFTMAX_REGS = 192;
  static constexpr int MIN_LAUNCH_REGS = (128 * CTRL_REGS + 256 * SOFTMAX_REGS + THREADS - 1) / THREADS;
  static constexpr int MAX_LAUNCH_REGS = SOFTMAX_REGS;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// TAIL: N is not a multiple of 128 (keys past N masked, rows past N not
// stored).  Grid (2·items, Hq, B) in clusters of (2, 1, 1), items of four
// query tiles; causal items heaviest first.  Tile pair 1 sees every K/V
// block tile pair 0 sees (and, with the causal mask, two more), so it is the
// last reader of every K/V unit.
template <bool CAUSAL, bool TAIL>
__global__ void __launch_bounds__(FwdPairCfg::THREADS, 1)
    fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdPairCfg;
  constexpr int D = C::D;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int n_items = (int)(gridDim.x >> 1);
  const int item = CAUSAL ? n_items - 1 - (int)(blockIdx.x >> 1) : (int)(blockIdx.x >> 1);
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int q_base = (b * p.Hq + h) * p.N;
  const int kv_base = (b * p.Hkv + h / p.G) * p.N;
  // K/V blocks of tile pair t: both CTAs take part in every product, the lower
  // tile's rows see the upper tile's diagonal block fully masked
  auto blocks = [&](int t) -> int { return CAUSAL ? min(4 * item + 2 * t + 2, p.n_qtiles) : p.n_qtiles; };
  const int n0 = blocks(0), n1 = blocks(1);  // n1 >= n0

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
  auto LBAR = [&](int i) -> uint32_t { return mapa_shared(BAR(i), 0); };  // the leader's copy
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(BAR(C::B_KVFULL + i), 1);
      mbar_init(BAR(C::B_KVEMPTY + i), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(C::B_SFULL + t), 1);
      mbar_init(BAR(C::B_PFULL + t), 8);
      mbar_init(BAR(C::B_PFULL2 + t), 8);
      mbar_init(BAR(C::B_ODONE + t), 1);
    }
    mbar_init(BAR(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before either side signals the other
  cluster_sync();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err, p.wait_cap};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<C::CTRL_REGS>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      if (leader) mbar_expect_tx(BAR(C::B_QFULL), 4 * C::Q_BYTES);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_2d_pair(sbase + C::Q_OFF + t * C::Q_BYTES + pn * C::PANEL, &tmQ, LBAR(C::B_QFULL), pn * 64,
                           q_base + (4 * item + 2 * t + (int)rank) * C::BM, pol_q);
      // units: K(0), V(0), K(1), V(1), ... of the blocks of tile pair 1
      bool ok = true;
      int kv_issued = 0;  // units whose loads this CTA issued
      for (int u = 0; u < 2 * n1 && ok; ++u) {
        const int j = u >> 1;
        const int slot = u % C::NSLOT;
        if (!mbar_wait(BAR(C::B_KVEMPTY + slot), ((u / C::NSLOT) & 1) ^ 1, wc, 61)) { ok = false; break; }
        if (leader) mbar_expect_tx(BAR(C::B_KVFULL + slot), 2 * C::UNIT_BYTES);
        const uint32_t dst = sbase + C::KV_OFF + slot * C::UNIT_BYTES;
        if (u & 1) {
          // columns 64·rank .. 64·rank + 63 of the 128-key V block
          tma_load_2d_pair(dst, &tmV, LBAR(C::B_KVFULL + slot), 64 * (int)rank, kv_base + j * C::BN, pol_kv);
        } else {
          // keys 64·rank .. 64·rank + 63 of the K block, both 64-column panels
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_2d_pair(dst + pn * C::KH_PANEL, &tmK, LBAR(C::B_KVFULL + slot), pn * 64,
                             kv_base + j * C::BN + 64 * (int)rank, pol_kv);
        }
        kv_issued = u + 1;
      }
      // both CTAs' loads complete on the leader's barriers: the leader waits
      // for every fill it armed before the pair's final cluster barrier
      // (immediate unless a CTA stopped early on a failed wait)
      if (leader) {
        mbar_wait_inflight(BAR(C::B_QFULL), 0, wc, 70);
        for (int sl = 0; sl < C::NSLOT && sl < kv_issued; ++sl) {
          const int last = kv_issued - 1 - (kv_issued - 1 - sl) % C::NSLOT;  // last unit loaded into slot sl
          mbar_wait_inflight(BAR(C::B_KVFULL + sl), (last / C::NSLOT) & 1, wc, 71);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only)
    setmaxnreg_dec<C::CTRL_REGS>();
    if (leader) {
      bool ok = mbar_wait_warp(BAR(C::B_QFULL), 0, wc, 62);
      tc_fence_after();
      int waited = -1;  // units whose arrival has been observed, in load order
      auto wait_upto = [&](int u) -> bool {
        while (waited < u) {
          ++waited;
          if (!mbar_wait_warp(BAR(C::B_KVFULL + waited % C::NSLOT), (waited / C::NSLOT) & 1, wc, 63)) return false;
        }
        tc_fence_after();
        return true;
      };
      auto release = [&](int u) { tc_commit_pair_w(BAR(C::B_KVEMPTY + u % C::NSLOT)); };
      const uint64_t dQ_k = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dKV_k = sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::KV_OFF, C::UNIT_BYTES, 1024);
      // S_t = Q_t · K_jᵀ (M = 256 rows of tile pair t, N = 128 keys, K = D)
      auto issue_s = [&](int t, int j) -> bool {
        const int u = 2 * j;
        if (!wait_upto(u)) return false;
        const uint64_t da0 = sdesc_add(dQ_k, t * C::Q_BYTES);
        const uint64_t db0 = sdesc_add(dKV_k, (u % C::NSLOT) * C::UNIT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_pair_w(tbase + C::S_COL + 128 * t, sdesc_add(da0, (kk >> 2) * C::PANEL + (kk & 3) * 32),
                        sdesc_add(db0, (kk >> 2) * C::KH_PANEL + (kk & 3) * 32), C::IDESC_S, kk > 0 ? 1u : 0u);
        tc_commit_pair_w(BAR(C::B_SFULL + t));
        if (t == 1) release(u);  // tile pair 1 is the last reader of K_j
        return true;
      };
      // O_t (+)= P_t V_j; half 0 covers keys 0..63, half 1 keys 64..127
      auto issue_pv = [&](int t, int j, int half) {
        const uint64_t db0 = sdesc_add(dKV_mn, ((2 * j + 1) % C::NSLOT) * C::UNIT_BYTES);
#pragma unroll
        for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
          mma_ts_pair_w(tbase + C::O_COL + 128 * t, tbase + C::S_COL + 128 * t + kk * 8, sdesc_add(db0, kk * 2048),
                        C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
      };
      if (ok) ok = issue_s(0, 0);
      if (ok) ok = issue_s(1, 0);
      for (int j = 0; j < n1 && ok; ++j) {
        for (int t = 0; t < 2; ++t) {
          if (j >= (t == 0 ? n0 : n1)) continue;
          if (!mbar_wait_warp(BAR(C::B_PFULL + t), j & 1, wc, 64)) { ok = false; break; }
          if (!wait_upto(2 * j + 1)) { ok = false; break; }
          issue_pv(t, j, 0);
          if (!mbar_wait_warp(BAR(C::B_PFULL2 + t), j & 1, wc, 65)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t, j, 1);
          tc_commit_pair_w(BAR(C::B_ODONE + t));
          if (t == 1) release(2 * j + 1);  // last reader of V_j
          // this tile pair's next S (P_t over S_t has been read by the PV above)
          if (j + 1 < (t == 0 ? n0 : n1)) {
            ok = issue_s(t, j + 1);
            if (!ok) break;
          }
        }
      }
      // no MMA may still be running when either CTA releases its TMEM
      tc_commit_pair_w(BAR(C::B_DRAIN));
      mbar_wait_inflight(BAR(C::B_DRAIN), 0, wc, 66);
    }
  } else if (warp < 4) {
    // idle warps of the control warpgroup: hand their registers to the softmax
    setmaxnreg_dec<C::CTRL_REGS>();
  } else {
    // ------------------------------------------------------------- softmax
    setmaxnreg_inc<C::SOFTMAX_REGS>();
    const int t = (warp - 4) >> 2;  // tile pair
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qt = 4 * item + 2 * t + (int)rank;  // this CTA's query tile of the pair
    const int q_row = qt * C::BM + row;
    const int n = t == 0 ? n0 : n1;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    const int scol = C::S_COL + 128 * t;
    const int ocol = C::O_COL + 128 * t;
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!mbar_wait_warp(BAR(C::B_SFULL + t), j & 1, wc, 67)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      tmem_ld32(tl + scol + 0, r0);
      tmem_ld32(tl + scol + 32, r1);
      tmem_ld32(tl + scol + 64, r2);
      tmem_ld32(tl + scol + 96, r3);
      tmem_ld_wait();
      reg_fence(r0);
      reg_fence(r1);
      reg_fence(r2);
      reg_fence(r3);
      float s[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(r0[c]);
        s[32 + c] = __uint_as_float(r1[c]);
        s[64 + c] = __uint_as_float(r2[c]);
        s[96 + c] = __uint_as_float(r3[c]);
      }
      if (CAUSAL && j >= qt) {
        // the diagonal block, or (lower tile of the pair) the upper tile's
        // diagonal block, which this tile's rows cannot see at all
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (j > qt || c > row) s[c] = -INFINITY;
      }
      if (TAIL && !CAUSAL && (j + 1) * C::BN > p.N) {
        const int lim = p.N - j * C::BN;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      const float mx = row_max128(s);
      const float m_new = fmaxf(m_ref, mx * sl2);
      float alpha = 1.f;
      bool warp_rescale = false;
      if (j == 0) {
        m_ref = m_new;
      } else {
        const bool need = m_new > m_ref + kRescaleTau;
        warp_rescale = __any_sync(0xffffffffu, need);
        if (need) {
          alpha = ex2(m_ref - m_new);
          m_ref = m_new;
          l *= alpha;
        }
      }
      const float neg_m = -m_ref;
      uint64_t rs2[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
      auto exp_half = [&](int base, uint32_t (&pk)[32]) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0, x1;
          f2_split(f2_fma(f2_make(s[base + 2 * c], s[base + 2 * c + 1]), f2_make(sl2, sl2), f2_make(neg_m, neg_m)),
                   x0, x1);
          const float a0 = ex2(x0);
          const float a1 = ex2(x1);
          rs2[c & 1] = f2_add(rs2[c & 1], f2_make(a0, a1));
          pk[c] = pack_bf16(a0, a1);
        }
      };
      {
        uint32_t pk[32];
        exp_half(0, pk);
        if (warp_rescale) {
          // O_t must hold the previous block's product before it is scaled,
          // and be scaled before this block's first PV half accumulates
          if (!mbar_wait_warp(BAR(C::B_ODONE + t), (j - 1) & 1, wc, 68)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int oc = 0; oc < D / 32; ++oc) {
            uint32_t ov[32];
            tmem_ld32(tl + ocol + oc * 32, ov);
            tmem_ld_wait();
            reg_fence(ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st32(tl + ocol + oc * 32, ov);
          }
        }
        tmem_st32(tl + scol, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LBAR(C::B_PFULL + t));
      }
      {
        uint32_t pk[32];
        exp_half(64, pk);
        tmem_st32(tl + scol + 32, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LBAR(C::B_PFULL2 + t));
      }
      float a, b2, c2, d2;
      f2_split(rs2[0], a, b2);
      f2_split(rs2[1], c2, d2);
      l += (a + b2) + (c2 + d2);
    }
    if (ok) ok = mbar_wait_warp(BAR(C::B_ODONE + t), (n - 1) & 1, wc, 69);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = p.o + ((size_t)q_base + q_row) * D;
      // tiles past N (the last item of a head with a tile count not a multiple
      // of four) take part in the pair's products but store nothing
      const bool store = q_row < p.N;
#pragma unroll
      for (int oc = 0; oc < D / 32; ++oc) {
        uint32_t ov[32];
        tmem_ld32(tl + ocol + oc * 32, ov);
        tmem_ld_wait();
        reg_fence(ov);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv_l, __uint_as_float(ov[2 * c + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + oc * 32);
        if (store) {
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      float lg;
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
      if (store) p.lse[(size_t)q_base + q_row] = (m_ref + lg) * kLn2;
    }
    tc_fence_before();
  }

  __syncthreads();
  // neither CTA frees its TMEM or leaves while the pair's products or the
  // other CTA's signals may still reach it
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa
