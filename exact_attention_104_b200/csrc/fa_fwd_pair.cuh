// Forward pass for d = 128 on CTA pairs (tcgen05 cta_group::2).
//
// Same arithmetic as fa_fwd_kernel (per-row running max, normaliser and
// output updated after every K/V block: "深度学习进阶（三十一）FlashAttention：IO
// 感知的精确注意力" §2.2), on a cluster of two CTAs that share every MMA —
// the Blackwell "2-CTA MMA" the handbook page "FlashAttention" lists for FA4
// in its version table, and the remedy for shared-memory traffic that the
// "Flash-Attention" concept page names among FA4's observations.
//
// The pair covers 256 query rows, 128 per CTA (CTA rank r owns query tile
// 2·pair + r).  The leader (rank 0) issues M = 256 products:
//   S = Q Kᵀ   A = each CTA's own Q tile; B = K split by keys: CTA r holds
//              keys 64·r .. 64·r + 63 of the tile (64 × 128, K-major)
//   O += P V   A = each CTA's own P in TMEM; B = V split by columns: CTA r
//              holds columns 64·r .. 64·r + 63 (128 keys × 64, MN-major)
// so each CTA loads and keeps half of every K/V tile: per 128-key tile a CTA
// reads 32 KB of K/V from L2 and, for the two products, 64 KB of operands
// from its shared memory, against 64 KB and 96 KB for a single CTA with the
// same 128 query rows.
// Roles in both CTAs: warp 0 TMA producer (its own halves; completion counted
// on the leader's barriers), warps 4-7 softmax of its own rows (thread = row;
// P handed to the leader's barriers, which count both CTAs' warps).  Warp 1
// of the leader issues the MMAs and commits to both CTAs' barriers at once.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

struct FwdPairCfg {
  static constexpr int D = 128;
  static constexpr int BM = 128;                 // query rows per CTA (the pair: 256)
  static constexpr int BN = 128;                 // keys per K/V tile
  static constexpr int THREADS = 256;
  static constexpr int PANEL = 128 * 128;        // 64 columns of a 128-row tile (bytes)
  static constexpr int KH_PANEL = 64 * 128;      // 64 columns of the 64-row K half
  static constexpr int Q_BYTES = BM * D * 2;     // 32 KB
  static constexpr int UNIT_BYTES = 16384;       // a K half (64 × 128) or a V half (128 × 64)
  static constexpr int NSLOT = 10;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = Q_BYTES;
  // one unit of padding after the ring: the operand reads of a unit stay
  // inside the allocation whatever the split of B between the CTAs
  static constexpr int BAR_OFF = KV_OFF + (NSLOT + 1) * UNIT_BYTES;
  static constexpr int B_QFULL = 0;
  static constexpr int B_KVFULL = 1;              // + slot (leader's copy counts both halves)
  static constexpr int B_KVEMPTY = 1 + NSLOT;     // + slot (both CTAs)
  static constexpr int B_SFULL = 1 + 2 * NSLOT;   // + {0,1} (both CTAs)
  static constexpr int B_PFULL = B_SFULL + 2;     // + {0,1}: P keys 0..63 (leader's copy, 8 warps)
  static constexpr int B_PFULL2 = B_PFULL + 2;    // + {0,1}: P keys 64..127
  static constexpr int B_ODONE = B_PFULL2 + 2;    // + {0,1} (both CTAs)
  static constexpr int B_DRAIN = B_ODONE + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0;    // S buffer x at S_COL + 128·x (P over its first 64 columns)
  static constexpr int O_COL = 256;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(256, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(256, D, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// TAIL: N is not a multiple of 128 (keys past N masked, rows past N not
// stored).  Grid (2·pairs, Hq, B) in clusters of (2, 1, 1); causal pairs
// heaviest first.
template <bool CAUSAL, bool TAIL>
__global__ void __launch_bounds__(FwdPairCfg::THREADS, 1)
    fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdPairCfg;
  using Ord = KVOrder;
  constexpr int D = C::D;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int n_pairs = (int)(gridDim.x >> 1);
  const int pair = CAUSAL ? n_pairs - 1 - (int)(blockIdx.x >> 1) : (int)(blockIdx.x >> 1);
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int qt = 2 * pair + (int)rank;  // this CTA's query tile
  const int q_base = (b * p.Hq + h) * p.N;
  const int kv_base = (b * p.Hkv + h / p.G) * p.N;
  // K/V tiles of the pair: both CTAs take part in every product, the lower
  // tile's rows see the upper tile's diagonal block fully masked
  const int n = CAUSAL ? min(2 * pair + 2, p.n_qtiles) : p.n_qtiles;

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::B_SFULL + i), 1);
      mbar_init(BAR(C::B_PFULL + i), 8);
      mbar_init(BAR(C::B_PFULL2 + i), 8);
      mbar_init(BAR(C::B_ODONE + i), 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      if (leader) mbar_expect_tx(BAR(C::B_QFULL), 2 * C::Q_BYTES);
#pragma unroll
      for (int pn = 0; pn < D / 64; ++pn)
        tma_load_2d_pair(sbase + C::Q_OFF + pn * C::PANEL, &tmQ, LBAR(C::B_QFULL), pn * 64, q_base + qt * C::BM,
                         pol_q);
      bool ok = true;
      for (int u = 0; u < 2 * n && ok; ++u) {
        bool is_v;
        int j;
        Ord::decode(u, n, is_v, j);
        const int slot = u % C::NSLOT;
        if (!mbar_wait(BAR(C::B_KVEMPTY + slot), ((u / C::NSLOT) & 1) ^ 1, wc, 61)) { ok = false; break; }
        if (leader) mbar_expect_tx(BAR(C::B_KVFULL + slot), 2 * C::UNIT_BYTES);
        const uint32_t dst = sbase + C::KV_OFF + slot * C::UNIT_BYTES;
        if (is_v) {
          // columns 64·rank .. 64·rank + 63 of the 128-key V tile
          tma_load_2d_pair(dst, &tmV, LBAR(C::B_KVFULL + slot), 64 * (int)rank, kv_base + j * C::BN, pol_kv);
        } else {
          // keys 64·rank .. 64·rank + 63 of the K tile, both 64-column panels
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_2d_pair(dst + pn * C::KH_PANEL, &tmK, LBAR(C::B_KVFULL + slot), pn * 64,
                             kv_base + j * C::BN + 64 * (int)rank, pol_kv);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only)
    if (leader) {
      bool ok = mbar_wait_warp(BAR(C::B_QFULL), 0, wc, 62);
      tc_fence_after();
      int k_ready = -1, v_ready = -1;
      auto wait_unit = [&](int u) -> bool {
        if (!mbar_wait_warp(BAR(C::B_KVFULL + u % C::NSLOT), (u / C::NSLOT) & 1, wc, 63)) return false;
        tc_fence_after();
        return true;
      };
      auto release_unit = [&](int u) { tc_commit_pair_w(BAR(C::B_KVEMPTY + u % C::NSLOT)); };
      auto need_k = [&](int j) -> bool {
        if (j <= k_ready) return true;
        k_ready = j;
        return wait_unit(Ord::unitK(j, n));
      };
      auto need_v = [&](int j) -> bool {
        if (j <= v_ready) return true;
        v_ready = j;
        return wait_unit(Ord::unitV(j, n));
      };
      const uint64_t dQ_k = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dKV_k = sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::KV_OFF, C::UNIT_BYTES, 1024);
      // S[scol] = Q · K_jᵀ   (M = 256 queries of the pair, N = 128 keys, K = D)
      auto issue_s = [&](int j, int scol) {
        const uint64_t db0 = sdesc_add(dKV_k, (Ord::unitK(j, n) % C::NSLOT) * C::UNIT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_pair_w(tbase + scol, sdesc_add(dQ_k, (kk >> 2) * C::PANEL + (kk & 3) * 32),
                        sdesc_add(db0, (kk >> 2) * C::KH_PANEL + (kk & 3) * 32), C::IDESC_S, kk > 0 ? 1u : 0u);
      };
      // O (+)= P(TMEM at scol) · V_j; half 0 covers keys 0..63, half 1 keys 64..127
      auto issue_pv = [&](int j, int scol, int half) {
        const uint64_t db0 = sdesc_add(dKV_mn, (Ord::unitV(j, n) % C::NSLOT) * C::UNIT_BYTES);
#pragma unroll
        for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
          mma_ts_pair_w(tbase + C::O_COL, tbase + scol + kk * 8, sdesc_add(db0, kk * 2048), C::IDESC_PV,
                        (j > 0 || kk > 0) ? 1u : 0u);
      };
      if (ok) {
        ok = need_k(0);
        if (ok) {
          issue_s(0, C::S_COL);
          tc_commit_pair_w(BAR(C::B_SFULL + 0));
          release_unit(Ord::unitK(0, n));
        }
        if (ok && n > 1) {
          ok = need_k(1);
          if (ok) {
            issue_s(1, C::S_COL + 128);
            tc_commit_pair_w(BAR(C::B_SFULL + 1));
            release_unit(Ord::unitK(1, n));
          }
        }
        for (int j = 0; j < n && ok; ++j) {
          const int x = j & 1;
          if (!mbar_wait_warp(BAR(C::B_PFULL + x), (j >> 1) & 1, wc, 64)) { ok = false; break; }
          tc_fence_after();
          if (!need_v(j)) { ok = false; break; }
          issue_pv(j, C::S_COL + 128 * x, 0);
          if (!mbar_wait_warp(BAR(C::B_PFULL2 + x), (j >> 1) & 1, wc, 65)) { ok = false; break; }
          tc_fence_after();
          issue_pv(j, C::S_COL + 128 * x, 1);
          tc_commit_pair_w(BAR(C::B_ODONE + x));
          release_unit(Ord::unitV(j, n));
          if (j + 2 < n) {
            if (!need_k(j + 2)) { ok = false; break; }
            issue_s(j + 2, C::S_COL + 128 * x);
            tc_commit_pair_w(BAR(C::B_SFULL + x));
            release_unit(Ord::unitK(j + 2, n));
          }
        }
      }
      // no MMA may still be running when either CTA releases its TMEM
      tc_commit_pair_w(BAR(C::B_DRAIN));
      mbar_wait_warp(BAR(C::B_DRAIN), 0, wc, 66);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int q_row = qt * C::BM + row;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;    // Σ P in fp32: the normaliser of the LSE
    float l_o = 0.f;  // Σ of the bf16-rounded P: the normaliser of O
    bool ok = true;
    auto odone_idx = [&](int jj) { return jj & 1; };
    auto odone_par = [&](int jj) -> uint32_t { return (jj >> 1) & 1; };
    for (int j = 0; j < n; ++j) {
      const int x = j & 1;
      const uint32_t par = (j >> 1) & 1;
      const int scol = C::S_COL + 128 * x;
      if (!mbar_wait_warp(BAR(C::B_SFULL + x), par, wc, 67)) { ok = false; break; }
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
          l_o *= alpha;
        }
      }
      const float neg_m = -m_ref;
      uint64_t rs2[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
      uint64_t ro2[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
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
          ro2[c & 1] = f2_add(ro2[c & 1], bf2_to_f2(pk[c]));
        }
      };
      {
        uint32_t pk[32];
        exp_half(0, pk);
        if (warp_rescale) {
          if (!mbar_wait_warp(BAR(C::B_ODONE + odone_idx(j - 1)), odone_par(j - 1), wc, 68)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int oc = 0; oc < D / 32; ++oc) {
            uint32_t ov[32];
            tmem_ld32(tl + C::O_COL + oc * 32, ov);
            tmem_ld_wait();
            reg_fence(ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st32(tl + C::O_COL + oc * 32, ov);
          }
        }
        tmem_st32(tl + scol, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LBAR(C::B_PFULL + x));
      }
      {
        uint32_t pk[32];
        exp_half(64, pk);
        tmem_st32(tl + scol + 32, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LBAR(C::B_PFULL2 + x));
      }
      float a, b2, c2, d2;
      f2_split(rs2[0], a, b2);
      f2_split(rs2[1], c2, d2);
      l += (a + b2) + (c2 + d2);
      f2_split(ro2[0], a, b2);
      f2_split(ro2[1], c2, d2);
      l_o += (a + b2) + (c2 + d2);
    }
    if (ok) ok = mbar_wait_warp(BAR(C::B_ODONE + odone_idx(n - 1)), odone_par(n - 1), wc, 69);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_o;
      __nv_bfloat16* orow = p.o + ((size_t)q_base + q_row) * D;
#pragma unroll
      for (int oc = 0; oc < D / 32; ++oc) {
        uint32_t ov[32];
        tmem_ld32(tl + C::O_COL + oc * 32, ov);
        tmem_ld_wait();
        reg_fence(ov);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv_l, __uint_as_float(ov[2 * c + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + oc * 32);
        if (!TAIL || q_row < p.N) {
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      float lg;
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
      if (!TAIL || q_row < p.N) p.lse[(size_t)q_base + q_row] = (m_ref + lg) * kLn2;
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
