// Persistent forward kernel for head dimensions 64 and 128 (two query tiles
// per work item).
//
// Same arithmetic as fa_fwd_kernel ("深度学习进阶（三十一）FlashAttention：IO 感知的
// 精确注意力" §2.2: per-row running max, normaliser and output updated after
// every K/V block), but one CTA per SM walks a list of work items
// (batch, head, pair of 128-row query tiles) so that one item's epilogue and
// the next item's Q/K loads and first QKᵀ overlap the running item:
//   * each query tile has its own Q buffer; it is reloaded as soon as the
//     tile's last QKᵀ of the item has completed;
//   * the next item's first QKᵀ for a tile is issued right after the tile's
//     last PV product, so the tensor pipe is fed while the softmax warpgroup
//     writes the finished tile out;
//   * at d = 64, P has TMEM columns of its own and each tile has its own MMA
//     warp, so a tile's next QKᵀ is issued as soon as its softmax has read S;
//   * with a causal mask the second tile of a pair sees one more K/V block
//     than the first (its diagonal block).  That block is processed first, so
//     both tiles finish an item in the same iteration;
//   * causal items are ordered heaviest first, dealt to CTAs in alternating
//     directions round by round; non-causal items are ordered head by head, so
//     concurrently running CTAs share K/V tiles in L2.
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner (at d = 64
// the MMA issuer of query tile 0, warp 2 that of tile 1), the other control
// warps idle, warps 4-7 / 8-11 softmax of query tile 0 / 1 (thread = query
// row).
#pragma once

#include "fa_fwd.cuh"

namespace fa {

template <int D>
struct FwdPCfg {
  using B = FwdCfg<D>;
  static_assert(B::NQ == 2, "persistent kernel covers two query tiles per item");
  static constexpr int BM = B::BM, BN = B::BN, CH = B::CH, NCH = B::NCH, PANEL = B::PANEL;
  static constexpr int THREADS = B::THREADS;
  static constexpr int Q_BYTES = B::Q_BYTES;
  static constexpr int SLOT_BYTES = B::SLOT_BYTES;
  static constexpr int NSLOT = B::NSLOT;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * Q_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSLOT * SLOT_BYTES;
  static constexpr int B_QFULL = 0;                  // + tile
  static constexpr int B_QEMPTY = 2;                 // + tile
  static constexpr int B_KVFULL = 4;                 // + slot
  static constexpr int B_KVEMPTY = 4 + NSLOT;        // + slot
  static constexpr int B_SFULL = 4 + 2 * NSLOT;      // + tile
  static constexpr int B_PFULL = B_SFULL + 2;        // + tile: P keys 0..63 in TMEM
  static constexpr int B_PFULL2 = B_PFULL + 2;       // + tile: P keys 64..127 in TMEM
  static constexpr int B_ODONE = B_PFULL2 + 2;       // + tile
  static constexpr int B_DRAIN = B_ODONE + 2;
  static constexpr int B_SFREE = B_DRAIN + 1;        // + tile: S read out of TMEM (SEP_P)
  static constexpr int NBAR = B_SFREE + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0;    // S of tile t at S_COL + 128·t
  static constexpr int O_COL = 256;  // O of tile t at O_COL + t·D
  // P (bf16, 64 columns for 128 keys): over the first 64 columns of its S
  // buffer, or, at d = 64 where TMEM has room, in columns of its own
  // (SEP_P).  Then a tile's next QKᵀ need not follow the PV that reads P: it
  // is issued as soon as the softmax has loaded S into registers.
  static constexpr bool SEP_P = (D == 64);
  static constexpr int P_COL = O_COL + 2 * D;  // SEP_P: P of tile t at P_COL + 64·t
  // One MMA warp per query tile (warps 1, 2) goes with SEP_P: each tile's
  // next QKᵀ is issued as soon as its softmax has read S, whatever the other
  // tile is doing.  Without SEP_P one MMA warp issues both tiles' products in
  // strict alternation, which keeps the two softmax warpgroups half a block
  // apart (measured faster at d = 128 than two independent issuers).
  static constexpr bool PER_TILE = SEP_P;
  static constexpr int MMA_WARPS = PER_TILE ? 2 : 1;
  static constexpr uint32_t IDESC_S = B::IDESC_S;
  static constexpr uint32_t IDESC_PV = B::IDESC_PV;
  // Register split (setmaxnreg): the item bookkeeping of the producer and MMA
  // warps needs more than the single-item kernel's control share.  Valid for a
  // launch allocation R with CTRL_REGS <= R <= SOFTMAX_REGS and
  // 128·CTRL_REGS + 256·SOFTMAX_REGS <= 384·R (checked on the host).
  static constexpr int CTRL_REGS = 120;
  static constexpr int SOFTMAX_REGS = 192;
  static constexpr bool REG_SPLIT = true;
  static constexpr int MIN_LAUNCH_REGS = (128 * CTRL_REGS + 256 * SOFTMAX_REGS + THREADS - 1) / THREADS;
  static constexpr int MAX_LAUNCH_REGS = SOFTMAX_REGS;
  // Exponentials moved from the MUFU to the FMA pipes (exp2_poly): the second
  // one of every kPolyPairs-th column pair, 1/8 of them at d = 64, where the
  // MUFU rather than the tensor pipe bounds a tile (+3 % measured); none at
  // d = 128, where every fraction tried (1/8, 1/4, 1/2) was slower.
  static constexpr int kPolyPairs = (D == 64) ? 4 : 0;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(!SEP_P || P_COL + 128 <= TMEM_COLS, "TMEM budget (separate P)");
};

struct FwdPParams {
  __nv_bfloat16* o;
  float* lse;
  int N, Hq, G, n_qtiles;
  int n_units;  // query-tile pairs per (batch, head)
  int BH;       // batch · query heads
  int n_items;  // n_units · BH (VARLEN: from the work table, see below)
  float scale_log2;
  long long wait_cap;
  int* err;
  // VARLEN only: packed sequences of T tokens per head, cu_seqlens, and the
  // work table of (sequence, tile pair) units with its header (hdr[0] units)
  const int2* table;
  const int* cu;
  const int* hdr;
  int T;
};

// One work item: query tiles qt0 (tile 0) and qt0 + 1 (tile 1, absent when
// qt0 is the last tile) of one (batch or sequence, head).  Iteration jj of
// the item multiplies by K/V block kv_block(jj); tile 0 takes part from
// iteration skew on, tile 1 in all.  qbase / kvbase are the rows of the
// sequence's first token in the Q (and O, LSE) and K/V tensors, len its
// length.
struct FwdItem {
  int h, qt0, n0, n1, skew, nit;
  int qbase, kvbase, len;
  __device__ int kv_block(int jj) const { return (skew && jj == 0) ? qt0 + 1 : jj - skew; }
  __device__ int first(int t) const { return t == 0 ? skew : 0; }
  __device__ bool has(int t) const { return t == 0 || n1 > 0; }
};

// ne: VARLEN work-table entries (hdr[0]).  Causal items go heaviest first
// across all heads; non-causal items head by head, so that CTAs running at
// the same time share a head's K/V tiles in L2.
template <bool CAUSAL, bool VARLEN>
__device__ __forceinline__ FwdItem fwd_item(int idx, const FwdPParams& p, int ne) {
  FwdItem w;
  int unit, n_qtiles;
  if (VARLEN) {
    int e;
    if (CAUSAL) {
      e = idx / p.Hq;
      w.h = idx % p.Hq;
    } else {
      w.h = idx / ne;
      e = idx % ne;
    }
    const int2 ent = p.table[e];
    unit = ent.y;
    const int start = p.cu[ent.x];
    w.len = p.cu[ent.x + 1] - start;
    w.qbase = w.h * p.T + start;
    w.kvbase = (w.h / p.G) * p.T + start;
    n_qtiles = (w.len + 127) / 128;
  } else {
    int bh;
    if (CAUSAL) {
      unit = p.n_units - 1 - idx / p.BH;  // heaviest (latest) query tiles first
      bh = idx % p.BH;
    } else {
      bh = idx / p.n_units;
      unit = idx % p.n_units;
    }
    const int b = bh / p.Hq;
    w.h = bh % p.Hq;
    w.len = p.N;
    w.qbase = bh * p.N;
    w.kvbase = (b * (p.Hq / p.G) + w.h / p.G) * p.N;
    n_qtiles = p.n_qtiles;
  }
  w.qt0 = 2 * unit;
  const bool has1 = w.qt0 + 1 < n_qtiles;
  w.n0 = CAUSAL ? w.qt0 + 1 : n_qtiles;
  w.n1 = has1 ? (CAUSAL ? w.qt0 + 2 : n_qtiles) : 0;
  w.skew = (CAUSAL && has1) ? 1 : 0;
  w.nit = w.n0 + w.skew;
  return w;
}

// Index of the k-th item of CTA c among G CTAs: round k covers items
// [k·G, (k+1)·G); causal rounds alternate direction so that every CTA gets a
// mix of heavier and lighter items.
template <bool CAUSAL>
__device__ __forceinline__ int fwd_item_index(int k, int c, int G) {
  return k * G + ((CAUSAL && (k & 1)) ? (G - 1 - c) : c);
}

// TAIL: N is not a multiple of 128 (keys past N masked, rows past N not stored).
// VARLEN: a packed batch of sequences (always with TAIL); items come from the
// work table, each with its own length and row bases.
template <int D, bool CAUSAL, bool TAIL, bool VARLEN = false>
__global__ void __launch_bounds__(FwdPCfg<D>::THREADS, 1)
    fa_fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const FwdPParams p) {
  using C = FwdPCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  static_assert(!VARLEN || TAIL, "packed sequences have ragged ends");
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int ne = VARLEN ? p.hdr[0] : 0;
  const int n_items = VARLEN ? ne * p.Hq : p.n_items;
  const int n_rounds = (n_items + G - 1) / G;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(C::B_QFULL + t), 1);
      mbar_init(BAR(C::B_QEMPTY + t), 1);
      mbar_init(BAR(C::B_SFULL + t), 1);
      mbar_init(BAR(C::B_PFULL + t), 4);
      mbar_init(BAR(C::B_PFULL2 + t), 4);
      mbar_init(BAR(C::B_ODONE + t), 1);
      mbar_init(BAR(C::B_SFREE + t), 4);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(BAR(C::B_KVFULL + i), 1);
      mbar_init(BAR(C::B_KVEMPTY + i), C::MMA_WARPS);  // released by every MMA warp
    }
    mbar_init(BAR(C::B_DRAIN), C::MMA_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
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
      int useq = 0;               // K/V units loaded so far (a unit is NCH chunks)
      int qloads[2] = {0, 0};     // Q tiles loaded so far, per tile buffer
      int kv_issued = 0;          // K/V chunk loads issued (chunk sequence numbers 0 .. kv_issued − 1)
      bool ok = true;
      for (int k = 0; k < n_rounds && ok; ++k) {
        const int idx = fwd_item_index<CAUSAL>(k, cta, G);
        if (idx >= n_items) continue;
        const FwdItem w = fwd_item<CAUSAL, VARLEN>(idx, p, ne);
        const int q_row_base = w.qbase;
        const int kv_row_base = w.kvbase;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!w.has(t)) continue;
          // the previous item's last QKᵀ of this tile must be done reading the buffer
          if (qloads[t] > 0 && !mbar_wait(BAR(C::B_QEMPTY + t), (qloads[t] - 1) & 1, wc, 41)) { ok = false; break; }
          mbar_expect_tx(BAR(C::B_QFULL + t), C::Q_BYTES);
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_2d_hint(sbase + C::Q_OFF + t * C::Q_BYTES + pn * C::PANEL, &tmQ, BAR(C::B_QFULL + t), pn * 64,
                             q_row_base + (w.qt0 + t) * C::BM, pol_q);
          ++qloads[t];
        }
        for (int u = 0; u < 2 * w.nit && ok; ++u) {
          const int kb = w.kv_block(u >> 1);
          const bool is_v = (u & 1);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            const int seq = (useq + u) * C::NCH + c;
            const int slot = seq % C::NSLOT;
            if (!mbar_wait(BAR(C::B_KVEMPTY + slot), ((seq / C::NSLOT) & 1) ^ 1, wc, 42)) { ok = false; break; }
            mbar_expect_tx(BAR(C::B_KVFULL + slot), C::SLOT_BYTES);
#pragma unroll
            for (int pp = 0; pp < C::CH / 64; ++pp)
              tma_load_2d_hint(sbase + C::KV_OFF + slot * C::SLOT_BYTES + pp * C::PANEL, is_v ? &tmV : &tmK,
                               BAR(C::B_KVFULL + slot), c * C::CH + pp * 64, kv_row_base + kb * C::BN, pol_kv);
            kv_issued = seq + 1;
          }
        }
        useq += 2 * w.nit;
      }
      // every load issued has landed before the CTA may exit (immediate unless
      // the CTA stopped early on a failed wait)
      for (int t = 0; t < 2; ++t)
        if (qloads[t] > 0) mbar_wait_inflight(BAR(C::B_QFULL + t), (qloads[t] - 1) & 1, wc, 53);
      for (int sl = 0; sl < C::NSLOT && sl < kv_issued; ++sl) {
        const int last = kv_issued - 1 - (kv_issued - 1 - sl) % C::NSLOT;  // last chunk loaded into slot sl
        mbar_wait_inflight(BAR(C::B_KVFULL + sl), (last / C::NSLOT) & 1, wc, 54);
      }
    }
  } else if (warp == 1 || (C::PER_TILE && warp == 2)) {
    if constexpr (C::PER_TILE) {
      // ------------------------------------------------ MMA issuers, one per tile
      // Warp 1 + t issues query tile t's products only (the whole warp runs the
      // role; one elected lane issues each instruction).  Both warps walk every
      // K/V unit of their items in load order and release each one (the slot's
      // empty barrier counts two arrivals); a unit the tile does not read (the
      // other tile's diagonal block, an item without tile 1) is released once
      // this fill of its slot has landed, so that no release can count towards
      // the slot's previous fill.
      setmaxnreg_dec<C::CTRL_REGS>();
      const int t = warp - 1;
      bool ok = true;
      int qfull_seen = 0;
      int p_seen = 0;  // P hand-overs consumed
      int s_cnt = 0;   // QKᵀ products issued into this tile's S buffer
      // Wait for the fill of unit U: a warp never lags a full fill behind a
      // slot, because the slot is refilled only after both warps released it.
      auto wait_unit = [&](int U) -> bool {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int seq = U * C::NCH + c;
          if (!mbar_wait_warp(BAR(C::B_KVFULL + seq % C::NSLOT), (seq / C::NSLOT) & 1, wc, 43)) return false;
        }
        tc_fence_after();
        return true;
      };
      auto release = [&](int U) {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) tc_commit_w(BAR(C::B_KVEMPTY + (U * C::NCH + c) % C::NSLOT));
      };
      const uint64_t dQ_t = sdesc_add(sdesc_sw128(sbase + C::Q_OFF, 16, 1024), t * C::Q_BYTES);
      const uint64_t dKV_k = sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::KV_OFF, C::PANEL, 1024);
      const uint32_t s_tm = tbase + C::S_COL + 128 * t;
      const uint32_t p_tm = tbase + (C::SEP_P ? C::P_COL + 64 * t : C::S_COL + 128 * t);
      const uint32_t o_tm = tbase + C::O_COL + t * D;
      // S_t = Q_t · Kᵀ for iteration jj of item w (its K unit is base + 2·jj)
      auto issue_s = [&](const FwdItem& w, int base, int jj) -> bool {
        // SEP_P: the softmax must have read the previous S out of the buffer
        // (otherwise the PV issued before this QKᵀ orders it after that read)
        if (C::SEP_P && s_cnt > 0) {
          if (!mbar_wait_warp(BAR(C::B_SFREE + t), (s_cnt - 1) & 1, wc, 51)) return false;
          tc_fence_after();
        }
        ++s_cnt;
        if (jj == w.first(t)) {
          if (!mbar_wait_warp(BAR(C::B_QFULL + t), qfull_seen & 1, wc, 44)) return false;
          ++qfull_seen;
        }
        const int U = base + 2 * jj;
        if (!wait_unit(U)) return false;
        uint64_t db0[C::NCH];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) db0[c] = sdesc_add(dKV_k, ((U * C::NCH + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int col = kk * 16;
          mma_ss_w(s_tm, sdesc_add(dQ_t, (kk >> 2) * C::PANEL + (kk & 3) * 32),
                   sdesc_add(db0[col / C::CH], ((col % C::CH) / 64) * C::PANEL + (kk & 3) * 32), C::IDESC_S,
                   kk > 0 ? 1u : 0u);
        }
        tc_commit_w(BAR(C::B_SFULL + t));
        if (jj == w.nit - 1) tc_commit_w(BAR(C::B_QEMPTY + t));  // last QKᵀ of this tile in the item
        release(U);
        return true;
      };
      // O_t (+)= P_t · V for one 64-key half of the P tile
      auto issue_pv = [&](int U, bool first, int half) {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint64_t db0 = sdesc_add(dKV_mn, ((U * C::NCH + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
          for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
            mma_ts_w(o_tm + c * C::CH, p_tm + kk * 8, sdesc_add(db0, kk * 2048), C::IDESC_PV,
                     (!first || kk > 0) ? 1u : 0u);
        }
      };

      int k = 0;
      while (k < n_rounds && fwd_item_index<CAUSAL>(k, cta, G) >= n_items) ++k;
      if (k < n_rounds) {
        FwdItem w = fwd_item<CAUSAL, VARLEN>(fwd_item_index<CAUSAL>(k, cta, G), p, ne);
        int base = 0;
        if (w.has(t)) ok = issue_s(w, base, w.first(t));
        while (ok) {
          int k2 = k + 1;
          while (k2 < n_rounds && fwd_item_index<CAUSAL>(k2, cta, G) >= n_items) ++k2;
          const bool has_next = k2 < n_rounds;
          FwdItem w2 = w;
          if (has_next) w2 = fwd_item<CAUSAL, VARLEN>(fwd_item_index<CAUSAL>(k2, cta, G), p, ne);
          const int base2 = base + 2 * w.nit;
          for (int jj = 0; jj < w.nit && ok; ++jj) {
            if (!w.has(t) || jj < w.first(t)) {
              // K and V units of this iteration that this tile does not read
              if (!wait_unit(base + 2 * jj) || !wait_unit(base + 2 * jj + 1)) { ok = false; break; }
              release(base + 2 * jj);
              release(base + 2 * jj + 1);
              continue;
            }
            // SEP_P: the tile's next QKᵀ of this item goes before its PV (the
            // next item's first one stays after it: it may wait for a Q load)
            if (C::SEP_P && jj + 1 < w.nit && !(ok = issue_s(w, base, jj + 1))) break;
            const int Uv = base + 2 * jj + 1;
            const bool first = (jj == w.first(t));
            if (!mbar_wait_warp(BAR(C::B_PFULL + t), p_seen & 1, wc, 45)) { ok = false; break; }
            if (!wait_unit(Uv)) { ok = false; break; }
            issue_pv(Uv, first, 0);
            if (!mbar_wait_warp(BAR(C::B_PFULL2 + t), p_seen & 1, wc, 46)) { ok = false; break; }
            tc_fence_after();
            issue_pv(Uv, first, 1);
            tc_commit_w(BAR(C::B_ODONE + t));
            ++p_seen;
            release(Uv);
            // this tile's next QKᵀ: the item's next iteration, or the next item's first
            if (jj + 1 < w.nit) {
              if (!C::SEP_P) ok = issue_s(w, base, jj + 1);
            } else if (has_next && w2.has(t)) {
              ok = issue_s(w2, base2, w2.first(t));
            }
          }
          if (!ok || !has_next) break;
          // the tile had no rows in this item, so its first QKᵀ of the next one is still due
          if (!w.has(t) && w2.has(t)) ok = issue_s(w2, base2, w2.first(t));
          w = w2;
          base = base2;
          k = k2;
        }
      }
      // no MMA of either warp may still be running when TMEM is released
      tc_commit_w(BAR(C::B_DRAIN));
      mbar_wait_inflight(BAR(C::B_DRAIN), 0, wc, 47);
    } else {
      // ---------------------------------------------------------- MMA issuer
      // (the whole warp runs this role; one elected lane issues each instruction)
      setmaxnreg_dec<C::CTRL_REGS>();
      bool ok = true;
      int waited = -1;           // K/V units whose arrival has been observed, in load order
      int qfull_seen[2] = {0, 0};
      int p_seen[2] = {0, 0};    // P hand-overs consumed per tile
      // Wait for every unit up to U in load order: a unit's slot barrier is only
      // ever waited on for its current fill, so the parity test is unambiguous.
      auto wait_upto = [&](int U) -> bool {
        while (waited < U) {
          ++waited;
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            const int seq = waited * C::NCH + c;
            if (!mbar_wait_warp(BAR(C::B_KVFULL + seq % C::NSLOT), (seq / C::NSLOT) & 1, wc, 43)) return false;
          }
        }
        tc_fence_after();
        return true;
      };
      auto release = [&](int U) {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) tc_commit_w(BAR(C::B_KVEMPTY + (U * C::NCH + c) % C::NSLOT));
      };
      const uint64_t dQ_k = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dKV_k = sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::KV_OFF, C::PANEL, 1024);
      // S_t = Q_t · Kᵀ for iteration jj of item w (its K unit is base + 2·jj)
      auto issue_s = [&](int t, const FwdItem& w, int base, int jj) -> bool {
        if (jj == w.first(t)) {
          if (!mbar_wait_warp(BAR(C::B_QFULL + t), qfull_seen[t] & 1, wc, 44)) return false;
          ++qfull_seen[t];
        }
        const int U = base + 2 * jj;
        if (!wait_upto(U)) return false;
        const uint64_t da0 = sdesc_add(dQ_k, t * C::Q_BYTES);
        uint64_t db0[C::NCH];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) db0[c] = sdesc_add(dKV_k, ((U * C::NCH + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int col = kk * 16;
          mma_ss_w(tbase + C::S_COL + 128 * t, sdesc_add(da0, (kk >> 2) * C::PANEL + (kk & 3) * 32),
                   sdesc_add(db0[col / C::CH], ((col % C::CH) / 64) * C::PANEL + (kk & 3) * 32), C::IDESC_S,
                   kk > 0 ? 1u : 0u);
        }
        tc_commit_w(BAR(C::B_SFULL + t));
        if (jj == w.nit - 1) tc_commit_w(BAR(C::B_QEMPTY + t));  // last QKᵀ of this tile in the item
        if (t == 1 || w.n1 == 0) release(U);                      // last reader of this K unit
        return true;
      };
      // O_t (+)= P_t · V for one 64-key half of the P tile
      auto issue_pv = [&](int t, int U, bool first, int half) {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint64_t db0 = sdesc_add(dKV_mn, ((U * C::NCH + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
          for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
            mma_ts_w(tbase + C::O_COL + t * D + c * C::CH, tbase + C::S_COL + 128 * t + kk * 8,
                     sdesc_add(db0, kk * 2048), C::IDESC_PV, (!first || kk > 0) ? 1u : 0u);
        }
      };

      int k = 0;
      while (k < n_rounds && fwd_item_index<CAUSAL>(k, cta, G) >= n_items) ++k;
      if (k < n_rounds) {
        FwdItem w = fwd_item<CAUSAL, VARLEN>(fwd_item_index<CAUSAL>(k, cta, G), p, ne);
        int base = 0;
        for (int t = 0; t < 2 && ok; ++t)
          if (w.has(t)) ok = issue_s(t, w, base, w.first(t));
        while (ok) {
          int k2 = k + 1;
          while (k2 < n_rounds && fwd_item_index<CAUSAL>(k2, cta, G) >= n_items) ++k2;
          const bool has_next = k2 < n_rounds;
          FwdItem w2 = w;
          if (has_next) w2 = fwd_item<CAUSAL, VARLEN>(fwd_item_index<CAUSAL>(k2, cta, G), p, ne);
          const int base2 = base + 2 * w.nit;
          for (int jj = 0; jj < w.nit && ok; ++jj) {
            for (int t = 0; t < 2; ++t) {
              if (!w.has(t) || jj < w.first(t)) continue;
              const int Uv = base + 2 * jj + 1;
              const bool first = (jj == w.first(t));
              if (!mbar_wait_warp(BAR(C::B_PFULL + t), p_seen[t] & 1, wc, 45)) { ok = false; break; }
              if (!wait_upto(Uv)) { ok = false; break; }
              issue_pv(t, Uv, first, 0);
              if (!mbar_wait_warp(BAR(C::B_PFULL2 + t), p_seen[t] & 1, wc, 46)) { ok = false; break; }
              tc_fence_after();
              issue_pv(t, Uv, first, 1);
              tc_commit_w(BAR(C::B_ODONE + t));
              ++p_seen[t];
              if (t == 1 || w.n1 == 0) release(Uv);  // last reader of this V unit
              // this tile's next QKᵀ: the item's next iteration, or the next item's first
              if (jj + 1 < w.nit) {
                ok = issue_s(t, w, base, jj + 1);
              } else if (has_next && w2.has(t)) {
                ok = issue_s(t, w2, base2, w2.first(t));
              }
              if (!ok) break;
            }
          }
          if (!ok || !has_next) break;
          // tile 1 had no rows in this item, so its first QKᵀ of the next one is still due
          if (!w.has(1) && w2.has(1)) ok = issue_s(1, w2, base2, 0);
          w = w2;
          base = base2;
          k = k2;
        }
      }
      // no MMA may still be running when TMEM is released
      tc_commit_w(BAR(C::B_DRAIN));
      mbar_wait_inflight(BAR(C::B_DRAIN), 0, wc, 47);
    }
  } else if (warp < 4) {
    // idle warps of the control warpgroup: hand their registers to the softmax
    setmaxnreg_dec<C::CTRL_REGS>();
  } else {
    // ------------------------------------------------------------- softmax
    setmaxnreg_inc<C::SOFTMAX_REGS>();
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    const int scol = C::S_COL + 128 * t;
    const int ocol = C::O_COL + t * D;
    const int pcol = C::SEP_P ? C::P_COL + 64 * t : scol;
    int done = 0;  // S tiles this warpgroup has finished (phase count of its barriers)
    bool ok = true;
    for (int k = 0; k < n_rounds && ok; ++k) {
      const int idx = fwd_item_index<CAUSAL>(k, cta, G);
      if (idx >= n_items) continue;
      const FwdItem w = fwd_item<CAUSAL, VARLEN>(idx, p, ne);
      if (!w.has(t)) continue;
      const int n = t == 0 ? w.n0 : w.n1;
      const int qt = w.qt0 + t;
      float m_ref = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t par = (done + j) & 1;
        if (!mbar_wait_warp(BAR(C::B_SFULL + t), par, wc, 48)) { ok = false; break; }
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
        if (C::SEP_P) {
          // S is in registers: the tile's next QKᵀ may overwrite the buffer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_SFREE + t));
        }
        float s[128];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = __uint_as_float(r0[c]);
          s[32 + c] = __uint_as_float(r1[c]);
          s[64 + c] = __uint_as_float(r2[c]);
          s[96 + c] = __uint_as_float(r3[c]);
        }
        const int kb = w.kv_block(w.first(t) + j);
        if (CAUSAL && kb == qt) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > row) s[c] = -INFINITY;
        }
        // ragged N: keys past the end of the sequence (the causal mask already
        // excludes them for every row < N)
        if (TAIL && !CAUSAL && (kb + 1) * C::BN > w.len) {
          const int lim = w.len - kb * C::BN;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        const float mx = row_max128(s);
        const float m_new = fmaxf(m_ref, mx * sl2);
        // conditional rescale against a stale reference max (see fa_fwd_kernel)
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
            // every kPolyPairs-th pair's second exponential on the FMA pipes
            const float a1 = (C::kPolyPairs > 0 && c % (C::kPolyPairs > 0 ? C::kPolyPairs : 1) == 0) ? exp2_poly(x1)
                                                                                                   : ex2(x1);
            rs2[c & 1] = f2_add(rs2[c & 1], f2_make(a0, a1));
            pk[c] = pack_bf16(a0, a1);
          }
        };
        {
          uint32_t pk[32];
          exp_half(0, pk);
          if (C::SEP_P && j > 0 && !warp_rescale) {
            // the previous block's PV must be done reading P before it is overwritten
            if (!mbar_wait_warp(BAR(C::B_ODONE + t), (done + j - 1) & 1, wc, 52)) { ok = false; break; }
            tc_fence_after();
          }
          if (warp_rescale) {
            // O must hold the previous block's product before it is scaled,
            // and be scaled before this block's first PV half accumulates
            if (!mbar_wait_warp(BAR(C::B_ODONE + t), (done + j - 1) & 1, wc, 49)) { ok = false; break; }
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
          tmem_st32(tl + pcol, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_PFULL + t));
        }
        {
          uint32_t pk[32];
          exp_half(64, pk);
          tmem_st32(tl + pcol + 32, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_PFULL2 + t));
        }
        float a, b2, c2, d2;
        f2_split(rs2[0], a, b2);
        f2_split(rs2[1], c2, d2);
        l += (a + b2) + (c2 + d2);
      }
      if (!ok) break;
      // epilogue: the item's last PV must be complete; the MMA warp overwrites
      // O with the next item's first PV only after this warpgroup hands over
      // that item's first P, i.e. after the loads below
      if (!mbar_wait_warp(BAR(C::B_ODONE + t), (done + n - 1) & 1, wc, 50)) { ok = false; break; }
      tc_fence_after();
      const int q_row = qt * C::BM + row;
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = p.o + ((size_t)w.qbase + q_row) * D;
#pragma unroll
      for (int oc = 0; oc < D / 32; ++oc) {
        uint32_t ov[32];
        tmem_ld32(tl + ocol + oc * 32, ov);
        tmem_ld_wait();
        reg_fence(ov);
        uint32_t wv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          wv[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv_l, __uint_as_float(ov[2 * c + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + oc * 32);
        if (!TAIL || q_row < w.len) {  // rows past a ragged end are computed, not stored
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
        }
      }
      float lg;
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
      if (!TAIL || q_row < w.len) p.lse[(size_t)w.qbase + q_row] = (m_ref + lg) * kLn2;
      done += n;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa
