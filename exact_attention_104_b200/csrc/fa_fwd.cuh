// Fused exact-attention forward pass for sm_100a.
//
// Computes O = softmax(s·Q Kᵀ [+ causal mask]) V and the per-row log-sum-exp,
// keeping the score and probability tiles on chip (TMEM / registers) as the
// FlashAttention pages describe: "深度学习进阶（三十一）FlashAttention：IO 感知的精确
// 注意力" §2.2 (fix a Q block, stream every K/V block, update the per-row running
// max m, normaliser d and output O after each block) and the "Flash-Attention"
// concept page, "Core idea" (tile into on-chip memory, write only O and a few
// per-row statistics).
//
// FwdCfg holds the tile shapes shared with the persistent kernel
// (fa_fwd_persistent.cuh), which handles d = 64 and 128 with two query tiles
// per work item.  fa_fwd_kernel below is the d = 256 kernel: one CTA owns one
// 128-row query tile of one (batch, head):
//   warp 0        TMA producer: the Q tile once, then K/V chunks through a ring
//   warp 1        MMA issuer + TMEM owner
//   warps 4-7     softmax warpgroup; thread = query row
// S = Q Kᵀ and O += P V both run on tcgen05 with fp32 accumulators in TMEM.
// P (bf16) is written back over the first half of its S columns and read by
// the PV MMA directly from TMEM.  The O rescale is conditional: a row keeps a
// stale reference max until the true max exceeds it by more than kRescaleTau
// (log2 units); l and O share that reference, so the result is unchanged.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr float kRescaleTau = 8.0f;

// NQ_: query tiles per CTA (two in the persistent kernel for d = 64, 128;
// one in fa_fwd_kernel).
template <int D, int NQ_ = (D <= 128) ? 2 : 1>
struct FwdCfg {
  static constexpr int BM = 128;                 // query rows per tile (MMA M)
  static constexpr int BN = 128;                 // keys per K/V tile (MMA N of QKᵀ)
  static constexpr int NQ = NQ_;                 // query tiles per CTA
  static constexpr int THREADS = 128 + 128 * NQ;
  static constexpr int CH = D < 128 ? D : 128;   // K/V chunk width in columns
  static constexpr int NCH = D / CH;             // chunks per K or V tile
  static constexpr int PANEL = 128 * 128;        // one 64-column panel of a 128-row tile (bytes)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int SLOT_BYTES = BN * CH * 2;
  static constexpr int NSLOT = (D == 64) ? 8 : 5;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = NQ * Q_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSLOT * SLOT_BYTES;
  // barrier indices
  static constexpr int B_QFULL = 0;
  static constexpr int B_KVFULL = 1;                 // + slot
  static constexpr int B_KVEMPTY = 1 + NSLOT;        // + slot
  static constexpr int B_SFULL = 1 + 2 * NSLOT;      // + {0,1}
  static constexpr int B_PFULL = B_SFULL + 2;        // + {0,1}: P keys 0..63 in TMEM
  static constexpr int B_PFULL2 = B_PFULL + 2;       // + {0,1}: P keys 64..127 in TMEM
  static constexpr int B_ODONE = B_PFULL2 + 2;       // + {0,1}
  static constexpr int B_DRAIN = B_ODONE + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align the base to 1024
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0;    // S buffer x at S_COL + 128*x
  static constexpr int O_COL = 256;  // O of query tile t at O_COL + t*D
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, CH, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL + NQ * D <= TMEM_COLS, "TMEM budget");
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int N, Hq, Hkv, G, n_qtiles;
  float scale_log2;
  long long wait_cap;
  int* err;
  // VARLEN only: packed sequences of T tokens per head, cu_seqlens, and the
  // work table of (sequence, query tile) units with its header (hdr[0] units)
  const int2* table;
  const int* cu;
  const int* hdr;
  int T;
  // DECODE only: Nq query rows per head against Nk keys; the G·Nq rows of a
  // kv head's query group (R of them) in n_rt tiles of 128; the key axis in
  // n_split splits of tiles_per_split 128-key tiles; partial results
  int Nq, Nk, R, n_rt, n_split, tiles_per_split;
  float* part_o;   // [n_split][B·Hkv·n_rt][128][d]
  float* part_ml;  // [n_split][B·Hkv·n_rt][128][2]: m (log2 units), l
};

// fa_fwd_kernel modes: one (batch, head, query tile) per CTA; a packed batch
// of sequences; decoding (a kv head's query group against one key split).
enum : int { kFwdDense = 0, kFwdVarlen = 1, kFwdDecode = 2 };

// Load order of the K/V tiles ("units"; each unit is NCH chunks) of the
// one-tile kernel: it keeps two S tiles in flight, so the MMA warp first uses
// K(0), K(1), V(0), K(2), V(1), ..., K(n-1), V(n-2), V(n-1).
struct KVOrder {
  __device__ static int unitK(int j, int n) { return j == 0 ? 0 : 2 * j - 1; }
  __device__ static int unitV(int j, int n) { return (j == n - 1) ? 2 * n - 1 : 2 * j + 2; }
  // inverse: unit u -> (is_v, j)
  __device__ static void decode(int u, int n, bool& is_v, int& j) {
    if (u == 0) { is_v = false; j = 0; }
    else if (u == 2 * n - 1) { is_v = true; j = n - 1; }
    else if (u & 1) { is_v = false; j = (u + 1) >> 1; }
    else { is_v = true; j = (u >> 1) - 1; }
  }
};

// Maximum of 128 values: eight independent chains of three-input max, then a
// small tree (short dependency chains keep the issue slots busy).
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float a = fmaxf(s[16 * k], s[16 * k + 1]);
#pragma unroll
    for (int i = 2; i < 16; i += 2) a = fmax3(a, s[16 * k + i], s[16 * k + i + 1]);
    acc[k] = a;
  }
  return fmaxf(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], fmax3(acc[5], acc[6], acc[7])));
}

// TAIL: N is not a multiple of 128 (keys past N masked, rows past N not stored).
// MODE kFwdVarlen: a packed batch of sequences (always with TAIL): a 1-D grid
// of at least table-entries × Hq CTAs; CTA i takes unit i (causal: heaviest
// first across heads, else head by head) and CTAs past the last unit exit at
// once.
// MODE kFwdDecode: grid (n_split, B·Hkv·n_rt); a CTA multiplies one 128-row
// tile of a kv head's query group (row r = g·Nq + i: query i of head
// hkv·G + g, at sequence position Nk − Nq + i) by the 128-key tiles of one
// key split, with a per-row position mask, and writes the split's
// unnormalised O with its reference max m and normaliser l for the combine
// kernel.  The group's rows are contiguous in q ([B, Hq, Nq, d], heads of a
// group adjacent), so one 128-row box loads them; every row of a K/V tile
// serves up to 128 query rows (the CUDA-core decode kernel serves 16).
template <int D, bool CAUSAL, bool TAIL, int MODE = kFwdDense>
__global__ void __launch_bounds__(FwdCfg<D, 1>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, 1>;
  using Ord = KVOrder;
  constexpr bool VARLEN = MODE == kFwdVarlen;
  constexpr bool DECODE = MODE == kFwdDecode;
  static_assert(!VARLEN || TAIL, "packed sequences have ragged ends");
  int h = 0, qt = 0, len = 0, q_base = 0, kv_base = 0, n = 0;
  int t0 = 0, rt = 0, rows_valid = C::BM;  // DECODE: first key tile, row tile, real rows of the tile
  if (DECODE) {
    const int unit = blockIdx.y;
    rt = unit % p.n_rt;
    const int hkv = (unit / p.n_rt) % p.Hkv;
    const int b = unit / (p.n_rt * p.Hkv);
    q_base = (b * p.Hq + hkv * p.G) * p.Nq + rt * C::BM;
    t0 = blockIdx.x * p.tiles_per_split;
    const int n_tiles = (p.Nk + C::BN - 1) / C::BN;
    n = min(n_tiles, t0 + p.tiles_per_split) - t0;
    kv_base = (b * p.Hkv + hkv) * p.Nk + t0 * C::BN;
    rows_valid = min(C::BM, p.R - rt * C::BM);
    len = p.Nk;
  } else if (VARLEN) {
    const int ne = p.hdr[0];
    const int idx = blockIdx.x;
    if (idx >= ne * p.Hq) return;  // no unit for this CTA (nothing shared has been touched)
    int e;
    if (CAUSAL) {
      e = idx / p.Hq;
      h = idx % p.Hq;
    } else {
      h = idx / ne;
      e = idx % ne;
    }
    const int2 ent = p.table[e];
    qt = ent.y;
    const int start = p.cu[ent.x];
    len = p.cu[ent.x + 1] - start;
    q_base = h * p.T + start;
    kv_base = (h / p.G) * p.T + start;
  } else {
    h = blockIdx.y;
    const int b = blockIdx.z;
    // causal: heaviest query tiles first so the tail of the grid is short
    qt = CAUSAL ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
    len = p.N;
    q_base = (b * p.Hq + h) * p.N;
    kv_base = (b * p.Hkv + h / p.G) * p.N;
  }
  if (!DECODE) n = CAUSAL ? qt + 1 : (len + C::BN - 1) / C::BN;  // K/V tiles this query tile sees
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
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
      mbar_init(BAR(C::B_PFULL + i), 4);
      mbar_init(BAR(C::B_PFULL2 + i), 4);
      mbar_init(BAR(C::B_ODONE + i), 1);
    }
    mbar_init(BAR(C::B_DRAIN), 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      const int q_row_base = q_base;
      const int kv_row_base = kv_base;
      mbar_expect_tx(BAR(C::B_QFULL), C::Q_BYTES);
#pragma unroll
      for (int pn = 0; pn < D / 64; ++pn)
        tma_load_2d_hint(sbase + C::Q_OFF + pn * C::PANEL, &tmQ, BAR(C::B_QFULL), pn * 64, q_row_base + qt * C::BM,
                         pol_q);
      bool ok = true;
      int kv_issued = 0;  // K/V chunk loads issued (sequence numbers 0 .. kv_issued − 1)
      for (int u = 0; u < 2 * n && ok; ++u) {
        bool is_v;
        int j;
        Ord::decode(u, n, is_v, j);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int seq = u * C::NCH + c;
          const int slot = seq % C::NSLOT;
          const int round = seq / C::NSLOT;
          if (!mbar_wait(BAR(C::B_KVEMPTY + slot), (round & 1) ^ 1, wc, 1)) { ok = false; break; }
          mbar_expect_tx(BAR(C::B_KVFULL + slot), C::SLOT_BYTES);
#pragma unroll
          for (int pp = 0; pp < C::CH / 64; ++pp)
            tma_load_2d_hint(sbase + C::KV_OFF + slot * C::SLOT_BYTES + pp * C::PANEL, is_v ? &tmV : &tmK,
                             BAR(C::B_KVFULL + slot), c * C::CH + pp * 64, kv_row_base + j * C::BN, pol_kv);
          kv_issued = seq + 1;
        }
      }
      // every load issued has landed before the CTA may exit (immediate unless
      // the CTA stopped early on a failed wait)
      mbar_wait_inflight(BAR(C::B_QFULL), 0, wc, 12);
      for (int sl = 0; sl < C::NSLOT && sl < kv_issued; ++sl) {
        const int last = kv_issued - 1 - (kv_issued - 1 - sl) % C::NSLOT;  // last chunk loaded into slot sl
        mbar_wait_inflight(BAR(C::B_KVFULL + sl), (last / C::NSLOT) & 1, wc, 13);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // (the whole warp runs this role; one elected lane issues each instruction)
    {
      bool ok = mbar_wait_warp(BAR(C::B_QFULL), 0, wc, 2);
      tc_fence_after();
      int k_ready = -1, v_ready = -1;
      auto wait_unit = [&](int u) -> bool {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int seq = u * C::NCH + c;
          if (!mbar_wait_warp(BAR(C::B_KVFULL + seq % C::NSLOT), (seq / C::NSLOT) & 1, wc, 3)) return false;
        }
        tc_fence_after();
        return true;
      };
      auto release_unit = [&](int u) {
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) tc_commit_w(BAR(C::B_KVEMPTY + (u * C::NCH + c) % C::NSLOT));
      };
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
      // Descriptors are built once; each MMA only adds a compile-time offset.
      const uint64_t dQ_k = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dKV_k = sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::KV_OFF, C::PANEL, 1024);
      // S[scol] = Q · K_jᵀ   (M=128 queries, N=128 keys, K=D)
      auto issue_s = [&](int j, int scol) {
        const int seq0 = Ord::unitK(j, n) * C::NCH;
        const uint64_t da0 = dQ_k;
        uint64_t db0[C::NCH];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) db0[c] = sdesc_add(dKV_k, ((seq0 + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int col = kk * 16;
          mma_ss_w(tbase + scol, sdesc_add(da0, (kk >> 2) * C::PANEL + (kk & 3) * 32),
                 sdesc_add(db0[col / C::CH], ((col % C::CH) / 64) * C::PANEL + (kk & 3) * 32), C::IDESC_S,
                 kk > 0 ? 1u : 0u);
        }
      };
      // O[:, c*CH..] (+)= P(TMEM at scol) · V_j[:, c*CH..]; half 0 covers keys
      // 0..63 of the tile, half 1 keys 64..127
      auto issue_pv = [&](int j, int scol, int ocol, int half) {
        const int seq0 = Ord::unitV(j, n) * C::NCH;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint64_t db0 = sdesc_add(dKV_mn, ((seq0 + c) % C::NSLOT) * C::SLOT_BYTES);
#pragma unroll
          for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
            mma_ts_w(tbase + ocol + c * C::CH, tbase + scol + kk * 8, sdesc_add(db0, kk * 2048), C::IDESC_PV,
                   (j > 0 || kk > 0) ? 1u : 0u);
        }
      };

      if (ok) {
        {
          // two S tiles in flight: S(j+2) is issued as soon as PV(j) has read P(j)
          ok = need_k(0);
          if (ok) {
            issue_s(0, C::S_COL);
            tc_commit_w(BAR(C::B_SFULL + 0));
            release_unit(Ord::unitK(0, n));
          }
          if (ok && n > 1) {
            ok = need_k(1);
            if (ok) {
              issue_s(1, C::S_COL + 128);
              tc_commit_w(BAR(C::B_SFULL + 1));
              release_unit(Ord::unitK(1, n));
            }
          }
          for (int j = 0; j < n && ok; ++j) {
            const int x = j & 1;
            if (!mbar_wait_warp(BAR(C::B_PFULL + x), (j >> 1) & 1, wc, 4)) { ok = false; break; }
            tc_fence_after();
            if (!need_v(j)) { ok = false; break; }
            issue_pv(j, C::S_COL + 128 * x, C::O_COL, 0);
            if (!mbar_wait_warp(BAR(C::B_PFULL2 + x), (j >> 1) & 1, wc, 10)) { ok = false; break; }
            tc_fence_after();
            issue_pv(j, C::S_COL + 128 * x, C::O_COL, 1);
            tc_commit_w(BAR(C::B_ODONE + x));
            release_unit(Ord::unitV(j, n));
            if (j + 2 < n) {
              if (!need_k(j + 2)) { ok = false; break; }
              issue_s(j + 2, C::S_COL + 128 * x);
              tc_commit_w(BAR(C::B_SFULL + x));
              release_unit(Ord::unitK(j + 2, n));
            }
          }
        }
      }
      // no MMA may still be running when TMEM is released
      tc_commit_w(BAR(C::B_DRAIN));
      mbar_wait_inflight(BAR(C::B_DRAIN), 0, wc, 8);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    {
      const int q_row = qt * C::BM + row;
      const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
      const float sl2 = p.scale_log2;
      const int ocol = C::O_COL;
      // DECODE: last key this row may see (absolute key index)
      const int row_last = DECODE ? (CAUSAL ? p.Nk - p.Nq + (rt * C::BM + row) % p.Nq : p.Nk - 1) : 0;
      float m_ref = -INFINITY;
      float l = 0.f;    // Σ P in fp32: the normaliser of the LSE
      float l_o = 0.f;  // Σ of the bf16-rounded P that the PV product used: the normaliser of O
      bool ok = true;
      // Completion of PV(j) is signalled on o_done[j & 1]: S(j+1) is issued
      // before PV(j), so a single barrier could run two phases ahead of a
      // waiter and make its parity test ambiguous.
      auto odone_idx = [&](int jj) { return jj & 1; };
      auto odone_par = [&](int jj) -> uint32_t { return (jj >> 1) & 1; };
      for (int j = 0; j < n; ++j) {
        const int x = j & 1;  // S buffer of K/V tile j
        const uint32_t par = (j >> 1) & 1;
        const int scol = C::S_COL + 128 * x;
        if (!mbar_wait_warp(BAR(C::B_SFULL + x), par, wc, 5)) { ok = false; break; }
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
        if (DECODE) {
          const int key0 = (t0 + j) * C::BN;
          if (key0 + C::BN - 1 > row_last) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (key0 + c > row_last) s[c] = -INFINITY;
          }
        }
        if (!DECODE && CAUSAL && j == qt) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > row) s[c] = -INFINITY;
        }
        // ragged N: keys past the end of the sequence (the causal mask already
        // excludes them for every row < N)
        if (!DECODE && TAIL && !CAUSAL && (j + 1) * C::BN > len) {
          const int lim = len - j * C::BN;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        const float mx = row_max128(s);
        const float m_new = fmaxf(m_ref, mx * sl2);
        // conditional rescale: keep the stale reference max unless the row max
        // grew by more than kRescaleTau; O itself is scaled after P is stored
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
        // P = 2^(s·scale·log2e − m_ref), rounded to bf16 and written over the
        // first 64 columns of S.  Keys 0..63 are handed to the MMA warp before
        // keys 64..127 are exponentiated, so the first half of the PV product
        // overlaps the second half of the exponentials.  Scale/shift and row
        // sums use packed fp32x2 instructions.  O is divided by the sum of the
        // rounded P, so that the weights it applies to V sum to one exactly:
        // with the very peaked rows of large logits the rounding of the
        // dominant P otherwise scales the whole row of O by up to 2^-9.
        // (a decoding row can see no key of this split at all: its reference
        // stays -inf and every P is 0)
        const float neg_m = (DECODE && m_ref == -INFINITY) ? 0.f : -m_ref;
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
            // O must hold the previous block's product before it is scaled,
            // and be scaled before this block's first PV half accumulates
            if (!mbar_wait_warp(BAR(C::B_ODONE + odone_idx(j - 1)), odone_par(j - 1), wc, 6)) { ok = false; break; }
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
          if (lane == 0) mbar_arrive(BAR(C::B_PFULL + x));
        }
        {
          uint32_t pk[32];
          exp_half(64, pk);
          tmem_st32(tl + scol + 32, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_PFULL2 + x));
        }
        float a, b2, c2, d2;
        f2_split(rs2[0], a, b2);
        f2_split(rs2[1], c2, d2);
        l += (a + b2) + (c2 + d2);
        f2_split(ro2[0], a, b2);
        f2_split(ro2[1], c2, d2);
        l_o += (a + b2) + (c2 + d2);
      }
      if (ok) ok = mbar_wait_warp(BAR(C::B_ODONE + odone_idx(n - 1)), odone_par(n - 1), wc, 7);
      if (ok && DECODE) {
        // this split's partial result: O scaled so that O / l is the average
        // under the rounded weights the PV product used, m and l in log2 units
        tc_fence_after();
        const size_t slot = ((size_t)blockIdx.x * gridDim.y + blockIdx.y) * C::BM + row;
        const float f = l_o > 0.f ? l / l_o : 0.f;
        float* po = p.part_o + slot * D;
#pragma unroll
        for (int oc = 0; oc < D / 32; ++oc) {
          uint32_t ov[32];
          tmem_ld32(tl + ocol + oc * 32, ov);
          tmem_ld_wait();
          reg_fence(ov);
          if (row < rows_valid) {
            float4* dst = reinterpret_cast<float4*>(po + oc * 32);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(ov[4 * c]) * f, __uint_as_float(ov[4 * c + 1]) * f,
                                   __uint_as_float(ov[4 * c + 2]) * f, __uint_as_float(ov[4 * c + 3]) * f);
          }
        }
        if (row < rows_valid) *reinterpret_cast<float2*>(p.part_ml + slot * 2) = make_float2(m_ref, l);
      } else if (ok) {
        tc_fence_after();
        const float inv_l = 1.f / l_o;
        __nv_bfloat16* orow = p.o + ((size_t)q_base + q_row) * D;
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
          if (!TAIL || q_row < len) {  // rows past a ragged end are computed, not stored
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          }
        }
        float lg;
        asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
        if (!TAIL || q_row < len) p.lse[(size_t)q_base + q_row] = (m_ref + lg) * kLn2;
      }
      tc_fence_before();
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa
