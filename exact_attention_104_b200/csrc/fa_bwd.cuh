// Exact-attention backward pass for sm_100a.
//
// The pages only state that the backward pass does not keep the probability
// matrix but recomputes it from Q, K, V and a few per-row statistics
// ("Flash-Attention" concept page, "Core idea").  The formulas are the chain
// rule on O = softmax(s·Q Kᵀ) V, with LSE saved by the forward pass:
//   P = exp(s·Q Kᵀ − LSE),  dV = Pᵀ dO,  dP = dO Vᵀ,  D = rowsum(dO ∘ O),
//   dS = P ∘ (dP − D),      dQ = s·dS K, dK = s·dSᵀ Q.
//
// Kernels:
//   fa_bwd_pre_kernel   D = rowsum(dO∘O), LSE·log2e, zero the fp32 dQ accumulator
//   fa_bwd_kernel       one CTA per (128-key tile, batch, kv head[, d-half]);
//                       streams 64-row query tiles of every query head of the
//                       GQA group; dK, dV accumulate in TMEM, dQ partials are
//                       added to the fp32 accumulator in global memory
//   fa_dq_convert_kernel dQ = bf16(s · accumulator)
//
// In fa_bwd_kernel every product runs on tcgen05 with fp32 TMEM accumulators:
//   Sᵀ = K Qᵀ, dPᵀ = V dOᵀ        (A, B from shared memory)
//   dV += Pᵀ dO, dK += dSᵀ Q       (A = bf16 Pᵀ / dSᵀ written back to TMEM; at
//                                  d = 64 dK reads dSᵀ from shared memory)
//   dQᵀ = Kᵀ dSᵀ                   (B = dSᵀ in smem; A = Kᵀ in TMEM at d <= 128,
//                                  the K tile read MN-major at d = 256)
// Roles: warp 0 TMA producer, warp 1 MMA issuer + TMEM owner, warps 4-7 compute
// (thread = key row: Pᵀ, dSᵀ), warps 8-11 drain (thread = d row of dQᵀ; at
// d <= 128 they also write each unit's Kᵀ into TMEM); at d <= 128 warps 12-15
// form a second compute warpgroup, the two groups taking 32 query columns of
// each step each.
// For d = 256, dK/dV/dQ do not fit TMEM for a full row, so two CTAs share a
// key tile, each owning 128 of the 256 output columns and both recomputing Sᵀ
// and dPᵀ over the full head dimension.
#pragma once

#include "fa_varlen.cuh"
#include "sm100.cuh"

namespace fa {

template <int D, int NCG_ = (D == 64 ? 2 : 1)>
struct BwdCfg {
  static constexpr int DH = D < 128 ? D : 128;  // output columns owned by one CTA
  static constexpr int NDH = D / DH;            // CTAs per key tile
  static constexpr int BR = 64;                 // query rows per step
  static constexpr int BC = 128;                // keys per CTA
  // compute warpgroups (BwdCfgOf picks them): two where the compute warps
  // rather than the tensor pipe bound a step, each group taking 32 of a
  // step's 64 query columns
  static constexpr int NCG = NCG_;
  static constexpr int CG_COLS = BR / NCG;
  static constexpr int A_HALF = NCG == 2 ? 32 : 16;  // TMEM columns between the two 16-query halves of Pᵀ / dSᵀ
  static constexpr int THREADS = 256 + 128 * NCG;
  static constexpr int KV_PANEL = BC * 128;     // 64 columns x 128 rows (bytes)
  static constexpr int Q_PANEL = BR * 128;      // 64 columns x 64 rows
  static constexpr int KV_BYTES = BC * D * 2;
  static constexpr int Q_BYTES = BR * D * 2;
  static constexpr int NSTAGE = (D == 64) ? 4 : (D == 128 ? 3 : 1);
  // dQᵀ = Kᵀ dSᵀ reads Kᵀ from TMEM (A operand of a TS product) instead of the
  // K tile in shared memory at every step: the drain warps write it once per
  // unit (32 KB less shared-memory traffic per step at d = 128).  At d = 64
  // TMEM has 64 columns to spare; at d = 128 they are the second Sᵀ buffer,
  // so Sᵀ is single-buffered there and each step's Sᵀ is issued right after
  // the previous step's dV product (the last reader of the buffer).
  static constexpr bool KT_TMEM = (D <= 128);
  static constexpr int ST_NBUF = (D == 128) ? 1 : 2;
  static constexpr int LA = (NSTAGE >= 2 && ST_NBUF == 2) ? 2 : 1;  // Sᵀ lookahead in steps
  // dK += dSᵀ Q with dSᵀ read from the shared-memory tile the dQᵀ product uses
  // (an SS product) instead of a bf16 copy in TMEM: at d = 64 this saved the
  // compute warps' TMEM store and was 2.7 % faster; at d = 128 it was no
  // faster (C3, C4) or slower (C2 +3.5 %), same box, alternated.
  static constexpr bool DK_SS = (D == 64);
  // d = 256 (one stage): a step's Q and dO tiles load in two halves.  Half A
  // is the two 64-column panels outside the CTA's own output columns (read
  // only by Sᵀ and dPᵀ, so it is free once dPᵀ is done); half B is the CTA's
  // own two panels and the row statistics (read until the dK product).  The
  // next step's half A loads while this step's softmax and gradient products
  // run, and Sᵀ / dPᵀ consume half A before half B.
  static constexpr bool HALVES = (NSTAGE == 1 && D == 256);
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = KV_BYTES;
  static constexpr int DS_OFF = 2 * KV_BYTES;   // dSᵀ: 128 key rows x 64 queries (bf16), 16 KB
  static constexpr int Q_OFF = DS_OFF + 16384;
  static constexpr int DO_OFF = Q_OFF + NSTAGE * Q_BYTES;
  static constexpr int LS_OFF = DO_OFF + NSTAGE * Q_BYTES;  // per stage: lse2[64], Dvec[64]
  // dQᵀ staging for the TMA reduce-add: STG_ROWS query rows x DH fp32,
  // row-major; at d = 64, where shared memory has room, two such buffers used
  // alternately, so that the next step's dQᵀ is staged while the previous
  // reduce still reads its buffer
  static constexpr int STG_ROWS = (D == 256) ? 32 : 64;
  static constexpr int STG_NBUF = (D == 64) ? 2 : 1;
  static constexpr int STG_OFF = LS_OFF + NSTAGE * 512 + ((1024 - (NSTAGE * 512) % 1024) % 1024);
  static constexpr int STG_BUF = STG_ROWS * DH * 4;
  static constexpr int STG_BYTES = STG_NBUF * STG_BUF;
  static constexpr int BAR_OFF = STG_OFF + STG_BYTES;
  static constexpr int B_KVFULL = 0;
  static constexpr int B_QFULL = 1;                  // + stage
  static constexpr int B_QEMPTY = 1 + NSTAGE;        // + stage
  static constexpr int B_SFULL = 1 + 2 * NSTAGE;     // + {0,1}
  static constexpr int B_DPFULL = B_SFULL + 2;
  static constexpr int B_PFULL = B_DPFULL + 1;   // + {0,1}: by step parity
  static constexpr int B_DSFULL = B_PFULL + 2;
  static constexpr int B_DQFULL = B_DSFULL + 1;
  static constexpr int B_DQEMPTY = B_DQFULL + 1;
  static constexpr int B_STGFREE = B_DQEMPTY + 1;  // staging may be overwritten
  static constexpr int B_STGFULL = B_STGFREE + 1;  // staging written by all drain threads
  static constexpr int B_ACC = B_STGFULL + 1;     // a unit's dK, dV accumulated
  static constexpr int B_KVEMPTY = B_ACC + 1;     // a unit's last product has read K, V
  static constexpr int B_DKFREE = B_KVEMPTY + 1;  // dK read out of TMEM (next unit may overwrite)
  static constexpr int B_DVFREE = B_DKFREE + 1;   // dV read out of TMEM
  static constexpr int B_UNITFULL = B_DVFREE + 1;   // + {0,1}: next unit index published
  static constexpr int B_UNITEMPTY = B_UNITFULL + 2; // + {0,1}: read by all nine consumer warps
  static constexpr int B_DRAIN = B_UNITEMPTY + 2;
  static constexpr int B_HAFULL = B_DRAIN + 1;    // half A of a step's Q and dO loaded
  static constexpr int B_HAEMPTY = B_HAFULL + 1;  // half A read by Sᵀ and dPᵀ
  static constexpr int B_QBFULL = B_HAEMPTY + 1;  // half B of Q and the row statistics loaded
  static constexpr int B_DOBFULL = B_QBFULL + 1;  // half B of dO loaded
  static constexpr int B_HBEMPTY = B_DOBFULL + 1; // half B read by the dV and dK products
  static constexpr int B_KTFULL = B_HBEMPTY + 1;  // a unit's Kᵀ written into TMEM
  static constexpr int NBAR = B_KTFULL + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int UNIT_OFF = MISC_OFF + 16;   // two unit-index slots
  static constexpr int SMEM_BYTES = UNIT_OFF + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int DK_COL = 0;
  static constexpr int DV_COL = DH;
  static constexpr int ST_COL = 2 * DH;        // ST_NBUF 64-column Sᵀ buffers
  static constexpr int DP_COL = 2 * DH + 128;  // dPᵀ (later dSᵀ bf16)
  static constexpr int DQ_COL = 2 * DH + 192;  // dQᵀ
  // Kᵀ (bf16, two keys per column): the free columns after dQᵀ at d = 64, the
  // unused second Sᵀ buffer at d = 128
  static constexpr int KT_COL = ST_NBUF == 2 ? 2 * DH + 256 : 2 * DH + 64;
  static constexpr uint32_t IDESC_ST = idesc_bf16_f32(128, BR, false, false);
  static constexpr uint32_t IDESC_DKV = idesc_bf16_f32(128, DH, false, true);
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, BR, true, true);
  static constexpr uint32_t IDESC_DQ_TS = idesc_bf16_f32(128, BR, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(DQ_COL + 64 <= TMEM_COLS, "TMEM budget");
  static_assert(!KT_TMEM || (KT_COL + 64 <= TMEM_COLS && (ST_NBUF == 1 || KT_COL >= DQ_COL + 64)), "TMEM budget (Kᵀ)");
  // Register split between the warpgroups (control: setmaxnreg.dec; compute
  // and drain: setmaxnreg.inc).  Valid for a launch allocation R with
  // CTRL_REGS <= R <= min(COMPUTE_REGS, DRAIN_REGS) and
  // 128·(CTRL_REGS + NCG·COMPUTE_REGS + DRAIN_REGS) <= THREADS·R; checked on the host.
  static constexpr int CTRL_REGS = NCG == 2 ? 96 : 104;
  static constexpr int COMPUTE_REGS = NCG == 2 ? 136 : 208;
  static constexpr int DRAIN_REGS = NCG == 2 ? 136 : 168;
  static constexpr bool REG_SPLIT = (D <= 128);  // d = 256 needs more than 104 in the MMA warp
  static constexpr int MIN_LAUNCH_REGS =
      (128 * (CTRL_REGS + NCG * COMPUTE_REGS + DRAIN_REGS) + THREADS - 1) / THREADS;
  static constexpr int MAX_LAUNCH_REGS = COMPUTE_REGS < DRAIN_REGS ? COMPUTE_REGS : DRAIN_REGS;
};

// The configuration a kernel instance uses: two compute warpgroups at d <= 128
// (measured, same box, backward main kernel: C3 −5.5 %, C4 −8.6 %, C2 causal
// −3.3 % time; non-causal C2 +4.3 % with Kᵀ read from shared memory, −1.4 % and
// −2.5 % with Kᵀ in TMEM), one at d = 256.
template <int D, bool CAUSAL>
using BwdCfgOf = BwdCfg<D, (D <= 128) ? 2 : 1>;

// ------------------------------------------------------------ preprocess
// The per-row workspace arrays (D, lse2 and the fp32 dQ accumulator) use a
// per-head row stride Np = N rounded up to 128, so every 64-row step starts on
// a 256-byte boundary and rows N..Np-1 of a head are padding that no other
// head shares.
//
// One group of D/8 threads per padded row: D_i = Σ_c dO_ic·O_ic in fp32 and
// lse2_i = LSE_i·log2e for i < N, zero for the padding rows.  Also zeroes
// the fp32 dQ accumulator and the main kernel's unit counter.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         const float* __restrict__ lse, float* __restrict__ dvec,
                                                         float* __restrict__ lse2, float* __restrict__ dqacc,
                                                         int* __restrict__ unit_counter, int N, int Np,
                                                         long long rows_p, long long dq_vec4) {
  constexpr int TPR = D / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  if (tid == 0) *unit_counter = 0;
  // zero the accumulator
  float4* acc4 = reinterpret_cast<float4*>(dqacc);
  for (long long i = tid; i < dq_vec4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  // row dots: rows are processed in rounds so that every lane of a group stays together
  const long long groups = nthreads / TPR;
  const long long gid = tid / TPR;
  const int sub = (int)(tid % TPR);
  for (long long r0 = 0; r0 < rows_p; r0 += groups) {
    const long long rp = r0 + gid;             // padded row (< 2^31, checked on the host)
    const unsigned head = (unsigned)rp / (unsigned)Np;
    const int i = (int)((unsigned)rp - head * (unsigned)Np);  // row within the head
    const bool real = rp < rows_p && gid < groups && i < N;
    const long long r = (long long)head * N + i;  // row of O, dO, LSE
    float acc = 0.f;
    if (real) {
      const uint4 ov = *reinterpret_cast<const uint4*>(o + r * D + sub * 8);
      const uint4 dv = *reinterpret_cast<const uint4*>(dout + r * D + sub * 8);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = __bfloat1622float2(o2[e]);
        const float2 c = __bfloat1622float2(d2[e]);
        acc = fmaf(a.x, c.x, acc);
        acc = fmaf(a.y, c.y, acc);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (rp < rows_p && gid < groups && sub == 0) {
      dvec[rp] = acc;
      lse2[rp] = real ? lse[r] * kLog2e : 0.f;
    }
  }
}

// dQ = bf16(s · accumulator), from the padded accumulator rows to the dense
// [B, Hq, N, d] output: one warp per row, lane = group of 4 columns.
template <int D>
__global__ void __launch_bounds__(256) fa_dq_convert_kernel(const float* __restrict__ dqacc,
                                                            __nv_bfloat16* __restrict__ dq, float scale,
                                                            long long rows, int N, int Np) {
  constexpr int V4 = D / 4;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = warp0; r < rows; r += nwarps) {
    const unsigned head = (unsigned)r / (unsigned)N;  // r < 2^31 (checked on the host)
    const long long rp = r + (long long)head * (Np - N);
    const float4* src = reinterpret_cast<const float4*>(dqacc) + rp * V4;
    uint2* dst = reinterpret_cast<uint2*>(dq) + r * V4;
#pragma unroll
    for (int c = lane; c < V4; c += 32) {
      const float4 a = src[c];
      uint2 w;
      w.x = pack_bf16(a.x * scale, a.y * scale);
      w.y = pack_bf16(a.z * scale, a.w * scale);
      dst[c] = w;
    }
  }
}

struct BwdParams {
  const float* lse2;
  const float* dvec;
  float* dqacc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N, Np, B, Hq, Hkv, G;  // Np: per-head row stride of lse2, dvec and dqacc
  int jt_band;               // key tiles per scheduling band (see bwd_unit)
  int n_units;               // key-tile units (x output-column halves at d = 256)
  int* unit_counter;         // next unclaimed unit (zeroed by fa_bwd_pre_kernel)
  float scale, scale_log2;
  long long wait_cap;
  int* err;
  // VARLEN only: packed sequences of T tokens per head (Tp padded workspace
  // rows per head), cu_seqlens, and the work table of (sequence, key tile)
  // units with its header (hdr[0] units)
  const int2* table;
  const int* cu;
  const int* hdr;
  int T, Tp;
};

// One unit of backward work: a 128-key tile (and, at d = 256, one half of the
// output columns) of one (batch, kv head), streamed against the 64-row query
// tiles of every query head of its GQA group (causal: only those at or after
// the diagonal).  Units are numbered so that key tiles come in bands of
// p.jt_band, earliest band first, head by head inside a band: CTAs running at
// the same time share Q/dO tiles in L2, and with a causal mask the heavy bands
// (early key tiles, more query steps) run first.
// len: the sequence's length; qrow(head) / qprow(head) / kvrow: rows of its
// first token in the Q/dO (and dQ output), padded workspace and K/V tensors.
struct BwdUnit {
  int jt, dh, hkv, i_start, per_head, n;
  int len, start, pstart, b;
};

// A packed batch's units (VARLEN; ne = hdr[0] table entries): causal units
// heaviest first across kv heads, non-causal ones kv head by kv head, the
// d-halves of a key tile adjacent.
template <int D, bool CAUSAL, bool VARLEN>
__device__ __forceinline__ BwdUnit bwd_unit(int idx, const BwdParams& p, int ne) {
  using C = BwdCfg<D>;
  BwdUnit u;
  if (VARLEN) {
    u.dh = idx % C::NDH;
    const int rest = idx / C::NDH;
    int e;
    if (CAUSAL) {
      e = rest / p.Hkv;
      u.hkv = rest % p.Hkv;
    } else {
      u.hkv = rest / ne;
      e = rest % ne;
    }
    const int2 ent = p.table[e];
    u.b = ent.x;
    u.jt = ent.y;
    u.start = p.cu[ent.x];
    u.len = p.cu[ent.x + 1] - u.start;
    u.pstart = varlen_pstart(ent.x, u.start);
  } else {
    const int n_kt = (p.N + C::BC - 1) / C::BC;
    const int U = C::NDH * p.Hkv * p.B;  // units per key tile
    const int bi = idx / (p.jt_band * U);
    const int wb = min(p.jt_band, n_kt - bi * p.jt_band);  // key tiles in this band
    const int rb = idx - bi * p.jt_band * U;
    const int bh = rb / (wb * C::NDH);
    const int rem = rb - bh * (wb * C::NDH);
    u.jt = bi * p.jt_band + rem / C::NDH;
    u.dh = rem % C::NDH;
    u.hkv = bh % p.Hkv;
    u.b = bh / p.Hkv;
    u.len = p.N;
    u.start = 0;
    u.pstart = 0;
  }
  const int nqt = (u.len + C::BR - 1) / C::BR;
  u.i_start = CAUSAL ? (u.jt * C::BC) / C::BR : 0;
  u.per_head = nqt - u.i_start;
  u.n = p.G * u.per_head;  // query steps
  return u;
}

// Row of query row 0 of query head `head` in Q / dO / dQ, and in the padded
// workspace arrays; row of key 0 of the unit's kv head in K / V / dK / dV.
template <bool VARLEN>
__device__ __forceinline__ int bwd_qrow(const BwdUnit& u, int head, const BwdParams& p) {
  return VARLEN ? head * p.T + u.start : (u.b * p.Hq + head) * p.N;
}
template <bool VARLEN>
__device__ __forceinline__ int bwd_qprow(const BwdUnit& u, int head, const BwdParams& p) {
  return VARLEN ? head * p.Tp + u.pstart : (u.b * p.Hq + head) * p.Np;
}
template <bool VARLEN>
__device__ __forceinline__ int bwd_kvrow(const BwdUnit& u, const BwdParams& p) {
  return VARLEN ? u.hkv * p.T + u.start : (u.b * p.Hkv + u.hkv) * p.N;
}

// TAIL: N is not a multiple of 128 (keys and queries past N get P = 0, rows past
// N are not stored).
//
// A CTA claims units one at a time from a global counter (the producer thread
// takes the next index with an atomic add and hands it to the other roles
// through a two-slot ring in shared memory), so the heaviest units spread over
// the SMs as the hardware block scheduler would spread CTAs; with fewer CTAs
// than units the kernel is persistent.  All step-level barriers
// count steps across units (g = steps of earlier units + s), so consecutive
// units form one pipeline; across a unit boundary K and V are reloaded once
// the unit's last product has read them (b_kvempty), and the next unit's first
// dV / dK products wait until the previous unit's accumulators have been read
// out of TMEM (b_dvfree / b_dkfree), so its epilogue overlaps the next unit's
// first loads and products.
// VARLEN: a packed batch of sequences (always with TAIL); units come from
// the work table, each with its own length and row bases.
template <int D, bool CAUSAL, bool TAIL, bool VARLEN = false>
__global__ void __launch_bounds__(BwdCfgOf<D, CAUSAL>::THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdCfgOf<D, CAUSAL>;
  static_assert(!VARLEN || TAIL, "packed sequences have ragged ends");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const int ne = VARLEN ? p.hdr[0] : 0;
  const int n_units = VARLEN ? ne * p.Hkv * C::NDH : p.n_units;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KVFULL), 1);
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(BAR(C::B_QFULL + i), 1);
      mbar_init(BAR(C::B_QEMPTY + i), 1);
    }
    mbar_init(BAR(C::B_SFULL + 0), 1);
    mbar_init(BAR(C::B_SFULL + 1), 1);
    mbar_init(BAR(C::B_DPFULL), 1);
    mbar_init(BAR(C::B_PFULL + 0), 4 * C::NCG);
    mbar_init(BAR(C::B_PFULL + 1), 4 * C::NCG);
    mbar_init(BAR(C::B_DSFULL), 4 * C::NCG);
    mbar_init(BAR(C::B_DQFULL), 1);
    mbar_init(BAR(C::B_DQEMPTY), 4);
    mbar_init(BAR(C::B_STGFREE), 1);
    mbar_init(BAR(C::B_STGFULL), 128);
    mbar_init(BAR(C::B_ACC), 1);
    mbar_init(BAR(C::B_KVEMPTY), 1);
    mbar_init(BAR(C::B_DKFREE), 4 * C::NCG);
    mbar_init(BAR(C::B_DVFREE), 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::B_UNITFULL + i), 1);
      mbar_init(BAR(C::B_UNITEMPTY + i), 5 + 4 * C::NCG);  // MMA warp, the compute warps, four drain warps
    }
    mbar_init(BAR(C::B_DRAIN), 1);
    for (int i = C::B_HAFULL; i <= C::B_HBEMPTY; ++i) mbar_init(BAR(i), 1);
    mbar_init(BAR(C::B_KTFULL), 4);
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

  auto step_head = [&](const BwdUnit& u, int s) { return u.hkv * p.G + s / u.per_head; };
  auto step_q0 = [&](const BwdUnit& u, int s) { return (u.i_start + s % u.per_head) * C::BR; };
  // unit-index ring: slot uc & 1 holds the index of this CTA's uc-th unit
  volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + C::UNIT_OFF);
  // consumer side (whole warp): the index of unit uc, or -1 on a failed wait
  auto next_unit = [&](int uc) -> int {
    if (!mbar_wait_warp(BAR(C::B_UNITFULL + (uc & 1)), (uc >> 1) & 1, wc, 26)) return -1;
    const int idx = unit_slot[uc & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(C::B_UNITEMPTY + (uc & 1)));
    return idx;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (C::REG_SPLIT) setmaxnreg_dec<C::CTRL_REGS>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      int gs = 0;  // steps loaded before this unit
      // loads issued so far: K/V tiles (one per unit), steps' Q/dO tiles (one
      // count per stage, or per half at d = 256)
      int kv_loads = 0, q_issued = 0, ha_issued = 0, qb_issued = 0, dob_issued = 0;
      bool ok = true;
      for (int uc = 0; ok; ++uc) {
        // claim the next unit and publish its index (an index past the end
        // tells every role to stop)
        const int idx = atomicAdd(p.unit_counter, 1);
        if (uc >= 2 && !mbar_wait(BAR(C::B_UNITEMPTY + (uc & 1)), ((uc >> 1) - 1) & 1, wc, 27)) break;
        unit_slot[uc & 1] = idx;
        mbar_arrive(BAR(C::B_UNITFULL + (uc & 1)));
        if (idx >= n_units) break;
        const BwdUnit u = bwd_unit<D, CAUSAL, VARLEN>(idx, p, ne);
        // Q, dO, lse2, D of step s of this unit into its stage
        auto load_q = [&](int s) -> bool {
          const int g = gs + s;
          if constexpr (C::HALVES) {
            const int q_row = bwd_qrow<VARLEN>(u, step_head(u, s), p) + step_q0(u, s);
            const int q_row_p = bwd_qprow<VARLEN>(u, step_head(u, s), p) + step_q0(u, s);
            const int own = 2 * u.dh, oth = 2 - own;
            if (!mbar_wait(BAR(C::B_HAEMPTY), (g & 1) ^ 1, wc, 40)) return false;
            // a unit's first step: the previous step (another unit, perhaps with
            // the other output half) may still read these panels as its half B
            if (s == 0 && !mbar_wait(BAR(C::B_HBEMPTY), (g & 1) ^ 1, wc, 45)) return false;
            mbar_expect_tx(BAR(C::B_HAFULL), 4 * C::Q_PANEL);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int pn = oth + j;
              tma_load_2d(sbase + C::Q_OFF + pn * C::Q_PANEL, &tmQ, BAR(C::B_HAFULL), pn * 64, q_row);
              tma_load_2d(sbase + C::DO_OFF + pn * C::Q_PANEL, &tmDO, BAR(C::B_HAFULL), pn * 64, q_row);
            }
            ha_issued = g + 1;
            if (!mbar_wait(BAR(C::B_HBEMPTY), (g & 1) ^ 1, wc, 41)) return false;
            mbar_expect_tx(BAR(C::B_QBFULL), 2 * C::Q_PANEL + 512);
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d(sbase + C::Q_OFF + (own + j) * C::Q_PANEL, &tmQ, BAR(C::B_QBFULL), (own + j) * 64, q_row);
            bulk_load(sbase + C::LS_OFF, p.lse2 + q_row_p, 256, BAR(C::B_QBFULL));
            bulk_load(sbase + C::LS_OFF + 256, p.dvec + q_row_p, 256, BAR(C::B_QBFULL));
            qb_issued = g + 1;
            mbar_expect_tx(BAR(C::B_DOBFULL), 2 * C::Q_PANEL);
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d(sbase + C::DO_OFF + (own + j) * C::Q_PANEL, &tmDO, BAR(C::B_DOBFULL), (own + j) * 64,
                          q_row);
            dob_issued = g + 1;
            return true;
          }
          const int st = g % C::NSTAGE;
          if (!mbar_wait(BAR(C::B_QEMPTY + st), ((g / C::NSTAGE) & 1) ^ 1, wc, 11)) return false;
          const int q_row = bwd_qrow<VARLEN>(u, step_head(u, s), p) + step_q0(u, s);
          const int q_row_p = bwd_qprow<VARLEN>(u, step_head(u, s), p) + step_q0(u, s);
          const uint32_t bar = BAR(C::B_QFULL + st);
          mbar_expect_tx(bar, 2 * C::Q_BYTES + 512);
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn) {
            tma_load_2d(sbase + C::Q_OFF + st * C::Q_BYTES + pn * C::Q_PANEL, &tmQ, bar, pn * 64, q_row);
            tma_load_2d(sbase + C::DO_OFF + st * C::Q_BYTES + pn * C::Q_PANEL, &tmDO, bar, pn * 64, q_row);
          }
          bulk_load(sbase + C::LS_OFF + st * 512, p.lse2 + q_row_p, 256, bar);
          bulk_load(sbase + C::LS_OFF + st * 512 + 256, p.dvec + q_row_p, 256, bar);
          q_issued = g + 1;
          return true;
        };
        // the first steps' tiles only need free stages: load them before K, V,
        // which wait for the previous unit's last product
        const int pre = u.n < C::NSTAGE ? u.n : C::NSTAGE;
        for (int s = 0; s < pre && ok; ++s) ok = load_q(s);
        if (!ok) break;
        if (uc > 0 && !mbar_wait(BAR(C::B_KVEMPTY), (uc - 1) & 1, wc, 18)) break;
        const int kv_row = bwd_kvrow<VARLEN>(u, p) + u.jt * C::BC;
        mbar_expect_tx(BAR(C::B_KVFULL), 2 * C::KV_BYTES);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) {
          tma_load_2d(sbase + C::K_OFF + pn * C::KV_PANEL, &tmK, BAR(C::B_KVFULL), pn * 64, kv_row);
          tma_load_2d(sbase + C::V_OFF + pn * C::KV_PANEL, &tmV, BAR(C::B_KVFULL), pn * 64, kv_row);
        }
        ++kv_loads;
        for (int s = pre; s < u.n && ok; ++s) ok = load_q(s);
        gs += u.n;
      }
      // every load issued has landed before the CTA may exit (immediate unless
      // the CTA stopped early on a failed wait)
      if (kv_loads > 0) mbar_wait_inflight(BAR(C::B_KVFULL), (kv_loads - 1) & 1, wc, 36);
      if constexpr (C::HALVES) {
        if (ha_issued > 0) mbar_wait_inflight(BAR(C::B_HAFULL), (ha_issued - 1) & 1, wc, 37);
        if (qb_issued > 0) mbar_wait_inflight(BAR(C::B_QBFULL), (qb_issued - 1) & 1, wc, 38);
        if (dob_issued > 0) mbar_wait_inflight(BAR(C::B_DOBFULL), (dob_issued - 1) & 1, wc, 39);
      } else {
        for (int st = 0; st < C::NSTAGE && st < q_issued; ++st) {
          const int last = q_issued - 1 - (q_issued - 1 - st) % C::NSTAGE;  // last step loaded into stage st
          mbar_wait_inflight(BAR(C::B_QFULL + st), (last / C::NSTAGE) & 1, wc, 10);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // (the whole warp runs this role; one elected lane issues each instruction)
    if (C::REG_SPLIT) setmaxnreg_dec<C::CTRL_REGS>();
    {
      bool ok = true;
      auto wait_q = [&](int g) -> bool {
        const bool r = mbar_wait_warp(BAR(C::B_QFULL + g % C::NSTAGE), (g / C::NSTAGE) & 1, wc, 13);
        tc_fence_after();
        return r;
      };
      // Descriptors are built once per unit; each MMA only adds a compile-time
      // offset (the issuing thread must keep up with 48-cycle MMAs).
      const uint64_t dK_k = sdesc_sw128(sbase + C::K_OFF, 16, 1024);
      const uint64_t dV_k = sdesc_sw128(sbase + C::V_OFF, 16, 1024);
      const uint64_t dQ_k = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dDO_k = sdesc_sw128(sbase + C::DO_OFF, 16, 1024);
      const uint64_t dDS_mn = sdesc_sw128(sbase + C::DS_OFF, 16384, 1024);
      const uint64_t dDS_k = sdesc_sw128(sbase + C::DS_OFF, 16, 1024);
      // Sᵀ / dPᵀ: [128 keys x 64 queries] = (K or V tile) · (Q or dO tile)ᵀ over D
      auto issue_xt = [&](uint64_t da0, uint64_t db0, uint32_t dtm) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(dtm, sdesc_add(da0, (kk >> 2) * C::KV_PANEL + (kk & 3) * 32),
                 sdesc_add(db0, (kk >> 2) * C::Q_PANEL + (kk & 3) * 32), C::IDESC_ST, kk > 0 ? 1u : 0u);
      };
      // dV or dK [128 keys x DH] += (Pᵀ or dSᵀ in TMEM) · (dO or Q tile)[:, dh half]
      auto issue_acc = [&](uint32_t atm, uint64_t db0, uint32_t dtm, bool first) {
#pragma unroll
        for (int kk = 0; kk < C::BR / 16; ++kk)
          mma_ts_w(dtm, atm + (kk >> 1) * C::A_HALF + (kk & 1) * 8, sdesc_add(db0, kk * 2048), C::IDESC_DKV,
                   (!first || kk > 0) ? 1u : 0u);
      };
      // dK += dSᵀ · Q tile[:, dh half], dSᵀ from TMEM or (DK_SS) from shared memory
      auto issue_dk = [&](uint64_t db0, bool first) {
        if constexpr (C::DK_SS) {
#pragma unroll
          for (int kk = 0; kk < C::BR / 16; ++kk)
            mma_ss_w(tbase + C::DK_COL, sdesc_add(dDS_k, kk * 32), sdesc_add(db0, kk * 2048), C::IDESC_DKV,
                     (!first || kk > 0) ? 1u : 0u);
        } else {
          issue_acc(tbase + C::DP_COL, db0, tbase + C::DK_COL, first);
        }
      };
      auto stage_bytes = [&](int g) -> uint32_t { return (uint32_t)(g % C::NSTAGE) * C::Q_BYTES; };
      auto q_off = [&](int g) -> uint64_t { return sdesc_add(dQ_k, stage_bytes(g)); };
      auto do_off = [&](int g) -> uint64_t { return sdesc_add(dDO_k, stage_bytes(g)); };
      int gs = 0;
      for (int uc = 0; ok; ++uc) {
        const int idx = next_unit(uc);
        if (idx < 0) { ok = false; break; }
        if (idx >= n_units) break;
        const BwdUnit u = bwd_unit<D, CAUSAL, VARLEN>(idx, p, ne);
        const int n = u.n;
        const uint64_t dQ_mn = sdesc_sw128(sbase + C::Q_OFF + (u.dh * C::DH / 64) * C::Q_PANEL, C::Q_PANEL, 1024);
        const uint64_t dDO_mn = sdesc_sw128(sbase + C::DO_OFF + (u.dh * C::DH / 64) * C::Q_PANEL, C::Q_PANEL, 1024);
        const uint64_t dKT_mn = sdesc_sw128(sbase + C::K_OFF + (u.dh * C::DH / 64) * C::KV_PANEL, C::KV_PANEL, 1024);
        // dQᵀ [128 d-rows x 64 queries] = K[:, dh half]ᵀ · dSᵀ over the 128 keys
        auto issue_dq = [&]() {
#pragma unroll
          for (int kk = 0; kk < C::BC / 16; ++kk) {
            if constexpr (C::KT_TMEM)
              mma_ts_w(tbase + C::DQ_COL, tbase + C::KT_COL + kk * 8, sdesc_add(dDS_mn, kk * 2048), C::IDESC_DQ_TS,
                       kk > 0 ? 1u : 0u);
            else
              mma_ss_w(tbase + C::DQ_COL, sdesc_add(dKT_mn, kk * 2048), sdesc_add(dDS_mn, kk * 2048), C::IDESC_DQ,
                       kk > 0 ? 1u : 0u);
          }
        };
        // Sᵀ buffer of step g
        auto st_col = [&](int g) -> uint32_t { return tbase + C::ST_COL + (C::ST_NBUF == 2 ? 64 * (g & 1) : 0); };
        if (!mbar_wait_warp(BAR(C::B_KVFULL), uc & 1, wc, 12)) { ok = false; break; }
        tc_fence_after();
        if constexpr (C::HALVES) {
          const int own = 2 * u.dh, oth = 2 - own;
          // Sᵀ or dPᵀ over the two 64-column panels pn0, pn0 + 1 of the head dimension
          auto issue_xt_half = [&](uint64_t da0, uint64_t db0, uint32_t dtm, int pn0, bool first) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss_w(dtm, sdesc_add(da0, (uint32_t)(pn0 + j) * C::KV_PANEL + kk * 32),
                         sdesc_add(db0, (uint32_t)(pn0 + j) * C::Q_PANEL + kk * 32), C::IDESC_ST,
                         (first && j == 0 && kk == 0) ? 0u : 1u);
          };
          for (int s = 0; s < n && ok; ++s) {
            const int g = gs + s;
            const uint32_t st_t = tbase + C::ST_COL + 64 * (g & 1);
            if (s == 0) {
              // a unit's first step; later steps' Sᵀ over half A was issued
              // during the step before, after its dV product
              if (!mbar_wait_warp(BAR(C::B_HAFULL), g & 1, wc, 42)) { ok = false; break; }
              tc_fence_after();
              issue_xt_half(dK_k, dQ_k, st_t, oth, true);
            }
            if (!mbar_wait_warp(BAR(C::B_QBFULL), g & 1, wc, 43)) { ok = false; break; }
            tc_fence_after();
            issue_xt_half(dK_k, dQ_k, st_t, own, false);
            tc_commit_w(BAR(C::B_SFULL + (g & 1)));
            issue_xt_half(dV_k, dDO_k, tbase + C::DP_COL, oth, true);
            if (!mbar_wait_warp(BAR(C::B_DOBFULL), g & 1, wc, 44)) { ok = false; break; }
            tc_fence_after();
            issue_xt_half(dV_k, dDO_k, tbase + C::DP_COL, own, false);
            tc_commit_w(BAR(C::B_DPFULL));
            tc_commit_w(BAR(C::B_HAEMPTY));
            if (!mbar_wait_warp(BAR(C::B_PFULL + (g & 1)), (g >> 1) & 1, wc, 14)) { ok = false; break; }
            if (s == 0 && uc > 0 && !mbar_wait_warp(BAR(C::B_DVFREE), (uc - 1) & 1, wc, 19)) { ok = false; break; }
            tc_fence_after();
            issue_acc(st_t, dDO_mn, tbase + C::DV_COL, s == 0);
            if (s + 1 < n) {
              // the next step's Sᵀ over half A (into the other Sᵀ buffer, whose
              // Pᵀ the dV product two steps back has read) while the compute
              // warps form dSᵀ: the tensor pipe would otherwise wait for them
              if (!mbar_wait_warp(BAR(C::B_HAFULL), (g + 1) & 1, wc, 48)) { ok = false; break; }
              tc_fence_after();
              issue_xt_half(dK_k, dQ_k, tbase + C::ST_COL + 64 * ((g + 1) & 1), oth, true);
            }
            if (!mbar_wait_warp(BAR(C::B_DSFULL), g & 1, wc, 15)) { ok = false; break; }
            if (s == 0 && uc > 0 && !mbar_wait_warp(BAR(C::B_DKFREE), (uc - 1) & 1, wc, 20)) { ok = false; break; }
            tc_fence_after();
            issue_dk(dQ_mn, s == 0);
            tc_commit_w(BAR(C::B_HBEMPTY));
            if (g > 0) {
              if (!mbar_wait_warp(BAR(C::B_DQEMPTY), (g - 1) & 1, wc, 16)) { ok = false; break; }
              tc_fence_after();
            }
            issue_dq();
            tc_commit_w(BAR(C::B_DQFULL));
          }
        } else {
          for (int k = 0; k < C::LA && k < n && ok; ++k) {
            ok = wait_q(gs + k);
            if (!ok) break;
            issue_xt(dK_k, q_off(gs + k), st_col(gs + k));
            tc_commit_w(BAR(C::B_SFULL + ((gs + k) & 1)));
          }
          if (!ok) break;
          issue_xt(dV_k, do_off(gs), tbase + C::DP_COL);
          tc_commit_w(BAR(C::B_DPFULL));
          for (int s = 0; s < n && ok; ++s) {
            const int g = gs + s;
            if (!mbar_wait_warp(BAR(C::B_PFULL + (g & 1)), (g >> 1) & 1, wc, 14)) { ok = false; break; }
            // the previous unit's dV must have been read out before it is overwritten
            if (s == 0 && uc > 0 && !mbar_wait_warp(BAR(C::B_DVFREE), (uc - 1) & 1, wc, 19)) { ok = false; break; }
            tc_fence_after();
            issue_acc(st_col(g), sdesc_add(dDO_mn, stage_bytes(g)), tbase + C::DV_COL, s == 0);
            if (C::ST_NBUF == 1 && s + 1 < n) {
              // one Sᵀ buffer: the next step's Sᵀ right after dV, the last
              // reader of this step's Pᵀ in it
              if (!wait_q(g + 1)) { ok = false; break; }
              issue_xt(dK_k, q_off(g + 1), st_col(g + 1));
              tc_commit_w(BAR(C::B_SFULL + ((g + 1) & 1)));
            }
            if (!mbar_wait_warp(BAR(C::B_DSFULL), g & 1, wc, 15)) { ok = false; break; }
            if (s == 0 && uc > 0 && !mbar_wait_warp(BAR(C::B_DKFREE), (uc - 1) & 1, wc, 20)) { ok = false; break; }
            tc_fence_after();
            issue_dk(sdesc_add(dQ_mn, stage_bytes(g)), s == 0);
            tc_commit_w(BAR(C::B_QEMPTY + g % C::NSTAGE));
            if (g > 0) {
              if (!mbar_wait_warp(BAR(C::B_DQEMPTY), (g - 1) & 1, wc, 16)) { ok = false; break; }
              tc_fence_after();
            }
            if (C::KT_TMEM && s == 0) {
              // this unit's Kᵀ is in TMEM
              if (!mbar_wait_warp(BAR(C::B_KTFULL), uc & 1, wc, 28)) { ok = false; break; }
              tc_fence_after();
            }
            issue_dq();
            tc_commit_w(BAR(C::B_DQFULL));
            // dPᵀ of the next step first: the compute warps are waiting for it
            if (s + 1 < n) {
              if (C::LA == 1 && C::ST_NBUF == 2 && !wait_q(g + 1)) { ok = false; break; }
              issue_xt(dV_k, do_off(g + 1), tbase + C::DP_COL);
              tc_commit_w(BAR(C::B_DPFULL));
            }
            if (C::ST_NBUF == 2 && s + C::LA < n) {
              const int g2 = g + C::LA;
              if (C::LA > 1 && !wait_q(g2)) { ok = false; break; }
              issue_xt(dK_k, q_off(g2), tbase + C::ST_COL + 64 * (g2 & 1));
              tc_commit_w(BAR(C::B_SFULL + (g2 & 1)));
            }
          }
        }
        if (!ok) break;
        tc_commit_w(BAR(C::B_ACC));      // this unit's dK, dV are complete
        tc_commit_w(BAR(C::B_KVEMPTY));  // and nothing reads its K, V any more
        gs += n;
      }
      tc_commit_w(BAR(C::B_DRAIN));
      mbar_wait_inflight(BAR(C::B_DRAIN), 0, wc, 17);
    }
  } else if (warp < 4) {
    // idle warps of the control warpgroup
    if (C::REG_SPLIT) setmaxnreg_dec<C::CTRL_REGS>();
  } else if ((warp >= 4 && warp < 8) || warp >= 12) {
    // ------------------------------------------- compute: Pᵀ and dSᵀ rows
    // With two compute warpgroups (d <= 128), warps 4-7 take query columns 0..31
    // of each step and warps 12-15 columns 32..63; each group writes its bf16
    // Pᵀ and dSᵀ into TMEM columns of its own Sᵀ / dPᵀ range (the products
    // read the two 16-query halves A_HALF columns apart), so neither group
    // overwrites columns the other has not read yet.
    if (C::REG_SPLIT) setmaxnreg_inc<C::COMPUTE_REGS>();
    constexpr int NC = C::CG_COLS;                      // query columns of this group
    const int cg = warp >= 12 ? 1 : 0;
    const int col0 = C::NCG == 2 ? 32 * cg : 0;         // first query column of this group
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within the tile
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int gs = 0;
    for (int uc = 0; ok; ++uc) {
      const int idx = next_unit(uc);
      if (idx < 0) { ok = false; break; }
      if (idx >= n_units) break;
      const BwdUnit u = bwd_unit<D, CAUSAL, VARLEN>(idx, p, ne);
      const int key = u.jt * C::BC + r;
      for (int s = 0; s < u.n; ++s) {
        const int g = gs + s;
        const int st = g % C::NSTAGE;
        const int q0 = step_q0(u, s) + col0;  // first query row of this group's columns
        const uint32_t stats_bar = C::HALVES ? BAR(C::B_QBFULL) : BAR(C::B_QFULL + st);
        if (!mbar_wait_warp(stats_bar, (g / C::NSTAGE) & 1, wc, 21)) { ok = false; break; }
        if (!mbar_wait_warp(BAR(C::B_SFULL + (g & 1)), (g >> 1) & 1, wc, 22)) { ok = false; break; }
        tc_fence_after();
        const float* lse2 = reinterpret_cast<const float*>(smem + C::LS_OFF + st * 512) + col0;
        const float* dv = lse2 + 64;
        uint32_t x0[32], x1[32];
        const int scol = C::ST_COL + (C::ST_NBUF == 2 ? 64 * (g & 1) : 0);
        tmem_ld32(tl + scol + col0, x0);
        if (NC == 64) tmem_ld32(tl + scol + 32, x1);
        tmem_ld_wait();
        reg_fence(x0);
        if (NC == 64) reg_fence(x1);
        float pr[NC];
        const bool diag = CAUSAL && (q0 < u.jt * C::BC + C::BC);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          pr[c] = ex2(fmaf(__uint_as_float(x0[c]), sl2, -lse2[c]));
          if (NC == 64) pr[(32 + c) % NC] = ex2(fmaf(__uint_as_float(x1[c]), sl2, -lse2[32 + c]));
        }
        if (diag) {
#pragma unroll
          for (int c = 0; c < NC; ++c)
            if (key > q0 + c) pr[c] = 0.f;
        }
        // ragged N: keys and queries past the end of the sequence contribute nothing
        if (TAIL && (key >= u.len || q0 + NC > u.len)) {
#pragma unroll
          for (int c = 0; c < NC; ++c)
            if (key >= u.len || q0 + c >= u.len) pr[c] = 0.f;
        }
        uint32_t pk[NC / 2];
#pragma unroll
        for (int c = 0; c < NC / 2; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
        if constexpr (NC == 64) {
          tmem_st32(tl + scol, pk);
        } else {
          tmem_st16(tl + scol + col0, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_PFULL + (g & 1)));

        if (!mbar_wait_warp(BAR(C::B_DPFULL), g & 1, wc, 23)) { ok = false; break; }
        // the previous dQᵀ product must be done reading the dSᵀ tile in smem
        if (g > 0 && !mbar_wait_warp(BAR(C::B_DQFULL), (g - 1) & 1, wc, 24)) { ok = false; break; }
        tc_fence_after();
        uint8_t* rowp = smem + C::DS_OFF + r * 128;
        // dSᵀ = Pᵀ ∘ (dPᵀ − D), 32 query columns at a time: bf16 into the smem
        // tile (B operand of dQᵀ; A operand of dK with DK_SS) and, without
        // DK_SS, over the consumed dPᵀ columns (A operand of dK)
#pragma unroll
        for (int h = 0; h < NC / 32; ++h) {
          const int hf = C::NCG == 2 ? cg : h;  // which 32 of the step's 64 query columns
          tmem_ld32(tl + C::DP_COL + 32 * hf, x0);
          tmem_ld_wait();
          reg_fence(x0);
          uint32_t dk16[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int q = 32 * h + 2 * c;  // this group's column index
            const float d0 = pr[q] * (__uint_as_float(x0[2 * c]) - dv[q]);
            const float d1 = pr[q + 1] * (__uint_as_float(x0[2 * c + 1]) - dv[q + 1]);
            dk16[c] = pack_bf16(d0, d1);
          }
          if (!C::DK_SS) tmem_st16(tl + C::DP_COL + C::A_HALF * hf, dk16);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int lch = 4 * hf + ch;
            const uint4 v = make_uint4(dk16[4 * ch], dk16[4 * ch + 1], dk16[4 * ch + 2], dk16[4 * ch + 3]);
            *reinterpret_cast<uint4*>(rowp + ((lch ^ (r & 7)) * 16)) = v;
          }
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_DSFULL));
      }
      if (!ok) break;
      // dK epilogue (scaled by s), this group's 32-column chunks of the CTA's
      // output columns; tcgen05.ld is warp-collective: every lane loads, only
      // rows < N are stored
      if (!mbar_wait_warp(BAR(C::B_ACC), uc & 1, wc, 25)) { ok = false; break; }
      tc_fence_after();
      __nv_bfloat16* dst = p.dk + ((size_t)bwd_kvrow<VARLEN>(u, p) + key) * D + u.dh * C::DH;
      constexpr int NOC = C::DH / 32 / C::NCG;  // chunks per group
#pragma unroll
      for (int h = 0; h < NOC; ++h) {
        const int oc = cg * NOC + h;
        uint32_t v[32];
        tmem_ld32(tl + C::DK_COL + oc * 32, v);
        tmem_ld_wait();
        reg_fence(v);
        if (h == NOC - 1) {
          // dK has been read out of TMEM: the next unit may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_DKFREE));
        }
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16(__uint_as_float(v[2 * c]) * p.scale, __uint_as_float(v[2 * c + 1]) * p.scale);
        uint4* d4 = reinterpret_cast<uint4*>(dst + oc * 32);
        if (!TAIL || key < u.len) {
#pragma unroll
          for (int c = 0; c < 4; ++c) d4[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      gs += u.n;
    }
    tc_fence_before();
  } else {
    // ------------------------- drain: dQᵀ -> smem staging -> TMA reduce-add
    if (C::REG_SPLIT) setmaxnreg_inc<C::DRAIN_REGS>();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // d row of dQᵀ, key row of dV
    const int dt = threadIdx.x - 256;   // 0..127 within the drain warpgroup
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    float* stg = reinterpret_cast<float*>(smem + C::STG_OFF);
    if (dt == 0) tma_prefetch_desc(&tmDQ);
    bool ok = true;
    int sub_seq = 0;  // staging uses so far
    int gs = 0;
    for (int uc = 0; ok; ++uc) {
      const int idx = next_unit(uc);
      if (idx < 0) { ok = false; break; }
      if (idx >= n_units) break;
      const BwdUnit u = bwd_unit<D, CAUSAL, VARLEN>(idx, p, ne);
      if constexpr (C::KT_TMEM) {
        // Kᵀ into TMEM, the A operand of the unit's dQᵀ products: lane r holds
        // column r of the K tile, keys 2c and 2c + 1 in column c (low half
        // first), gathered from the 128B-swizzled tile.  The previous unit's
        // last dQᵀ is complete: its K tile was replaced only after that.
        if (!mbar_wait_warp(BAR(C::B_KVFULL), uc & 1, wc, 29)) { ok = false; break; }
        if (quarter * 32 < C::DH) {
          const uint8_t* kp = smem + C::K_OFF + (r >> 6) * C::KV_PANEL + (r & 7) * 2;
          const int cb = (r & 63) >> 3;  // 16-byte chunk of column r in a key row
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t w[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int k0 = 64 * h + 2 * c;
              const uint32_t lo = *reinterpret_cast<const uint16_t*>(kp + k0 * 128 + ((cb ^ (k0 & 7)) << 4));
              const uint32_t hi = *reinterpret_cast<const uint16_t*>(kp + (k0 + 1) * 128 + ((cb ^ ((k0 + 1) & 7)) << 4));
              w[c] = lo | (hi << 16);
            }
            tmem_st32(tl + C::KT_COL + 32 * h, w);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_KTFULL));
      }
      for (int s = 0; s < u.n && ok; ++s) {
        const int g = gs + s;
        if (!mbar_wait_warp(BAR(C::B_DQFULL), g & 1, wc, 31)) { ok = false; break; }
        tc_fence_after();
        uint32_t x0[32], x1[32];
        tmem_ld32(tl + C::DQ_COL, x0);
        tmem_ld32(tl + C::DQ_COL + 32, x1);
        tmem_ld_wait();
        reg_fence(x0);
        reg_fence(x1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_DQEMPTY));
        const int q_row = bwd_qprow<VARLEN>(u, step_head(u, s), p) + step_q0(u, s);  // padded accumulator row
#pragma unroll
        for (int sub = 0; sub < 64 / C::STG_ROWS; ++sub) {
          const int buf = C::STG_NBUF == 2 ? (sub_seq & 1) : 0;
          // the reduce that last read this staging buffer must be done reading
          // it (with two buffers the previous reduce may still be in flight)
          if (dt == 0) {
            bulk_wait_read<C::STG_NBUF - 1>();
            mbar_arrive(BAR(C::B_STGFREE));
          }
          if (!mbar_wait_warp(BAR(C::B_STGFREE), sub_seq & 1, wc, 33)) { ok = false; break; }
          float* sb = stg + buf * (C::STG_BUF / 4);
          if (r < C::DH) {
#pragma unroll
            for (int qq = 0; qq < C::STG_ROWS; ++qq) {
              const int c = sub * C::STG_ROWS + qq;
              sb[qq * C::DH + r] = __uint_as_float(c < 32 ? x0[c] : x1[c - 32]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(BAR(C::B_STGFULL));
          if (dt == 0) {
            if (!mbar_wait(BAR(C::B_STGFULL), sub_seq & 1, wc, 34)) { ok = false; break; }
            tma_reduce_add_2d(&tmDQ, sbase + C::STG_OFF + buf * C::STG_BUF, u.dh * C::DH, q_row + sub * C::STG_ROWS);
            bulk_commit_group();
          }
          ++sub_seq;
        }
      }
      if (!ok) break;
      // dV epilogue
      if (!mbar_wait_warp(BAR(C::B_ACC), uc & 1, wc, 32)) { ok = false; break; }
      tc_fence_after();
      __nv_bfloat16* dst = p.dv + ((size_t)bwd_kvrow<VARLEN>(u, p) + u.jt * C::BC + r) * D + u.dh * C::DH;
#pragma unroll
      for (int oc = 0; oc < C::DH / 32; ++oc) {
        uint32_t v[32];
        tmem_ld32(tl + C::DV_COL + oc * 32, v);
        tmem_ld_wait();
        reg_fence(v);
        if (oc == C::DH / 32 - 1) {
          // dV has been read out of TMEM: the next unit may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_DVFREE));
        }
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = pack_bf16(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
        uint4* d4 = reinterpret_cast<uint4*>(dst + oc * 32);
        if (!TAIL || u.jt * C::BC + r < u.len) {
#pragma unroll
          for (int c = 0; c < 4; ++c) d4[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      gs += u.n;
    }
    if (dt == 0) bulk_wait_all();
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa
