// Decoding: a few queries (the last Nq positions of the sequence) against a
// long cached K/V of Nk keys, split over the key axis.
//
// Same arithmetic as the forward pass (per-row running max, normaliser and
// output updated block by block: "深度学习进阶（三十一）FlashAttention：IO 感知的
// 精确注意力" §2.2), but with Nq ≤ 16 query rows per head there is almost no
// reuse of a K/V tile, so the pass is bound by reading K and V from HBM, not
// by arithmetic: the products run on the CUDA cores and the work is spread
// over the key axis instead ("split-KV").
//
//   fa_decode_split_kernel    one CTA per (key split, batch, kv head, row
//                             group): the R ≤ RMAX query rows of the GQA group
//                             (G heads × Nq queries) against the split's keys,
//                             64-key tiles double-buffered with cp.async;
//                             writes a partial O (fp32, unnormalised) and the
//                             split's running max m and normaliser l (log2 units)
//   fa_decode_combine_kernel  O = Σ_s 2^(m_s − M) O_s / Σ_s 2^(m_s − M) l_s,
//                             LSE = (M + log2 Σ_s 2^(m_s − M) l_s)·ln 2
//
// Query row r of a head is the sequence position Nk − Nq + r; with the causal
// mask it sees keys 0 .. Nk − Nq + r.
#pragma once

#include "sm100.cuh"

namespace fa {

struct DecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, Nq, d]
  const __nv_bfloat16* k;  // [B, Hkv, Nk, d]
  const __nv_bfloat16* v;
  __nv_bfloat16* o;        // [B, Hq, Nq, d]
  float* lse;              // [B, Hq, Nq]
  float* part_o;           // [n_split][units][RMAX][d]
  float* part_ml;          // [n_split][units][RMAX][2]: m, l
  int B, Hq, Hkv, G, Nq, Nk, R;   // R = G·Nq rows per (batch, kv head)
  int n_rg;                // row groups of RMAX rows
  int n_split, tiles_per_split;
  float scale_log2;
};

template <int D, int RMAX>
struct DecCfg {
  static constexpr int THREADS = 256;
  static constexpr int KT = 64;                  // keys per tile
  static constexpr int ROW_BYTES = D * 2 + 16;   // padded K/V row in shared memory
  static constexpr int TILE_BYTES = KT * ROW_BYTES;
  static constexpr int Q_OFF = 0;                                  // fp32 [RMAX][D]
  static constexpr int K_OFF = Q_OFF + RMAX * D * 4;               // 2 stages
  static constexpr int V_OFF = K_OFF + 2 * TILE_BYTES;             // 2 stages
  static constexpr int S_OFF = V_OFF + 2 * TILE_BYTES;             // fp32 [RMAX][KT]: scores, then P
  static constexpr int ST_OFF = S_OFF + RMAX * KT * 4;             // fp32 m, l, alpha [RMAX] each
  static constexpr int SMEM_BYTES = ST_OFF + 3 * RMAX * 4;
  static constexpr int SR = RMAX * KT / THREADS;                   // score rows per thread (≥ 1)
  static constexpr int PV_ITEMS = RMAX * (D / 2);                  // (row, column pair) items
  static constexpr int PR = (PV_ITEMS + THREADS - 1) / THREADS;    // items per thread
  static_assert(RMAX % 4 == 0 && SR >= 1, "four rows per 64-key tile at least");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// two bf16 in one 32-bit word -> two floats (exact)
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Query row r of row group rg -> (head within the group g, query index i).
__device__ __forceinline__ void dec_row(const DecodeParams& p, int rg, int r, int RMAX, int& g, int& i) {
  const int rr = rg * RMAX + r;
  g = rr / p.Nq;
  i = rr - g * p.Nq;
}

template <int D, int RMAX, bool CAUSAL>
__global__ void __launch_bounds__(DecCfg<D, RMAX>::THREADS)
    fa_decode_split_kernel(const DecodeParams p) {
  using C = DecCfg<D, RMAX>;
  extern __shared__ __align__(16) uint8_t smem[];
  float* Qs = reinterpret_cast<float*>(smem + C::Q_OFF);
  float* S = reinterpret_cast<float*>(smem + C::S_OFF);
  float* m_s = reinterpret_cast<float*>(smem + C::ST_OFF);
  float* l_s = m_s + RMAX;
  float* a_s = l_s + RMAX;
  const uint32_t sbase = smem_u32(smem);

  const int tid = threadIdx.x;
  const int split = blockIdx.x;
  const int unit = blockIdx.y;  // (batch, kv head, row group)
  const int rg = unit % p.n_rg;
  const int hkv = (unit / p.n_rg) % p.Hkv;
  const int b = unit / (p.n_rg * p.Hkv);
  const int rows = min(RMAX, p.R - rg * RMAX);  // real rows of this group

  // query rows, pre-scaled to log2 units
  for (int e = tid; e < RMAX * D; e += C::THREADS) {
    const int r = e / D, c = e - r * D;
    float x = 0.f;
    if (r < rows) {
      int g, i;
      dec_row(p, rg, r, RMAX, g, i);
      const int h = hkv * p.G + g;
      x = __bfloat162float(p.q[((size_t)(b * p.Hq + h) * p.Nq + i) * D + c]) * p.scale_log2;
    }
    Qs[e] = x;
  }
  if (tid < RMAX) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }

  const int n_tiles = (p.Nk + C::KT - 1) / C::KT;
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(n_tiles, t0 + p.tiles_per_split);
  const size_t kv_base = (size_t)(b * p.Hkv + hkv) * p.Nk;

  // K and V tile t into stage st: 16-byte chunks, rows past Nk zero-filled
  // (their source address is clamped to a valid row and nothing is read)
  auto load_tile = [&](int t, int st) {
    constexpr int CHUNKS = C::KT * D / 8;
    for (int e = tid; e < CHUNKS; e += C::THREADS) {
      const int row = e / (D / 8), ch = e - row * (D / 8);
      const int key = t * C::KT + row;
      const bool in = key < p.Nk;
      const size_t src = (kv_base + (in ? key : 0)) * D + ch * 8;
      const uint32_t off = (uint32_t)(row * C::ROW_BYTES + ch * 16);
      cp_async16(sbase + C::K_OFF + st * C::TILE_BYTES + off, p.k + src, in ? 16u : 0u);
      cp_async16(sbase + C::V_OFF + st * C::TILE_BYTES + off, p.v + src, in ? 16u : 0u);
    }
    cp_async_commit();
  };

  // output accumulators: item = tid + THREADS·j -> (row, column pair)
  float acc[C::PR][2];
#pragma unroll
  for (int j = 0; j < C::PR; ++j) acc[j][0] = acc[j][1] = 0.f;

  const int warp = tid >> 5, lane = tid & 31;
  const int kk = tid % C::KT;          // key of this thread in the score phase
  const int r0 = tid / C::KT;          // first score row of this thread
  if (t0 < t1) load_tile(t0, 0);
  for (int t = t0; t < t1; ++t) {
    const int st = (t - t0) & 1;
    if (t + 1 < t1) {
      load_tile(t + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    // scores S[r][kk] = Q_r · K_kk (log2 units), masked
    {
      const uint8_t* krow = smem + C::K_OFF + st * C::TILE_BYTES + kk * C::ROW_BYTES;
      float s[C::SR];
#pragma unroll
      for (int j = 0; j < C::SR; ++j) s[j] = 0.f;
#pragma unroll 4
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 kv4 = *reinterpret_cast<const uint4*>(krow + ch * 16);
        const float kf[8] = {bf_lo(kv4.x), bf_hi(kv4.x), bf_lo(kv4.y), bf_hi(kv4.y),
                             bf_lo(kv4.z), bf_hi(kv4.z), bf_lo(kv4.w), bf_hi(kv4.w)};
#pragma unroll
        for (int j = 0; j < C::SR; ++j) {
          const float4* qv = reinterpret_cast<const float4*>(Qs + (r0 + 4 * j) * D + ch * 8);
          const float4 qa = qv[0], qb = qv[1];
          s[j] = fmaf(qa.x, kf[0], s[j]);
          s[j] = fmaf(qa.y, kf[1], s[j]);
          s[j] = fmaf(qa.z, kf[2], s[j]);
          s[j] = fmaf(qa.w, kf[3], s[j]);
          s[j] = fmaf(qb.x, kf[4], s[j]);
          s[j] = fmaf(qb.y, kf[5], s[j]);
          s[j] = fmaf(qb.z, kf[6], s[j]);
          s[j] = fmaf(qb.w, kf[7], s[j]);
        }
      }
      const int key = t * C::KT + kk;
#pragma unroll
      for (int j = 0; j < C::SR; ++j) {
        const int r = r0 + 4 * j;
        bool vis = (r < rows) && (key < p.Nk);
        if (CAUSAL && vis) {
          int g, i;
          dec_row(p, rg, r, RMAX, g, i);
          vis = key <= p.Nk - p.Nq + i;
        }
        S[r * C::KT + kk] = vis ? s[j] : -INFINITY;
      }
    }
    __syncthreads();

    // online softmax, one warp per row: P over S, running m and l, rescale factor
    for (int r = warp; r < rows; r += C::THREADS / 32) {
      float* sr = S + r * C::KT;
      const float x0 = sr[lane], x1 = sr[lane + 32];
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_s[r];
      const float m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {  // a row that has seen no visible key yet keeps m = -inf, l = 0
        p0 = ex2(x0 - m_new);
        p1 = ex2(x1 - m_new);
        alpha = ex2(m_old - m_new);
      }
      float sum = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      sr[lane] = p0;
      sr[lane + 32] = p1;
      if (lane == 0) {
        l_s[r] = l_s[r] * alpha + sum;
        m_s[r] = m_new;
        a_s[r] = alpha;
      }
    }
    __syncthreads();

    // O[r][2cp..2cp+1] = alpha_r·O + Σ_kk P[r][kk]·V[kk][2cp..2cp+1]
    {
      const uint8_t* vt = smem + C::V_OFF + st * C::TILE_BYTES;
#pragma unroll
      for (int j = 0; j < C::PR; ++j) {
        const int item = tid + C::THREADS * j;
        if (item < C::PV_ITEMS) {
          const int r = item / (D / 2), cp = item - r * (D / 2);
          if (r < rows) {
            const float* pr = S + r * C::KT;
            float o0 = acc[j][0] * a_s[r], o1 = acc[j][1] * a_s[r];
#pragma unroll 8
            for (int key = 0; key < C::KT; ++key) {
              const uint32_t w = *reinterpret_cast<const uint32_t*>(vt + key * C::ROW_BYTES + cp * 4);
              const float pk = pr[key];
              o0 = fmaf(pk, bf_lo(w), o0);
              o1 = fmaf(pk, bf_hi(w), o1);
            }
            acc[j][0] = o0;
            acc[j][1] = o1;
          }
        }
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
  }

  // partial results of this split
  const size_t units = (size_t)p.B * p.Hkv * p.n_rg;
  float* po = p.part_o + ((size_t)split * units + unit) * RMAX * D;
#pragma unroll
  for (int j = 0; j < C::PR; ++j) {
    const int item = tid + C::THREADS * j;
    if (item < C::PV_ITEMS) {
      const int r = item / (D / 2), cp = item - r * (D / 2);
      if (r < rows) *reinterpret_cast<float2*>(po + r * D + 2 * cp) = make_float2(acc[j][0], acc[j][1]);
    }
  }
  if (tid < rows) {
    float* pml = p.part_ml + (((size_t)split * units + unit) * RMAX + tid) * 2;
    pml[0] = m_s[tid];
    pml[1] = l_s[tid];
  }
}

// One CTA per (batch, kv head, row group); thread = (row, column pair).
template <int D, int RMAX>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecodeParams p) {
  const int unit = blockIdx.x;
  const int rg = unit % p.n_rg;
  const int hkv = (unit / p.n_rg) % p.Hkv;
  const int b = unit / (p.n_rg * p.Hkv);
  const int rows = min(RMAX, p.R - rg * RMAX);
  const size_t units = (size_t)p.B * p.Hkv * p.n_rg;
  for (int item = threadIdx.x; item < rows * (D / 2); item += blockDim.x) {
    const int r = item / (D / 2), cp = item - r * (D / 2);
    float M = -INFINITY;
    for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, p.part_ml[(((size_t)s * units + unit) * RMAX + r) * 2]);
    float L = 0.f, o0 = 0.f, o1 = 0.f;
    for (int s = 0; s < p.n_split; ++s) {
      const size_t base = ((size_t)s * units + unit) * RMAX + r;
      const float ms = p.part_ml[base * 2];
      if (ms == -INFINITY) continue;  // no visible key in this split
      const float wgt = ex2(ms - M);
      L = fmaf(wgt, p.part_ml[base * 2 + 1], L);
      const float2 po = *reinterpret_cast<const float2*>(p.part_o + base * D + 2 * cp);
      o0 = fmaf(wgt, po.x, o0);
      o1 = fmaf(wgt, po.y, o1);
    }
    int g, i;
    dec_row(p, rg, r, RMAX, g, i);
    const int h = hkv * p.G + g;
    const size_t orow = (size_t)(b * p.Hq + h) * p.Nq + i;
    const float inv = 1.f / L;
    *reinterpret_cast<uint32_t*>(p.o + orow * D + 2 * cp) = pack_bf16(o0 * inv, o1 * inv);
    if (cp == 0) {
      float lg;
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(L));
      p.lse[orow] = (M + lg) * kLn2;
    }
  }
}

}  // namespace fa
