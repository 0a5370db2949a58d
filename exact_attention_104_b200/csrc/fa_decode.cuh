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
  // K/V rows are stored unpadded; the 16-byte chunk c of tile row k sits at
  // chunk position c ^ (k & 7), so that eight consecutive rows reading one
  // chunk, and one row's eight consecutive chunks, hit distinct banks
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int TILE_BYTES = KT * ROW_BYTES;
  // score phase: thread = (key, part); part p sums the chunks p, p + PARTS, ...
  static constexpr int PARTS = THREADS / KT;
  static constexpr int CH_PER_PART = D / 8 / PARTS;
  // PV phase: thread = (8-column chunk, group of 4 rows, key group)
  static constexpr int NCH = D / 8;
  static constexpr int NRG4 = RMAX / 4;
  static constexpr int KG = THREADS / (NCH * NRG4);   // key groups
  static constexpr int KPG = KT / KG;                  // keys per group (key = group + KG·j)
  static constexpr int Q_OFF = 0;                                  // fp32 [RMAX][D], log2 units
  static constexpr int K_OFF = Q_OFF + RMAX * D * 4;               // 2 stages
  static constexpr int V_OFF = K_OFF + 2 * TILE_BYTES;             // 2 stages
  static constexpr int SP_OFF = V_OFF + 2 * TILE_BYTES;            // fp32 [PARTS][RMAX][KT]: partial scores
  static constexpr int PT_OFF = SP_OFF + PARTS * RMAX * KT * 4;    // fp32 [KT][RMAX]: P, key-major
  static constexpr int ST_OFF = PT_OFF + KT * RMAX * 4;            // fp32 m, l, alpha [RMAX] each
  static constexpr int SMEM_BYTES = ST_OFF + 3 * RMAX * 4;
  static constexpr int RED_BYTES = KG * RMAX * D * 4;              // final sum over key groups (over K/V)
  static_assert(RMAX % 4 == 0 && CH_PER_PART >= 1 && NCH % 8 == 0, "tile shape");
  static_assert(KG >= 1 && KT % KG == 0 && THREADS % (NCH * NRG4) == 0, "PV thread map");
  static_assert(RED_BYTES <= 4 * TILE_BYTES, "key-group sums fit over the K/V stages");
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
  float* SP = reinterpret_cast<float*>(smem + C::SP_OFF);
  float* PT = reinterpret_cast<float*>(smem + C::PT_OFF);
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

  // query rows, pre-scaled to log2 units (rows past `rows` are zero)
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
    constexpr int CHUNKS = C::KT * C::NCH;
    for (int e = tid; e < CHUNKS; e += C::THREADS) {
      const int row = e / C::NCH, ch = e - row * C::NCH;
      const int key = t * C::KT + row;
      const bool in = key < p.Nk;
      const size_t src = (kv_base + (in ? key : 0)) * D + ch * 8;
      const uint32_t off = (uint32_t)(row * C::ROW_BYTES + ((ch ^ (row & 7)) << 4));
      cp_async16(sbase + C::K_OFF + st * C::TILE_BYTES + off, p.k + src, in ? 16u : 0u);
      cp_async16(sbase + C::V_OFF + st * C::TILE_BYTES + off, p.v + src, in ? 16u : 0u);
    }
    cp_async_commit();
  };

  const int warp = tid >> 5, lane = tid & 31;
  // score phase map
  const int ks = tid % C::KT;     // tile row (key) of this thread
  const int part = tid / C::KT;   // warp-uniform
  // PV phase map
  const int c8 = tid % C::NCH;
  const int g4 = (tid / C::NCH) % C::NRG4;
  const int kg = tid / (C::NCH * C::NRG4);
  // O accumulators of rows 4·g4 .. 4·g4+3, columns 8·c8 .. 8·c8+7, as fp32 pairs
  uint64_t acc[4][4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[rr][i] = 0;
  const uint64_t zero2 = 0;

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

    // partial scores of this thread's part of the head dimension, all rows
    {
      const uint8_t* krow = smem + C::K_OFF + st * C::TILE_BYTES + ks * C::ROW_BYTES;
      uint64_t s2[RMAX];
#pragma unroll
      for (int r = 0; r < RMAX; ++r) s2[r] = 0;
#pragma unroll
      for (int i = 0; i < C::CH_PER_PART; ++i) {
        const int ch = part + C::PARTS * i;
        const uint4 w = *reinterpret_cast<const uint4*>(krow + ((ch ^ (ks & 7)) << 4));
        const uint64_t k01 = bf2_to_f2(w.x), k23 = bf2_to_f2(w.y), k45 = bf2_to_f2(w.z), k67 = bf2_to_f2(w.w);
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
          const ulonglong2* qv = reinterpret_cast<const ulonglong2*>(Qs + r * D + ch * 8);
          const ulonglong2 qa = qv[0], qb = qv[1];
          s2[r] = f2_fma(qa.x, k01, s2[r]);
          s2[r] = f2_fma(qa.y, k23, s2[r]);
          s2[r] = f2_fma(qb.x, k45, s2[r]);
          s2[r] = f2_fma(qb.y, k67, s2[r]);
        }
      }
      float* sp = SP + part * RMAX * C::KT + ks;
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        float lo, hi;
        f2_split(s2[r], lo, hi);
        sp[r * C::KT] = lo + hi;
      }
    }
    __syncthreads();

    // one warp per row: sum the parts, mask, online softmax; P stored key-major
    for (int r = warp; r < RMAX; r += C::THREADS / 32) {
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int pp = 0; pp < C::PARTS; ++pp) {
        x0 += SP[(pp * RMAX + r) * C::KT + lane];
        x1 += SP[(pp * RMAX + r) * C::KT + lane + 32];
      }
      int last = -1;  // last visible key of this row (-1: a padding row sees none)
      if (r < rows) {
        last = p.Nk - 1;
        if (CAUSAL) {
          int g, i;
          dec_row(p, rg, r, RMAX, g, i);
          last = p.Nk - p.Nq + i;
        }
      }
      const int key0 = t * C::KT + lane;
      if (key0 > last) x0 = -INFINITY;
      if (key0 + 32 > last) x1 = -INFINITY;
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
      PT[lane * RMAX + r] = p0;
      PT[(lane + 32) * RMAX + r] = p1;
      if (lane == 0) {
        l_s[r] = l_s[r] * alpha + sum;
        m_s[r] = m_new;
        a_s[r] = alpha;
      }
    }
    __syncthreads();

    // O[r][cols] = alpha_r·O + Σ_key P[r][key]·V[key][cols] over this thread's keys
    {
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const float a = a_s[4 * g4 + rr];
        const uint64_t a2 = f2_make(a, a);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rr][i] = f2_fma(acc[rr][i], a2, zero2);
      }
      const uint8_t* vt = smem + C::V_OFF + st * C::TILE_BYTES;
#pragma unroll 4
      for (int j = 0; j < C::KPG; ++j) {
        const int key = kg + C::KG * j;
        const uint4 w = *reinterpret_cast<const uint4*>(vt + key * C::ROW_BYTES + ((c8 ^ (key & 7)) << 4));
        const uint64_t v01 = bf2_to_f2(w.x), v23 = bf2_to_f2(w.y), v45 = bf2_to_f2(w.z), v67 = bf2_to_f2(w.w);
        const float4 p4 = *reinterpret_cast<const float4*>(PT + key * RMAX + 4 * g4);
        const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const uint64_t p2 = f2_make(pr[rr], pr[rr]);
          acc[rr][0] = f2_fma(p2, v01, acc[rr][0]);
          acc[rr][1] = f2_fma(p2, v23, acc[rr][1]);
          acc[rr][2] = f2_fma(p2, v45, acc[rr][2]);
          acc[rr][3] = f2_fma(p2, v67, acc[rr][3]);
        }
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
  }

  // sum the key groups' partial outputs (over the K/V stages, all reads done),
  // then write this split's unnormalised O, m and l
  float* red = reinterpret_cast<float*>(smem + C::K_OFF);  // [KG][RMAX][D]
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    float o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) f2_split(acc[rr][i], o[2 * i], o[2 * i + 1]);
    float4* dst = reinterpret_cast<float4*>(red + ((size_t)kg * RMAX + 4 * g4 + rr) * D + 8 * c8);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
  __syncthreads();
  const size_t units = (size_t)p.B * p.Hkv * p.n_rg;
  float* po = p.part_o + ((size_t)split * units + unit) * RMAX * D;
  for (int item = tid; item < rows * (D / 4); item += C::THREADS) {
    const int r = item / (D / 4), c4 = item - r * (D / 4);
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < C::KG; ++g) {
      const float4 x = reinterpret_cast<const float4*>(red + ((size_t)g * RMAX + r) * D)[c4];
      sum.x += x.x;
      sum.y += x.y;
      sum.z += x.z;
      sum.w += x.w;
    }
    reinterpret_cast<float4*>(po + r * D)[c4] = sum;
  }
  if (tid < rows) {
    float* pml = p.part_ml + (((size_t)split * units + unit) * RMAX + tid) * 2;
    pml[0] = m_s[tid];
    pml[1] = l_s[tid];
  }
}

// Rows of a combine CTA: a row group of up to 16 rows is one CTA, the
// 128-row groups of the tensor-core path are spread over 8 CTAs.
constexpr int kCombineRows = 16;

// One CTA per (batch, kv head, row group, chunk of kCombineRows rows);
// thread = (row, column pair).
template <int D, int RMAX>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecodeParams p) {
  const int unit = blockIdx.x;
  const int rg = unit % p.n_rg;
  const int hkv = (unit / p.n_rg) % p.Hkv;
  const int b = unit / (p.n_rg * p.Hkv);
  const int r0 = blockIdx.y * kCombineRows;
  const int rows = min(RMAX, p.R - rg * RMAX) - r0;  // rows of this chunk (may be <= 0)
  const size_t units = (size_t)p.B * p.Hkv * p.n_rg;
  for (int item = threadIdx.x; item < min(rows, kCombineRows) * (D / 2); item += blockDim.x) {
    const int r = r0 + item / (D / 2), cp = item % (D / 2);
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
