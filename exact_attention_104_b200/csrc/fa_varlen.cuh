// Packed batches of sequences with different lengths ("varlen").
//
// nseq sequences lie back to back along the token axis of every head
// (q, o, dout, dq: [Hq, T, d]; k, v, dk, dv: [Hkv, T, d]); sequence b owns
// tokens cu[b] .. cu[b+1]-1 and attends only to itself.  The attention
// kernels are the fixed-length ones with a VARLEN flag: a work unit names a
// (sequence, tile) pair from a table instead of a (batch, tile) pair, and
// every length, row base and mask comes from that sequence.  Ragged batches
// are what the "Flash-Attention" concept page lists under "Design space and
// trade-offs": they change which tiles exist and how work balances.
//
// fa_varlen_plan_kernel (one CTA, first kernel of every varlen call) checks
// cu_seqlens and writes the work table, sorted heaviest first by a counting
// sort on the unit's weight (its number of 128-key tiles, or of 64-row query
// steps in the backward).  With an invalid cu_seqlens it records
// kDevBadSeqlens and publishes zero units, so that no later kernel of the
// call touches memory through it.
#pragma once

#include "sm100.cuh"

namespace fa {

// Workspace header of a varlen call (first 256 bytes): hdr[0] = number of
// table entries, hdr[1] = 1 if cu_seqlens passed the checks.
constexpr int kVarlenHdrBytes = 256;
constexpr int kVarlenMaxSeqlen = 1 << 20;
constexpr int kPlanThreads = 1024;

// First padded workspace row of sequence b in each head of the backward's
// per-row arrays (D, lse2, fp32 dQ accumulator): 256·b + cu[b] rounded up to
// 64.  Every 64-row step then starts 256-byte aligned, and the padded
// regions (128-row multiples) of consecutive sequences never overlap:
// 256·b + ceil64(cu[b]) + pad128(len) <= 256·(b+1) + ceil64(cu[b+1]).
__device__ __host__ __forceinline__ int varlen_pstart(int b, int cu_b) { return 256 * b + ((cu_b + 63) & ~63); }

// Padded rows per head of the backward workspace arrays.
__host__ __forceinline__ long long varlen_tp(int nseq, int T) {
  return ((long long)T + 256LL * nseq + 63) / 64 * 64;
}

// Weight (sort key) of unit u of a sequence with nt 128-row tiles.
//   forward (tpu tiles per unit): causal -> key tiles seen by its last tile,
//                                 else all nt key tiles;
//   backward (unit = one key tile): causal -> query tiles at or after it,
//                                 else all nt.
__device__ __forceinline__ int varlen_key(int u, int nt, int tpu, bool bwd, bool causal) {
  if (!causal) return nt;
  if (bwd) return nt - u;
  const int last = (u + 1) * tpu;
  return last < nt ? last : nt;
}

// Exclusive prefix sum over the block (kPlanThreads threads); returns this
// thread's offset and, through *total, the block sum.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of the warp sums
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  *total = warp_sums[32];
  __syncthreads();
  return r;
}

// One CTA of kPlanThreads threads; dynamic shared memory 2·(max_key+1) ints.
// table receives (sequence, unit) pairs, heaviest first.
__global__ void __launch_bounds__(kPlanThreads) fa_varlen_plan_kernel(const int* __restrict__ cu, int nseq, int T,
                                                                      int max_seqlen, int max_key, int tpu, int bwd,
                                                                      int causal, int2* __restrict__ table,
                                                                      int* __restrict__ hdr, int* __restrict__ err) {
  extern __shared__ int plan_smem[];
  __shared__ int bad;
  __shared__ int warp_sums[33];
  const int nb = max_key + 1;
  int* cnt = plan_smem;        // units per key, later the fill cursor
  int* base = plan_smem + nb;  // first table slot of each key
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = kPlanThreads / 32;
  for (int i = tid; i < nb; i += kPlanThreads) cnt[i] = 0;
  if (tid == 0) bad = (cu[0] != 0 || cu[nseq] != T) ? 1 : 0;
  __syncthreads();
  for (int b = tid; b < nseq; b += kPlanThreads) {
    const int len = cu[b + 1] - cu[b];
    if (len < 0 || len > max_seqlen) atomicOr(&bad, 1);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      hdr[0] = 0;
      hdr[1] = 0;
      atomicCAS(err, 0, kDevBadSeqlens);
    }
    return;
  }
  // histogram of unit weights: one warp per sequence, lanes over its units
  for (int b = warp; b < nseq; b += nwarps) {
    const int len = cu[b + 1] - cu[b];
    const int nt = (len + 127) / 128;
    const int nu = (nt + tpu - 1) / tpu;
    for (int u = lane; u < nu; u += 32) atomicAdd(&cnt[varlen_key(u, nt, tpu, bwd, causal)], 1);
  }
  __syncthreads();
  // exclusive scan in descending key order: base[k] = Σ_{k' > k} cnt[k']
  const int chunk = (nb + kPlanThreads - 1) / kPlanThreads;
  const int i0 = tid * chunk;
  int local = 0;
  for (int i = i0; i < i0 + chunk && i < nb; ++i) local += cnt[max_key - i];
  int total = 0;
  int off = block_exclusive_scan(local, warp_sums, &total);
  for (int i = i0; i < i0 + chunk && i < nb; ++i) {
    base[max_key - i] = off;
    off += cnt[max_key - i];
  }
  __syncthreads();
  for (int i = tid; i < nb; i += kPlanThreads) cnt[i] = 0;
  __syncthreads();
  for (int b = warp; b < nseq; b += nwarps) {
    const int len = cu[b + 1] - cu[b];
    const int nt = (len + 127) / 128;
    const int nu = (nt + tpu - 1) / tpu;
    for (int u = lane; u < nu; u += 32) {
      const int k = varlen_key(u, nt, tpu, bwd, causal);
      table[base[k] + atomicAdd(&cnt[k], 1)] = make_int2(b, u);
    }
  }
  if (tid == 0) {
    hdr[0] = total;
    hdr[1] = 1;
  }
}

// Largest b in [0, nseq) with key(b) <= x, for a non-decreasing key.
template <class Key>
__device__ __forceinline__ int varlen_search(int nseq, int x, Key key) {
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (key(mid) <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Backward preprocess of a varlen call (see fa_bwd_pre_kernel): D and
// LSE·log2e for every real token, zero for the padding rows of each
// sequence's region, the fp32 dQ accumulator zeroed and the unit counter
// reset.  Padded row rp = head·Tp + rr; its sequence is the last one whose
// region starts at or before rr.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_varlen_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
    float* __restrict__ dvec, float* __restrict__ lse2, float* __restrict__ dqacc, int* __restrict__ unit_counter,
    const int* __restrict__ cu, const int* __restrict__ hdr, int nseq, int T, int Tp, long long rows_p,
    long long dq_vec4) {
  constexpr int TPR = D / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  if (tid == 0) *unit_counter = 0;
  if (hdr[1] == 0) return;  // invalid cu_seqlens: the main kernel has no units
  float4* acc4 = reinterpret_cast<float4*>(dqacc);
  for (long long i = tid; i < dq_vec4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long groups = nthreads / TPR;
  const long long gid = tid / TPR;
  const int sub = (int)(tid % TPR);
  for (long long r0 = 0; r0 < rows_p; r0 += groups) {
    const long long rp = r0 + gid;  // < 2^31 (checked on the host)
    const bool in_range = rp < rows_p && gid < groups;
    int head = 0, b = 0, i = 0;
    bool real = false;
    if (in_range) {
      head = (int)(rp / Tp);
      const int rr = (int)(rp - (long long)head * Tp);
      b = varlen_search(nseq, rr, [&](int s) { return varlen_pstart(s, cu[s]); });
      i = rr - varlen_pstart(b, cu[b]);
      real = i >= 0 && i < cu[b + 1] - cu[b];
    }
    const long long r = (long long)head * T + (real ? cu[b] + i : 0);
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
    if (in_range && sub == 0) {
      dvec[rp] = acc;
      lse2[rp] = real ? lse[r] * kLog2e : 0.f;
    }
  }
}

// dQ = bf16(s · accumulator) of a varlen call: token row r = head·T + t of
// the dense [Hq, T, d] output reads padded row head·Tp + pstart(b) + t - cu[b].
template <int D>
__global__ void __launch_bounds__(256) fa_dq_convert_varlen_kernel(const float* __restrict__ dqacc,
                                                                   __nv_bfloat16* __restrict__ dq, float scale,
                                                                   const int* __restrict__ cu,
                                                                   const int* __restrict__ hdr, int nseq, int T,
                                                                   int Tp, long long rows) {
  constexpr int V4 = D / 4;
  if (hdr[1] == 0) return;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = warp0; r < rows; r += nwarps) {
    const int head = (int)(r / T);
    const int t = (int)(r - (long long)head * T);
    const int b = varlen_search(nseq, t, [&](int s) { return cu[s]; });
    const long long rp = (long long)head * Tp + varlen_pstart(b, cu[b]) + (t - cu[b]);
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

}  // namespace fa
