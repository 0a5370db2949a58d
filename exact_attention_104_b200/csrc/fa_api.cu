// Host side of libfa_b200.so: argument checks, TMA descriptor encoding and
// kernel launches behind the C ABI declared in include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_pair.cuh"
#include "fa_fwd_persistent.cuh"
#include "fa_varlen.cuh"

// Scratch of fa_bwd_noalloc: a fixed device array instead of a caller buffer.
// Host code must not pass this symbol to a kernel (on the host it names a
// stand-in, not device memory); noalloc_scratch() resolves its device address.
static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<long long> g_wait_cap{1LL << 31};  // may be set from any host thread

// pending one-shot profiling events of this host thread (fa_profile_next)
thread_local cudaEvent_t t_prof_start = nullptr;
thread_local cudaEvent_t t_prof_stop = nullptr;

struct ProfileScope {
  cudaEvent_t start, stop;
  cudaStream_t stream;
  explicit ProfileScope(cudaStream_t s) : start(t_prof_start), stop(t_prof_stop), stream(s) {
    t_prof_start = t_prof_stop = nullptr;
    if (start) cudaEventRecord(start, stream);
  }
  ~ProfileScope() {
    if (stop) cudaEventRecord(stop, stream);
  }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view [rows, d] of a bf16 tensor; boxes of 64 columns (128 bytes, the
// swizzle span) by `box_rows` rows, 128-byte swizzled in shared memory.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, int d, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view [rows, d] of an fp32 tensor, unswizzled boxes of box_cols x box_rows
// (used as the destination of TMA reduce-adds).
bool make_map_f32(CUtensorMap* m, const void* ptr, uint64_t rows, int d, int box_cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
  bool checked = false;
  bool sm100 = false;
  int sms = 0;
  int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Checks for an sm_100 device and resolves the error word's device address
// (once per device, with that device current).
fa_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.checked) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_err) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    di.sm100 = (major == 10 && minor == 0);
    di.sms = sms;
    di.err = static_cast<int*>(p);
    di.checked = true;
  }
  if (!di.sm100) return FA_ERR_UNSUPPORTED;
  *out = &di;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
Range span(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return Range{a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// N rounded up to a whole number of 128-row tiles.
long long pad128(long long n) { return (n + 127) / 128 * 128; }

// Size checks shared by both passes.  Returns FA_OK, or the status to report;
// sets *empty for a problem with nothing to compute.
fa_status check_sizes(int B, int Hq, int Hkv, int N, int d, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) {
    *empty = true;
    return FA_OK;
  }
  if (B > 65535 || Hq > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  if ((long long)B * Hq * pad128(N) >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// The per-warpgroup register split (setmaxnreg) of a kernel is only valid for
// a launch allocation inside [C::MIN_LAUNCH_REGS, C::MAX_LAUNCH_REGS]: below
// the minimum an increase would wait forever, outside the window an
// increase/decrease would go the wrong way.  Checked before every launch.
template <class C, class Kern>
bool reg_split_fits(Kern kern) {
  cudaFuncAttributes fattr;
  if (cudaFuncGetAttributes(&fattr, kern) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const int r = (fattr.numRegs + 7) & ~7;  // allocation granularity
  return r >= C::MIN_LAUNCH_REGS && r <= C::MAX_LAUNCH_REGS;
}

// grid_units > 0 (VARLEN): a 1-D grid of that many CTAs instead of
// (query tiles, Hq, B).
template <int D, bool CAUSAL, bool TAIL, bool VARLEN = false>
fa_status launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const fa::FwdParams& p,
                     int B, int Hq, cudaStream_t stream, long long grid_units = 0) {
  using C = fa::FwdCfg<D, 1>;
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, TAIL, VARLEN ? fa::kFwdVarlen : fa::kFwdDense>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  const dim3 grid = VARLEN ? dim3((unsigned)grid_units) : dim3((p.n_qtiles + C::NQ - 1) / C::NQ, Hq, B);
  ProfileScope prof(stream);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Two query tiles per item (d = 64, 128): one persistent CTA per SM walks the
// item list.  d = 256: one CTA per 128-row query tile (launch_fwd).
template <int D, bool CAUSAL, bool TAIL, bool VARLEN = false>
fa_status launch_fwd_persistent(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const fa::FwdParams& fp, int B, int Hq, int sms, cudaStream_t stream) {
  using C = fa::FwdPCfg<D>;
  auto kern = fa::fa_fwd_persistent_kernel<D, CAUSAL, TAIL, VARLEN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  if (!reg_split_fits<C>(kern)) return FA_ERR_UNSUPPORTED;
  fa::FwdPParams p{};
  p.o = fp.o;
  p.lse = fp.lse;
  p.N = fp.N;
  p.Hq = fp.Hq;
  p.G = fp.G;
  p.n_qtiles = fp.n_qtiles;
  p.n_units = (fp.n_qtiles + 1) / 2;
  p.BH = B * Hq;
  const long long items = (long long)p.n_units * p.BH;
  if (items >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  p.n_items = (int)items;
  p.scale_log2 = fp.scale_log2;
  p.wait_cap = fp.wait_cap;
  p.err = fp.err;
  p.table = fp.table;
  p.cu = fp.cu;
  p.hdr = fp.hdr;
  p.T = fp.T;
  // VARLEN: the item count is only known on the device; one CTA per SM
  const int grid = (!VARLEN && p.n_items < sms) ? p.n_items : sms;
  ProfileScope prof(stream);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// d = 128 on CTA pairs (cta_group::2): clusters of two CTAs, each CTA two
// 128-row query tiles, each K/V block split between the two (fa_fwd_pair).

template <bool CAUSAL, bool TAIL>
fa_status launch_fwd_pair(const void* k, const CUtensorMap& tq, const CUtensorMap& tv, const fa::FwdParams& p,
                          int B, int Hq, uint64_t kvrows, cudaStream_t stream) {
  using C = fa::FwdPairCfg;
  auto kern = fa::fa_fwd_pair_kernel<CAUSAL, TAIL>;
  if (!reg_split_fits<C>(kern)) return FA_ERR_UNSUPPORTED;
  CUtensorMap tk_half;  // K halves: 64-key boxes
  if (!make_map(&tk_half, k, kvrows, C::D, 64)) return FA_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  const int items = (p.n_qtiles + 3) / 4;  // four query tiles per cluster
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * (unsigned)items, (unsigned)Hq, (unsigned)B);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfileScope prof(stream);
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk_half, tv, p) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// d = 64, 128: one persistent CTA per SM walks the key-tile units; d = 256:
// one CTA per unit (its one query/dO stage leaves nothing to overlap).
#ifndef FA_BWD_PERSISTENT
#define FA_BWD_PERSISTENT 1
#endif

// dq_rows: rows of the fp32 dQ accumulator; units: work units, or (VARLEN)
// an upper bound on them (the kernel reads the true count from the table).
template <int D, bool CAUSAL, bool TAIL, bool VARLEN>
fa_status launch_bwd_kernel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const fa::BwdParams& p, uint64_t dq_rows, long long units,
                            int sms, cudaStream_t stream) {
  using C = fa::BwdCfgOf<D, CAUSAL>;
  auto kern = fa::fa_bwd_kernel<D, CAUSAL, TAIL, VARLEN>;
  if (C::REG_SPLIT && !reg_split_fits<C>(kern)) return FA_ERR_UNSUPPORTED;
  CUtensorMap tdq;
  if (!make_map_f32(&tdq, p.dqacc, dq_rows, D, C::DH, C::STG_ROWS)) return FA_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  const bool persistent = FA_BWD_PERSISTENT && D <= 128;
  const dim3 grid((unsigned)(persistent && units > sms ? sms : units));
  ProfileScope prof(stream);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool CAUSAL, bool TAIL>
fa_status launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, fa::BwdParams p, int B, int Hkv, int sms, cudaStream_t stream) {
  using C = fa::BwdCfg<D>;
  const long long units = (long long)((p.N + C::BC - 1) / C::BC) * C::NDH * Hkv * B;
  if (units >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  p.n_units = (int)units;
  return launch_bwd_kernel<D, CAUSAL, TAIL, false>(tq, tk, tv, tdo, p, (uint64_t)B * p.Hq * p.Np, units, sms,
                                                   stream);
}

template <int D>
fa_status launch_bwd_pre(const void* o, const void* dout, const float* lse, float* dvec, float* lse2, float* dqacc,
                         int* unit_counter, int N, int Np, long long rows_p, int sms, cudaStream_t stream) {
  const long long dq_vec4 = rows_p * D / 4;
  long long want = rows_p * (D / 8);
  if (dq_vec4 > want) want = dq_vec4;
  long long blocks = (want + 255) / 256;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  fa::fa_bwd_pre_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, dvec, lse2, dqacc,
      unit_counter, N, Np, rows_p, dq_vec4);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Device address of g_fa_noalloc_scratch on the current device, looked up
// once per device (with that device current) and cached.
fa_status noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return FA_OK;
}

// ----------------------------------------------------------------- varlen
// Checks shared by the varlen entry points; *empty for nothing to compute.
fa_status varlen_sizes(int nseq, int Hq, int Hkv, int T, int max_seqlen, int d, float scale, bool* empty) {
  *empty = false;
  if (nseq < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (nseq == 0 || T == 0) {
    *empty = true;
    return FA_OK;
  }
  if (max_seqlen < 1) return FA_ERR_INVALID_ARG;
  if (max_seqlen > fa::kVarlenMaxSeqlen) return FA_ERR_UNSUPPORTED;
  if (Hq > 65535) return FA_ERR_UNSUPPORTED;
  if ((long long)Hq * fa::varlen_tp(nseq, T) >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  // work units (one per 128-row tile, at most T/128 + nseq) times heads
  if (((long long)(T + 127) / 128 + nseq) * Hq * 2 >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Upper bound on the work-table entries (one per 128-row tile of a sequence).
long long varlen_max_entries(int nseq, int T) { return (long long)(T + 127) / 128 + nseq; }
size_t varlen_table_bytes(int nseq, int T) { return round256(8 * (size_t)varlen_max_entries(nseq, T)); }

// The first kernel of a varlen call: check cu_seqlens and write the work table
// of (sequence, unit) pairs, heaviest first, behind the header.
fa_status launch_varlen_plan(const int* cu, int nseq, int T, int max_seqlen, int tpu, bool bwd, bool causal,
                             uint8_t* ws, int* err, cudaStream_t s) {
  const int max_key = (max_seqlen + 127) / 128;
  const size_t smem = 2 * (size_t)(max_key + 1) * sizeof(int);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(fa::fa_varlen_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return FA_ERR_CUDA;
  int* hdr = reinterpret_cast<int*>(ws);
  int2* table = reinterpret_cast<int2*>(ws + fa::kVarlenHdrBytes);
  fa::fa_varlen_plan_kernel<<<1, fa::kPlanThreads, smem, s>>>(cu, nseq, T, max_seqlen, max_key, tpu, bwd ? 1 : 0,
                                                              causal ? 1 : 0, table, hdr, err);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

namespace fa {
// One thread waits on a barrier nothing arrives on; the bounded wait gives up.
__global__ void selftest_wait_kernel(long long cap, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
    const WaitCtx wc{&abort_flag, err, cap};
    mbar_wait(smem_u32(&bar), 0, wc, 99);
  }
}
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n, int poly) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = poly ? exp2_poly(x[i]) : ex2(x[i]);
}
}  // namespace fa

// ------------------------------------------------------------------ decode
// Split plan of a decode call (a pure function of the sizes, so that
// fa_decode_workspace_bytes needs no device).
//  * R = G·Nq <= 16 query rows per kv head: the CUDA-core kernel, row groups
//    of RMAX (4, 8 or 16) rows, 64-key tiles, enough key splits for about
//    kDecodeCtas CTAs in all;
//  * R > 16: the tensor-core kernel (fa_fwd_kernel, decode mode), row tiles
//    of 128 rows, 128-key tiles, and about one CTA per SM of a B200
//    (kDecodeTcCtas) in all: every CTA streams its key range once at HBM
//    speed, so one wave with few, long splits keeps the partial results small.
#ifndef FA_DECODE_CTAS
#define FA_DECODE_CTAS 1024
#endif
constexpr int kDecodeCtas = FA_DECODE_CTAS;
constexpr int kDecodeTcCtas = 148;
constexpr int kDecodeMaxSplit = 256;
struct DecodePlan {
  bool tc = false;  // tensor-core kernel
  int rmax = 4, n_rg = 1, n_split = 1, tiles_per_split = 1;
  size_t part_o_bytes = 0, part_ml_bytes = 0;
};

fa_status decode_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, bool* empty) {
  *empty = false;
  if (B < 0 || Nq < 0 || Nk < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Nq == 0) {
    *empty = true;
    return FA_OK;
  }
  if (Nk == 0) return FA_ERR_INVALID_ARG;              // a query with no key at all
  if (causal && Nq > Nk) return FA_ERR_INVALID_ARG;   // queries before the first key
  if (Nq > 256) return FA_ERR_UNSUPPORTED;            // decoding sizes; use fa_fwd for long query blocks
  if (B > 65535 || Hq > 65535) return FA_ERR_UNSUPPORTED;
  if ((long long)B * Hq * Nq >= (1LL << 31) || (long long)B * Hkv * Nk >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

DecodePlan decode_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  DecodePlan pl;
  const long long R = (long long)(Hq / Hkv) * Nq;
  pl.tc = R > 16;
  pl.rmax = pl.tc ? 128 : (R <= 4 ? 4 : (R <= 8 ? 8 : 16));
  pl.n_rg = (int)((R + pl.rmax - 1) / pl.rmax);
  const long long units = (long long)B * Hkv * pl.n_rg;
  const int n_tiles = pl.tc ? (Nk + 127) / 128 : (Nk + 63) / 64;
  long long want = pl.tc ? kDecodeTcCtas / units : (kDecodeCtas + units - 1) / units;
  if (want < 1) want = 1;
  int n_split = (int)std::min<long long>({want, (long long)n_tiles, (long long)kDecodeMaxSplit});
  pl.tiles_per_split = (n_tiles + n_split - 1) / n_split;
  pl.n_split = (n_tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
  const size_t rows = (size_t)pl.n_split * units * pl.rmax;
  pl.part_o_bytes = round256(rows * d * 4);
  pl.part_ml_bytes = round256(rows * 2 * 4);
  return pl;
}

template <int D, int RMAX, bool CAUSAL>
fa_status launch_decode_split(const fa::DecodeParams& p, unsigned units, cudaStream_t s) {
  using C = fa::DecCfg<D, RMAX>;
  auto kern = fa::fa_decode_split_kernel<D, RMAX, CAUSAL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  ProfileScope prof(s);
  kern<<<dim3((unsigned)p.n_split, units), C::THREADS, C::SMEM_BYTES, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The tensor-core split kernel of a decode call with R > 16 rows per kv head.
template <int D, bool CAUSAL>
fa_status launch_decode_tc(const fa::DecodeParams& dp, const void* q, const void* k, const void* v, float scale,
                           const DeviceInfo* di, unsigned units, cudaStream_t s) {
  using C = fa::FwdCfg<D, 1>;
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, true, fa::kFwdDecode>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, (uint64_t)dp.B * dp.Hq * dp.Nq, D, 128) ||
      !make_map(&tk, k, (uint64_t)dp.B * dp.Hkv * dp.Nk, D, 128) ||
      !make_map(&tv, v, (uint64_t)dp.B * dp.Hkv * dp.Nk, D, 128))
    return FA_ERR_CUDA;
  fa::FwdParams p{};
  p.Hq = dp.Hq;
  p.Hkv = dp.Hkv;
  p.G = dp.G;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  p.Nq = dp.Nq;
  p.Nk = dp.Nk;
  p.R = dp.R;
  p.n_rt = dp.n_rg;
  p.n_split = dp.n_split;
  p.tiles_per_split = dp.tiles_per_split;
  p.part_o = dp.part_o;
  p.part_ml = dp.part_ml;
  ProfileScope prof(s);
  kern<<<dim3((unsigned)dp.n_split, units), C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status launch_decode(const fa::DecodeParams& p, int rmax, bool causal, unsigned units, cudaStream_t s) {
  fa_status st;
  switch (rmax) {
    case 128: st = FA_OK; break;  // the tensor-core split kernel was launched by the caller
    case 4: st = causal ? launch_decode_split<D, 4, true>(p, units, s) : launch_decode_split<D, 4, false>(p, units, s); break;
    case 8: st = causal ? launch_decode_split<D, 8, true>(p, units, s) : launch_decode_split<D, 8, false>(p, units, s); break;
    default: st = causal ? launch_decode_split<D, 16, true>(p, units, s) : launch_decode_split<D, 16, false>(p, units, s); break;
  }
  if (st != FA_OK) return st;
  const dim3 cgrid(units, (unsigned)((rmax + fa::kCombineRows - 1) / fa::kCombineRows));
  switch (rmax) {
    case 128: fa::fa_decode_combine_kernel<D, 128><<<cgrid, 256, 0, s>>>(p); break;
    case 4: fa::fa_decode_combine_kernel<D, 4><<<cgrid, 256, 0, s>>>(p); break;
    case 8: fa::fa_decode_combine_kernel<D, 8><<<cgrid, 256, 0, s>>>(p); break;
    default: fa::fa_decode_combine_kernel<D, 16><<<cgrid, 256, 0, s>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device wait timed out";
    case FA_ERR_DEVICE_CHECK: return "device-side check failed (debug build)";
  }
  return "unknown status";
}

fa_status fa_profile_next(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr)) return FA_ERR_INVALID_ARG;
  t_prof_start = static_cast<cudaEvent_t>(start_event);
  t_prof_stop = static_cast<cudaEvent_t>(stop_event);
  return FA_OK;
}

fa_status fa_selftest_wait_timeout(long long cap_cycles, void* stream) {
  if (cap_cycles < 1 || cap_cycles > (1LL << 31)) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  fa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cap_cycles, di->err);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_selftest_exp2(const float* x, float* y, long long n, int use_poly, void* stream) {
  if (n < 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return FA_ERR_INVALID_ARG;
  if (overlap(span(x, (size_t)n * 4), span(y, (size_t)n * 4))) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  long long blocks = (n + 255) / 256;
  if (blocks > (long long)di->sms * 8) blocks = (long long)di->sms * 8;
  fa::selftest_exp2_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, use_poly);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_set_wait_cap(long long cycles) {
  if (cycles < 0) return FA_ERR_INVALID_ARG;
  g_wait_cap.store(cycles == 0 ? (1LL << 31) : cycles, std::memory_order_relaxed);
  return FA_OK;
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  bool empty = false;
  if (check_sizes(B, Hq, Hkv, N, d, 1.f, &empty) != FA_OK) return 0;
  const size_t rows_p = (size_t)B * Hq * pad128(N);  // per-head stride N rounded up to 128
  return 2 * round256(rows_p * 4) + round256(rows_p * (size_t)d * 4) + 256;  // + the unit counter
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int d, int causal, float scale, void* stream) {
  bool empty = false;
  fa_status st = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)B * Hq * N * d * 2, kvbytes = (size_t)B * Hkv * N * d * 2;
  const Range rq = span(q, qbytes), rk = span(k, kvbytes), rv = span(v, kvbytes);
  const Range ro = span(o, qbytes), rl = span(lse, (size_t)B * Hq * N * 4);
  for (Range out : {ro, rl})
    for (Range in : {rq, rk, rv})
      if (overlap(out, in)) return FA_ERR_INVALID_ARG;
  if (overlap(ro, rl)) return FA_ERR_INVALID_ARG;

  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;

  CUtensorMap tq, tk, tv;
  const uint64_t qrows = (uint64_t)B * Hq * N, kvrows = (uint64_t)B * Hkv * N;
  if (!make_map(&tq, q, qrows, d, 128) || !make_map(&tk, k, kvrows, d, 128) || !make_map(&tv, v, kvrows, d, 128))
    return FA_ERR_CUDA;
  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (N + 127) / 128;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tail = (N % 128) != 0;
  // one kernel instance per (d, causal, ragged tail)
  auto dispatch = [&](auto dtag) -> fa_status {
    constexpr int D = decltype(dtag)::value;
    if constexpr (D <= 128) {
      if (causal) return tail ? launch_fwd_persistent<D, true, true>(tq, tk, tv, p, B, Hq, di->sms, s)
                              : launch_fwd_persistent<D, true, false>(tq, tk, tv, p, B, Hq, di->sms, s);
      return tail ? launch_fwd_persistent<D, false, true>(tq, tk, tv, p, B, Hq, di->sms, s)
                  : launch_fwd_persistent<D, false, false>(tq, tk, tv, p, B, Hq, di->sms, s);
    } else {
      if (causal) return tail ? launch_fwd<D, true, true>(tq, tk, tv, p, B, Hq, s)
                              : launch_fwd<D, true, false>(tq, tk, tv, p, B, Hq, s);
      return tail ? launch_fwd<D, false, true>(tq, tk, tv, p, B, Hq, s) : launch_fwd<D, false, false>(tq, tk, tv, p, B, Hq, s);
    }
  };
  switch (d) {
    case 64: return dispatch(std::integral_constant<int, 64>{});
    case 128: return dispatch(std::integral_constant<int, 128>{});
    case 256: return dispatch(std::integral_constant<int, 256>{});
  }
  return FA_ERR_UNSUPPORTED;
}

fa_status fa_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                      int N, int d, int causal, float scale, void* stream) {
  bool empty = false;
  fa_status st = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)B * Hq * N * d * 2, kvbytes = (size_t)B * Hkv * N * d * 2;
  const Range rq = span(q, qbytes), rk = span(k, kvbytes), rv = span(v, kvbytes);
  const Range ro = span(o, qbytes), rl = span(lse, (size_t)B * Hq * N * 4);
  for (Range out : {ro, rl})
    for (Range in : {rq, rk, rv})
      if (overlap(out, in)) return FA_ERR_INVALID_ARG;
  if (overlap(ro, rl)) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;
  const uint64_t qrows = (uint64_t)B * Hq * N, kvrows = (uint64_t)B * Hkv * N;
  // the item of the last query tiles reads up to three tiles past N
  if (qrows + 3 * 128 >= (1ULL << 31)) return FA_ERR_UNSUPPORTED;
  CUtensorMap tq, tv;
  if (!make_map(&tq, q, qrows, d, 128) || !make_map(&tv, v, kvrows, d, 128)) return FA_ERR_CUDA;
  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (N + 127) / 128;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tail = (N % 128) != 0;
  if (causal) return tail ? launch_fwd_pair<true, true>(k, tq, tv, p, B, Hq, kvrows, s)
                          : launch_fwd_pair<true, false>(k, tq, tv, p, B, Hq, kvrows, s);
  return tail ? launch_fwd_pair<false, true>(k, tq, tv, p, B, Hq, kvrows, s)
              : launch_fwd_pair<false, false>(k, tq, tv, p, B, Hq, kvrows, s);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream) {
  bool empty = false;
  fa_status st = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)lse, dout, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_bytes(B, Hq, Hkv, N, d);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  const size_t rows = (size_t)B * Hq * N;
  const size_t qbytes = rows * d * 2, kvbytes = (size_t)B * Hkv * N * d * 2;
  const Range ins[6] = {span(q, qbytes), span(k, kvbytes), span(v, kvbytes),
                        span(o, qbytes), span(lse, rows * 4), span(dout, qbytes)};
  const Range outs[4] = {span(dq, qbytes), span(dk, kvbytes), span(dv, kvbytes), span(workspace, need)};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 6; ++j)
      if (overlap(outs[i], ins[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], outs[j])) return FA_ERR_INVALID_ARG;
  }

  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;

  // workspace: D, lse2 (B·Hq·Np fp32 each), the dQ accumulator (B·Hq·Np·d fp32)
  // and the main kernel's unit counter
  const int Np = (int)pad128(N);
  const size_t rows_p = (size_t)B * Hq * Np;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dvec = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + round256(rows_p * 4));
  float* dqacc = reinterpret_cast<float*>(ws + 2 * round256(rows_p * 4));
  int* unit_counter = reinterpret_cast<int*>(ws + 2 * round256(rows_p * 4) + round256(rows_p * (size_t)d * 4));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  switch (d) {
    case 64: st = launch_bwd_pre<64>(o, dout, lse, dvec, lse2, dqacc, unit_counter, N, Np, (long long)rows_p, di->sms, s); break;
    case 128: st = launch_bwd_pre<128>(o, dout, lse, dvec, lse2, dqacc, unit_counter, N, Np, (long long)rows_p, di->sms, s); break;
    default: st = launch_bwd_pre<256>(o, dout, lse, dvec, lse2, dqacc, unit_counter, N, Np, (long long)rows_p, di->sms, s); break;
  }
  if (st != FA_OK) return st;

  CUtensorMap tq, tk, tv, tdo;
  const uint64_t kvrows = (uint64_t)B * Hkv * N;
  if (!make_map(&tq, q, rows, d, 64) || !make_map(&tdo, dout, rows, d, 64) || !make_map(&tk, k, kvrows, d, 128) ||
      !make_map(&tv, v, kvrows, d, 128))
    return FA_ERR_CUDA;
  fa::BwdParams p{};
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dqacc = dqacc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.N = N;
  p.Np = Np;
  p.B = B;
  p.unit_counter = unit_counter;
  {
    // Causal: key tiles in bands, heaviest band first (see fa_bwd_kernel).  More
    // bands shorten the tail of heavy CTAs dispatched last; fewer keep the
    // concurrently running CTAs on fewer heads (Q/dO reuse in L2).  The band
    // count is a rule fitted to measurements (same box, fa_bwd call time):
    // 128 (b, kv head) units per key tile: 4 bands +3.2 % over head-major;
    // 32 units: 2 bands +4 %; 16 units (N = 16384): head-major best, 4 bands −4 %.
    const int n_kt = (N + 127) / 128;
    const int units = (d == 256 ? 2 : 1) * Hkv * B;
    const int bands = !causal ? 1 : (units >= 64 ? 4 : (units > 16 ? 2 : 1));
    p.jt_band = (n_kt + bands - 1) / bands;
  }
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.scale = scale;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  const bool tail = (N % 128) != 0;
  auto main_kernel = [&](auto dtag) -> fa_status {
    constexpr int D = decltype(dtag)::value;
    if (causal) return tail ? launch_bwd_main<D, true, true>(tq, tk, tv, tdo, p, B, Hkv, di->sms, s)
                            : launch_bwd_main<D, true, false>(tq, tk, tv, tdo, p, B, Hkv, di->sms, s);
    return tail ? launch_bwd_main<D, false, true>(tq, tk, tv, tdo, p, B, Hkv, di->sms, s)
                : launch_bwd_main<D, false, false>(tq, tk, tv, tdo, p, B, Hkv, di->sms, s);
  };
  switch (d) {
    case 64: st = main_kernel(std::integral_constant<int, 64>{}); break;
    case 128: st = main_kernel(std::integral_constant<int, 128>{}); break;
    default: st = main_kernel(std::integral_constant<int, 256>{}); break;
  }
  if (st != FA_OK) return st;

  long long blocks = ((long long)rows + 7) / 8;  // 8 warps (rows) per block
  if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
  __nv_bfloat16* dq16 = static_cast<__nv_bfloat16*>(dq);
  switch (d) {
    case 64: fa::fa_dq_convert_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, rows, N, Np); break;
    case 128: fa::fa_dq_convert_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, rows, N, Np); break;
    default: fa::fa_dq_convert_kernel<256><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, rows, N, Np); break;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  int host = 0;
  const int zero = 0;
  if (cudaMemcpy(&host, di->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (host != 0 && cudaMemcpy(di->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return FA_ERR_CUDA;
  if (host == 0) return FA_OK;
  if ((host & 0xff) == fa::kDevCheck) return FA_ERR_DEVICE_CHECK;
  if ((host & 0xff) == fa::kDevBadSeqlens) return FA_ERR_INVALID_ARG;
  return FA_ERR_TIMEOUT;
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                         int causal, float scale, void* stream) {
  bool empty = false;
  fa_status st = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  const size_t need = fa_bwd_workspace_bytes(B, Hq, Hkv, N, d);
  if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  // argument and device checks first, so that a bad pointer reports
  // FA_ERR_INVALID_ARG and a non-sm_100 device FA_ERR_UNSUPPORTED before the
  // scratch array's address is looked up
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)lse, dout, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, scratch,
                (size_t)FA_NOALLOC_SCRATCH_BYTES, stream);
}

size_t fa_fwd_varlen_workspace_bytes(int nseq, int Hq, int Hkv, int T, int max_seqlen, int d) {
  bool empty = false;
  if (varlen_sizes(nseq, Hq, Hkv, T, max_seqlen, d, 1.f, &empty) != FA_OK) return 0;
  if (empty) return fa::kVarlenHdrBytes;
  return fa::kVarlenHdrBytes + varlen_table_bytes(nseq, T);
}

size_t fa_bwd_varlen_workspace_bytes(int nseq, int Hq, int Hkv, int T, int max_seqlen, int d) {
  bool empty = false;
  if (varlen_sizes(nseq, Hq, Hkv, T, max_seqlen, d, 1.f, &empty) != FA_OK) return 0;
  if (empty) return fa::kVarlenHdrBytes;
  const size_t rows_p = (size_t)Hq * fa::varlen_tp(nseq, T);
  // header, work table, D and lse2 rows, fp32 dQ accumulator, unit counter
  return fa::kVarlenHdrBytes + varlen_table_bytes(nseq, T) + 2 * round256(rows_p * 4) +
         round256(rows_p * (size_t)d * 4) + 256;
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int nseq, int Hq, int Hkv, int T, int max_seqlen, int d, int causal, float scale,
                        void* workspace, size_t workspace_bytes, void* stream) {
  bool empty = false;
  fa_status st = varlen_sizes(nseq, Hq, Hkv, T, max_seqlen, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse || !cu_seqlens || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  const size_t need = fa_fwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)Hq * T * d * 2, kvbytes = (size_t)Hkv * T * d * 2;
  const Range ins[4] = {span(q, qbytes), span(k, kvbytes), span(v, kvbytes), span(cu_seqlens, 4 * (size_t)(nseq + 1))};
  const Range outs[3] = {span(o, qbytes), span(lse, (size_t)Hq * T * 4), span(workspace, need)};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 4; ++j)
      if (overlap(outs[i], ins[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return FA_ERR_INVALID_ARG;
  }
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = launch_varlen_plan(cu_seqlens, nseq, T, max_seqlen, d <= 128 ? 2 : 1, false, causal != 0, ws, di->err, s);
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, (uint64_t)Hq * T, d, 128) || !make_map(&tk, k, (uint64_t)Hkv * T, d, 128) ||
      !make_map(&tv, v, (uint64_t)Hkv * T, d, 128))
    return FA_ERR_CUDA;
  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = 0;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  p.table = reinterpret_cast<const int2*>(ws + fa::kVarlenHdrBytes);
  p.cu = cu_seqlens;
  p.hdr = reinterpret_cast<const int*>(ws);
  p.T = T;
  const long long grid_units = varlen_max_entries(nseq, T) * Hq;  // d = 256: one CTA per (tile, head)
  auto dispatch = [&](auto dtag) -> fa_status {
    constexpr int D = decltype(dtag)::value;
    if constexpr (D <= 128) {
      return causal ? launch_fwd_persistent<D, true, true, true>(tq, tk, tv, p, 1, Hq, di->sms, s)
                    : launch_fwd_persistent<D, false, true, true>(tq, tk, tv, p, 1, Hq, di->sms, s);
    } else {
      return causal ? launch_fwd<D, true, true, true>(tq, tk, tv, p, 1, Hq, s, grid_units)
                    : launch_fwd<D, false, true, true>(tq, tk, tv, p, 1, Hq, s, grid_units);
    }
  };
  switch (d) {
    case 64: return dispatch(std::integral_constant<int, 64>{});
    case 128: return dispatch(std::integral_constant<int, 128>{});
    default: return dispatch(std::integral_constant<int, 256>{});
  }
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens, int nseq, int Hq,
                        int Hkv, int T, int max_seqlen, int d, int causal, float scale, void* workspace,
                        size_t workspace_bytes, void* stream) {
  bool empty = false;
  fa_status st = varlen_sizes(nseq, Hq, Hkv, T, max_seqlen, d, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !cu_seqlens || !workspace)
    return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)lse, dout, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  const size_t rows = (size_t)Hq * T;
  const size_t qbytes = rows * d * 2, kvbytes = (size_t)Hkv * T * d * 2;
  const Range ins[7] = {span(q, qbytes),  span(k, kvbytes),    span(v, kvbytes),
                        span(o, qbytes),  span(lse, rows * 4), span(dout, qbytes),
                        span(cu_seqlens, 4 * (size_t)(nseq + 1))};
  const Range outs[4] = {span(dq, qbytes), span(dk, kvbytes), span(dv, kvbytes), span(workspace, need)};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 7; ++j)
      if (overlap(outs[i], ins[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], outs[j])) return FA_ERR_INVALID_ARG;
  }
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;

  // workspace: header | work table | D | lse2 | fp32 dQ accumulator | unit counter
  const int Tp = (int)fa::varlen_tp(nseq, T);
  const size_t rows_p = (size_t)Hq * Tp;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t tb = varlen_table_bytes(nseq, T);
  float* dvec = reinterpret_cast<float*>(ws + fa::kVarlenHdrBytes + tb);
  float* lse2 = reinterpret_cast<float*>(ws + fa::kVarlenHdrBytes + tb + round256(rows_p * 4));
  float* dqacc = reinterpret_cast<float*>(ws + fa::kVarlenHdrBytes + tb + 2 * round256(rows_p * 4));
  int* unit_counter = reinterpret_cast<int*>(ws + fa::kVarlenHdrBytes + tb + 2 * round256(rows_p * 4) +
                                             round256(rows_p * (size_t)d * 4));
  const int* hdr = reinterpret_cast<const int*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  st = launch_varlen_plan(cu_seqlens, nseq, T, max_seqlen, 1, true, causal != 0, ws, di->err, s);
  if (st != FA_OK) return st;
  {
    const long long dq_vec4 = (long long)rows_p * d / 4;
    long long want = (long long)rows_p * (d / 8);
    if (dq_vec4 > want) want = dq_vec4;
    long long blocks = (want + 255) / 256;
    if (blocks > (long long)di->sms * 8) blocks = (long long)di->sms * 8;
    if (blocks < 1) blocks = 1;
    auto pre = [&](auto kern) {
      kern<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(o),
                                            static_cast<const __nv_bfloat16*>(dout), lse, dvec, lse2, dqacc,
                                            unit_counter, cu_seqlens, hdr, nseq, T, Tp, (long long)rows_p, dq_vec4);
    };
    switch (d) {
      case 64: pre(fa::fa_bwd_pre_varlen_kernel<64>); break;
      case 128: pre(fa::fa_bwd_pre_varlen_kernel<128>); break;
      default: pre(fa::fa_bwd_pre_varlen_kernel<256>); break;
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }

  CUtensorMap tq, tk, tv, tdo;
  const uint64_t kvrows = (uint64_t)Hkv * T;
  if (!make_map(&tq, q, rows, d, 64) || !make_map(&tdo, dout, rows, d, 64) || !make_map(&tk, k, kvrows, d, 128) ||
      !make_map(&tv, v, kvrows, d, 128))
    return FA_ERR_CUDA;
  fa::BwdParams p{};
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dqacc = dqacc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.N = T;
  p.Np = Tp;
  p.B = 1;
  p.jt_band = 1;
  p.n_units = 0;
  p.unit_counter = unit_counter;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.scale = scale;
  p.scale_log2 = scale * fa::kLog2e;
  p.wait_cap = g_wait_cap.load(std::memory_order_relaxed);
  p.err = di->err;
  p.table = reinterpret_cast<const int2*>(ws + fa::kVarlenHdrBytes);
  p.cu = cu_seqlens;
  p.hdr = hdr;
  p.T = T;
  p.Tp = Tp;
  auto main_kernel = [&](auto dtag) -> fa_status {
    constexpr int D = decltype(dtag)::value;
    const long long units = varlen_max_entries(nseq, T) * Hkv * fa::BwdCfg<D>::NDH;  // upper bound
    return causal ? launch_bwd_kernel<D, true, true, true>(tq, tk, tv, tdo, p, rows_p, units, di->sms, s)
                  : launch_bwd_kernel<D, false, true, true>(tq, tk, tv, tdo, p, rows_p, units, di->sms, s);
  };
  switch (d) {
    case 64: st = main_kernel(std::integral_constant<int, 64>{}); break;
    case 128: st = main_kernel(std::integral_constant<int, 128>{}); break;
    default: st = main_kernel(std::integral_constant<int, 256>{}); break;
  }
  if (st != FA_OK) return st;

  long long blocks = ((long long)rows + 7) / 8;  // 8 warps (rows) per block
  if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
  __nv_bfloat16* dq16 = static_cast<__nv_bfloat16*>(dq);
  switch (d) {
    case 64: fa::fa_dq_convert_varlen_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, cu_seqlens, hdr, nseq, T, Tp, (long long)rows); break;
    case 128: fa::fa_dq_convert_varlen_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, cu_seqlens, hdr, nseq, T, Tp, (long long)rows); break;
    default: fa::fa_dq_convert_varlen_kernel<256><<<(unsigned)blocks, 256, 0, s>>>(dqacc, dq16, scale, cu_seqlens, hdr, nseq, T, Tp, (long long)rows); break;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  bool empty = false;
  if (decode_sizes(B, Hq, Hkv, Nq, Nk, d, 1.f, 0, &empty) != FA_OK || empty) return 0;
  const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, d);
  return pl.part_o_bytes + pl.part_ml_bytes;
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Nq, int Nk, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  bool empty = false;
  fa_status st = decode_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)o, (const void*)lse})
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  const size_t need = fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)B * Hq * Nq * d * 2, kvbytes = (size_t)B * Hkv * Nk * d * 2;
  const Range ins[3] = {span(q, qbytes), span(k, kvbytes), span(v, kvbytes)};
  const Range outs[3] = {span(o, qbytes), span(lse, (size_t)B * Hq * Nq * 4), span(workspace, need)};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 3; ++j)
      if (overlap(outs[i], ins[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return FA_ERR_INVALID_ARG;
  }
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;

  const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, d);
  fa::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.part_o_bytes);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.R = p.G * Nq;
  p.n_rg = pl.n_rg;
  p.n_split = pl.n_split;
  p.tiles_per_split = pl.tiles_per_split;
  p.scale_log2 = scale * fa::kLog2e;
  const long long n_units = (long long)B * Hkv * pl.n_rg;
  if (n_units > 65535) return FA_ERR_UNSUPPORTED;  // grid.y of the split kernel
  const unsigned units = (unsigned)n_units;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.tc) {
    if ((long long)B * Hq * Nq >= (1LL << 31) - 128) return FA_ERR_UNSUPPORTED;  // row index of the last Q box
    auto tc = [&](auto dtag) -> fa_status {
      constexpr int D = decltype(dtag)::value;
      return causal ? launch_decode_tc<D, true>(p, q, k, v, scale, di, units, s)
                    : launch_decode_tc<D, false>(p, q, k, v, scale, di, units, s);
    };
    switch (d) {
      case 64: st = tc(std::integral_constant<int, 64>{}); break;
      case 128: st = tc(std::integral_constant<int, 128>{}); break;
      default: st = tc(std::integral_constant<int, 256>{}); break;
    }
    if (st != FA_OK) return st;
  }
  switch (d) {
    case 64: return launch_decode<64>(p, pl.rmax, causal != 0, units, s);
    case 128: return launch_decode<128>(p, pl.rmax, causal != 0, units, s);
    default: return launch_decode<256>(p, pl.rmax, causal != 0, units, s);
  }
}

}  // extern "C"
