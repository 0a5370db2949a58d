/*
 * fa.h — C ABI of libfa_b200.so: exact scaled-dot-product attention
 * (forward and backward) for NVIDIA B200 (sm_100a).
 *
 * What it computes.  For every batch b and query head h, with key/value head
 * g = h / (Hq / Hkv) (grouped-query attention; contiguous groups):
 *
 *     S   = scale · Q[b,h] · K[b,g]ᵀ            (N × N, never stored)
 *     S_ij = -inf  where causal and j > i
 *     P   = softmax(S) row-wise                  (never stored)
 *     O[b,h]   = P · V[b,g]
 *     LSE[b,h,i] = log Σ_j exp(S_ij)             (natural log)
 *
 * The standard definition is on the page "FlashAttention" (LLM inference
 * handbook, kernel-optimization chapter), section "attention 为什么一开始就很慢";
 * the tiled online-softmax evaluation that keeps S and P on chip is section
 * 2.2 of "深度学习进阶（三十一）FlashAttention：IO 感知的精确注意力"; the backward
 * pass recomputes P from Q, K and the saved LSE ("Flash-Attention" concept
 * page, "Core idea") and returns the chain-rule gradients dQ, dK, dV.
 *
 * Layouts (all row-major, contiguous, 16-byte aligned device pointers):
 *   q, o, dout, dq : bf16 [B, Hq,  N, d]
 *   k, v, dk, dv   : bf16 [B, Hkv, N, d]
 *   lse            : fp32 [B, Hq,  N]
 * N is any positive length.  The kernels work in 128-row tiles; when N is not
 * a multiple of 128, keys past N are masked out of every row and query rows
 * past N are neither stored nor given any weight in the gradients.
 *
 * Ownership.  The caller allocates every buffer (device memory) and keeps it
 * alive until the work on `stream` has finished.  No call allocates or frees
 * memory.  The library's only device memory of its own is static: a 4-byte
 * error word and the FA_NOALLOC_SCRATCH_BYTES (64 MiB) scratch array of
 * fa_bwd_noalloc, both held by every device that loads the library, whether
 * or not it ever calls fa_bwd_noalloc.
 * `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  Every call only enqueues work and returns; errors found on the
 * device are reported by fa_device_status().
 *
 * Errors.  Arguments are checked before anything is enqueued:
 *   FA_ERR_INVALID_ARG  null or misaligned pointer, negative size, Hq not a
 *                       multiple of Hkv, non-finite or non-positive scale,
 *                       an output overlapping an input or another output,
 *                       workspace too small;
 *   FA_ERR_UNSUPPORTED  d not in {64, 128, 256}, sizes beyond the index
 *                       limits (B, Hq ≤ 65535, B·Hq·Np < 2^31 with Np = N
 *                       rounded up to 128), or no sm_100 device;
 *   FA_ERR_CUDA         a CUDA launch or attribute call failed;
 *   FA_ERR_TIMEOUT      (fa_device_status only) a kernel gave up a bounded
 *                       wait and returned early; its outputs are invalid;
 *   FA_ERR_DEVICE_CHECK (fa_device_status, debug builds only) a device-side
 *                       check of a bulk-copy coordinate or address failed
 *                       and the copy was skipped; outputs are invalid.  The
 *                       library is a debug build when compiled with
 *                       -DFA_DEBUG (python -m exact_attention_104_b200.build
 *                       --debug writes libfa_b200_debug.so).
 * A problem with B == 0 or N == 0 is empty: nothing is enqueued, FA_OK.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4,
  FA_ERR_DEVICE_CHECK = 5
} fa_status;

/* Forward pass: writes O (bf16) and LSE (fp32, natural log).
 * One fused kernel; S and P stay on chip.  `causal` != 0 masks keys after
 * the query.  `scale` multiplies the scores before masking and softmax
 * (usually 1/sqrt(d)). */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                 void* stream);

/* The same forward pass (same arguments, layouts, results within the same
 * rounding) computed on pairs of CTAs that share every tensor-core product
 * (tcgen05 cta_group::2, the "2-CTA MMA" of FA4 in the version table of the
 * handbook page "FlashAttention"): a cluster of two CTAs takes four query
 * tiles of 128 rows, each CTA two of them, and each CTA loads only half of
 * every K/V block.  d = 128 only (other d: FA_ERR_UNSUPPORTED).  On B200 it
 * measured 12-26 % slower than fa_fwd, which therefore does not use it. */
fa_status fa_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                      void* stream);

/* Bytes of device workspace fa_bwd needs: two fp32 [B,Hq,Np] row vectors
 * (D = rowsum(dO∘O) and LSE·log2 e) and an fp32 [B,Hq,Np,d] dQ accumulator,
 * each rounded up to 256 bytes, where Np = N rounded up to a multiple of 128
 * (per-head padding rows keep every tile aligned and private to its head),
 * plus 256 bytes for the counter the main kernel's CTAs claim work from.
 * Returns 0 for invalid sizes. */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/* Backward pass: given q, k, v, the forward outputs o and lse, and the output
 * gradient dout, writes dq, dk, dv (bf16).  dk and dv are summed over the
 * query heads that share a key/value head.  `workspace` (device, 256-byte
 * aligned, at least fa_bwd_workspace_bytes) is scratch owned by the caller;
 * its contents on entry do not matter, and it is in use until the call's
 * kernels have finished, so calls that may run at the same time (on
 * different streams) need separate workspaces.  Enqueues three kernels on
 * `stream`. */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv,
                 int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the current device's error
 * word.  FA_ERR_DEVICE_CHECK if a debug build's device-side check failed,
 * else FA_ERR_TIMEOUT if a kernel abandoned a bounded wait since the last
 * call, FA_ERR_CUDA if the stream reported a CUDA error, else FA_OK. */
fa_status fa_device_status(void* stream);

/* Static English description of a status code; never NULL. */
const char* fa_status_string(fa_status s);

/* Cycle budget (SM clock cycles) after which a kernel's wait on an on-chip
 * barrier gives up, records FA_ERR_TIMEOUT and returns.  0 restores the
 * default (2^31 cycles, about one second).  Affects later launches only. */
fa_status fa_set_wait_cap(long long cycles);

/* One-shot profiling hook for the calling host thread: the next fa_fwd,
 * fa_bwd or fa_fwd_decode call records `start_event` on its stream
 * immediately before its main kernel (fa_fwd's fused kernel; fa_bwd's
 * dK/dV/dQ kernel, after the preprocessing kernel; fa_fwd_decode's split
 * kernel, before the combine kernel) and `stop_event` immediately after it,
 * then forgets both.  The events are cudaEvent_t handles owned by the caller;
 * NULL for both cancels a pending request. */
fa_status fa_profile_next(void* start_event, void* stop_event);

/* Self-test of the failure path: launches one tiny kernel whose single
 * thread waits, through the same bounded mbarrier wait the attention kernels
 * use, on an on-chip barrier that nothing ever arrives on.  After
 * `cap_cycles` SM cycles (must be in [1, 2^31]) the wait gives up, records
 * FA_ERR_TIMEOUT in the device error word and the kernel returns normally;
 * fa_device_status() then reports FA_ERR_TIMEOUT once.  Nothing faults or
 * hangs, and the context stays usable. */
fa_status fa_selftest_wait_timeout(long long cap_cycles, void* stream);

/* Self-test of the device exponentials: y[i] = 2^x[i] for n floats (device
 * pointers, 16-byte aligned), computed with the MUFU instruction
 * (use_poly = 0) or with the FMA-pipe polynomial the softmax can use
 * (use_poly = 1). */
fa_status fa_selftest_exp2(const float* x, float* y, long long n, int use_poly, void* stream);

/* ------------------------------------------------------------------------
 * Decoding: Nq query rows per head against Nk cached keys and values.
 *
 * The queries are the last Nq positions of an Nk-long sequence: query row i
 * sits at position Nk - Nq + i, and with `causal` != 0 it sees keys
 * 0 .. Nk - Nq + i (so its result is row Nk - Nq + i of fa_fwd over the whole
 * sequence).  Same per-row online softmax as fa_fwd ("深度学习进阶（三十一）
 * FlashAttention：IO 感知的精确注意力" §2.2); the key axis is split over
 * CTAs and the partial results are merged with their running maxima and
 * normalisers, since with few query rows the pass is bound by reading K, V.
 *
 * Layouts: q, o bf16 [B, Hq, Nq, d]; k, v bf16 [B, Hkv, Nk, d]; lse fp32
 * [B, Hq, Nq] (natural log).  `workspace` (device, 256-byte aligned, at least
 * fa_decode_workspace_bytes) holds the per-split partial results.
 * Errors as for fa_fwd, plus FA_ERR_INVALID_ARG for Nk == 0 with Nq > 0 and
 * for causal with Nq > Nk, and FA_ERR_UNSUPPORTED for Nq > 256 (use fa_fwd).
 * Two kernels are enqueued on `stream`; B == 0 or Nq == 0 is a no-op. */
size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d);
fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Packed batches of sequences with different lengths ("varlen").
 *
 * `nseq` independent sequences are stored back to back along the token axis
 * of every head: sequence b owns tokens cu_seqlens[b] .. cu_seqlens[b+1] - 1,
 * and T = cu_seqlens[nseq] tokens in all.  Each sequence attends only to its
 * own keys (with `causal` != 0, key j of the sequence is masked for query i
 * of the sequence when j > i, positions counted from the sequence's first
 * token), so the result for every sequence is exactly that of one fa_fwd /
 * fa_bwd call on its own tokens.  Ragged batches are the case the
 * "Flash-Attention" concept page names under "Design space and trade-offs"
 * (they change which tiles are legal and how work balances) and "Known
 * limits" (continuous batching).
 *
 * Layouts (head-major: [B, H, N, d] with B = 1, N = T and the sequences
 * concatenated along N):
 *   q, o, dout, dq : bf16 [Hq,  T, d]
 *   k, v, dk, dv   : bf16 [Hkv, T, d]
 *   lse            : fp32 [Hq,  T]
 *   cu_seqlens     : int32 [nseq + 1] in DEVICE memory: cu_seqlens[0] = 0,
 *                    non-decreasing, cu_seqlens[nseq] = T (empty sequences
 *                    are allowed)
 * `max_seqlen` (host) must bound every sequence length, 1 <= max_seqlen <=
 * 2^20.  Because cu_seqlens lives on the device it is checked by the
 * library's first kernel: if it breaks any rule above, no attention kernel
 * computes anything, the outputs are left untouched and fa_device_status()
 * reports FA_ERR_INVALID_ARG.
 *
 * Scheduling: the first kernel of each call turns cu_seqlens into a table of
 * (sequence, tile) work units in the workspace, heaviest first, which the
 * attention kernels deal out.  Units of equal weight may come in any order,
 * so the backward's dQ, like fa_bwd's, is not bitwise reproducible.
 *
 * Workspace: device, 256-byte aligned, at least the size the matching
 * *_workspace_bytes function returns (0 for invalid sizes); it is in use
 * until the call's kernels have finished.  Other errors as for fa_fwd and
 * fa_bwd; T == 0 (or nseq == 0) is an empty problem.
 * fa_fwd_varlen enqueues two kernels, fa_bwd_varlen four. */
size_t fa_fwd_varlen_workspace_bytes(int nseq, int Hq, int Hkv, int T, int max_seqlen, int d);
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens, int nseq, int Hq, int Hkv, int T, int max_seqlen,
                        int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                        void* stream);

size_t fa_bwd_varlen_workspace_bytes(int nseq, int Hq, int Hkv, int T, int max_seqlen, int d);
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv,
                        const int* cu_seqlens, int nseq, int Hq, int Hkv, int T, int max_seqlen,
                        int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Size in bytes of the fixed device scratch array used by fa_bwd_noalloc. */
#define FA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Backward pass without caller-provided scratch.  (The FlashAttention pages
 * have no counterpart to this entry point; it exists for callers, not for
 * the method.)
 *
 * Same arguments, layouts and results as fa_bwd, minus the workspace.  It is
 * meant for callers that cannot hand the library a device buffer: code that
 * runs inside a host framework which owns all device memory and offers its
 * plugins no allocator, or a latency-critical loop where calling cudaMalloc
 * (which can synchronise the whole device) is not acceptable.  Instead of a
 * workspace it uses one file-scope device array of FA_NOALLOC_SCRATCH_BYTES
 * (64 MiB), which every GPU that loads the library holds until the process
 * exits.  Nothing is allocated or freed per call.
 *
 * Limit: the problem's fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) must not
 * exceed FA_NOALLOC_SCRATCH_BYTES (for d = 128 that is B·Hq·Np ≤ 129,024
 * padded query rows, i.e. 1008 heads of up to 128 rows); larger problems
 * return FA_ERR_UNSUPPORTED and enqueue nothing.
 *
 * Set-up: the first call on each device, with that device current, looks up
 * the array's device address (cudaGetSymbolAddress).  Make that first call
 * before any stream capture on that device.
 *
 * Sharing: all calls on a device use the same array, and it keeps whatever
 * the last call left in it (the dQ accumulator is zeroed by every call before
 * use).  Two calls whose work overlaps on the GPU — different streams, or
 * different host threads without ordering — race on the array and give wrong
 * results; order them on one stream or with events. */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv,
                         int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
