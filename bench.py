"""Benchmark: exact attention forward + backward on B200, through the C ABI.

One step = one forward pass (fa_fwd) and one backward pass (fa_bwd) over the
whole workload, with inputs resident in HBM.  The default workload is the
long causal sequence B=1, Hq=Hkv=16, N=16384, d=128, bf16, seeded synthetic
N(0,1) inputs.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME|all] [--no-e2e] [--no-cpu-baseline]

(--workload all prints one line per reference workload.)

Multi-GPU (launched by torchrun): every rank runs its own independent problem
of the same size (weak scaling; attention over distinct batches needs no data
exchange), timed with CUDA events, max over ranks.

--impl reference times the fp64 CPU oracle on this host's cores on a bounded
sample of the same workload (one strided block of query rows of one head per
step).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd and fwd+bwd TFLOPS (bf16) and % of B200 dense BF16 tensor peak"
NOMINAL_PEAK_TFLOPS = 2250.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        try:
            lines = open(self.out.name).read().strip().splitlines()
        except Exception:
            lines = []
        os.unlink(self.out.name)
        mhz, maxes, reasons, power = [], [], set(), []
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            mhz.append(sm)
            maxes.append(smax)
            try:
                power.append(float(parts[3]))
            except ValueError:
                pass
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(mhz), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------- CPU oracle
_CPU_INPUTS = {}

# Largest score block (query rows x keys) the CPU sample materialises per step:
# every row of a head for N <= 2048, a strided block of rows beyond.
CPU_BLOCK_ENTRIES = 1 << 22


def cpu_sample_rows(w, step: int):
    """Query rows and head of CPU-sample step ``step``: head ``step % Hq`` of
    batch 0, rows ``off, off + stride, ...`` with ``stride = N / R`` and the
    offset rotating from step to step, R = min(N, CPU_BLOCK_ENTRIES / N)."""
    import numpy as np
    n_rows = max(1, min(w.N, CPU_BLOCK_ENTRIES // w.N))
    stride = max(1, w.N // n_rows)
    off = (step // w.Hq) % stride
    return step % w.Hq, np.arange(off, w.N, stride)[:n_rows]


def cpu_sample_flops(w, rows) -> float:
    """FLOPs of the forward+backward share of the given query rows, in the
    metric's convention: 3.5 x 4·d per visible (query, key) pair."""
    import numpy as np
    visible = float(np.sum(np.asarray(rows) + 1)) if w.causal else float(len(rows)) * w.N
    return 3.5 * 4.0 * w.d * visible


def cpu_oracle_sample(w, seconds: float, max_steps: int | None = None, first_step: int = 0):
    """Time the fp64 oracle's forward+backward share (oracle.head_backward_rows)
    of strided query-row blocks of single heads of the workload until
    ``seconds`` of CPU work have been spent (or ``max_steps`` blocks).
    Returns (TFLOPS, blocks, elapsed seconds, rows per block)."""
    import numpy as np

    import oracle
    from exact_attention_104_b200.workloads import make_inputs

    key = (w.name, w.seed)
    if key not in _CPU_INPUTS:
        _CPU_INPUTS.clear()
        _CPU_INPUTS[key] = make_inputs(w, "cpu")
    q, k, v, do = _CPU_INPUTS[key]
    G = w.G
    steps, t_total, flops, n_rows = 0, 0.0, 0.0, 0
    while True:
        h, rows = cpu_sample_rows(w, first_step + steps)
        n_rows = len(rows)
        sl = lambda t, hh: t[0, hh].float().numpy().astype(np.float64)  # noqa: E731
        qs, dos = sl(q, h), sl(do, h)
        ks, vs = sl(k, h // G), sl(v, h // G)
        t0 = time.perf_counter()
        oracle.head_backward_rows(qs, ks, vs, dos, w.scale, w.causal, rows)
        t_total += time.perf_counter() - t0
        flops += cpu_sample_flops(w, rows)
        steps += 1
        if t_total >= seconds or (max_steps is not None and steps >= max_steps):
            break
    return flops / t_total / 1e12, steps, t_total, n_rows


def run_reference(args, w, rank, world):
    """The reference arm: the fp64 oracle on the host cores, one strided block
    of query rows of one head of the workload per step.  Rank 0 only."""
    if rank != 0:
        return
    for i in range(args.warmup):
        cpu_oracle_sample(w, 0.0, max_steps=1, first_step=i)
    total, flops, n_rows = 0.0, 0.0, 0
    for i in range(args.steps):
        h, rows = cpu_sample_rows(w, args.warmup + i)
        _, _, t, n_rows = cpu_oracle_sample(w, 0.0, max_steps=1, first_step=args.warmup + i)
        total += t
        flops += cpu_sample_flops(w, rows)
    value = flops / total / 1e12
    cores = _blas_threads()
    sample = (f"per step: {n_rows} strided query rows of one head (batch 0) of {w.describe()}, their share "
              "of the forward and backward (oracle.head_backward_rows) in fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- decode
def decode_oracle_sample(w, seconds: float, max_batches: int | None = None):
    """Time the fp64 oracle's suffix attention on whole batch entries (all
    heads of one b) of a decode workload.  Returns (TFLOPS, batches, seconds)."""
    import oracle
    from exact_attention_104_b200.workloads import make_decode_inputs

    key = (w.name, w.seed)
    if key not in _CPU_INPUTS:
        _CPU_INPUTS.clear()
        _CPU_INPUTS[key] = make_decode_inputs(w, "cpu")
    q, k, v = _CPU_INPUTS[key]
    done, t_total = 0, 0.0
    while True:
        b = done % w.B
        sl = lambda t: t[b:b + 1].double().numpy()  # noqa: E731
        t0 = time.perf_counter()
        oracle.attention_forward_suffix(sl(q), sl(k), sl(v), w.scale, w.causal)
        t_total += time.perf_counter() - t0
        done += 1
        if t_total >= seconds or (max_batches is not None and done >= max_batches):
            break
    return w.fwd_flops() / w.B * done / t_total / 1e12, done, t_total


def decode_split_kernel_name(w) -> str:
    """The kernel fa_fwd_decode runs before its combine kernel: the CUDA-core
    split kernel for at most 16 query rows per kv head (G·Nq), else the
    tensor-core forward kernel in its decode mode."""
    return "fa_decode_split_kernel" if w.G * w.Nq <= 16 else "fa_fwd_kernel (decode mode)"


def run_decode(args, w, rank, world, local_rank):
    """One step = one fa_fwd_decode call over the whole decode workload (all
    batch entries and heads), K and V resident in HBM.  Reported in the same
    TFLOPS metric; the roofline is HBM bandwidth, since every step must read
    the whole K/V cache once."""
    import torch
    import torch.distributed as dist

    from exact_attention_104_b200 import binding
    from exact_attention_104_b200.workloads import make_decode_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    stream = torch.cuda.current_stream()
    q, k, v = make_decode_inputs(w, dev, seed=w.seed + 7919 * rank)
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.Nq, dtype=torch.float32, device=dev)
    ws_bytes = binding.fa_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step(prof=None):
        if prof is not None:
            binding.fa_profile_next(*prof)
        st = binding.fa_fwd_decode(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, w.scale, ws,
                                   ws_bytes, stream)
        if st:
            raise binding.FAError(st, "fa_fwd_decode")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        return reduce_max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    K = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    k_ev = [(ev(), ev()) for _ in range(K)]
    start, stop = ev(), ev()
    for e in [x for pair in k_ev for x in pair] + [start, stop]:
        e.record(stream)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        barrier()
        start.record(stream)
        for i in range(K):
            step(k_ev[i])
        stop.record(stream)
        barrier()
    clocks = clk.summary()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms_step = max_over_ranks(start.elapsed_time(stop)) / K
    ms_split = max_over_ranks(sum(a.elapsed_time(b) for a, b in k_ev) / K)
    F = w.fwd_flops()
    value = F * world / (ms_step * 1e-3) / 1e12
    peaks = _peaks()
    gbs = w.hbm_bytes() / (ms_split * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        # a decoding step's own data is its query rows and its outputs; the K/V
        # cache stays on the device between steps
        def e2e_compute(ins, outs, extra):
            (q_,) = ins
            o_, lse_ = outs
            (ws_,) = extra
            st = binding.fa_fwd_decode(q_, k, v, o_, lse_, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, w.scale,
                                       ws_, ws_bytes, stream)
            if st:
                raise binding.FAError(st, "fa_fwd_decode")

        e2e = run_e2e(dev, stream, (q,), (o, lse), (ws,), e2e_compute, F, world, barrier, max_over_ranks, K)
        if binding.fa_device_status(stream) != 0:
            raise RuntimeError("device error in the end-to-end region")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tflops, nb, secs = decode_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": tflops, "unit": "TFLOPS", "cores": _blas_threads(), "kind": "oracle",
               "sample": f"{nb} batch entries (all heads) of {w.describe()}, fp64, {secs:.1f} s"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "causal": w.causal, "global_batch": w.B * world, "parallelism": f"dp{world}",
                   "l2": f"K/V {2 * w.B * w.Hkv * w.Nk * w.d * 2 / 2**20:.0f} MiB per step (> 126 MiB L2: no flush "
                         "needed)" if 4 * w.B * w.Hkv * w.Nk * w.d > 126 * 2**20 else "K/V fit in L2"},
        "roofline": {"kernel": decode_split_kernel_name(w), "bound": "hbm", "achieved": gbs,
                     "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "peak_source": peaks["source"] + " HBM copy (MEASURED_PEAKS.json)",
                     "bytes_per_launch": w.hbm_bytes(), "ms_per_launch": ms_split,
                     "traffic": MEASURED_DECODE_TRAFFIC.get(w.name)},
        "ms": {"split_kernel": ms_split, "call": ms_step},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_decode_reference(args, w, rank):
    """The reference arm for a decode workload: the fp64 oracle on one batch
    entry (all heads) per step.  Rank 0 only."""
    if rank != 0:
        return
    for _ in range(args.warmup):
        decode_oracle_sample(w, 0.0, max_batches=1)
    total = 0.0
    for _ in range(args.steps):
        total += decode_oracle_sample(w, 0.0, max_batches=1)[2]
    value = w.fwd_flops() / w.B * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"one batch entry (all heads) of {w.describe()} per step, fp64"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- varlen
def run_varlen(args, w, rank, world, local_rank):
    """One step = fa_fwd_varlen + fa_bwd_varlen over a packed batch of
    sequences of different lengths ([H, T, d] tensors), inputs resident in
    HBM.  FLOPs: 4·d per visible (query, key) pair of each sequence and query
    head, 3.5x for forward + backward (the fixed-length convention)."""
    import torch
    import torch.distributed as dist

    from exact_attention_104_b200 import binding
    from exact_attention_104_b200.workloads import make_varlen_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    stream = torch.cuda.current_stream()
    q, k, v, do, cu = make_varlen_inputs(w, dev)
    nseq, T = len(w.lengths), w.T
    o = torch.empty_like(q)
    lse = torch.empty(w.Hq, T, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fws = binding.fa_fwd_varlen_workspace_bytes(nseq, w.Hq, w.Hkv, T, w.max_seqlen, w.d)
    bws = binding.fa_bwd_varlen_workspace_bytes(nseq, w.Hq, w.Hkv, T, w.max_seqlen, w.d)
    fw = torch.empty(fws, dtype=torch.uint8, device=dev)
    bw = torch.empty(bws, dtype=torch.uint8, device=dev)

    def step(fprof=None, bprof=None):
        if fprof is not None:
            binding.fa_profile_next(*fprof)
        st = binding.fa_fwd_varlen(q, k, v, o, lse, cu, nseq, w.Hq, w.Hkv, T, w.max_seqlen, w.d, w.causal, w.scale,
                                   fw, fws, stream)
        if st:
            raise binding.FAError(st, "fa_fwd_varlen")
        if bprof is not None:
            binding.fa_profile_next(*bprof)
        st = binding.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu, nseq, w.Hq, w.Hkv, T, w.max_seqlen, w.d,
                                   w.causal, w.scale, bw, bws, stream)
        if st:
            raise binding.FAError(st, "fa_bwd_varlen")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    K = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    f_ev = [(ev(), ev()) for _ in range(K)]
    b_ev = [(ev(), ev()) for _ in range(K)]
    start, stop = ev(), ev()
    for e in [x for pair in f_ev + b_ev for x in pair] + [start, stop]:
        e.record(stream)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        barrier()
        start.record(stream)
        for i in range(K):
            step(f_ev[i], b_ev[i])
        stop.record(stream)
        barrier()
    clocks = clk.summary()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    mo = lambda x: reduce_max_over_ranks(x, world, dev)  # noqa: E731
    ms_step = mo(start.elapsed_time(stop)) / K
    ms_fwd = mo(sum(a.elapsed_time(b) for a, b in f_ev) / K)
    ms_bwd = mo(sum(a.elapsed_time(b) for a, b in b_ev) / K)
    F = w.fwd_flops()
    value = 3.5 * F * world / (ms_step * 1e-3) / 1e12
    peaks = _peaks()
    bwd_tflops = 2.5 * F / (ms_bwd * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        def e2e_compute(ins, outs, extra):
            q_, k_, v_, do_, cu_ = ins
            o_, lse_, dq_, dk_, dv_ = outs
            fw_, bw_ = extra
            st = binding.fa_fwd_varlen(q_, k_, v_, o_, lse_, cu_, nseq, w.Hq, w.Hkv, T, w.max_seqlen, w.d, w.causal,
                                       w.scale, fw_, fws, stream)
            if st:
                raise binding.FAError(st, "fa_fwd_varlen")
            st = binding.fa_bwd_varlen(q_, k_, v_, o_, lse_, do_, dq_, dk_, dv_, cu_, nseq, w.Hq, w.Hkv, T,
                                       w.max_seqlen, w.d, w.causal, w.scale, bw_, bws, stream)
            if st:
                raise binding.FAError(st, "fa_bwd_varlen")

        e2e = run_e2e(dev, stream, (q, k, v, do, cu), (o, lse, dq, dk, dv), (fw, bw), e2e_compute, 3.5 * F,
                      world, barrier, mo, K)
        if binding.fa_device_status(stream) != 0:
            raise RuntimeError("device error in the end-to-end region")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "sequences": len(w.lengths), "T": T, "max_seqlen": w.max_seqlen,
                   "lengths": list(w.lengths), "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "causal": w.causal,
                   "parallelism": f"dp{world}",
                   "l2": _l2_note(q, k, v, o, do)},
        "fwd_tflops": F / (ms_fwd * 1e-3) / 1e12,
        "bwd_tflops": bwd_tflops,
        "ms": {"fwd_kernel": ms_fwd, "bwd_main_kernel": ms_bwd},
        "roofline": {"kernel": "fa_bwd_kernel (packed-batch mode)", "bound": "tensor", "achieved": bwd_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": bwd_tflops / peaks["bf16_tflops"],
                     "peak_source": peaks["source"] + " bf16 burst (MEASURED_PEAKS.json)",
                     "flops_per_launch": 2.5 * F, "ms_per_launch": ms_bwd, "traffic": None},
        "cpu_baseline": None,
        "e2e": e2e,
        "gpu_launches": 6 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- e2e
def run_e2e(dev, stream, ins0, outs0, extra0, compute, step_flops, world, barrier, max_over_ranks, K):
    """The step through the public C ABI with its data on the host: every step
    copies that step's inputs from pinned host memory to the device, runs the
    step's kernels (``compute(ins, outs, extra)`` enqueues them on ``stream``)
    and copies its outputs back.  As in a training loop, the copies of
    neighbouring steps overlap the kernels: H2D and D2H run on their own
    streams (the GPU's copy engines) over three sets of device buffers, with
    events ordering each buffer's reuse, so that both copy directions can stay
    busy while the kernels run.  The timed region runs from the first H2D to
    the last D2H."""
    import torch

    host_in = [t.cpu().pin_memory() for t in ins0]
    n_sets = 3
    sets = [(list(ins0), list(outs0), list(extra0))]
    for _ in range(n_sets - 1):
        sets.append(([torch.empty_like(t) for t in ins0], [torch.empty_like(t) for t in outs0],
                     [torch.empty_like(t) for t in extra0]))
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs0] for _ in range(n_sets)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_h2d = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
    in_ready = [ev() for _ in range(n_sets)]
    comp_done = [ev() for _ in range(n_sets)]
    out_done = [ev() for _ in range(n_sets)]

    def step(i):
        b = i % n_sets
        ins, outs, extra = sets[b]
        with torch.cuda.stream(s_h2d):
            if i >= n_sets:
                s_h2d.wait_event(comp_done[b])  # this buffer's previous step no longer reads its inputs
            for hsrc, ddst in zip(host_in, ins):
                ddst.copy_(hsrc, non_blocking=True)
            in_ready[b].record(s_h2d)
        stream.wait_event(in_ready[b])
        if i >= n_sets:
            stream.wait_event(out_done[b])  # its previous outputs have reached the host
        compute(ins, outs, extra)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(comp_done[b])
            for hdst, dsrc in zip(host_out[b], outs):
                hdst.copy_(dsrc, non_blocking=True)
            out_done[b].record(s_d2h)

    ke = max(3, min(K, 30))
    for i in range(n_sets):  # warm-up
        step(i)
    torch.cuda.synchronize()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_h2d)
    for i in range(ke):
        step(i)
    s_d2h.wait_stream(stream)
    t1.record(s_d2h)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1)) / ke
    return {"value": step_flops * world / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ke,
            "overlap": "H2D of later steps and D2H of earlier ones overlap the kernels of step i (3 buffer sets)"}


# ------------------------------------------------------------------- ours
L2_BYTES = 126 * 2**20

# dram__bytes_read.sum + dram__bytes_write.sum of one fa_bwd_kernel launch, from one ncu
# capture of the current kernel (summarised under profiles/).  An entry must be
# removed whenever fa_bwd_kernel changes.
MEASURED_TRAFFIC = {"long_b1_h16_n16384_d128_causal": 631.6e6, "wide_b2_h8_n8192_d256_bigqk": 626.3e6}

# The same for one fa_decode_split_kernel launch (also summarised under profiles/);
# reset to None whenever that kernel changes.
MEASURED_DECODE_TRAFFIC = {"decode_b8_hq32_hkv8_nk32768_d128": 1079.4e6,
                           "decode_b8_hq32_hkv8_nq32_nk32768_d128": 1079.0e6}


def _l2_note(*tensors) -> str:
    nbytes = sum(t.numel() * t.element_size() for t in tensors)
    mib = nbytes / 2**20
    if nbytes > L2_BYTES:
        return f"inputs larger than L2 (Q,K,V,O,dO {mib:.0f} MiB in all > 126 MiB L2; no flush needed)"
    return f"inputs fit in L2 ({mib:.1f} MiB; not flushed: a small parity-sized case, not a bench line)"


def reduce_max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values of x (a per-rank elapsed time): every
    multi-GPU figure is timed on the slowest rank.  ``device`` holds the
    one-element tensor the collective reduces (a CUDA device under NCCL)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def logit_extremes(q, k, scale: float, causal: bool, rows_per_chunk: int = 2048):
    """Largest |q·k| and |s·q·k| over every visible (query, key) pair of batch 0, query
    head 0 (its kv head is 0), computed on the host in fp32 from the bf16 inputs.  A
    record of how peaked the softmax rows are (the d = 256 workload's Q, K ~ N(0, 9)
    is there to give raw logits far above 100)."""
    import numpy as np
    qh = q[0, 0].float().cpu().numpy()
    kh = k[0, 0].float().cpu().numpy()
    n = qh.shape[0]
    best = 0.0
    for r0 in range(0, n, rows_per_chunk):
        s = qh[r0:r0 + rows_per_chunk] @ kh.T
        if causal:
            rows = np.arange(r0, min(n, r0 + rows_per_chunk))[:, None]
            s = np.where(np.arange(n)[None, :] <= rows, s, 0.0)
        best = max(best, float(np.abs(s).max()))
    return {"max_abs_raw": best, "max_abs_scaled": best * scale,
            "sample": "batch 0, query head 0, all visible (query, key) pairs, fp32 on the host"}


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from exact_attention_104_b200 import binding
    from exact_attention_104_b200.workloads import make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    stream = torch.cuda.current_stream()

    # independent problem per rank (weak scaling): same shape, rank-specific seed
    q, k, v, do = make_inputs(w, dev, seed=w.seed + 7919 * rank)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scale = w.scale

    def fwd(prof=None):
        if prof is not None:
            binding.fa_profile_next(*prof)
        st = binding.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, w.causal, scale, stream)
        if st:
            raise binding.FAError(st, "fa_fwd")

    def bwd(prof=None):
        if prof is not None:
            binding.fa_profile_next(*prof)
        st = binding.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, N, d, w.causal, scale, ws, ws_bytes,
                            stream)
        if st:
            raise binding.FAError(st, "fa_bwd")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        return reduce_max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")

    # timed region: K whole steps, plus per-kernel events on the same stream
    K = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    f_ev = [(ev(), ev()) for _ in range(K)]
    b_ev = [(ev(), ev()) for _ in range(K)]
    start, stop = ev(), ev()
    for e in [x for pair in f_ev + b_ev for x in pair] + [start, stop]:
        e.record(stream)  # creates the event handles before the timed region
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        barrier()
        start.record(stream)
        for i in range(K):
            fwd(f_ev[i])
            bwd(b_ev[i])
        stop.record(stream)
        barrier()
    clocks = clk.summary()
    if binding.fa_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms_total = max_over_ranks(start.elapsed_time(stop))
    ms_fwd_kernel = max_over_ranks(sum(a.elapsed_time(b) for a, b in f_ev) / K)
    ms_bwd_kernel = max_over_ranks(sum(a.elapsed_time(b) for a, b in b_ev) / K)

    F = w.fwd_flops()
    step_flops = 3.5 * F
    ms_step = ms_total / K
    value = step_flops * world * K / (ms_total * 1e-3) / 1e12
    fwd_tflops = F / (ms_fwd_kernel * 1e-3) / 1e12
    bwd_main_tflops = 2.5 * F / (ms_bwd_kernel * 1e-3) / 1e12
    peaks = _peaks()

    # separate fwd-only and bwd-only throughput (whole calls), outside the main timed region
    def time_calls(fn, reps):
        barrier()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        barrier()
        return max_over_ranks(a.elapsed_time(b)) / reps

    reps = max(3, min(K, 50))
    ms_fwd_call = time_calls(fwd, reps)
    ms_bwd_call = time_calls(bwd, reps)

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        def e2e_compute(ins, outs, extra):
            q_, k_, v_, do_ = ins
            o_, lse_, dq_, dk_, dv_ = outs
            (ws_,) = extra
            st = binding.fa_fwd(q_, k_, v_, o_, lse_, B, Hq, Hkv, N, d, w.causal, scale, stream)
            if st:
                raise binding.FAError(st, "fa_fwd")
            st = binding.fa_bwd(q_, k_, v_, o_, lse_, do_, dq_, dk_, dv_, B, Hq, Hkv, N, d, w.causal, scale, ws_,
                                ws_bytes, stream)
            if st:
                raise binding.FAError(st, "fa_bwd")

        e2e = run_e2e(dev, stream, (q, k, v, do), (o, lse, dq, dk, dv), (ws,), e2e_compute, step_flops, world,
                      barrier, max_over_ranks, K)
        if binding.fa_device_status(stream) != 0:
            raise RuntimeError("device error in the end-to-end region")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tflops, blocks, secs, n_rows = cpu_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": tflops, "unit": "TFLOPS", "cores": _blas_threads(), "kind": "oracle",
               "sample": f"{blocks} blocks of {n_rows} strided query rows of one head (batch 0) of "
                         f"{w.describe()}, their share of the forward and backward in fp64, {secs:.1f} s"}

    # dominant kernel: the backward dK/dV/dQ kernel (2.5x the forward FLOPs)
    bwd_main_flops = 2.5 * F
    roof = {
        "kernel": "fa_bwd_kernel",
        "bound": "tensor",
        "achieved": bwd_main_tflops,
        "peak": peaks["bf16_tflops"],
        "unit": "TFLOP/s",
        "frac": bwd_main_tflops / peaks["bf16_tflops"],
        "peak_source": peaks["source"] + " bf16 burst (MEASURED_PEAKS.json)",
        "flops_per_launch": bwd_main_flops,
        "ms_per_launch": ms_bwd_kernel,
        "traffic": args.traffic_bytes if args.traffic_bytes else MEASURED_TRAFFIC.get(w.name),
    }
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "causal": w.causal,
                   "qk_std": w.qk_std, "global_batch": B * world, "seq_len": N,
                   "parallelism": f"dp{world} (independent problem per GPU)",
                   "l2": _l2_note(q, k, v, o, do)},
        "fwd_tflops": fwd_tflops,
        "bwd_tflops": 2.5 * F / (ms_bwd_call * 1e-3) / 1e12,
        "fwd_bwd_tflops": value / world,
        "pct_of_peak": {"fwd_vs_2250_nominal": fwd_tflops / NOMINAL_PEAK_TFLOPS,
                        "fwd_vs_measured": fwd_tflops / peaks["bf16_tflops"],
                        "fwd_bwd_vs_2250_nominal": value / world / NOMINAL_PEAK_TFLOPS,
                        "fwd_bwd_vs_measured": value / world / peaks["bf16_tflops"]},
        "ms": {"fwd_kernel": ms_fwd_kernel, "bwd_main_kernel": ms_bwd_kernel, "fwd_call": ms_fwd_call,
               "bwd_call": ms_bwd_call},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 4 * K,
        "clocks": clocks,
    }
    if rank == 0:
        line["logits"] = logit_extremes(q, k, scale, w.causal)
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--traffic-bytes", type=float, default=0.0,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture, if known")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from exact_attention_104_b200.workloads import BENCH_WORKLOAD, DECODE_WORKLOADS, VARLEN_WORKLOADS, WORKLOADS

    names = (list(WORKLOADS) + list(DECODE_WORKLOADS) + list(VARLEN_WORKLOADS) if args.workload == "all"
             else [args.workload or BENCH_WORKLOAD])
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        for name in names:
            if name in DECODE_WORKLOADS:
                run_decode_reference(args, DECODE_WORKLOADS[name], rank)
            elif name in VARLEN_WORKLOADS:
                if rank == 0:
                    print(json.dumps({"impl": "reference", "workload": name,
                                      "unavailable": "the reference arm times fixed-length workloads"}), flush=True)
            else:
                run_reference(args, WORKLOADS[name], rank, world)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        for name in names:
            if name in DECODE_WORKLOADS:
                run_decode(args, DECODE_WORKLOADS[name], rank, world, local_rank)
            elif name in VARLEN_WORKLOADS:
                run_varlen(args, VARLEN_WORKLOADS[name], rank, world, local_rank)
            else:
                run_ours(args, WORKLOADS[name], rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
