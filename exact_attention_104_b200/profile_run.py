"""Run a few attention calls on one synthetic shape, for a profiler to capture.

    python -m exact_attention_104_b200.profile_run fwd B H N d causal qk_std [calls]
    python -m exact_attention_104_b200.profile_run bwd B H N d causal qk_std [calls]

``fwd`` runs ``calls`` forward calls (default 4); ``bwd`` runs one forward and
``calls`` backward calls (default 3).  Inputs are the seeded standard-normal
tensors of ``workloads.make_inputs`` (Q and K times qk_std), one kv head per
query head.  Exits non-zero if a call or the device status reports an error.
"""

import sys

import torch

from . import binding
from .workloads import Workload, make_inputs


def main(argv):
    if len(argv) < 7:
        print(__doc__)
        return 2
    kind = argv[0]
    B, H, N, d = (int(x) for x in argv[1:5])
    causal = argv[5] in ("1", "true", "True")
    qk_std = float(argv[6])
    calls = int(argv[7]) if len(argv) > 7 else (4 if kind == "fwd" else 3)
    w = Workload("profile", B, H, H, N, d, causal, qk_std, 777)
    q, k, v, do = make_inputs(w, "cuda")
    if kind == "fwd":
        for _ in range(calls):
            binding.attention_forward(q, k, v, causal=causal, scale=w.scale)
    elif kind == "bwd":
        o, lse = binding.attention_forward(q, k, v, causal=causal, scale=w.scale)
        for _ in range(calls):
            binding.attention_backward(q, k, v, o, lse, do, causal=causal, scale=w.scale)
    else:
        print(__doc__)
        return 2
    torch.cuda.synchronize()
    status = binding.fa_device_status()
    if status != binding.FA_OK:
        print("device status", status)
        return 1
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
