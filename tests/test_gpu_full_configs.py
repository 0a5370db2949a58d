"""GPU parity at the full sizes of the five reference workloads (C2 in both
masking modes), plus the d = 64 and ragged-length workloads, in the launch
configuration bench.py times.  The oracle computes sampled outputs one head at
a time: O and LSE for sampled query rows, dQ for the same rows and dK, dV for
sampled key rows (every query row contributes to those, so the oracle computes
the full probability columns).

The sampled (batch, kv head) units always include the first and the last unit
the persistent schedulers deal: the forward deals (batch 0, head 0) first
(with a causal mask, its last query tiles, the heaviest) and the last head of
the last batch entry last; the backward claims key tile 0 of (batch 0, kv
head 0) first and the last key tile band of (B-1, Hkv-1) last.  Two more
units are drawn at random (seeded), so at least four are checked per
workload wherever it has four.  Three more shapes give every CTA of the
persistent forward several work items (d = 64 and 128, causal with an odd
tile count and GQA, and a ragged d = 64 case)."""

import numpy as np
import pytest

from exact_attention_104_b200.workloads import WORKLOADS, Workload

from _parity import assert_within_tolerance, compare_sampled, run_gpu

pytestmark = pytest.mark.gpu


def sampled_units(w, seed):
    units = [(0, 0), (w.B - 1, w.Hkv - 1)]
    rng = np.random.default_rng(seed)
    total = w.B * w.Hkv
    while len(set(units)) < min(4, total):
        u = int(rng.integers(total))
        units.append((u // w.Hkv, u % w.Hkv))
    return sorted(set(units))


@pytest.mark.parametrize("name", list(WORKLOADS), ids=list(WORKLOADS))
def test_full_size_workload_sampled_parity(name):
    w = WORKLOADS[name]
    seed = sum(map(ord, name)) % 1000
    units = sampled_units(w, seed)
    assert (0, 0) in units and (w.B - 1, w.Hkv - 1) in units
    g = run_gpu(w)
    err = compare_sampled(w, g, units, n_rows=40, seed=seed)
    print(name, units, err)
    assert_within_tolerance(err)


# Several work items per CTA in every mode of the persistent forward: at
# d = 64 (one MMA warp per query tile) and d = 128, causal with an odd tile
# count (the last item of every head has no second tile, and the causal
# items start with the second tile's diagonal block), GQA 4:1.
MANY_ITEMS = [Workload(f"many_items_d{d}_causal", 4, 16, 4, 1920, d, True, 1.0, 4100 + d) for d in (64, 128)] + \
             [Workload("many_items_d64_ragged", 3, 16, 8, 1000, 64, False, 1.0, 4200)]


@pytest.mark.parametrize("w", MANY_ITEMS, ids=lambda w: w.name)
def test_many_items_per_cta_sampled_parity(w):
    units = sampled_units(w, 5)
    err = compare_sampled(w, run_gpu(w), units, n_rows=40, seed=5)
    print(w.name, units, err)
    assert_within_tolerance(err)
