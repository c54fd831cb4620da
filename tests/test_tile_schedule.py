"""Host logic of the bf16 step's static tile schedule (fdllm_plan_tile_schedule).

When the (row group, head) tiles of a step outnumber the SMs, the step runs
one persistent CTA per bin of this schedule, so the schedule must list every
tile exactly once (a missing tile leaves rows unattended, a repeated one
writes the cache twice) and should keep the bins' summed costs level. These
checks need no GPU: the packing is host code in the library.
"""
import heapq

import numpy as np
import pytest

import kv_cache_attention_flash_b200 as F
from kv_cache_attention_flash_b200 import _lib


def _loads(cost, n_heads, bin_start, tiles):
    return np.array([sum(cost[t // n_heads] for t in tiles[bin_start[i]:bin_start[i + 1]])
                     for i in range(len(bin_start) - 1)])


def _lpt_makespan(cost, n_heads, n_bins):
    items = sorted((c for c in cost for _ in range(n_heads)), reverse=True)
    heap = [(0.0, b) for b in range(n_bins)]
    for w in items:
        load, b = heapq.heappop(heap)
        heapq.heappush(heap, (load + w, b))
    return max(load for load, _ in heap)


def _cases():
    rng = np.random.default_rng(11)
    out = [
        # modelled per-group tile times of a 32-sequence divergent batch
        ([155.4, 141.0, 121.0, 112.4, 110.6, 107.5, 104.3, 98.0, 94.8, 91.7, 82.2, 79.1], 32, 148),
        ([100.0], 1, 1),
        ([5.0, 5.0, 5.0], 7, 160),            # more bins than tiles: some stay empty
        ([0.0, 0.0], 4, 3),                    # zero costs
    ]
    for _ in range(60):
        ng = int(rng.integers(1, 40))
        nh = int(rng.integers(1, 64))
        if ng * nh > 1024:
            continue
        P = int(rng.integers(1, 161))
        c = np.sort(rng.uniform(40, 350, ng))[::-1]
        if rng.random() < 0.3:
            c = np.round(c / 10) * 10          # many equal costs
        out.append((c.tolist(), nh, P))
    return out


@pytest.mark.parametrize("case", range(len(_cases())))
def test_schedule_is_a_partition_ordered_and_no_worse_than_lpt(case):
    cost, nh, P = _cases()[case]
    bin_start, tiles = F.fdllm_plan_tile_schedule(cost, nh, P)
    n = len(cost) * nh
    assert bin_start[0] == 0 and bin_start[-1] == n
    assert np.all(np.diff(bin_start) >= 0)
    assert sorted(tiles.tolist()) == list(range(n))
    for i in range(P):                          # costliest tile first within a bin
        c = [cost[t // nh] for t in tiles[bin_start[i]:bin_start[i + 1]]]
        assert c == sorted(c, reverse=True)
    loads = _loads(cost, nh, bin_start, tiles)
    lower = max(max(cost), sum(cost) * nh / P)
    assert loads.max() >= lower - 1e-9
    assert loads.max() <= _lpt_makespan(cost, nh, P) + 1e-9


def test_divergent_batch_is_near_level():
    cost = [155.4, 141.0, 121.0, 112.4, 110.6, 107.5, 104.3, 98.0, 94.8, 91.7, 82.2, 79.1]
    bin_start, tiles = F.fdllm_plan_tile_schedule(cost, 32, 148)
    loads = _loads(cost, 32, bin_start, tiles)
    assert loads.max() <= 1.05 * loads.mean()
    assert loads.max() < _lpt_makespan(cost, 32, 148) - 10.0   # level where LPT is not


def test_deterministic():
    cost = [90.0, 80.0, 80.0, 75.5, 60.0]
    a = F.fdllm_plan_tile_schedule(cost, 20, 37)
    b = F.fdllm_plan_tile_schedule(cost, 20, 37)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("args,status", [
    (([1.0], 1, 161), _lib.FDLLM_ERR_UNSUPPORTED),          # too many bins
    (([1.0] * 2, 513, 10), _lib.FDLLM_ERR_UNSUPPORTED),     # too many heads / tiles
    (([1.0] * 5, 250, 10), _lib.FDLLM_ERR_UNSUPPORTED),     # 1250 tiles
    (([-1.0], 4, 2), _lib.FDLLM_ERR_INVALID_ARG),
    (([float("nan")], 4, 2), _lib.FDLLM_ERR_INVALID_ARG),
    (([float("inf")], 4, 2), _lib.FDLLM_ERR_INVALID_ARG),
    (([1.0], 0, 2), _lib.FDLLM_ERR_INVALID_ARG),
    (([1.0], 4, 0), _lib.FDLLM_ERR_INVALID_ARG),
    (([], 4, 2), _lib.FDLLM_ERR_INVALID_ARG),
])
def test_rejects_out_of_range(args, status):
    with pytest.raises(F.FdllmError) as ei:
        F.fdllm_plan_tile_schedule(*args)
    assert ei.value.status == status
