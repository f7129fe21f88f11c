"""Load balance of the persistent kernels' work assignment (CPU only).

Both kernels number their work items heaviest first, the backward as (key tile
kt = k / BH, head k % BH) with n_qtiles - kt steps, the forward as (query tile
qt = n_qtiles - 1 - k / BH, head k % BH) with qt + 1 key tiles, and deal them to
min(items, 148) CTAs in a zigzag: CTA b takes item r * n + b in even rounds r and
r * n + (n - 1 - b) in odd ones.  This restates that rule (the kernels' item_of) and
checks two properties on every workload: each item is dealt exactly once, and the
longest CTA is as short as greedy longest-processing-time scheduling makes it."""
import heapq

import pytest

from causal_attention_fwd_attn_b200 import workloads as wl

SMS = 148


def zigzag(n_items, n_ctas):
    out = []
    for b in range(n_ctas):
        mine, r = [], 0
        while True:
            k = r * n_ctas + ((n_ctas - 1 - b) if r & 1 else b)
            if k >= n_items:
                break
            mine.append(k)
            r += 1
        out.append(mine)
    return out


def lpt_makespan(costs, n):
    loads = [0] * n
    for c in sorted(costs, reverse=True):
        heapq.heapreplace(loads, loads[0] + c)
    return max(loads)


@pytest.mark.parametrize("w", wl.WORKLOADS[1:], ids=lambda w: w.name)
@pytest.mark.parametrize("kernel", ["fwd", "bwd"])
def test_zigzag_deal_matches_lpt(w, kernel):
    BH, nq = w.B * w.H, -(-w.T // 128)
    n_items = BH * nq
    n_ctas = min(n_items, SMS)
    if kernel == "bwd":
        cost = lambda k: nq - k // BH            # key tile kt sees query tiles kt .. nq-1
    else:
        cost = lambda k: (nq - 1 - k // BH) + 1  # query tile qt sees key tiles 0 .. qt
    dealt = zigzag(n_items, n_ctas)
    flat = sorted(k for mine in dealt for k in mine)
    assert flat == list(range(n_items))
    makespan = max(sum(cost(k) for k in mine) for mine in dealt)
    assert makespan == lpt_makespan([cost(k) for k in range(n_items)], n_ctas)
    ideal = sum(cost(k) for k in range(n_items)) / n_ctas
    assert makespan < ideal + 3
