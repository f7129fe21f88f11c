"""Model check of the forward kernel's mbarrier protocol (CPU only).

The forward (attn_fwd.cu) runs three roles per CTA over the CTA's item sequence: a
TMA producer (Q per item into one of kQBufs buffers, K/V tiles into a ring), an MMA
issuer (the item's Q copied into tensor memory before its first score product, which
frees the shared-memory Q buffer; score products two key tiles ahead of the P V
products, S buffer g & 1 for the CTA's g-th key tile) and the softmax warps (one row per thread, every key tile in
order, the item's epilogue at its end).  Every wait is an mbarrier parity wait, which
is only sound if the waiter is never two phases ahead of the barrier (the parity of
phase k + 2 equals that of phase k).  This test restates each role's sequence of
waits and arrivals, runs them against every CTA's item sequence of every workload and
several edge shapes, and checks that all roles finish and that every parity wait
resolves to the phase it is meant for.  MMA completions are modelled as immediate;
the soundness argument for each barrier does not depend on timing."""
import pytest

from causal_attention_fwd_attn_b200 import workloads as wl

SMS = 148


class Bar:
    def __init__(self, count):
        self.count, self.arrivals, self.done = count, 0, 0

    def arrive(self):
        self.arrivals += 1
        if self.arrivals == self.count:
            self.arrivals = 0
            self.done += 1


def simulate(items, d, causal, n_kv, rescale, item_relative_rescale=False):
    """items: query-tile index of each of the CTA's items.  Returns (finished, errors).
    item_relative_rescale plants a plausible mistake for the sensitivity check: the
    rescale wait names the P V phase by the tile's index within its item."""
    q_bufs, stages = (2, 4) if d == 64 else (1, 3)
    bars = {}
    for b in range(2):
        for name, count in (("q_full", 1), ("q_empty", 1), ("s_full", 1), ("p_full", 4)):
            bars[f"{name}{b}"] = Bar(count)
    for s in range(stages):
        for name in ("k_full", "v_full", "kv_empty"):
            bars[f"{name}{s}"] = Bar(1)
    bars["pv_done"], bars["o_done"], bars["o_free"] = Bar(1), Bar(1), Bar(4)
    tiles = [qt + 1 if causal else n_kv for qt in items]
    seq = [(it, n) for it in range(len(items)) for n in range(tiles[it])]

    def producer():
        g = 0
        for item in range(len(items)):
            qb, use = item % q_bufs, item // q_bufs
            if use:
                yield f"q_empty{qb}", use - 1
            bars[f"q_full{qb}"].arrive()
            for _ in range(tiles[item]):
                st, u = g % stages, g // stages
                if u:
                    yield f"kv_empty{st}", u - 1
                bars[f"k_full{st}"].arrive()
                bars[f"v_full{st}"].arrive()
                g += 1

    def mma():
        order = [("s", g) for g in range(min(2, len(seq)))]
        for g in range(len(seq)):
            order.append(("pv", g))
            if g + 2 < len(seq):
                order.append(("s", g + 2))
        for kind, g in order:
            item, n = seq[g]
            st, qb = g % stages, item % q_bufs
            if kind == "s":
                if n == 0:
                    yield f"q_full{qb}", item // q_bufs
                    bars[f"q_empty{qb}"].arrive()    # Q copied to tensor memory
                yield f"k_full{st}", g // stages
                if g >= 2:
                    yield "pv_done", g - 2
                bars[f"s_full{g & 1}"].arrive()
            else:
                yield f"p_full{g & 1}", g >> 1
                yield f"v_full{st}", g // stages
                if n == 0 and item > 0:
                    yield "o_free", item - 1
                bars["pv_done"].arrive()
                bars[f"kv_empty{st}"].arrive()
                if n == tiles[item] - 1:
                    bars["o_done"].arrive()

    def softmax():
        g = 0
        for item in range(len(items)):
            for n in range(tiles[item]):
                yield f"s_full{g & 1}", g >> 1
                if rescale and n > 0:
                    yield "pv_done", (n - 1) if item_relative_rescale else g - 1
                for _ in range(4):
                    bars[f"p_full{g & 1}"].arrive()
                g += 1
            yield "o_done", item
            for _ in range(4):
                bars["o_free"].arrive()

    roles = [producer(), mma(), softmax()]
    waiting = [None] * len(roles)
    finished = [False] * len(roles)
    errors = []
    progress = True
    while progress:
        progress = False
        for i, role in enumerate(roles):
            while not finished[i]:
                if waiting[i] is not None:
                    name, phase = waiting[i]
                    b = bars[name]
                    passes = (b.done & 1) != (phase & 1)   # what the hardware checks
                    if passes != (b.done > phase) or b.done > phase + 1:
                        errors.append((i, name, phase, b.done))
                    if not passes:
                        break
                try:
                    waiting[i] = next(role)
                    progress = True
                except StopIteration:
                    finished[i] = True
    return all(finished), errors


def cta_items(b, n_ctas, n_items, BH, nq):
    """The kernel's item_of: heaviest first, dealt in a zigzag; the query tile of each."""
    out, r = [], 0
    while True:
        k = r * n_ctas + ((n_ctas - 1 - b) if r & 1 else b)
        if k >= n_items:
            return out
        out.append(nq - 1 - k // BH)
        r += 1


SHAPES = [(w.B, w.H, w.T, w.d, 1) for w in wl.WORKLOADS] + [
    (4, 16, 1024, 64, 0), (1, 2, 300, 128, 0), (3, 5, 257, 64, 1), (1, 2, 1, 64, 1),
    (1, 2, 129, 64, 0), (2, 40, 1000, 64, 1), (1, 1, 640, 128, 1)]


def run_all(shape, rescale, **kw):
    B, H, T, d, causal = shape
    BH, nq = B * H, -(-T // 128)
    n_items = BH * nq
    n_ctas = min(n_items, SMS)
    bad = []
    for b in range(n_ctas):
        ok, errors = simulate(cta_items(b, n_ctas, n_items, BH, nq), d, causal, nq, rescale, **kw)
        if not ok or errors:
            bad.append((b, ok, errors[:2]))
    return bad


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}h{}t{}d{}c{}".format(*s))
@pytest.mark.parametrize("rescale", [False, True])
def test_forward_protocol_finishes_without_aliased_waits(shape, rescale):
    assert run_all(shape, rescale) == []


def test_model_catches_a_misnamed_phase():
    """The model is sensitive: naming the rescale's P V phase by the tile's index within
    its item (instead of over the CTA's key tiles) is flagged on the GPT-2-small
    workload."""
    w = wl.WORKLOADS[1]
    assert run_all((w.B, w.H, w.T, w.d, 1), True, item_relative_rescale=True)
