"""Model check of the forward kernel's mbarrier protocol (CPU only).

The forward (attn_fwd.cu) runs three roles per CTA over the CTA's item sequence: a
TMA producer (Q per item into one of kQBufs buffers, K/V tiles into a ring), an MMA
issuer (the item's Q copied into tensor memory before its first score product, which
frees the shared-memory Q buffer; score products one (d = 64, two CTAs per SM) or two
(d = 128) key tiles ahead of the P V products, S buffer g mod the buffer count for the
CTA's g-th key tile) and the softmax warps (one row per thread, every key tile in
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


def simulate(items, d, causal, n_kv, rescale, item_relative_rescale=False, seed=None,
             rescale_every=1, s_bufs=None):
    """items: query-tile index of each of the CTA's items.  Returns (finished, errors).
    With rescale, the softmax rescales O (waiting for the previous tile's P V) on every
    rescale_every-th key tile of the CTA, past an item's first.

    Tensor-core work is modelled as an in-order pipe: the MMA role issues products and
    commits, and a separate pipe role completes them one at a time (a commit arrives
    once every product issued before it has completed).  With seed None every role
    runs as far as it can in a fixed order; with a seed the next role to take one step
    (the pipe included) is drawn at random, which reaches schedules where the pipe
    lags far behind the MMA issuer.  Planted mistakes for the sensitivity checks:
    item_relative_rescale names the rescale's P V phase by the tile's index within its
    item; s_bufs = 3 runs the score products three tiles ahead with the same single
    P V-done barrier (the softmax's wait for P V(g-1) can then be two phases ahead)."""
    import collections
    import random
    # d = 64: two CTAs per SM, each with one S buffer and a two-stage K/V ring
    q_bufs, stages, s_bufs_kernel = (2, 2, 1) if d == 64 else (1, 3, 2)
    s_bufs = s_bufs or s_bufs_kernel
    bars = {}
    for b in range(2):
        for name in ("q_full", "q_empty"):
            bars[f"{name}{b}"] = Bar(1)
    for b in range(s_bufs):
        bars[f"s_full{b}"], bars[f"p_full{b}"] = Bar(1), Bar(4)
    for s in range(stages):
        for name in ("k_full", "v_full", "kv_empty"):
            bars[f"{name}{s}"] = Bar(1)
    bars["pv_done"], bars["o_done"], bars["o_free"] = Bar(1), Bar(1), Bar(4)
    tiles = [qt + 1 if causal else n_kv for qt in items]
    seq = [(it, n) for it in range(len(items)) for n in range(tiles[it])]
    pipe = collections.deque()   # commits in issue order

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
        order = [("s", g) for g in range(min(s_bufs, len(seq)))]
        for g in range(len(seq)):
            order.append(("pv", g))
            if g + s_bufs < len(seq):
                order.append(("s", g + s_bufs))
        for kind, g in order:
            item, n = seq[g]
            st, qb, sb = g % stages, item % q_bufs, g % s_bufs
            if kind == "s":
                if n == 0:
                    yield f"q_full{qb}", item // q_bufs
                    pipe.append(f"q_empty{qb}")    # Q copied to tensor memory
                yield f"k_full{st}", g // stages
                if g >= s_bufs:
                    yield "pv_done", g - s_bufs
                pipe.append(f"s_full{sb}")
            else:
                yield f"p_full{sb}", g // s_bufs
                yield f"v_full{st}", g // stages
                if n == 0 and item > 0:
                    yield "o_free", item - 1
                pipe.append("pv_done")
                pipe.append(f"kv_empty{st}")
                if n == tiles[item] - 1:
                    pipe.append("o_done")

    def softmax():
        g = 0
        for item in range(len(items)):
            for n in range(tiles[item]):
                yield f"s_full{g % s_bufs}", g // s_bufs
                if rescale and n > 0 and g % rescale_every == 0:
                    yield "pv_done", (n - 1) if item_relative_rescale else g - 1
                for _ in range(4):
                    bars[f"p_full{g % s_bufs}"].arrive()
                g += 1
            yield "o_done", item
            for _ in range(4):
                bars["o_free"].arrive()

    roles = [producer(), mma(), softmax()]
    waiting = [None] * len(roles)
    finished = [False] * len(roles)
    errors = []

    def ready(i):
        """Checks role i's pending wait (recording a wrong pass); True if it may step."""
        if finished[i]:
            return False
        if waiting[i] is None:
            return True
        name, phase = waiting[i]
        b = bars[name]
        passes = (b.done & 1) != (phase & 1)   # what the hardware checks
        if passes != (b.done > phase) or b.done > phase + 1:
            errors.append((i, name, phase, b.done))
        return passes

    def step(i):
        try:
            waiting[i] = next(roles[i])
        except StopIteration:
            finished[i] = True

    if seed is None:
        progress = True
        while progress:
            progress = False
            while pipe:
                bars[pipe.popleft()].arrive()
                progress = True
            for i in range(len(roles)):
                while ready(i):
                    step(i)
                    progress = True
    else:
        rng = random.Random(seed)
        while True:
            choices = [i for i in range(len(roles)) if ready(i)]
            if pipe:
                choices.append(-1)
            if not choices:
                break
            i = rng.choice(choices)
            if i < 0:
                bars[pipe.popleft()].arrive()
            else:
                step(i)
    return all(finished) and not pipe, errors


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


RANDOM_SHAPES = [(1, 2, 1000, 64, 1), (1, 2, 1000, 128, 1), (1, 3, 700, 128, 0), (2, 3, 600, 64, 0)]


@pytest.mark.parametrize("shape", RANDOM_SHAPES, ids=lambda s: "b{}h{}t{}d{}c{}".format(*s))
def test_forward_protocol_under_random_schedules(shape):
    """Random interleavings of the roles and of the tensor pipe's completions (the
    pipe may lag the MMA issuer by many products), several CTAs' item sequences."""
    B, H, T, d, causal = shape
    BH, nq = B * H, -(-T // 128)
    n_items = BH * nq
    n_ctas = min(n_items, SMS)
    for b in range(0, n_ctas, max(1, n_ctas // 4)):
        items = cta_items(b, n_ctas, n_items, BH, nq)
        for seed in range(12):
            ok, errors = simulate(items, d, causal, nq, True, seed=seed,
                                  rescale_every=1 + seed % 4)
            assert ok and not errors, (b, seed, errors[:2])


def test_random_schedules_catch_three_buffers_on_one_pv_barrier():
    """Sensitivity: with the score products three tiles ahead (three S buffers) and the
    same single P V-done barrier, the pipe can still be on P V(g-2) when the softmax of
    tile g waits for P V(g-1); random schedules flag it, the kernel's two buffers not."""
    bad = good = 0
    for seed in range(40):
        _, errors = simulate([7, 6, 5], 128, 1, 8, True, seed=seed, rescale_every=3, s_bufs=3)
        bad += bool(errors)
        ok, errors = simulate([7, 6, 5], 128, 1, 8, True, seed=seed, rescale_every=3)
        good += ok and not errors
    assert bad > 0 and good == 40
