"""Model check of the dK/dV kernel's mbarrier protocol (CPU only).

The dK/dV kernel (attn_bwd.cu) runs five roles per CTA over the CTA's item sequence
(an item is one (head, key tile); its steps are the query tiles it meets): a TMA
producer (K, V per item; Q with its row statistics and dO per step, in rings), an MMA
issuer (S^T, dP^T, dV, dK, dQ per step in a fixed order), the compute warps (P^T and
dS^T), the drain warps (dQ out of tensor memory, staged, reduce-added; the item's dK,
dV at its end), all counting steps across items.  This test restates each role's
waits and arrivals for the four configurations the kernel instantiates (head
dimension 64 / 128, default / precise mode) and runs them against every CTA's item
sequence of several workloads.  Tensor-core work completes through an in-order pipe
that runs as a role of its own, and TMA loads complete in any order; with a seed the
roles, the pipe and the loads are stepped in random order.  Every parity wait must
resolve to the phase it is meant for (never two phases away from the barrier) and
every role must finish."""
import collections
import random

import pytest

SMS = 148


class Bar:
    def __init__(self, count):
        self.count, self.arrivals, self.done = count, 0, 0

    def arrive(self):
        self.arrivals += 1
        if self.arrivals == self.count:
            self.arrivals = 0
            self.done += 1


def config(d, precise):
    """The kernel's BwdCfg choices that shape the protocol."""
    stage_own = not precise
    return dict(
        SQ=3 if (d == 64 and not precise) else 2,   # Q stages
        SD=1 if d == 128 else 2,                    # dO stages
        p_alias_s=not (d == 64 and not precise),    # P^T over S^T
        separate_dq=d == 64,                        # dQ has tensor-memory columns of its own
        stage_own=stage_own,                        # dQ staging buffer of its own
        stage_in_q=precise and d == 128,            # dQ staged in Q's stage
    )


def simulate(steps, d, precise, seed=None, q_empty_count=None):
    """steps: number of query-tile steps of each of the CTA's items.  Returns
    (finished, errors).  q_empty_count overrides the Q-empty barrier's arrival count
    (a planted mistake for the sensitivity check)."""
    c = config(d, precise)
    SQ, SD = c["SQ"], c["SD"]
    bars = collections.defaultdict(lambda: None)

    def mk(name, count):
        bars[name] = Bar(count)

    for s in range(3):
        mk(f"q_full{s}", 1)
        mk(f"q_empty{s}", q_empty_count or (2 if c["stage_in_q"] else 1))
    for s in range(2):
        mk(f"do_full{s}", 1)
        mk(f"do_empty{s}", 1)
    mk("kv_full", 1)
    mk("kv_empty", 1)
    for name, count in (("s_full", 1), ("s_free", 8), ("dp_full", 1), ("p_full", 8),
                        ("p_free", 1), ("ds_full", 8), ("ds_free", 1), ("dq_full", 1),
                        ("dq_free", 4), ("stage_done", 1), ("acc_done", 1), ("acc_free", 4)):
        mk(name, count)
    mk("always", 1)              # a wait that always passes: a point where the role may pause
    pipe = collections.deque()   # tensor-core commits, in issue order
    loads = []                   # TMA loads in flight (complete in any order)
    n_items = len(steps)

    def producer():
        g = 0
        for r in range(n_items):
            if r > 0:
                yield "kv_empty", r - 1
            loads.append("kv_full")
            for _ in range(steps[r]):
                sq, uq = g % SQ, g // SQ
                if uq:
                    yield f"q_empty{sq}", uq - 1
                loads.append(f"q_full{sq}")
                sd, ud = g % SD, g // SD
                if ud:
                    yield f"do_empty{sd}", ud - 1
                loads.append(f"do_full{sd}")
                g += 1

    def mma():
        if n_items == 0:
            return
        yield "kv_full", 0
        yield "q_full0", 0
        pipe.append("s_full")
        yield "do_full0", 0
        pipe.append("dp_full")
        g = 0
        for r in range(n_items):
            have_next = r + 1 < n_items
            for n in range(steps[r]):
                last = n + 1 == steps[r]
                next_step = not last or have_next
                s_late = c["stage_in_q"] or last

                def issue_s():
                    if last:
                        yield "kv_full", r + 1
                    yield f"q_full{(g + 1) % SQ}", (g + 1) // SQ
                    pipe.append("s_full")

                def s_cols_free():
                    yield ("p_free" if c["p_alias_s"] else "s_free"), g

                if not c["p_alias_s"] and next_step and not s_late:
                    yield from s_cols_free()
                    yield from issue_s()
                yield "p_full", g
                if n == 0 and r > 0:
                    yield "acc_free", r - 1
                pipe.append("p_free")                 # dV_g
                pipe.append(f"do_empty{g % SD}")
                if c["p_alias_s"] and next_step and not s_late:
                    yield from s_cols_free()
                    yield from issue_s()
                yield "ds_full", g
                if c["separate_dq"] and g > 0:
                    yield "dq_free", g - 1
                pipe.append("dq_full")                # dK_g, dQ_g
                pipe.append("ds_free")
                pipe.append(f"q_empty{g % SQ}")
                if last:
                    pipe.append("acc_done")
                    pipe.append("kv_empty")
                if s_late and next_step:
                    yield from s_cols_free()
                    yield from issue_s()
                if next_step:
                    if not c["separate_dq"]:
                        yield "dq_free", g
                    yield f"do_full{(g + 1) % SD}", (g + 1) // SD
                    pipe.append("dp_full")            # dP_{g+1}
                g += 1

    def compute(warps):
        g = 0
        for r in range(n_items):
            for _ in range(steps[r]):
                sq = g % SQ
                yield "s_full", g
                if not c["p_alias_s"]:
                    for _ in range(warps):
                        bars["s_free"].arrive()
                yield f"q_full{sq}", g // SQ
                if not c["p_alias_s"] and g > 0:
                    yield "p_free", g - 1
                for _ in range(warps):
                    bars["p_full"].arrive()
                yield "dp_full", g
                staged = not c["stage_own"] and not c["stage_in_q"]
                if g > 0:
                    yield ("stage_done" if staged else "ds_free"), g - 1
                for _ in range(warps):
                    bars["ds_full"].arrive()
                g += 1

    def drain():
        g = 0
        for r in range(n_items):
            for _ in range(steps[r]):
                yield "dq_full", g
                for _ in range(4):
                    bars["dq_free"].arrive()
                # staging rounds and their reduces (the warps' own handshake)
                yield "always", -1
                if not c["stage_own"]:
                    bars[f"q_empty{g % SQ}" if c["stage_in_q"] else "stage_done"].arrive()
                g += 1
            yield "acc_done", r
            for _ in range(4):
                bars["acc_free"].arrive()

    roles = [producer(), mma(), drain()] + [compute(1) for _ in range(8)]
    waiting = [None] * len(roles)
    finished = [False] * len(roles)
    errors = []

    def ready(i):
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
            while pipe or loads:
                bars[(pipe or loads).popleft() if pipe else loads.pop(0)].arrive()
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
            if loads:
                choices.append(-2)
            if not choices:
                break
            i = rng.choice(choices)
            if i == -1:
                bars[pipe.popleft()].arrive()
            elif i == -2:
                bars[loads.pop(rng.randrange(len(loads)))].arrive()
            else:
                step(i)
    return all(finished) and not pipe and not loads, errors


def cta_steps(b, n_ctas, n_items, BH, nq, causal):
    """The kernel's item_of (heaviest first, zigzag) and each item's step count."""
    out, r = [], 0
    while True:
        k = r * n_ctas + ((n_ctas - 1 - b) if r & 1 else b)
        if k >= n_items:
            return out
        kt = k // BH
        out.append(nq - (kt if causal else 0))
        r += 1


SHAPES = [(8, 12, 1024, 1), (4, 16, 2048, 1), (2, 16, 4096, 1), (1, 32, 8000, 1),
          (4, 16, 1024, 0), (2, 40, 1000, 1), (1, 2, 129, 1), (1, 2, 1, 1)]


def ctas_of(shape):
    B, H, T, causal = shape
    BH, nq = B * H, -(-T // 128)
    n_items = BH * nq
    n_ctas = min(n_items, SMS)
    return [cta_steps(b, n_ctas, n_items, BH, nq, causal) for b in range(n_ctas)]


@pytest.mark.parametrize("d,precise", [(64, False), (64, True), (128, False), (128, True)])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}h{}t{}c{}".format(*s))
def test_backward_protocol_finishes_without_aliased_waits(shape, d, precise):
    for steps in ctas_of(shape):
        ok, errors = simulate(steps, d, precise)
        assert ok and not errors, (steps[:4], errors[:2])


@pytest.mark.parametrize("d,precise", [(64, False), (64, True), (128, False), (128, True)])
def test_backward_protocol_under_random_schedules(d, precise):
    """Random interleavings of the roles, the tensor pipe's completions and the TMA
    loads, on several CTAs' item sequences with two to four items each."""
    for shape in ((2, 16, 1024, 1), (4, 16, 1024, 0), (2, 40, 1000, 1)):
        ctas = ctas_of(shape)
        for b in range(0, len(ctas), max(1, len(ctas) // 3)):
            for seed in range(6):
                ok, errors = simulate(ctas[b], d, precise, seed=seed)
                assert ok and not errors, (shape, b, seed, errors[:2])


def test_model_catches_a_single_arrival_q_empty():
    """Sensitivity: with dQ staged in Q's stage two parties release the stage (the MMA
    commit and the drain); a Q-empty barrier that counts one arrival lets the
    producer's parity waits run ahead, which the model flags."""
    flagged = False
    for seed in range(20):
        ok, errors = simulate([8, 7, 6], 128, True, seed=seed, q_empty_count=1)
        flagged |= bool(errors) or not ok
    assert flagged
