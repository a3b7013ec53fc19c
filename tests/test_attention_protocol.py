"""CPU model of the barrier schedule of the persistent six-deep-ring attention
kernel (attn_block_tc_persistent_kernel): the TMA producer, the MMA issuer and
four softmax warps, with TMA completions in any order and tensor-core commits
completing in issue order, interleaved at random.  Every wait is written as
in the kernel — the phase it expects follows from the tile counter carried
across items (ring stage g % 6, S/P buffer g % 2) or from the item count — and
the model checks that all roles finish (no deadlock) and that no wait ever
finds its barrier two or more phases past the expected one (an mbarrier
parity wait could not tell those apart).

The model follows the kernel's order of operations; it does not execute the
kernel's code (GPU parity covers that)."""

from __future__ import annotations

import random

import pytest

ST = 6   # K/V ring depth of the persistent kernel


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def passed(bar, k):
    """The wait for phase k (k = -1: the phase before the first), checked
    against what an mbarrier parity wait answers: true when the barrier's
    current phase has the other parity.  The two agree only while the barrier
    is at phase k or k + 1."""
    ideal = bar.done > k
    parity = (bar.done & 1) != (k & 1)
    assert ideal == parity, f"{bar.done} phases done while waiting for phase {k}"
    return ideal


def run(tiles_per_item, seed):
    rnd = random.Random(seed)
    kv_full = [Bar(1) for _ in range(ST)]
    kv_empty = [Bar(1) for _ in range(ST)]
    s_full = [Bar(1) for _ in range(2)]
    s_empty = [Bar(4) for _ in range(2)]
    p_full = [Bar(4) for _ in range(2)]
    o_ready, q_full, o_final, q_empty = Bar(1), Bar(4), Bar(1), Bar(1)
    pipe, tma = [], []                   # in-order MMA commits; outstanding TMA
    live = [n for n in tiles_per_item if n > 0]   # items without keys are skipped

    def producer():
        g = 0
        for n in live:
            for _ in range(n):
                while not passed(kv_empty[g % ST], g // ST - 1):
                    yield
                tma.append(kv_full[g % ST])
                g += 1
                yield

    def mma():
        g = 0
        for idx, n in enumerate(live):
            while not passed(q_full, idx):
                yield
            g0 = g

            def ready(t):
                gt = g0 + t
                return passed(kv_full[gt % ST], gt // ST) and passed(s_empty[gt & 1],
                                                                    (gt >> 1) - 1)

            def issue_qk(t):
                pipe.append(s_full[(g0 + t) & 1])
                if t == n - 1:
                    pipe.append(q_empty)

            while not ready(0):
                yield
            issue_qk(0)
            for t in range(n):
                gt = g0 + t
                first = t + 1 < n and ready(t + 1)
                if first:
                    issue_qk(t + 1)
                while not passed(p_full[gt & 1], gt >> 1):
                    yield
                pipe.extend([kv_empty[gt % ST], o_ready] + ([o_final] if t + 1 == n else []))
                if not first and t + 1 < n:
                    while not ready(t + 1):
                        yield
                    issue_qk(t + 1)
                yield
            g += n

    def softmax_warp():
        g = 0
        if live:
            q_full.arrive()
        for idx, n in enumerate(live):
            for t in range(n):
                gt = g + t
                while not passed(s_full[gt & 1], gt >> 1):
                    yield
                s_empty[gt & 1].arrive()
                yield
                if t > 0 and rnd.random() < 0.3:       # an O rescale
                    while not passed(o_ready, gt - 1):
                        yield
                if gt > 0:                              # the one P buffer is free
                    while not passed(o_ready, gt - 1):
                        yield
                p_full[gt & 1].arrive()
                yield
            g += n
            if idx + 1 < len(live):                     # next item's Q
                while not passed(q_empty, idx):
                    yield
                q_full.arrive()
            while not passed(o_final, idx):             # this item's output
                yield
            yield

    roles = [producer(), mma()] + [softmax_warp() for _ in range(4)]
    alive = list(range(len(roles)))
    for _ in range(500000):
        if not (alive or pipe or tma):
            return
        x = rnd.random()
        if pipe and x < 0.2:
            pipe.pop(0).arrive()
        elif tma and x < 0.4:
            tma.pop(rnd.randrange(len(tma))).arrive()
        elif alive:
            i = rnd.choice(alive)
            try:
                next(roles[i])
            except StopIteration:
                alive.remove(i)
    raise AssertionError("the roles did not finish: deadlock")


@pytest.mark.parametrize("seed", range(4))
def test_persistent_schedule_finishes_without_ambiguous_waits(seed):
    rng = random.Random(seed)
    for trial in range(150):
        items = [rng.choice([0, 0, 1, 2, 3, 5, 7, 12, 13])
                 for _ in range(rng.randint(1, 6))]
        run(items, seed * 1000 + trial)


def test_parity_wait_flags_a_barrier_two_phases_ahead():
    """The checker itself: a wait whose barrier is two phases past the
    expected one is reported (an mbarrier parity wait would pass it wrongly)."""
    b = Bar(1)
    for _ in range(3):
        b.arrive()
    assert passed(b, 2) is True
    with pytest.raises(AssertionError):
        passed(b, 1)          # two phases behind: the parity wait would not pass
    with pytest.raises(AssertionError):
        passed(b, 4)          # one phase ahead: the parity wait would pass early
