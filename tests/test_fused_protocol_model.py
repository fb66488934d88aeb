"""A randomized model of the fused decode + matmul kernel's stage protocol.

The kernel (csrc/qamw_decode_gemm.cu) hands its stages over through
mbarriers whose waits test only the parity of a phase. Such a wait is right
only if the waiter is never two phases behind or ahead of the barrier. This
model runs the kernel's roles as coroutines in a random interleaving, with
every barrier counted as the hardware counts it (arrivals and transaction
bytes), and checks that:
- every wait sees the phase it means;
- no phase gets more arrivals than its count;
- every stage holds the unit its consumer expects when the wait passes.

Modelled roles:
- the word-copy warp: unit i into word stage i % SW;
- the activation-copy warp: unit i into stage i % SA, bytes on the operand
  stage's full barrier;
- 2 decode groups of 8 warps: unit i in group i % 2;
- 1 or 2 MMA issuers, each committing to the stage's empty barrier;
- the copies landing and the MMAs completing in any order the hardware
  allows (commits in issue order per issuer).
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._maybe_flip()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0
        self._maybe_flip()

    def _maybe_flip(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):   # try_wait.parity: the phase with this parity has completed
        return (self.phase & 1) != parity


def run(units, SA, SW, n_issuers, seed, shared_stage=False):
    rnd = random.Random(seed)
    groups, wpg = 2, 8
    full_w = [Bar(1) for _ in range(SW)]
    empty_w = [Bar(wpg) for _ in range(SW)]
    full_a = [Bar(wpg + 1) for _ in range(SA)]          # the group's warps + the activation warp
    empty_a = [Bar(n_issuers) for _ in range(SA)]       # one commit per MMA issuer
    words = [None] * SW
    acts = [None] * SA
    tiles = [[None] * wpg for _ in range(SA)]
    done_by = [[None] * n_issuers for _ in range(SA)]   # last unit each issuer finished per stage
    landing, commits = [], []

    def word_warp():
        for i in range(units):
            s = i % SW
            if i >= SW:
                while not empty_w[s].done(((i // SW) - 1) & 1):
                    yield
            full_w[s].arrive_expect_tx(1)
            landing.append(("w", s, i))
            yield

    def act_warp():
        sx, px = 0, 0
        for i in range(units):
            if i >= SA:
                while not empty_a[sx].done(px ^ 1):
                    yield
                assert all(d == i - SA for d in done_by[sx])
            full_a[sx].arrive_expect_tx(1)
            landing.append(("x", sx, i))
            yield
            sx += 1
            if sx == SA:
                sx, px = 0, px ^ 1

    def decode_warp(grp, w):
        i, sw, qw, qa = grp, grp, 0, 0
        st = 0 if shared_stage else grp   # the operand stage this group fills (a planted mistake: 0 for both)
        while i < units:
            while not full_w[sw].done(qw & 1):
                yield
            assert words[sw] == i
            yield
            empty_w[sw].arrive()                        # words in registers
            if qa > 0:
                while not empty_a[st].done((qa & 1) ^ 1):
                    yield
            assert all(d == i - SA for d in done_by[st]) if i >= SA else True
            yield
            tiles[st][w] = i
            full_a[st].arrive()
            i += groups
            qa += 1
            sw += groups
            if sw >= SW:
                sw, qw = sw - SW, qw + 1

    def mma_warp(mi):
        sa, pa = 0, 0
        for i in range(units):
            while not full_a[sa].done(pa):
                yield
            assert all(t == i for t in tiles[sa]) and acts[sa] == i
            commits.append((mi, sa, i))
            yield
            sa += 1
            if sa == SA:
                sa, pa = 0, pa ^ 1

    roles = [word_warp(), act_warp()] + [mma_warp(m) for m in range(n_issuers)]
    roles += [decode_warp(g, w) for g in range(groups) for w in range(wpg)]
    steps = 0
    while roles or landing or commits:
        steps += 1
        assert steps < 2_000_000, "no progress: a wait never passes"
        r = rnd.random()
        if landing and r < 0.2:
            kind, s, i = landing.pop(rnd.randrange(len(landing)))
            if kind == "w":
                words[s] = i
                full_w[s].complete_tx(1)
            else:
                acts[s] = i
                full_a[s].complete_tx(1)
            continue
        if commits and r < 0.35:
            j = rnd.randrange(len(commits))
            mi, s, i = commits[j]
            if any(c[0] == mi and c[2] < i for c in commits):
                continue                                  # an issuer's commits complete in order
            commits.pop(j)
            done_by[s][mi] = i
            empty_a[s].arrive()
            continue
        if not roles:
            continue
        role = rnd.choice(roles)
        try:
            next(role)
        except StopIteration:
            roles.remove(role)


@pytest.mark.parametrize("SW", [2, 4, 8])
@pytest.mark.parametrize("n_issuers", [1, 2])
def test_stage_protocol_has_no_parity_aliasing(SW, n_issuers):
    for units in (1, 2, 3, 5, 8, 13, 29):
        for seed in range(6):
            run(units, 2, SW, n_issuers, seed)


def test_the_model_catches_two_groups_on_one_stage():
    """A planted mistake: both decode groups fill operand stage 0. The model
    must fail (a wrong tile under a passed wait, an over-arrival, or a wait
    that never passes), or it would not be checking anything."""
    failures = 0
    for seed in range(6):
        try:
            run(8, 2, 4, 1, seed, shared_stage=True)
        except AssertionError:
            failures += 1
    assert failures == 6
