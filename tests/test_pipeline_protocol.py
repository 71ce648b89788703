"""The mbarrier protocol of the prefill GEMM engine (prefill.cuh, pf_gemm),
model-checked on the CPU over random interleavings: producer warps, two MMA
issuers and the token-tile loader, with the kernel's stage and slot counts.

An mbarrier phase wait by parity is only sound if the barrier can never be
two phases ahead of the waiter (the parity would read as "not done" and the
wait would spin until its time limit), and the roles must never wait on each
other in a cycle.  Each role below takes exactly the waits and arrivals the
kernel does, in the same order."""
import random

import pytest

STAGES, BSLOTS, ISSUERS = 3, 4, 2  # kPfStages, kPfBSlots, kPfIssuers


class Bar:
    def __init__(self, count):
        self.count, self.arrived, self.done = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived, self.done = 0, self.done + 1

    def ready(self, phase):
        """Wait for phase `phase` (0, 1, 2, ... of this barrier)."""
        assert self.done <= phase + 1, "barrier two phases ahead of its waiter"
        return self.done > phase


def run(nchunks, warps, seed, loader_waits=True, producers_wait=True):
    rnd = random.Random(seed)
    full = [Bar(warps) for _ in range(STAGES)]
    empty = [Bar(ISSUERS) for _ in range(STAGES)]
    bfull = [Bar(1) for _ in range(BSLOTS)]
    bempty = [Bar(ISSUERS) for _ in range(BSLOTS)]
    prod = [0] * warps           # next chunk of each producer warp
    iss = [0] * ISSUERS          # next chunk of each issuer
    load = 0                     # next chunk of the loader
    inflight = []                # async completions: MMA commits and TMA bytes
    for _ in range(200000):
        moves = []
        for w in range(warps):
            g = prod[w]
            if g < nchunks and (g < STAGES or not producers_wait or empty[g % STAGES].ready(g // STAGES - 1)):
                moves.append(("p", w))
        for q in range(ISSUERS):
            g = iss[q]
            if g < nchunks and bfull[g % BSLOTS].ready(g // BSLOTS) and full[g % STAGES].ready(g // STAGES):
                moves.append(("i", q))
        if load < nchunks and (load < BSLOTS or not loader_waits or bempty[load % BSLOTS].ready(load // BSLOTS - 1)):
            moves.append(("l", 0))
        if inflight:
            moves.append(("c", 0))
        if not moves:
            done = all(p == nchunks for p in prod) and all(i == nchunks for i in iss) and load == nchunks
            assert done, "deadlock"
            return
        kind, who = rnd.choice(moves)
        if kind == "p":
            g = prod[who]
            full[g % STAGES].arrive()
            prod[who] += 1
        elif kind == "i":
            g = iss[who]
            inflight.append(("mma", g))
            iss[who] += 1
        elif kind == "l":
            inflight.append(("tma", load))
            load += 1
        else:
            what, g = inflight.pop(rnd.randrange(len(inflight)) if rnd.random() < 0.5 else 0)
            if what == "mma":
                empty[g % STAGES].arrive()
                bempty[g % BSLOTS].arrive()
            else:
                bfull[g % BSLOTS].arrive()
    raise AssertionError("did not finish")


@pytest.mark.parametrize("nchunks", [1, 2, 3, 5, 8, 17, 40])
def test_prefill_pipeline_protocol(nchunks):
    for seed in range(60):
        run(nchunks, warps=3, seed=seed)


@pytest.mark.parametrize("broken", ["loader_waits", "producers_wait"])
def test_protocol_check_is_not_vacuous(broken):
    """Dropping a wait the kernel takes (the loader's on `bempty`, or the
    producers' on `empty`) lets a barrier run two phases ahead of a waiter:
    the model must catch it."""
    caught = False
    for seed in range(300):
        try:
            run(24, warps=2, seed=seed, **{broken: False})
        except AssertionError:
            caught = True
            break
    assert caught
