"""The expert residency cache (host policy, moe_cache_*): a bounded number of
slots, the experts a token routes to are made resident, least recently used
slots are refilled first and never one the current token needs.  Checked
against a reference written independently below, on random and on the
decode-loop routing (27% of experts reused between consecutive tokens)."""
import numpy as np
import pytest

from quantised_expert_ffn_moe_b200 import moeq, synth


class RefCache:
    """Plain reference: a dict of resident experts with last-use times."""

    def __init__(self, n_experts, n_slots):
        self.n_slots = n_slots
        self.where = {}                    # expert -> slot
        self.last = [None] * n_slots       # slot -> last use time (None: empty)
        self.time = 0
        self.hits = self.misses = 0

    def plan(self, ids):
        self.time += 1
        for e in ids:
            if e in self.where:
                self.last[self.where[e]] = self.time
        slots, fills = [], []
        for e in ids:
            if e in self.where:
                self.hits += 1
            else:
                self.misses += 1
                empty = [s for s in range(self.n_slots) if self.last[s] is None]
                if empty:
                    s = empty[0]
                else:
                    free = [s for s in range(self.n_slots) if self.last[s] != self.time]
                    s = min(free, key=lambda t: (self.last[t], t))
                    old = [x for x, y in self.where.items() if y == s][0]
                    del self.where[old]
                self.where[e] = s
                self.last[s] = self.time
                fills.append((e, s))
            slots.append(self.where[e])
        return slots, fills


def _check_against_reference(n_experts, n_slots, seqs):
    c, r = moeq.ExpertCache(n_experts, n_slots), RefCache(n_experts, n_slots)
    resident = {}
    for ids in seqs:
        ids = [int(e) for e in ids]
        got = c.plan(ids)
        assert got == r.plan(ids)
        slots, fills = got
        assert len(set(slots)) == len(slots)          # distinct slots within a token
        for e, s in fills:                             # a refilled slot loses its old expert
            for x in [x for x, y in resident.items() if y == s]:
                assert x not in ids                     # never one this token needs
                del resident[x]
            resident[e] = s
        for e, s in zip(ids, slots):
            assert resident[e] == s
    assert c.stats() == (r.hits, r.misses)
    return c.stats()


@pytest.mark.parametrize("n_slots", [10, 11, 32, 200])
def test_random_routing_matches_reference(n_slots):
    rng = np.random.default_rng(n_slots)
    seqs = [rng.choice(512, size=10, replace=False) for _ in range(300)]
    _check_against_reference(512, n_slots, seqs)


def test_decode_loop_reuse_sets_the_hit_rate():
    """With as many slots as routed experts, the hit rate is the reuse
    between consecutive tokens (27% requested); more slots only add hits."""
    E, k, T = 512, 10, 2000
    _, sets = synth.repeat_logit_bias(E, k, T, 0.27, seed=3)
    hits, misses = _check_against_reference(E, k, sets)
    reuse = np.mean([len(set(sets[t]) & set(sets[t - 1])) / k for t in range(1, T)])
    assert hits == pytest.approx(reuse * k * (T - 1), abs=1)
    assert hits + misses == k * T
    more = _check_against_reference(E, 4 * k, sets)[0]
    assert more >= hits


def test_every_expert_resident_gives_only_hits_after_warmup():
    c = moeq.ExpertCache(16, 16)
    for e in range(16):
        c.plan([e])
    rng = np.random.default_rng(0)
    for _ in range(50):
        _, fills = c.plan([int(x) for x in rng.choice(16, size=4, replace=False)])
        assert fills == []
    assert c.stats() == (200, 16)


def test_bad_arguments_are_rejected():
    with pytest.raises(moeq.MoeError):
        moeq.ExpertCache(8, 9)
    with pytest.raises(moeq.MoeError):
        moeq.ExpertCache(0, 1)
    c = moeq.ExpertCache(8, 2)
    with pytest.raises(moeq.MoeError):
        c.plan([1, 2, 3])          # more ids than slots
    with pytest.raises(moeq.MoeError):
        c.plan([1, 1])             # repeated id
    with pytest.raises(moeq.MoeError):
        c.plan([8])                # out of range
    assert c.stats() == (0, 0)     # rejected calls change nothing
    assert c.plan([3, 5]) == ([0, 1], [(3, 0), (5, 1)])
