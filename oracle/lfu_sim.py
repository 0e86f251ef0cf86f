"""Reference simulation of the per-layer 16-slot LFU expert cache.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.

Source: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
(blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": per token the CPU
checks the 8 selected ids against a 16-slot LFU cache of that layer; hits
reuse the resident buffer, misses fetch the expert blob.  The pages give no
more than that; the policy below is this library's reading of it:

  * counts live only while an expert is resident: insert -> 1, hit -> +1;
  * a step is one token's k ids at one layer; within a step hits are taken
    first, then misses, each in the step's order; a global tick advances by
    one per access and stamps the slot used;
  * a miss fills the lowest-index empty slot, else evicts, among slots not
    used by the current step, the one with the smallest (count, last tick,
    slot index);
  * a prefill chunk is split into steps: its distinct experts at that layer,
    those already resident first (ascending id), then the rest (ascending
    id), k at a time.

Every access is logged as (layer, step, expert, hit, slot); `step` counts
the steps of that layer from 0.

Lookahead prefetch (an option of this library, not of the pages, which
report speculative reads as tried and rejected): `prefetch(layer, P)` stages
up to P experts of a layer -- the non-resident ones with the most accesses so
far in the run (hits and misses; ties to the lower id), each into the slot a
miss would take (the victim rule above, slots taken by this prefetch
excluded), stopping at the first candidate whose victim slot holds an expert
with count >= the candidate's access total.  A prefetched expert enters with
count 0 and the tick advances; the prefetch is one more step of the layer
and each staged expert is logged with hit = 2.
"""
from __future__ import annotations


class LFUSim:
    def __init__(self, n_layers: int, n_slots: int):
        self.n_slots = n_slots
        self.expert = [[-1] * n_slots for _ in range(n_layers)]
        self.count = [[0] * n_slots for _ in range(n_layers)]
        self.last = [[0] * n_slots for _ in range(n_layers)]
        self.steps = [0] * n_layers
        self.tick = 0
        self.log = []
        self.freq = [dict() for _ in range(n_layers)]   # accesses per expert over the run

    def resident(self, layer: int):
        return {e for e in self.expert[layer] if e >= 0}

    def slot_of(self, layer: int, e: int) -> int:
        try:
            return self.expert[layer].index(e)
        except ValueError:
            return -1

    def step(self, layer: int, ids):
        """One step: ids are distinct experts. Returns {expert: slot}."""
        ids = [int(e) for e in ids]
        assert len(set(ids)) == len(ids), "ids of one step must be distinct"
        assert len(ids) <= self.n_slots
        st = self.steps[layer]
        self.steps[layer] += 1
        used = set()
        where = {}
        hits = [e for e in ids if self.slot_of(layer, e) >= 0]
        misses = [e for e in ids if self.slot_of(layer, e) < 0]
        for e in hits + misses:
            self.freq[layer][e] = self.freq[layer].get(e, 0) + 1
        for e in hits:
            s = self.slot_of(layer, e)
            self.tick += 1
            self.count[layer][s] += 1
            self.last[layer][s] = self.tick
            used.add(s)
            where[e] = s
            self.log.append((layer, st, e, 1, s))
        for e in misses:
            s = self._victim(layer, used)
            self.tick += 1
            self.expert[layer][s] = e
            self.count[layer][s] = 1
            self.last[layer][s] = self.tick
            used.add(s)
            where[e] = s
            self.log.append((layer, st, e, 0, s))
        return where

    def _victim(self, layer: int, used) -> int:
        ex = self.expert[layer]
        for s in range(self.n_slots):
            if ex[s] < 0:
                return s
        best = None
        for s in range(self.n_slots):
            if s in used:
                continue
            key = (self.count[layer][s], self.last[layer][s], s)
            if best is None or key < best:
                best = key
        return best[2]

    def prefetch(self, layer: int, P: int):
        """One lookahead prefetch of up to P experts; returns [(expert, slot)]."""
        if P <= 0:
            return []
        res = self.resident(layer)
        fr = self.freq[layer]
        cand = sorted((e for e in fr if fr[e] > 0 and e not in res), key=lambda e: (-fr[e], e))
        st = self.steps[layer]
        self.steps[layer] += 1
        used, out = set(), []
        for e in cand:
            if len(out) == P:
                break
            s = self._victim(layer, used)
            if self.expert[layer][s] >= 0 and self.count[layer][s] >= fr[e]:
                break
            self.tick += 1
            self.expert[layer][s] = e
            self.count[layer][s] = 0
            self.last[layer][s] = self.tick
            used.add(s)
            out.append((e, s))
            self.log.append((layer, st, e, 2, s))
        return out

    def chunk_steps(self, layer: int, distinct, width: int):
        """Order a chunk's distinct experts into steps (resident first)."""
        res = self.resident(layer)
        d = sorted(set(int(e) for e in distinct))
        order = [e for e in d if e in res] + [e for e in d if e not in res]
        return [order[i:i + width] for i in range(0, len(order), width)]
