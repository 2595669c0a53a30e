"""Naive reference simulator of the per-layer LFU expert cache, used to pin the
oracle's incremental implementation.

It keeps the whole selection history and, at every miss, rescans it to
recount each resident expert's frequency and recency, instead of keeping
counters.  Policy (from "El milagro de la IA de 2GB en Apple Silicon", section
"Mas inteligente que tu RAM": a miss replaces the least frequently used
expert currently held; readings where the pages are silent: ties go to the
least recently used, then the lower id; experts of the current wave are never
evicted; empty slots fill lowest first; waves of at most S distinct experts in
ascending id order; frequency counts every (token, k) selection so far, the
current call's included).
"""


LFU, LRU, LFU_DECAY, LFU_IN_CACHE = 0, 1, 2, 3


class NaiveLfu:
    """policy: LFU (the pages' rule), LRU (victim by recency, then id),
    LFU_DECAY (the frequency of every earlier call is halved, with the integer
    floor, at each call whose step is a positive multiple of `period`),
    LFU_IN_CACHE (frequency counts only selections made after the expert's
    last eviction)."""

    def __init__(self, E, S, policy=LFU, period=0):
        self.E, self.S = E, S
        self.policy, self.period = policy, period
        self.selections = []      # every (step, expert) selection, one per pair
        self.calls = []           # (step, [experts selected, one per pair]) per call
        self.events = []          # ("sel", e) per pair at call start, ("evict", e) at evictions
        self.wave_uses = []       # (step, expert) for each expert of each finished wave
        self.slots = [None] * S   # slot -> expert

    def _freq(self, e):
        if self.policy == LFU_DECAY:
            c = 0                 # replay the history call by call
            for step, sel in self.calls:
                if self.period > 0 and step > 0 and step % self.period == 0:
                    c //= 2
                c += sum(1 for x in sel if x == e)
            return c
        if self.policy == LFU_IN_CACHE:
            c = 0
            for kind, x in self.events:
                if x != e:
                    continue
                c = 0 if kind == "evict" else c + 1
            return c
        return sum(1 for _, x in self.selections if x == e)

    def _key(self, e):
        if self.policy == LRU:
            return (self._recency(e), e)
        return (self._freq(e), self._recency(e), e)

    def _recency(self, e):
        steps = [s + 1 for s, x in self.wave_uses if x == e]
        return max(steps) if steps else 0

    def plan(self, ids, step):
        """ids: list of T lists of K ids.  Returns (pair_slot, events) with
        events = list of (expert, slot, hit, victim, wave) in ascending id."""
        for row in ids:
            for e in row:
                self.selections.append((step, int(e)))
                self.events.append(("sel", int(e)))
        self.calls.append((step, [int(e) for row in ids for e in row]))
        distinct = sorted({int(e) for row in ids for e in row})
        events, slot_of_wave = [], {}
        for w in range(0, len(distinct), self.S):
            wave = distinct[w:w + self.S]
            for e in wave:
                if e in self.slots:
                    s = self.slots.index(e)
                    events.append((e, s, 1, -1, w // self.S))
                    slot_of_wave[e] = s
                    continue
                if None in self.slots:
                    s, victim = self.slots.index(None), -1
                else:
                    cands = [x for x in self.slots if x not in wave]
                    victim = min(cands, key=self._key)
                    s = self.slots.index(victim)
                    self.events.append(("evict", victim))
                self.slots[s] = e
                slot_of_wave[e] = s
                events.append((e, s, 0, victim, w // self.S))
            for e in wave:
                self.wave_uses.append((step, e))
        pair_slot = [[slot_of_wave[int(e)] for e in row] for row in ids]
        return pair_slot, events
