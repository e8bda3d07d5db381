"""The q* split and the shared LRU expert cache, step by step.

Test infrastructure (see oracle/__init__.py).

What the pages fix:
* all routed weights live in a host pool (the source of truth); the rest of
  GPU memory is one cache shared by every MoE layer, one slot per
  (layer, expert) ([paperlens] "設計: 2階建てのエキスパート記憶", paper §3);
* during decode one LRU shared across all MoE layers follows the router
  ([techfeed] "セマンティック認識キャッシング"; [leadeas]
  "VRAMをキャッシュとして使う ― 帯域幅適応的なCPU-GPU協調実行");
* with m missed experts in a step, about m * B_P / B_H of them go to the GPU
  cache and the rest are executed where the weights already are ([techfeed]
  "帯域適応型実行（q*ポリシー）"); on this GPU those are read zero-copy from
  the host pool by the expert kernel and not inserted;
* prefill loads every expert of layer l+1 while layer l computes, from the
  same slot pool, with two layers' worth of slots; with fewer slots it falls
  back to on-demand ([paperlens] "プレフィル: 全層ダブルバッファと「意味の錨」",
  paper §3.1);
* the first request meets a cold, empty cache ([techfeed] "弾性メモリ管理");
* the memory given to expert slots can grow or shrink at safe points without
  reloading the model, which is correct because what the cache holds never
  changes a result ([techfeed] "弾性メモリ管理").

Readings taken where the pages are silent:
* q* = floor((2 m B_P + B_H) / (2 B_H)) -- m B_P / B_H rounded half up, in
  exact integers of MB/s -- clamped to [0, m];
* one lookup per unique (layer, expert) per call, in ascending expert order;
  hits are stamped first (ascending e), then the staged misses are inserted
  (ascending e), each with a fresh stamp;
* the misses staged are the first min(q*, C - hits) in ascending e; the rest
  are streamed and do not enter the cache;
* an insertion takes the lowest-index free slot, else evicts the entry with
  the smallest stamp that is not pinned; pinned = touched or inserted in this
  call (decode), or belonging to layer l or l+1 (prefill call of layer l);
* prefill with C >= 2E: a call for layer l loads layer l if the previous call
  did not already prefetch it, then prefetches layer l+1 (if l+1 < L), all E
  experts each, no q*; with C < 2E a prefill call follows the decode rules
  for its routed experts; a call with T = 0 changes nothing;
* optional predictive prefetch: right after the decode lookup of layer l,
  the experts that layer (l+1) mod L was routed to in its last decode call and
  that are not resident are staged, ascending e, as staged inserts (fresh
  stamps), never evicting what layer l's lookup touched or inserted; resident
  ones are left untouched; only decode calls record their routing and
  prefetch; a resize clears the record;
* a resize to C' slots between layer calls keeps the min(C', resident)
  most recently stamped entries with their stamps; a survivor whose slot is
  below C' stays there, the others move, in ascending order of their old
  slot, to the lowest free slots below C'; the clock is kept and the
  layer-ahead prefetch state is cleared.

For the miss-rate comparison with engines that pin a fixed hot subset
([techfeed] "セマンティック認識キャッシング" sets the shared LRU against such
static placements), `static_hot_placement` gives the best static placement of
C slots in hindsight and `static_placement_misses` its misses.

A predictive prefetch (`ExpertCache.prefetch`, a policy simulation of the
next layer staged during the current one) inserts like a staged miss.

Pins (tests/test_oracle_cache.py): q* against the table derived from the
pages' two B_P:B_H profiles (tests/golden/qstar_profiles.txt) and the bound
|q* - m B_P / B_H| <= 1/2; q* = 0 at B_P = 0 and q* = m at B_P >= B_H; with
one access per step and B_P = B_H the hit/miss sequence equals a textbook
move-to-front LRU list; misses are never fewer than Belady's optimal policy;
C >= L*E gives only compulsory misses; C = 0 makes every lookup a streamed
miss; a resize equals a move-to-front list truncated at each shrink; a
prefetch equals an insert at the most-recent end of that list; the best static
placement equals the brute-force minimum over all placements.
"""
from __future__ import annotations

HIT, STAGED, STREAMED = 0, 1, 2
DECODE, PREFILL = 0, 1


def qstar(m: int, bp_mbps: int, bh_mbps: int) -> int:
    """Number of the m missed experts to stage into the GPU cache."""
    if m <= 0:
        return 0
    q = (2 * m * bp_mbps + bh_mbps) // (2 * bh_mbps)
    return max(0, min(m, q))


def static_hot_placement(key_counts: dict, C: int) -> set:
    """The C keys with the most lookups, ties to the lower key: on a trace known
    in advance, no static placement of C slots misses less (every lookup of a
    pinned key hits, every other lookup misses, whatever the order)."""
    order = sorted(key_counts, key=lambda k: (-key_counts[k], k))
    return set(order[:max(C, 0)])


def static_placement_misses(batches, hot: set):
    """(lookups, misses) of a static placement over lookup batches (each an
    iterable of unique keys): nothing is ever inserted or evicted."""
    lookups = misses = 0
    for batch in batches:
        for key in batch:
            lookups += 1
            misses += key not in hot
    return lookups, misses


class ExpertCache:
    """C slots shared by L layers of E experts; keys are layer * E + e."""

    def __init__(self, L: int, E: int, C: int, bp_mbps: int = 1, bh_mbps: int = 1):
        self.L, self.E, self.C = L, E, C
        self.bp, self.bh = bp_mbps, bh_mbps
        self.key_of = [-1] * C   # slot -> key
        self.stamp = [0] * C     # slot -> last-use stamp (0 = never / free)
        self.slot_of = {}        # key -> slot
        self.clock = 0
        self.prefetched = -1     # layer whose experts the last prefill call loaded ahead
        self.n = dict(lookups=0, hits=0, misses=0, staged=0, streamed=0, layer_calls=0, prefetched=0)
        # predictive prefetch (opt-in): after the decode lookup of layer l,
        # stage the experts layer (l+1) mod L was routed to in its last decode call
        self.prefetch_on = False
        self.last_routed = {}    # layer -> experts of its last decode call

    # --- primitives -------------------------------------------------------
    def _touch(self, slot: int):
        self.clock += 1
        self.stamp[slot] = self.clock

    def _victim(self, pinned: set) -> int:
        for s in range(self.C):
            if self.key_of[s] < 0:
                return s
        best = None
        for s in range(self.C):
            if s in pinned:
                continue
            if best is None or self.stamp[s] < self.stamp[best]:
                best = s
        assert best is not None, "no unpinned slot"
        return best

    def _insert(self, key: int, pinned: set) -> int:
        s = self._victim(pinned)
        old = self.key_of[s]
        if old >= 0:
            del self.slot_of[old]
        self.key_of[s] = key
        self.slot_of[key] = s
        self._touch(s)
        pinned.add(s)
        return s

    # --- one lookup batch -------------------------------------------------
    def _batch(self, layer: int, experts, pinned: set, limit_q: bool):
        """Look up `experts` (ascending) of `layer`. Returns (kinds, m, q*, q_stage)."""
        kinds = {}
        misses = []
        for e in experts:
            key = layer * self.E + e
            if key in self.slot_of:
                s = self.slot_of[key]
                self._touch(s)
                pinned.add(s)
                kinds[e] = HIT
            else:
                misses.append(e)
        h = len(experts) - len(misses)
        m = len(misses)
        if limit_q:
            q = qstar(m, self.bp, self.bh)
            q_stage = min(q, self.C - h)
        else:
            q = -1
            q_stage = m
        for e in misses[:q_stage]:
            self._insert(layer * self.E + e, pinned)
            kinds[e] = STAGED
        for e in misses[q_stage:]:
            kinds[e] = STREAMED
        self.n["lookups"] += len(experts)
        self.n["hits"] += h
        self.n["misses"] += m
        self.n["staged"] += q_stage
        self.n["streamed"] += m - q_stage
        return kinds, m, q, q_stage

    # --- one layer call ---------------------------------------------------
    def forward(self, layer: int, mode: int, counts):
        """Cache work of one layer call whose routed experts have `counts`
        tokens each. Returns a record: lookups [(layer, e, kind)] in lookup
        order, this layer's kind per routed expert, m, q*, q_stage."""
        E = self.E
        if sum(int(c) for c in counts) == 0:
            return dict(lookups=[], kinds={}, m=0, qstar=0, qstage=0, n_cur=0)
        self.n["layer_calls"] += 1
        routed = [e for e in range(E) if counts[e] > 0]
        if mode == DECODE or self.C < 2 * E:
            pinned = set()
            kinds, m, q, qs = self._batch(layer, routed, pinned, True)
            self.prefetched = -1
            if mode == DECODE:
                nxt = (layer + 1) % self.L
                if self.prefetch_on and nxt in self.last_routed:
                    self._prefetch(nxt, self.last_routed[nxt], pinned)
                self.last_routed[layer] = routed
            look = [(layer, e, kinds[e]) for e in routed]
            return dict(lookups=look, kinds=kinds, m=m, qstar=q, qstage=qs, n_cur=len(look))
        look = []
        m = qs = 0
        if self.prefetched != layer:
            kinds, m, _, qs = self._batch(layer, list(range(E)), set(), False)
            look += [(layer, e, kinds[e]) for e in range(E)]
        n_cur = len(look)
        if layer + 1 < self.L:
            pinned = {self.slot_of[layer * E + e] for e in range(E)}
            nk, _, _, _ = self._batch(layer + 1, list(range(E)), pinned, False)
            look += [(layer + 1, e, nk[e]) for e in range(E)]
            self.prefetched = layer + 1
        else:
            self.prefetched = -1
        # every expert of this layer is resident now: all are read from slots
        return dict(lookups=look, kinds={e: HIT for e in routed}, m=m, qstar=-1, qstage=qs,
                    n_cur=n_cur)

    # --- predictive prefetch (a policy simulation) -------------------------
    def prefetch(self, layer: int, experts, pinned_keys=()) -> int:
        """Stage the non-resident `experts` of `layer` ahead of its lookup, in
        ascending e, each with a fresh stamp (as staged inserts); the keys in
        `pinned_keys` (the layer computing meanwhile) are not evicted. Returns
        the number of blobs copied; only the `prefetched` counter changes."""
        return self._prefetch(layer, experts, {self.slot_of[k] for k in pinned_keys if k in self.slot_of})

    def _prefetch(self, layer: int, experts, pinned: set) -> int:
        """prefetch() with the pinned slots given; `pinned` grows by the inserts."""
        n = 0
        for e in sorted(set(int(x) for x in experts)):
            key = layer * self.E + e
            if key in self.slot_of:
                continue
            if len(pinned) >= self.C:
                break
            self._insert(key, pinned)
            n += 1
        self.n["prefetched"] += n
        return n

    # --- elastic capacity -------------------------------------------------
    def resize(self, C_new: int):
        """Change the capacity to C_new slots at a safe point (between calls)."""
        res = [s for s in range(self.C) if self.key_of[s] >= 0]
        res.sort(key=lambda s: -self.stamp[s])          # most recent first
        keep = sorted(res[:C_new])                      # ascending old slot
        key_of, stamp = [-1] * C_new, [0] * C_new
        movers = []
        for s in keep:
            if s < C_new:
                key_of[s], stamp[s] = self.key_of[s], self.stamp[s]
            else:
                movers.append(s)
        free = [s for s in range(C_new) if key_of[s] < 0]
        for s, t in zip(movers, free):
            key_of[t], stamp[t] = self.key_of[s], self.stamp[s]
        self.C = C_new
        self.key_of, self.stamp = key_of, stamp
        self.slot_of = {k: s for s, k in enumerate(key_of) if k >= 0}
        self.prefetched = -1
        self.last_routed = {}

    def contents(self):
        """(key_of [C], stamp [C]) as lists."""
        return list(self.key_of), list(self.stamp)
