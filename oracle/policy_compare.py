"""Miss rate of the shared LRU (with the q* admission) against the best
static placement of the same number of slots, on the 43-layer NVFP4 decode
trace (batch 1; per layer a Markov chain that keeps each of the k experts with
p = 0.8, else draws Zipf(1.1)), at the capacities of the mixed workload.

Part of the test infrastructure (it runs the oracle only). The pages set the
shared LRU's miss rate against engines that pin a fixed hot subset
([techfeed] "セマンティック認識キャッシング"); the static placement here is the
best one in hindsight (the most-used keys of the whole trace), so it is a lower
bound for any static policy. The routed experts of a step are the trace's
chosen experts (the bias that realises the trace in the benchmark makes them
the top-k).

    python -m oracle.policy_compare [steps]
"""
from __future__ import annotations

import sys

import numpy as np

import ftgen
from oracle import cache


def run(steps: int = 512, fracs=(0.10, 0.20, 0.37, 0.60), profile=(52700, 77300)):
    wl = ftgen.workload("trace_nvfp4")
    L, E, k = wl.L, wl.E, wl.k
    ex = wl.extra
    traces = [ftgen.markov_trace(steps, 1, E, k, ex["p_reuse"], ex["zipf_s"], wl.seed("trace", 0, l))
              for l in range(L)]
    batches = [[l * E + int(e) for e in sorted(set(traces[l][st][0].tolist()))]
               for st in range(steps) for l in range(L)]
    counts = {}
    for b in batches:
        for key in b:
            counts[key] = counts.get(key, 0) + 1
    # profiled placement: per layer the experts the routing prior ranks first
    # (the Zipf ranks of the permutation the layer's trace draws from), C/L of
    # them, the first C mod L layers one more
    ranks = [ftgen.expert_permutation(E, ftgen.subseed("pi", wl.seed("trace", 0, l))) for l in range(L)]
    half = steps // 2
    rows = []
    for f in fracs:
        C = int(f * L * E)
        c = cache.ExpertCache(L, E, C, *profile)
        for st in range(steps):
            if st == half:
                n_half = dict(c.n)
            for l in range(L):
                cnt = np.zeros(E, int)
                cnt[traces[l][st][0]] = 1
                c.forward(l, cache.DECODE, cnt)
        lru = c.n["misses"] / c.n["lookups"]
        lru_half = (c.n["misses"] - n_half["misses"]) / (c.n["lookups"] - n_half["lookups"])
        prior = set()
        for l in range(L):
            take = C // L + (1 if l < C % L else 0)
            prior |= {l * E + int(e) for e in ranks[l][:take]}
        _, m_prior = cache.static_placement_misses(batches, prior)
        look, m_best = cache.static_placement_misses(batches, cache.static_hot_placement(counts, C))
        # the same LRU with the predictive prefetch: after layer l's lookup,
        # layer l+1's experts of its last call are staged (the reuse of the
        # Markov trace); cost: every prefetched blob crosses the link
        cp = cache.ExpertCache(L, E, C, *profile)
        cp.prefetch_on = True
        for st in range(steps):
            for l in range(L):
                cnt = np.zeros(E, int)
                cnt[traces[l][st][0]] = 1
                cp.forward(l, cache.DECODE, cnt)
        pf_miss = cp.n["misses"] / cp.n["lookups"]
        link_lru = c.n["misses"] / steps          # blobs over the link per step (staged + streamed)
        link_pf = (cp.n["misses"] + cp.n["prefetched"]) / steps
        rows.append((C, f, lru, lru_half, m_prior / look, m_best / look, pf_miss, link_lru, link_pf))
    return rows


if __name__ == "__main__":
    steps = int(sys.argv[1]) if len(sys.argv) > 1 else 512
    rows = run(steps)
    print(f"43-layer NVFP4 trace, {steps} steps at batch 1, B_P:B_H = 52.7:77.3; static placements pre-loaded")
    print("| slots | capacity | shared LRU (cold start) | shared LRU, second half | static, profiled | static, best in hindsight |")
    print("|---|---|---|---|---|---|")
    for C, f, lru, lru_half, st_prior, st_best, *_ in rows:
        print(f"| {C} | {100 * f:.0f}% | {100 * lru:.1f}% | {100 * lru_half:.1f}% | {100 * st_prior:.1f}% | "
              f"{100 * st_best:.1f}% |")
    print()
    print("| slots | capacity | LRU miss rate | LRU + prefetch miss rate | link blobs per step, LRU | with prefetch |")
    print("|---|---|---|---|---|---|")
    for C, f, lru, _, _, _, pf, link_lru, link_pf in rows:
        print(f"| {C} | {100 * f:.0f}% | {100 * lru:.1f}% | {100 * pf:.1f}% | {link_lru:.1f} | {link_pf:.1f} |")
