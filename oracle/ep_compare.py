"""Expert parallelism against replicas on the 43-layer NVFP4 decode trace, as
a cache-and-link simulation of the oracle.

Part of the test infrastructure (it runs the oracle only). G devices each
serve their own stream of `batch` tokens per step (per device, layer and
token a Markov chain that keeps each of the k experts with p = 0.8, else
draws Zipf(1.1)), each with the same number of slots:

* replicas: every device caches any (layer, expert) of its own stream in one
  shared LRU with the q* admission;
* expert parallelism (oracle/ep.py): device o owns experts [o E/G, (o+1) E/G)
  of every layer and caches only those, for the rows all G streams route to
  them;
* the same with the decode prefetch on every owner (after its lookup for
  layer l it stages layer l+1's experts of its last call); a prefetched blob
  crosses the owner's link during layer l and counts there.

A miss costs a blob over the device's own host link either way (staged or
streamed). Replicas run independently: each device's step takes its own
blobs over its link, and the devices' rates add up. Expert-parallel devices
exchange rows at every layer, so a layer call takes, on the link, the largest
number of blobs any one owner moves. The step times that follow at a given
link rate are a model, not a measurement. The pages put
the miss cost on the bus ([wiki] "FreeToken：エッジネイティブMoEセットアップ
ガイドと比較") and note that a datacenter interconnect hides moves between
devices ([ainew] "UC バークレーと MIT、MoE モデルを一般ハードウェアで動かす推論
エンジン「FreeToken」公開", opening paragraph).

    python -m oracle.ep_compare [steps] [batch]
"""
from __future__ import annotations

import sys

import numpy as np

import ftgen
from oracle import cache


def run(steps: int = 256, gs=(1, 2, 4, 8), fracs=(0.10, 0.37), profile=(52700, 77300), link_gbs=55.6, batch=1):
    wl = ftgen.workload("trace_nvfp4")
    L, E, k = wl.L, wl.E, wl.k
    ex = wl.extra
    blob = wl.slot_bytes
    rows = []
    for G in gs:
        # stream g, layer l: chosen experts per step and token; a layer's
        # expert popularity (the Zipf ranks) is the model's, the same on every
        # device; the streams differ
        pis = [ftgen.expert_permutation(E, ftgen.subseed("pi", wl.seed("trace", 0, l))) for l in range(L)]
        tr = [[ftgen.markov_trace(steps, batch, E, k, ex["p_reuse"], ex["zipf_s"], wl.seed("ep_trace", g, l),
                                  pi=pis[l])
               for l in range(L)] for g in range(G)]
        for f in fracs:
            C = int(f * L * E)
            rep = [cache.ExpertCache(L, E, C, *profile) for _ in range(G)]
            own = [cache.ExpertCache(L, E // G, C, *profile) for _ in range(G)]
            own_pf = [cache.ExpertCache(L, E // G, C, *profile) for _ in range(G)]
            for c in own_pf:
                c.prefetch_on = True
            blobs_rep = np.zeros(G)  # per device, over all steps
            link_ep = link_pf = 0
            for st in range(steps):
                for l in range(L):
                    m_rep, per_owner = [], [np.zeros(E // G, int) for _ in range(G)]
                    for g in range(G):
                        cnt = np.zeros(E, int)
                        for t in range(batch):
                            for e in tr[g][l][st][t]:
                                cnt[int(e)] += 1
                                per_owner[int(e) // (E // G)][int(e) % (E // G)] += 1
                        m_rep.append(rep[g].forward(l, cache.DECODE, cnt)["m"])
                    m_own = [own[o].forward(l, cache.DECODE, per_owner[o])["m"] for o in range(G)]
                    m_pf = []
                    for o in range(G):
                        before = own_pf[o].n["prefetched"]
                        m = own_pf[o].forward(l, cache.DECODE, per_owner[o])["m"]
                        m_pf.append(m + own_pf[o].n["prefetched"] - before)
                    blobs_rep += m_rep
                    link_ep += max(m_own)
                    link_pf += max(m_pf)
            miss_rep = sum(c.n["misses"] for c in rep) / sum(c.n["lookups"] for c in rep)
            miss_ep = sum(c.n["misses"] for c in own) / sum(c.n["lookups"] for c in own)
            miss_pf = sum(c.n["misses"] for c in own_pf) / sum(c.n["lookups"] for c in own_pf)
            # tokens per second on the link model (`batch` tokens per device per step)
            sec = blob / (link_gbs * 1e9)
            tps_rep = sum(batch * steps / (b * sec) for b in blobs_rep if b) if blobs_rep.all() else float("inf")
            tps_ep = G * batch * steps / (link_ep * sec) if link_ep else float("inf")
            tps_pf = G * batch * steps / (link_pf * sec) if link_pf else float("inf")
            rows.append((G, C, f, miss_rep, miss_ep, blobs_rep.mean() / steps, link_ep / steps, tps_rep, tps_ep,
                         miss_pf, link_pf / steps, tps_pf))
    return rows


if __name__ == "__main__":
    steps = int(sys.argv[1]) if len(sys.argv) > 1 else 256
    batch = int(sys.argv[2]) if len(sys.argv) > 2 else 1
    rows = run(steps, batch=batch)
    print(f"43-layer NVFP4 trace, {steps} steps, {batch} token(s) per device per step, B_P:B_H = 52.7:77.3, "
          f"link model 55.6 GB/s per device")
    print("| devices | slots per device | capacity | miss rate, replicas | miss rate, expert parallel | "
          "link blobs per step, replicas (mean device) | expert parallel (slowest owner per layer) | "
          "tokens/s on the link model, replicas | expert parallel |")
    print("|---|---|---|---|---|---|---|---|---|")
    for G, C, f, mr, me, lr, le, tr, te, *_ in rows:
        print(f"| {G} | {C} | {100 * f:.0f}% | {100 * mr:.1f}% | {100 * me:.1f}% | {lr:.1f} | {le:.1f} | "
              f"{tr:.1f} | {te:.1f} |")
    print()
    print("| devices | capacity | expert parallel: miss rate | with prefetch | link blobs per step (slowest owner) | "
          "with prefetch | tokens/s on the link model | with prefetch |")
    print("|---|---|---|---|---|---|---|---|")
    for G, C, f, mr, me, lr, le, tr, te, mp, lp, tp in rows:
        print(f"| {G} | {100 * f:.0f}% | {100 * me:.1f}% | {100 * mp:.1f}% | {le:.1f} | {lp:.1f} | {te:.1f} | "
              f"{tp:.1f} |")
