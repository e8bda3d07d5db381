"""Seeded synthetic inputs for the routed-MoE layer.

This module is shared by the CPU oracle and the CUDA path's tests and bench;
it holds none of the layer's arithmetic (no routing, no expert math, no cache
policy). It only draws random numbers and lays them out in the slot-blob
format of include/ft_moe.h:

* expert blobs: fp32 / bf16 weights drawn N(0, 0.02); NVFP4 blobs drawn as
  random e2m1 codes and random positive e4m3 block scales, plus one fp32
  tensor scale per matrix that brings the weight scale to about 0.02;
* router weights N(0, 0.02), hidden states N(0, 1), one row per sub-seed so a
  single token can be redrawn;
* router biases: the Zipf(s) log-probability of each expert's rank under a
  seeded permutation, and the per-layer Markov routing trace with its +beta
  bias on the chosen experts.

The workload shapes follow the pages' model: 43 layers x 256 routed experts,
top-6 (DeepSeek-V4-Flash, [paperlens] "MoEは扉を開けると同時に、別の扉を閉める",
paper §1), a shared cache at 37% of the pool ([techfeed]
"セマンティック認識キャッシング") and the B_P:B_H profiles 52.7:77.3 and 11.8:47.5
([techfeed] "帯域適応型実行（q*ポリシー）").
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np
import torch

MASTER_SEED = 20260817

W_F32, W_BF16, W_NVFP4 = 0, 1, 2
WTYPE_NAMES = {W_F32: "f32", W_BF16: "bf16", W_NVFP4: "nvfp4"}

# e4m3 codes used for random block scales: exponent fields 6..8, any mantissa
# (positive, finite, normal codes; magnitudes between one half and four).
_SCALE_CODES = np.array([(e << 3) | m for e in (6, 7, 8) for m in range(8)], dtype=np.uint8)
# Nominal fp32 tensor scale: picked by hand so that a random code times a random
# block scale times this is about 0.02 in root-mean-square.
NVFP4_TENSOR_SCALE = 0.0035


def subseed(*parts) -> int:
    """63-bit seed derived from the master seed and any labels (config name,
    layer, expert, step, token, attempt...)."""
    h = hashlib.blake2b(repr((MASTER_SEED,) + parts).encode(), digest_size=8)
    return int.from_bytes(h.digest(), "little") & ((1 << 63) - 1)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def slot_bytes(d: int, d_ff: int, wtype: int) -> int:
    n = 3 * d * d_ff
    if wtype == W_F32:
        return 4 * n
    if wtype == W_BF16:
        return 2 * n
    if wtype == W_NVFP4:
        return n // 2 + n // 16
    raise ValueError(wtype)


def expert_blob(d: int, d_ff: int, wtype: int, seed: int, device="cpu") -> torch.Tensor:
    """Random slot blob of one (layer, expert) as a flat uint8 tensor."""
    g = _gen(seed, device)
    n = 3 * d * d_ff
    if wtype == W_F32:
        w = torch.randn(n, generator=g, device=device, dtype=torch.float32).mul_(0.02)
        return w.view(torch.uint8)
    if wtype == W_BF16:
        w = torch.randn(n, generator=g, device=device, dtype=torch.float32).mul_(0.02)
        return w.to(torch.bfloat16).view(torch.uint8)
    if wtype == W_NVFP4:
        codes = torch.randint(0, 256, (n // 2,), generator=g, device=device, dtype=torch.uint8)
        pick = torch.randint(0, len(_SCALE_CODES), (n // 16,), generator=g, device=device)
        scales = torch.as_tensor(_SCALE_CODES, device=device)[pick]
        return torch.cat([codes, scales])
    raise ValueError(wtype)


def tensor_scales(seed: int) -> np.ndarray:
    """Per-matrix fp32 tensor scales (gate, up, down) of an NVFP4 blob: the
    nominal scale times a seeded factor in [0.75, 1.25)."""
    r = np.random.default_rng(seed)
    return (NVFP4_TENSOR_SCALE * r.uniform(0.75, 1.25, size=3)).astype(np.float32)


def act_dtype(wtype: int) -> torch.dtype:
    return torch.float32 if wtype == W_F32 else torch.bfloat16


def router_weight(E: int, d: int, wtype: int, seed: int) -> torch.Tensor:
    """W_r [E, d], N(0, 0.02), fp32 for fp32 experts else bf16 (CPU tensor)."""
    w = torch.randn(E, d, generator=_gen(seed), dtype=torch.float32).mul_(0.02)
    return w.to(act_dtype(wtype))


def hidden_row(d: int, wtype: int, seed: int, token: int, attempt: int = 0) -> torch.Tensor:
    g = _gen(subseed("row", seed, token, attempt))
    return torch.randn(d, generator=g, dtype=torch.float32).to(act_dtype(wtype))


def hidden(T: int, d: int, wtype: int, seed: int, attempts=None) -> torch.Tensor:
    """x [T, d] ~ N(0, 1); row t is drawn from its own sub-seed and attempt
    number, so a caller can redraw single tokens."""
    out = torch.empty(T, d, dtype=act_dtype(wtype))
    for t in range(T):
        a = 0 if attempts is None else int(attempts[t])
        out[t] = hidden_row(d, wtype, seed, t, a)
    return out


def expert_permutation(E: int, seed: int) -> np.ndarray:
    """pi: pi[r] = the expert of Zipf rank r+1."""
    return np.random.default_rng(seed).permutation(E)


def zipf_log_bias(E: int, s: float, seed: int) -> np.ndarray:
    """b[e] = ln p(rank(e)) for p(r) = r^-s / sum_r' r'^-s, ranks 1..E assigned
    by a seeded permutation. fp32 [E]."""
    pi = expert_permutation(E, seed)
    r = np.arange(1, E + 1, dtype=np.float64)
    logp = -s * np.log(r) - np.log(np.sum(r ** -s))
    b = np.empty(E, dtype=np.float64)
    b[pi] = logp
    return b.astype(np.float32)


def _zipf_draw(rng, pi, cdf, exclude) -> int:
    while True:
        r = int(np.searchsorted(cdf, rng.random(), side="right"))
        e = int(pi[min(r, len(pi) - 1)])
        if e not in exclude:
            return e


def markov_trace(steps: int, T: int, E: int, k: int, p_reuse: float, s: float, seed: int,
                 pi: np.ndarray | None = None) -> np.ndarray:
    """Per-token routing trace of one layer, int32 [steps, T, k]: each of the
    k expert positions keeps the previous step's expert with probability
    p_reuse, else draws Zipf(s) over the permutation pi (no duplicates within a
    token). Step 0 draws all k fresh."""
    rng = np.random.default_rng(seed)
    if pi is None:
        pi = expert_permutation(E, subseed("pi", seed))
    w = np.arange(1, E + 1, dtype=np.float64) ** -s
    cdf = np.cumsum(w) / w.sum()
    out = np.empty((steps, T, k), dtype=np.int32)
    for t in range(T):
        prev = None
        for st in range(steps):
            chosen: list[int] = []
            keep = [prev is not None and rng.random() < p_reuse for _ in range(k)]
            if prev is not None:
                chosen = [int(prev[j]) for j in range(k) if keep[j]]
            cur = []
            for j in range(k):
                if prev is not None and keep[j]:
                    cur.append(int(prev[j]))
                else:
                    e = _zipf_draw(rng, pi, cdf, set(chosen))
                    chosen.append(e)
                    cur.append(e)
            out[st, t] = cur
            prev = out[st, t]
    return out


def trace_bias(chosen: np.ndarray, base: np.ndarray, beta: float = 8.0) -> np.ndarray:
    """Per-token router bias [T, E] fp32 realising one trace step: the base
    log-bias plus beta on each token's chosen experts."""
    T = chosen.shape[0]
    b = np.repeat(base[None, :].astype(np.float32), T, axis=0)
    for t in range(T):
        b[t, chosen[t]] += np.float32(beta)
    return b


@dataclass
class Workload:
    """One synthetic workload recipe (sizes, seeds, cache and link settings)."""
    name: str
    L: int
    E: int
    k: int
    d: int
    d_ff: int
    wtype: int
    cache_slots: int
    bp_mbps: int = 52700
    bh_mbps: int = 77300
    batches: tuple = (1,)
    steps: int = 1
    extra: dict = field(default_factory=dict)

    @property
    def slot_bytes(self) -> int:
        return slot_bytes(self.d, self.d_ff, self.wtype)

    def seed(self, *parts) -> int:
        return subseed(self.name, *parts)


def workload(name: str) -> Workload:
    """The five workloads: tiny fp32 layer; single-layer BF16 decode; single-
    layer BF16 prefill; 43-layer NVFP4 decode trace; 43-layer mixed NVFP4."""
    E, k, d, d_ff = 256, 6, 4096, 1536
    if name == "tiny_f32":
        return Workload(name, L=1, E=8, k=2, d=64, d_ff=128, wtype=W_F32, cache_slots=4,
                        batches=(16,), steps=1)
    if name == "decode_bf16":
        return Workload(name, L=1, E=E, k=k, d=d, d_ff=d_ff, wtype=W_BF16,
                        cache_slots=int(0.37 * E), batches=(1, 4, 16), steps=64,
                        extra={"zipf_s": 1.1})
    if name == "prefill_bf16":
        return Workload(name, L=1, E=E, k=k, d=d, d_ff=d_ff, wtype=W_BF16,
                        cache_slots=2 * E, batches=(4096,), steps=1)
    if name == "trace_nvfp4":
        return Workload(name, L=43, E=E, k=k, d=d, d_ff=d_ff, wtype=W_NVFP4,
                        cache_slots=int(0.37 * 43 * E), batches=(1,), steps=512,
                        extra={"zipf_s": 1.1, "p_reuse": 0.8, "beta": 8.0})
    if name == "mixed_nvfp4":
        return Workload(name, L=43, E=E, k=k, d=d, d_ff=d_ff, wtype=W_NVFP4,
                        cache_slots=int(0.37 * 43 * E), batches=(1, 2, 4, 8), steps=1024,
                        extra={"zipf_s": 1.1, "p_reuse": 0.8, "beta": 8.0, "prefill_T": 8192,
                               "cache_fracs": (0.10, 0.20, 0.37, 0.60),
                               "profiles": ((11800, 47500), (52700, 77300))})
    raise KeyError(name)


WORKLOADS = ("tiny_f32", "decode_bf16", "prefill_bf16", "trace_nvfp4", "mixed_nvfp4")
