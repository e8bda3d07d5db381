"""Expert parallelism: the routed-MoE layer with its experts split among the
ranks of a process group, one rank per GPU.

Rank r of G owns experts [r E/G, (r+1) E/G) of every layer: its slot cache,
its share of the host expert pool and its host link serve only those, so G
ranks bring G host links to the misses. The router is replicated; each rank
routes its own tokens. Per layer call every rank takes the same steps in the
same order, with empty blocks where it has nothing to send:

1. route its tokens and pack the rows (t, j) it sends, owner by owner, in
   its expert-permutation order (expert ascending, then t*k + j) -- ops.dispatch;
2. exchange the per-owner row counts (an all-to-all of one integer per pair);
3. exchange the rows and their expert ids (all-to-all with those splits);
4. run the experts it owns on the rows it received, blocks of ranks 0..G-1
   one after the other -- ops.experts;
5. send every output row back the way its input came (all-to-all, splits
   swapped);
6. combine its tokens' k outputs in rank order -- ops.combine.

Each output row is the same function of the same input row as on one GPU and
the combine adds in the same order. The routing of a token depends only on its
own row and on its batch size class: batches of up to 32 tokens and larger
ones sum the router logits with two different kernels, whose fp32 results can
differ in the last bit, so a token whose k-th and (k+1)-th logits lie within
that rounding (about sqrt(d) * 2^-24 * sum_i |x_i W_ei|) may route differently
when its rank holds a batch of the other size class than one GPU would. Away
from such near-ties the layer's result does not depend on G, and with equal
batch size classes it is the one-GPU result bit for bit.

Before any row moves, the ranks agree (one all-reduce of a flag) that every
owner can take the rows sent to it (ops.max_rows, when the ops object has
one); otherwise every rank raises the same error and no rank is left waiting
in a later exchange.

The pages serve one GPU and give no split; this one follows the layer's
definition ([wiki] "FreeToken：エッジネイティブMoEセットアップガイドと比較":
each token passes through a few of many experts, and a miss costs a move over
the bus; [ainew] "UC バークレーと MIT、MoE モデルを一般ハードウェアで動かす推論
エンジン「FreeToken」公開": in a datacenter NVLink hides moves between devices).

This module moves data and sizes between the compute steps with
torch.distributed (NCCL between GPUs); the compute steps are the `ops`
object's. An ops object provides

    dispatch(layer, x, bias) -> (rows [n, d], eids [n] int64,
                                 send_counts: list of G ints, state)
    experts(layer, mode, rows [m, d], eids [m] int64) -> out [m, d]
    combine(out_back [n, d], state) -> y [T, d]
    max_rows (optional attribute): the most rows experts() takes in one call

where rows are sent in the order described in step 1, `state` is whatever
the combine needs from the dispatch (the inverse order and the weights), and
experts() keeps the row order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def owned_experts(E: int, G: int, rank: int) -> range:
    """The experts of every layer that `rank` owns when E experts are split
    among G ranks."""
    if E % G:
        raise ValueError(f"{G} ranks do not divide {E} experts")
    n = E // G
    return range(rank * n, (rank + 1) * n)


class ExpertParallelLayer:
    """One rank's side of the expert-parallel layer call."""

    def __init__(self, ops, n_experts: int, group=None):
        self.ops = ops
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E = n_experts
        self.owned = owned_experts(n_experts, self.G, self.rank)

    def _exchange(self, send, send_counts, recv_counts):
        """All-to-all of the first axis of `send`, split by send_counts among
        the ranks; returns the blocks received, in rank order."""
        out = send.new_empty((sum(recv_counts),) + tuple(send.shape[1:]))
        dist.all_to_all_single(out, send.contiguous(), recv_counts, send_counts, group=self.group)
        return out

    def forward(self, layer: int, mode: int, x, bias=None):
        """The layer on this rank's tokens x [T, d] (T may be 0)."""
        rows, eids, send_counts, state = self.ops.dispatch(layer, x, bias)
        send_counts = [int(n) for n in send_counts]
        if len(send_counts) != self.G or sum(send_counts) != rows.shape[0]:
            raise ValueError("dispatch: one count per rank, summing to the rows sent")
        sc = torch.tensor(send_counts, dtype=torch.int64, device=rows.device)
        rc = torch.empty_like(sc)
        dist.all_to_all_single(rc, sc, group=self.group)
        recv_counts = [int(n) for n in rc.tolist()]
        # every rank takes the same collective steps: agree on the owners'
        # capacity before the rows move, so that all raise or none does
        cap = getattr(self.ops, "max_rows", None)
        ok = torch.tensor([1 if cap is None or sum(recv_counts) <= cap else 0], dtype=torch.int64,
                          device=rows.device)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN, group=self.group)
        if int(ok.item()) == 0:
            raise ValueError(f"an owner cannot take the rows sent to it this call (this rank receives "
                             f"{sum(recv_counts)}, takes at most {cap})")
        recv_rows = self._exchange(rows, send_counts, recv_counts)
        recv_eids = self._exchange(eids, send_counts, recv_counts)
        out = self.ops.experts(layer, mode, recv_rows, recv_eids)
        back = self._exchange(out, recv_counts, send_counts)
        return self.ops.combine(back, state)


class CudaEpOps:
    """The compute steps on this rank's GPU, every one a library call.

    ctx is this rank's context whose n_experts are the experts it owns
    (owned_experts(E, G, rank), local ids 0..E/G-1, with their host pool,
    slots and LRU) and whose max_tokens bounds the rows it can receive;
    routers[l] is layer l's full router [E, d] on this GPU (replicated). All
    calls are enqueued on `stream`, which must be the context's compute
    stream and the stream torch.distributed runs on (torch's current stream
    when the layer is called). max_rows is the context's max_tokens (the most
    rows one ft_moe_expert_rows call takes); ExpertParallelLayer checks it on
    every rank before the rows are exchanged."""

    def __init__(self, ctx, routers, n_experts: int, top_k: int, d_model: int, wtype: int, group=None, stream=None,
                 max_rows=None):
        from . import (FT_ROUTE_STATIC_MAX_TOKENS, FT_W_F32, ft_ep_combine, ft_ep_pack, ft_ep_pack_scratch_bytes,
                       ft_moe_expert_rows, ft_route_topk_static)
        self._route, self._pack, self._rows, self._combine = (ft_route_topk_static, ft_ep_pack,
                                                              ft_moe_expert_rows, ft_ep_combine)
        self._scratch_bytes = ft_ep_pack_scratch_bytes
        self.route_chunk = FT_ROUTE_STATIC_MAX_TOKENS
        self.ctx, self.routers = ctx, routers
        self.E, self.k, self.d, self.wtype = n_experts, top_k, d_model, wtype
        self.act_dtype = torch.float32 if wtype == FT_W_F32 else torch.bfloat16
        self.G = dist.get_world_size(group)
        self.base = owned_experts(n_experts, self.G, dist.get_rank(group)).start
        self.stream = stream
        self.max_rows = max_rows  # the context's max_tokens: rows ft_moe_expert_rows takes per call
        self.scratch = None

    def dispatch(self, layer, x, bias):
        T, dev, k = x.shape[0], x.device, self.k
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        per_token = 1 if (bias is not None and bias.dim() == 2) else 0
        for t0 in range(0, T, self.route_chunk):  # routing is per token: chunks are exact
            t1 = min(T, t0 + self.route_chunk)
            b = bias[t0:t1] if per_token else bias
            self._route(x[t0:t1], self.routers[layer], b, per_token, t1 - t0, self.E, self.d, k, self.wtype,
                        ids[t0:t1], w[t0:t1], self.stream)
        n = T * k
        need = self._scratch_bytes(T, k, self.E)
        if self.scratch is None or self.scratch.numel() < need:
            self.scratch = torch.empty(need, dtype=torch.uint8, device=dev)
        rows = torch.empty((n, self.d), dtype=self.act_dtype, device=dev)
        eids = torch.empty(n, dtype=torch.int32, device=dev)
        counts = torch.empty(self.G, dtype=torch.int64, device=dev)
        inv = torch.empty(n, dtype=torch.int32, device=dev)
        self._pack(ids, T, k, self.E, self.G, x, self.d, self.wtype, rows, eids, counts, inv, None, self.scratch,
                   self.stream)
        return rows, eids, counts.tolist(), (w, inv, T)

    def experts(self, layer, mode, rows, eids):
        n = rows.shape[0]
        out = torch.empty((n, self.d), dtype=torch.float32, device=rows.device)
        self._rows(self.ctx, layer, mode, rows, eids, self.base, n, out)
        return out

    def combine(self, back, state):
        w, inv, T = state
        y = torch.empty((T, self.d), dtype=self.act_dtype, device=back.device)
        self._combine(back, w, inv, T, self.k, self.d, self.wtype, y, self.stream)
        return y
