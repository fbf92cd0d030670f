"""Tensor parallelism across processes: one process per GPU, each rank holding
only its own shards (Diffusers "Tensor parallelism" page, opening paragraph
and the paragraph under the "Colwise and rowwise" table).

Rank r keeps the colwise shard of the projection that opens the pair (W_up,r
and b_up,r, or the heads of W_qkv it owns) and the rowwise shard of the one
that closes it (W_down,r or W_o,r).  Its colwise output never leaves the rank;
the rowwise projection yields a partial sum of the layer output, and a single
AllReduce(sum) at the block boundary adds the partials of all ranks.  The
rowwise bias is added once, after the sum, on every rank (so every rank ends
with the same replicated output, ready for the next layer).

The per-rank compute runs in the CUDA kernels of libtp
(``tp_mlp_rank_partial`` / ``tp_attn_rank_partial`` write the fp32 partial,
``tp_reduce_partials`` adds the bias and rounds once); the exchange is
``torch.distributed.all_reduce`` (NCCL over NVLink on GPUs).  Nothing here
computes: ``allreduce_layer`` only sequences partial -> AllReduce -> finish,
which the CPU tests drive with gloo ranks and host-side partials.
"""
from __future__ import annotations

import torch

from . import (TP_COLWISE, TP_ROWWISE, _check, tp_attn_rank_partial, tp_attn_rank_workspace_bytes,
               tp_mlp_rank_partial, tp_mlp_rank_workspace_bytes, tp_reduce_partials, tp_shard_bias,
               tp_shard_qkv_heads, tp_shard_weight)


def allreduce_layer(partial, finish, group=None):
    """One layer pair under TP across processes: this rank's partial (no
    rowwise bias), ONE AllReduce(sum) over the group, then ``finish`` (bias
    once + rounding) on the summed tensor.  Returns finish's result."""
    import torch.distributed as dist
    part = partial()
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    # (without a process group there is one rank, whose partial is the sum)
    return finish(part)


def ulysses_attention(qkv_local, pack, attend, unpack, group=None):
    """Ulysses attention ("Context parallelism" page): U ranks each hold M/U
    tokens with every head.  ``pack`` groups this rank's [Q | K | V] columns by
    destination head group ([U, M/U, ...], e.g. tp_shard_packed_all with
    TP_ROWWISE and blocks [1, 1, 1]); one all-to-all gives every rank all M
    tokens of its H/U heads (rank order = token order); ``attend`` runs the
    attention on them ([M, (H/U)*d] out, viewed as [U, M/U, ...]); the
    reverse all-to-all returns each rank its tokens' rows of every head group,
    which ``unpack`` puts back in head order (tp_unshard_rowwise_all)."""
    import torch.distributed as dist
    send = pack(qkv_local)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    out = attend(recv)
    back = torch.empty_like(out)
    dist.all_to_all_single(back, out, group=group)
    return unpack(back)


def ring_attention(q_local, kv_local, attend_block, merge, group=None):
    """Ring attention ("Context parallelism" page): R ranks each hold a block
    of tokens.  R steps: attend this rank's queries to the key/value block it
    currently holds (``attend_block`` -> (O_b, lse_b), e.g.
    tp_sdpa_block_stats), then pass the block on to the next rank and take the
    previous rank's.  ``merge`` combines the R results (tp_attn_merge); their
    order differs between ranks and does not change the result."""
    import torch.distributed as dist
    R, rank = dist.get_world_size(group), dist.get_rank(group)
    parts = []
    kv = kv_local
    for step in range(R):
        parts.append(attend_block(q_local, kv))
        if step + 1 < R:
            nxt = torch.empty_like(kv)
            ops = [dist.P2POp(dist.isend, kv, (rank + 1) % R, group), dist.P2POp(dist.irecv, nxt, (rank - 1) % R, group)]
            for req in dist.batch_isend_irecv(ops):
                req.wait()
            kv = nxt
    return merge(parts)


class MlpRank:
    """Rank ``rank`` of a ``tp_degree``-way MLP pair: cuts its own shards from
    the full weights once (as sharded loading would), then runs its partial."""

    def __init__(self, W_up, b_up, W_down, b_down, tp_degree: int, rank: int, stream=None):
        F, D = W_up.shape
        self.D, self.F, self.T, self.rank = D, F, tp_degree, rank
        Fs = F // tp_degree
        dev = W_up.device
        self.w_up = torch.empty((Fs, D), dtype=torch.int16, device=dev)
        self.w_down = torch.empty((D, Fs), dtype=torch.int16, device=dev)
        self.b_up = None if b_up is None else torch.empty((Fs,), dtype=torch.int16, device=dev)
        _check(tp_shard_weight(W_up, F, D, TP_COLWISE, tp_degree, rank, self.w_up, stream), "tp_shard_weight W_up")
        _check(tp_shard_weight(W_down, D, F, TP_ROWWISE, tp_degree, rank, self.w_down, stream),
               "tp_shard_weight W_down")
        if b_up is not None:
            _check(tp_shard_bias(b_up, F, tp_degree, rank, self.b_up, stream), "tp_shard_bias b_up")
        self.b_down = b_down  # replicated; added once after the sum
        self._ws = None

    def partial(self, X, out=None, stream=None):
        M = X.shape[0]
        nb = tp_mlp_rank_workspace_bytes(M, self.D, self.F, self.T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=X.device)
        part = out if out is not None else torch.empty((M, self.D), dtype=torch.float32, device=X.device)
        _check(tp_mlp_rank_partial(X, M, self.D, self.F, self.w_up, self.b_up, self.w_down, self.T, part, self._ws,
                                   nb, stream), "tp_mlp_rank_partial")
        return part

    def finish(self, summed, out=None, stream=None):
        M = summed.shape[0]
        Y = out if out is not None else torch.empty((M, self.D), dtype=torch.int16, device=summed.device)
        _check(tp_reduce_partials(summed, M, self.D, 1, self.b_down, Y, stream), "tp_reduce_partials")
        return Y

    def forward(self, X, group=None):
        return allreduce_layer(lambda: self.partial(X), self.finish, group)


class AttnRank:
    """Rank ``rank`` of a ``tp_degree``-way attention block (heads split)."""

    def __init__(self, W_qkv, W_o, heads: int, tp_degree: int, rank: int, stream=None):
        D = W_qkv.shape[1]
        self.D, self.heads, self.T, self.rank = D, heads, tp_degree, rank
        Ds = D // tp_degree
        dev = W_qkv.device
        self.w_qkv = torch.empty((3 * Ds, D), dtype=torch.int16, device=dev)
        self.w_o = torch.empty((D, Ds), dtype=torch.int16, device=dev)
        _check(tp_shard_qkv_heads(W_qkv, D, heads, tp_degree, rank, self.w_qkv, stream), "tp_shard_qkv_heads")
        _check(tp_shard_weight(W_o, D, D, TP_ROWWISE, tp_degree, rank, self.w_o, stream), "tp_shard_weight W_o")
        self._ws = None

    def partial(self, X, out=None, stream=None):
        M = X.shape[0]
        nb = tp_attn_rank_workspace_bytes(M, self.D, self.heads, self.T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=X.device)
        part = out if out is not None else torch.empty((M, self.D), dtype=torch.float32, device=X.device)
        _check(tp_attn_rank_partial(X, M, self.D, self.w_qkv, self.w_o, self.heads, self.T, part, self._ws, nb,
                                    stream), "tp_attn_rank_partial")
        return part

    def finish(self, summed, out=None, stream=None):
        M = summed.shape[0]
        Y = out if out is not None else torch.empty((M, self.D), dtype=torch.int16, device=summed.device)
        _check(tp_reduce_partials(summed, M, self.D, 1, None, Y, stream), "tp_reduce_partials")
        return Y

    def forward(self, X, group=None):
        return allreduce_layer(lambda: self.partial(X), self.finish, group)
