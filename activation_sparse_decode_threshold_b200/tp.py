"""Tensor-parallel neuron sharding of the sparse FFN across ranks.

Each rank holds a shard of every layer's neurons -- its rows of W_gate, W_up,
U and c and its columns of W_down -- and the full V, so that it predicts
exactly its own neurons of the full predictor.  Per layer every rank computes
its share of y on the same residual (``pi_sparse_ffn_decode_partial``), the
shares are summed with one all-reduce of d floats (``torch.distributed``: NCCL
across GPUs, gloo on the host), and every rank adds the sum to its copy of the
residual (``pi_residual_add``).  This module only splits weights and sequences
the calls; every step of the FFN runs in the library's kernels.

Neurons are dealt to the ranks by descending profiled frequency in snake
order, so each shard holds the same number of neurons (up to one) and a
balanced share of the hot ones -- the rule the neuron table applies to strips,
applied across ranks.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B
from . import synth


def shard_neurons(freq: np.ndarray, world: int) -> list[np.ndarray]:
    """Original neuron indices of each rank's shard (ascending), dealt by
    descending frequency (ties: lower index) in snake order."""
    F = int(freq.shape[0])
    order = sorted(range(F), key=lambda i: (-float(freq[i]), i))
    out = [[] for _ in range(world)]
    for k, i in enumerate(order):
        rnd, pos = divmod(k, world)
        out[pos if rnd % 2 == 0 else world - 1 - pos].append(i)
    return [np.array(sorted(s), dtype=np.int64) for s in out]


def shard_expert(e: synth.ExpertWeights, idx: np.ndarray) -> synth.ExpertWeights:
    """The shard of one expert holding neurons `idx` (original order kept)."""
    ix = torch.as_tensor(idx, device=e.U.device)
    take = (lambda t: None if t is None else t.index_select(0, ix).contiguous())
    # W_down: d x F for float formats (columns), neuron-major F x d/2 for INT4 (rows)
    if e.s_down is not None:
        w_down = take(e.w_down)
    else:
        w_down = e.w_down.index_select(1, ix).contiguous()
    return synth.ExpertWeights(
        w_gate=take(e.w_gate), w_up=take(e.w_up), w_down=w_down, c=take(e.c), U=take(e.U),
        V=e.V, freq=e.freq[idx], s_gate=take(e.s_gate), s_up=take(e.s_up), s_down=take(e.s_down),
        sU=take(e.sU), sV=e.sV)


def shard_layer(lw: synth.LayerWeights, shards: list[list[np.ndarray]], rank: int) -> synth.LayerWeights:
    """Rank `rank`'s shard of a layer; shards[e][rank] are expert e's neurons."""
    return synth.LayerWeights([shard_expert(e, shards[k][rank]) for k, e in enumerate(lw.experts)],
                              lw.router, dict(lw.meta, rank=rank))


class ShardedDecoder:
    """One rank's handle on its neuron shard of every layer of a stack."""

    def __init__(self, cfg: synth.FFNConfig, rank: int, world: int, group=None, device: int = 0,
                 active=None, layers=None):
        self.cfg, self.rank, self.world, self.group = cfg, rank, world, group
        self.device = device
        L = cfg.n_layers
        self.shards = []
        handle = None
        for l in range(L):
            lw = layers[l] if layers is not None else synth.make_layer(cfg, l, "cuda", active)
            sh = [shard_neurons(e.freq, world) for e in lw.experts]
            self.shards.append(sh)
            part = shard_layer(lw, sh, rank)
            if handle is None:
                F_local = int(sh[0][rank].shape[0])
                assert all(int(s[rank].shape[0]) == F_local for s in sh), "experts shard unevenly"
                handle = B.pi_ffn_create(L, cfg.d, F_local, cfg.rank, act=cfg.act, w_dtype=cfg.wdtype,
                                         pred_dtype=cfg.pdtype, n_experts=cfg.n_experts,
                                         top_k=cfg.top_k, device=device)
            B.pi_ffn_load_layer(handle, l, part.experts, part.router,
                                np.stack([e.freq for e in part.experts]).astype(np.float32))
            del lw, part
        self.h = handle
        self.y = torch.empty(cfg.d, device="cuda", dtype=torch.float32)
        self.stats = torch.zeros(4, device="cuda", dtype=torch.int32)

    def layer(self, resid: torch.Tensor, l: int, all_reduce=None) -> torch.Tensor:
        """One layer on every rank: r <- r + sum over ranks of this layer's y."""
        B.pi_sparse_ffn_decode_partial(self.h, l, resid, self.y, self.stats)
        if self.world > 1:
            all_reduce(self.y)
        B.pi_residual_add(self.h, resid, self.y)
        return resid

    def decode(self, resid: torch.Tensor, all_reduce=None, trace: list | None = None) -> torch.Tensor:
        for l in range(self.cfg.n_layers):
            if trace is not None:
                trace.append(resid.detach().clone())
            self.layer(resid, l, all_reduce)
        return resid

    def close(self):
        if self.h:
            torch.cuda.synchronize()
            B.pi_ffn_destroy(self.h)
            self.h = None


def nccl_all_reduce(group=None):
    import torch.distributed as dist
    return lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def host_all_reduce(group=None):
    """All-reduce of a device tensor through host memory (the gloo backend)."""
    import torch.distributed as dist

    def f(t: torch.Tensor):
        h = t.detach().to("cpu")
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
        t.copy_(h)
    return f
