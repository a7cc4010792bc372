"""Tensor-parallel neuron sharding, host side (CPU): the dealing rule, the
sharded weights, and -- on the fp64 oracle -- that the layer output is the
sum of the shards' outputs, each shard predicting its own neurons with the
full predictor.  The multi-process composition runs on gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from activation_sparse_decode_threshold_b200 import synth, tp


def test_shard_neurons_partition_and_balance():
    rng = np.random.default_rng(3)
    F = 1001
    freq = rng.random(F)
    for world in (1, 2, 3, 8):
        sh = tp.shard_neurons(freq, world)
        allidx = np.concatenate(sh)
        assert np.array_equal(np.sort(allidx), np.arange(F))          # a partition
        sizes = [s.size for s in sh]
        assert max(sizes) - min(sizes) <= 1
        mass = [freq[s].sum() for s in sh]
        assert max(mass) - min(mass) <= freq.max() + 1e-12              # snake dealing balances
        for s in sh:
            assert np.all(np.diff(s) > 0)


def test_shard_neurons_snake_order_by_hand():
    freq = np.array([0.1, 0.9, 0.5, 0.7, 0.3, 0.2])
    # ranking 1 (0.9), 3 (0.7), 2 (0.5), 4 (0.3), 5 (0.2), 0 (0.1); snake over 2 ranks:
    # round 0: rank0 <- 1, rank1 <- 3; round 1: rank1 <- 2, rank0 <- 4; round 2: rank0 <- 5, rank1 <- 0
    sh = tp.shard_neurons(freq, 2)
    assert sh[0].tolist() == [1, 4, 5] and sh[1].tolist() == [0, 2, 3]


@pytest.mark.parametrize("name", ["reglu-f16", "relu-f16", "moe-int4", "drelu-bf16-i8pred"])
def test_layer_output_is_the_sum_of_shard_outputs(name):
    cfgs = {
        "reglu-f16": synth.small(synth.CONFIGS["llama7b"], n_layers=1, d=64, F=90, rank=16),
        "relu-f16": synth.small(synth.CONFIGS["falcon40b"], n_layers=1, d=64, F=90, rank=16),
        "moe-int4": synth.small(synth.CONFIGS["mixtral47b"], n_layers=1, d=64, F=96, rank=16, n_experts=3),
        "drelu-bf16-i8pred": synth.small(synth.CONFIGS["mistral7b"], n_layers=1, d=64, F=90, rank=16,
                                         pdtype="i8row"),
    }
    cfg = cfgs[name]
    lw = synth.make_layer(cfg, 0, "cpu")
    n = synth.to_numpy

    def ox(e):
        return oracle.Expert(act=cfg.act, wdtype=cfg.wdtype, pdtype=cfg.pdtype, w_gate=n(e.w_gate),
                             w_up=n(e.w_up), w_down=n(e.w_down), c=n(e.c), U=n(e.U), V=n(e.V),
                             s_gate=n(e.s_gate), s_up=n(e.s_up), s_down=n(e.s_down), sU=n(e.sU), sV=n(e.sV))
    router = None if lw.router is None else n(lw.router)
    full = [ox(e) for e in lw.experts]
    r = synth.token_input(cfg, 5).double().numpy()
    ref = oracle.decode_layer(r, full, router)
    for world in (2, 3):
        sh = [tp.shard_neurons(e.freq, world) for e in lw.experts]
        y = np.zeros_like(r)
        for k in range(world):
            part = tp.shard_layer(lw, sh, k)
            res = oracle.decode_layer(r, [ox(e) for e in part.experts], router)
            assert res.experts == ref.experts
            y += res.y
            for slot, e_id in enumerate(ref.experts):    # each shard predicts its own neurons
                assert np.array_equal(res.mask[slot], ref.mask[slot][sh[e_id][k]])
        assert np.allclose(y, ref.y, rtol=1e-12, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = torch.full((8,), float(rank + 1))
        tp.host_all_reduce()(t)
        out[rank] = t.tolist()
    finally:
        dist.destroy_process_group()


def test_host_all_reduce_sums_over_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_gloo_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0] == [3.0] * 8 and out[1] == [3.0] * 8
