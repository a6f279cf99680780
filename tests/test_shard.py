"""N_out-sharded (column-parallel) weight quantization, on CPU with gloo.

gamma is a per-tensor scale ("BitNet b1.58: How Ternary Weights Cut LLM
Memory by 82% Without Losing Accuracy", section "How ternary quantization
works during training"). When a layer's rows are split across ranks, each
rank forms the exact gamma bins of its rows, an all-reduce sums them (integer
sums: exact, independent of order), and each rank quantizes its rows with the
gamma of the whole tensor. This checks that decomposition with the oracle on
two gloo ranks: the summed bins give the unsharded gamma bit for bit, and the
ranks' packed rows are the unsharded packing's rows.
"""

import os
import socket

import numpy as np
import pytest

import oracle
from sparse_linear_layers_fwd_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(rows, k, seed):
    w = synth.latent_weights(rows, k, seed=seed, tag="shard")
    # a few magnitudes far outside the usual window: subnormals, large values
    w[0, :4] = np.array([0x0001, 0x8003, 0x7F00, 0x4400], dtype=np.uint16)
    return w


CASES = [(6, 8, 37, 256, 17), (2, 4, 20, 384, 9), (8, 16, 11, 512, 1), (4, 4, 9, 128, 4)]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        out = []
        for (n, m, rows, k, split) in CASES:
            w = _layer(rows, k, seed=rows)
            lo, hi = (0, split) if rank == 0 else (split, rows)
            shard = w[lo:hi]
            bins = torch.tensor([int(b) for b in oracle.gamma_bins(shard)], dtype=torch.int64)
            dist.all_reduce(bins, op=dist.ReduceOp.SUM)
            gamma = oracle.gamma_from_bins([int(b) for b in bins.tolist()], w.size)
            mask = oracle.nm_mask(shard, n, m)
            codes = oracle.ternary_codes(shard, gamma, mask)
            cb, mb = oracle.pack_weights(codes, mask, n, m)
            out.append((float(gamma), cb, mb))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_sharded_gamma_bins_allreduce_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for ci, (n, m, rows, k, split) in enumerate(CASES):
        w = _layer(rows, k, seed=rows)
        cb, mb, gamma, _, _ = oracle.quantize_weights(w, n, m)
        g0, cb0, mb0 = res[0][ci]
        g1, cb1, mb1 = res[1][ci]
        assert np.float32(g0) == gamma and np.float32(g1) == gamma
        assert np.array_equal(np.concatenate([cb0, cb1]), cb)
        assert np.array_equal(np.concatenate([mb0, mb1]), mb)


def test_gamma_bins_add_over_row_splits():
    # the exact bins are additive over any row split (the property the
    # all-reduce relies on), including splits of a single row
    w = _layer(13, 256, seed=5)
    full = oracle.gamma_bins(w)
    for split in (1, 6, 12):
        a, b = oracle.gamma_bins(w[:split]), oracle.gamma_bins(w[split:])
        assert all(int(x) + int(y) == int(z) for x, y, z in zip(a, b, full))
