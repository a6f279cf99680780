"""Host logic of bench.py across ranks, on CPU with the gloo backend.

Each rank of a multi-GPU bench runs its own independent layer (weak
scaling, no collective on the data path); only the timing is combined: the
slowest rank's time, and the units of all ranks over that time.
"""

import importlib.util
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        b = _bench()
        ms_local = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms = b.max_over_ranks(ms_local, world, "cpu")
        value = b.whole_job_value("decode", 100, world, ms)
        data = b.make_layers_data("decode", rank)
        w_head = np.asarray(data[0][0][:2, :8]).copy()
        q.put((rank, ms, value, w_head))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda o: o[0])
    b = _bench()
    for rank, ms, value, _ in out:
        assert ms == 15.0                                   # max over ranks on every rank
        layers = b.WORKLOADS["decode"]["layers"]
        expect = b.step_bytes(layers, b.is_fused("decode")) * 100 * world / (15.0e-3) / 1e9
        assert value == pytest.approx(expect, rel=1e-12)    # all ranks' bytes / slowest time
    # independent inputs per rank
    assert not np.array_equal(out[0][3], out[1][3])


def test_single_rank_is_identity():
    b = _bench()
    assert b.max_over_ranks(3.5, 1, "cpu") == 3.5
    layers = b.WORKLOADS["prefill"]["layers"]
    v = b.whole_job_value("prefill", 10, 1, 2.0)
    assert v == pytest.approx(b.step_ops(layers) * 10 / 2.0e-3 / 1e12)


def test_reference_arm_other_ranks_do_nothing(capsys):
    b = _bench()

    class A:
        workload = "decode"
        steps = 1
        warmup = 3
        reference_seconds = 1.0

    b.run_reference(A(), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_entropy_workload_accounting():
    # the bench's own size formulas against the oracle's format sizes, and
    # the oracle step of the entropy workload on a small layer
    import oracle
    b = _bench()
    for (n, m) in [(2, 4), (6, 8), (8, 16), (4, 4)]:
        for k in (128, 2560):
            assert b.entropy_bytes(3, k, n, m) == 3 * oracle.entropy_row_bytes(k, n, m)
            assert b.packed_bytes(3, k, n, m) == 3 * (oracle.codes_row_bytes(k, n, m) + oracle.meta_row_bytes(k, n, m))
    layers = b.WORKLOADS["decode_entropy"]["layers"]
    assert b.workload_mode("decode_entropy") == "entropy"
    (n_out, k, n, m, ts) = layers[0]
    want = b.qw_bytes(n_out, k, n, m) + b.pe_bytes(n_out, k, n, m) + sum(
        2 * t * k + b.entropy_bytes(n_out, k, n, m) + 4 + 2 * t * n_out for t in ts)
    assert b.step_bytes(layers, "entropy") == want
    from sparse_linear_layers_fwd_b200 import synth
    w = synth.latent_weights(8, 256, seed=1, tag="ent_step")
    x = synth.activations(2, 256, seed=1, tag="ent_step")
    b.oracle_step([(w, [x], 6, 8)], 8, "entropy")
