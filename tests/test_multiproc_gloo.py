"""The multi-GPU host path, on the CPU: two ranks over gloo.

The layer shards by sequence with no data-path collective (each rank runs its
own sequences; only the step time crosses ranks, as the maximum over ranks).
These tests start two processes with a gloo process group on 127.0.0.1 and
check, without a GPU:
  - that `batch_shard` covers a global batch exactly once, in order, and that
    the fp64 oracle run on each rank's shard and gathered on rank 0 equals
    the oracle run on the whole batch bit for bit (sequences are
    independent, so sharding cannot change a result);
  - that `max_over_ranks` returns the slowest rank's time on every rank;
  - the weak-scaling aggregate the bench reports.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2
B_GLOBAL = 5   # not a multiple of the world size: the shards differ in size


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_args(inp, s, lo, hi):
    """The oracle's layer arguments for sequences [lo, hi) of a batch."""
    cut = lambda t: None if t is None else t[lo:hi].double().numpy()   # noqa: E731
    return (cut(inp["xBC"]), inp["w"].double().numpy(), None, cut(inp["conv_state"]),
            cut(inp["dt_raw"]), inp["A"].double().numpy(), inp["dt_bias"].double().numpy(),
            inp["D"].double().numpy(), cut(inp["init_state"]), s.H, s.P, s.G, s.N)


def _worker(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from ssd_selective_scan_b200 import shard, synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        s = synth.CONFIGS[0].with_(b=B_GLOBAL, L=96)
        inp = synth.layer_inputs(s, 1234, conv_state=True, init_state=True)
        lo, hi = shard.batch_shard(B_GLOBAL, rank, WORLD)
        y, fs, cs = oracle.layer_prefill(*_layer_args(inp, s, lo, hi), nthreads=1)
        # gather the shards (padded to the largest shard) on every rank
        n_max = -(-B_GLOBAL // WORLD)
        def gather(a):
            pad = np.zeros((n_max,) + a.shape[1:], dtype=a.dtype)
            pad[: a.shape[0]] = a
            t = torch.from_numpy(pad)
            parts = [torch.empty_like(t) for _ in range(WORLD)]
            dist.all_gather(parts, t)
            sizes = [shard.batch_shard(B_GLOBAL, r, WORLD) for r in range(WORLD)]
            return np.concatenate([p.numpy()[: b - a_] for p, (a_, b) in zip(parts, sizes)])
        y_all, fs_all, cs_all = gather(y), gather(fs), gather(cs)
        # the slowest rank's time, as the bench takes it
        t_max = shard.max_over_ranks(10.0 + rank)
        if rank == 0:
            np.savez(os.path.join(out_dir, "gathered.npz"), y=y_all, fs=fs_all, cs=cs_all,
                     t_max=np.array([t_max]))
        else:
            np.savez(os.path.join(out_dir, f"tmax{rank}.npz"), t_max=np.array([t_max]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_batch_shard_covers_the_batch_once():
    sys.path.insert(0, ROOT)
    from ssd_selective_scan_b200 import shard
    for b in range(0, 12):
        for world in range(1, 6):
            spans = [shard.batch_shard(b, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == b
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.batch_shard(4, 2, 2)


def test_aggregate_is_all_ranks_tokens_over_the_slowest_step():
    sys.path.insert(0, ROOT)
    from ssd_selective_scan_b200 import shard
    assert shard.aggregate_tokens_per_s(16384, 1, 1.0) == pytest.approx(16384e3)
    assert shard.aggregate_tokens_per_s(16384, 8, 2.0) == pytest.approx(8 * 16384 / 2e-3)
    assert shard.rank_seed(20260001, 3) == 20260004
    assert shard.max_over_ranks(3.5) == 3.5   # no process group: identity


def test_two_gloo_ranks_shard_the_layer_without_changing_it(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True, start_method="spawn")
    got = np.load(tmp_path / "gathered.npz")

    sys.path.insert(0, ROOT)
    import oracle
    from ssd_selective_scan_b200 import synth
    s = synth.CONFIGS[0].with_(b=B_GLOBAL, L=96)
    inp = synth.layer_inputs(s, 1234, conv_state=True, init_state=True)
    y, fs, cs = oracle.layer_prefill(*_layer_args(inp, s, 0, B_GLOBAL), nthreads=1)
    assert np.array_equal(got["y"], y)
    assert np.array_equal(got["fs"], fs)
    assert np.array_equal(got["cs"], cs)
    # every rank saw the slowest rank's time
    assert got["t_max"][0] == 10.0 + WORLD - 1
    for r in range(1, WORLD):
        assert np.load(tmp_path / f"tmax{r}.npz")["t_max"][0] == 10.0 + WORLD - 1
