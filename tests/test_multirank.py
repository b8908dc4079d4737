"""The N-GPU benchmark shards independent sequences across ranks with no collective on
the data path.  This checks that host logic on CPU with two gloo ranks: the ranks draw
disjoint sequences, each rank's result equals the matching slice of one single-process
run over the union (the units are independent), and the max-over-ranks time reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, wl_kw, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from long_context_kv_kvc_b200 import synth
    from oracle import oracle as O

    wl = synth.scaled(synth.LLAMA8B_32K, **wl_kw)
    seeds = bench.rank_seeds(wl, rank)
    inp = synth.make_inputs(wl, seeds=seeds)
    ref = O.compress(inp["q"], inp["k"], inp["v"], window=wl.window, n_sink=wl.n_sink,
                     pool_kernel=wl.pool_kernel, kv_budget=wl.kv_budget, threads=1)
    np.save(os.path.join(result_dir, f"idx{rank}.npy"), ref["idx"])
    np.save(os.path.join(result_dir, f"seeds{rank}.npy"), np.array(seeds))
    t = torch.tensor([10.0 * (rank + 1)], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    np.save(os.path.join(result_dir, f"tmax{rank}.npy"), t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_batches(tmp_path):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    wl_kw = dict(B=2, Hq=8, Hkv=2, N=700, kv_budget=120, n_hubs=8)
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), wl_kw, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)

    import bench
    from long_context_kv_kvc_b200 import synth
    from oracle import oracle as O

    wl = synth.scaled(synth.LLAMA8B_32K, **wl_kw)
    s0 = np.load(tmp_path / "seeds0.npy")
    s1 = np.load(tmp_path / "seeds1.npy")
    assert not set(s0) & set(s1)
    # one process over the union of both ranks' sequences
    union = synth.scaled(synth.LLAMA8B_32K, **dict(wl_kw, B=4))
    inp = synth.make_inputs(union, seeds=tuple(s0) + tuple(s1))
    ref = O.compress(inp["q"], inp["k"], inp["v"], window=wl.window, n_sink=wl.n_sink,
                     pool_kernel=wl.pool_kernel, kv_budget=wl.kv_budget)
    assert np.array_equal(np.load(tmp_path / "idx0.npy"), ref["idx"][:2])
    assert np.array_equal(np.load(tmp_path / "idx1.npy"), ref["idx"][2:])
    for r in range(world):
        assert float(np.load(tmp_path / f"tmax{r}.npy")[0]) == 20.0
    assert bench.rank_seeds(wl, 0) == (0, 1) and bench.rank_seeds(wl, 3) == (6, 7)


def test_algorithmic_bytes_of_the_128k_workload():
    import bench
    from long_context_kv_kvc_b200 import synth
    ab = bench.algorithmic_bytes(synth.LLAMA8B_128K_B4)
    assert ab["k_read"] == 1_073_741_824
    assert ab["q_read"] == 1_048_576
    assert ab["gather"] == 134_217_728
    assert ab["idx"] == 524_288
    assert ab["total"] == 1_073_741_824 + 1_048_576 + 134_217_728 + 524_288


def test_clock_summary():
    import bench
    rows = [["0", "1900", "1965", "800.0", "0x0", "Not Active", "Not Active", "Not Active", "Active"],
            ["0", "1800", "1965", "900.0", "0x4", "Not Active", "Not Active", "Not Active", "Not Active"],
            ["0", "600", "1965", "100.0", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]]
    c = bench.summarize_clocks(rows)
    assert c["sm_mhz"] == 1850 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
