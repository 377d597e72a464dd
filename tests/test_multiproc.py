"""The data-parallel (weak scaling) path across ranks, on CPU with the gloo backend.

Two ranks each draw their shard of a global batch and run the oracle's sparse path on it;
the union of the shards' supports and outputs must equal the unsharded run, and the
max-over-ranks timing reduction must return the slowest rank's time.  This is the host
logic bench.py uses for --gpus N (the GPU path runs the same shards through libspa.so)."""
import os
import tempfile

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from synth import SMALL, decode_inputs
from synth.shard import batch_range, global_config


def _worker(rank, world, init_file, out_dir):
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank, world_size=world)
    try:
        base = SMALL["c2s"].with_(B=1, N=3000, n_clusters=4)
        gcfg = global_config(base, world)
        x = decode_inputs(gcfg, batch=batch_range(base, rank, world), threads=1)
        res = oracle.decode(base, x, with_output=True)   # the shard alone, as a rank sees it
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"),
                 idx=np.concatenate([r["idx"] for r in res]), counts=np.array([len(r["idx"]) for r in res]),
                 out=np.stack([r["out"] for r in res]))
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)    # each rank's "device time"
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        assert t.item() == float(world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reassemble_the_global_batch():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        init_file = os.path.join(d, "pg")
        mp.spawn(_worker, args=(world, init_file, d), nprocs=world, join=True)
        base = SMALL["c2s"].with_(B=1, N=3000, n_clusters=4)
        gcfg = global_config(base, world)
        full = oracle.decode(gcfg, decode_inputs(gcfg, threads=1))
        per_rank = base.U
        for r in range(world):
            z = np.load(os.path.join(d, f"rank{r}.npz"))
            ref = full[r * per_rank:(r + 1) * per_rank]
            np.testing.assert_array_equal(z["counts"], [len(x["idx"]) for x in ref])
            np.testing.assert_array_equal(z["idx"], np.concatenate([x["idx"] for x in ref]))
            np.testing.assert_allclose(z["out"], np.stack([x["out"] for x in ref]), rtol=0, atol=0)
