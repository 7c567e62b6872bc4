"""World-size-2 gloo tests of the data-parallel path (CPU, no GPU).

Each rank takes its own batch shard (same W, rank-seeded data), computes its
gradients (here with the fp64 oracle), and all-reduces dW; the result must
equal the oracle's dW over the concatenated global batch, and the per-row
gradients must equal the matching rows of the global computation.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from non_linear_matrix_persistent_b200 import Workload
from non_linear_matrix_persistent_b200.inputs import make_shard_inputs

W0 = Workload("dp", B=2, H=2, T=9, K=4, V=6, h0_range=0.5, backward=True, seed=3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from non_linear_matrix_persistent_b200 import parallel
    from oracle import oracle
    r, ws = parallel.init("gloo", timeout_s=60)
    assert (r, ws) == (rank, world)
    x = make_shard_inputs(W0, rank)
    g = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dY"], nthreads=1)
    dW = torch.from_numpy(g["dW"])
    parallel.allreduce_dW(dW)
    t_max = parallel.max_over_ranks(float(rank + 1))
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), dW=dW.numpy(), dk=g["dk"], t_max=t_max)
    import torch.distributed as dist
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_dW_allreduce_matches_global_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    from oracle import oracle
    shards = [make_shard_inputs(W0, r) for r in range(world)]
    assert torch.equal(shards[0]["W"], shards[1]["W"])
    assert not torch.equal(shards[0]["k"], shards[1]["k"])
    cat = {n: torch.cat([s[n] for s in shards]) for n in ("k", "v", "q", "f", "H0", "dY")}
    g = oracle.backward(cat["k"], cat["v"], cat["q"], cat["f"], shards[0]["W"], cat["H0"], cat["dY"])
    for r in range(world):
        res = np.load(os.path.join(str(tmp_path), "rank%d.npz" % r))
        np.testing.assert_allclose(res["dW"], g["dW"], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(res["dk"], g["dk"][r * W0.B:(r + 1) * W0.B])
        assert float(res["t_max"]) == float(world)


# ---------------------------------------------------------------- heads sharded
# Topology-aware tensor parallelism: each rank holds whole k / q head groups and
# their heads; nothing is exchanged, and the ranks' results are slices of the
# single-process result.

W_TP = Workload("tp", B=2, H=4, T=7, K=4, V=6, h0_range=0.5, backward=True, qk_heads=2, seed=8)


def _tp_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from non_linear_matrix_persistent_b200 import make_inputs, parallel
    from oracle import oracle
    r, ws = parallel.init("gloo", timeout_s=60)
    x = parallel.head_shard(make_inputs(W_TP), r, ws)
    y, HT = oracle.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], nthreads=1)
    g = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dY"], nthreads=1)
    np.savez(os.path.join(out_dir, "tp%d.npz" % r), y=y, HT=HT, **g)
    import torch.distributed as dist
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_head_shards_need_no_exchange(tmp_path):
    from non_linear_matrix_persistent_b200 import make_inputs
    from oracle import oracle
    world = 2
    mp.start_processes(_tp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    x = make_inputs(W_TP)
    y, HT = oracle.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], nthreads=1)
    g = oracle.backward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], x["dY"], nthreads=1)
    res = [np.load(os.path.join(str(tmp_path), "tp%d.npz" % r)) for r in range(world)]
    for n, ref in dict(y=y, HT=HT, dv=g["dv"], df=g["df"], dH0=g["dH0"], dk=g["dk"], dq=g["dq"]).items():
        np.testing.assert_array_equal(np.concatenate([r[n] for r in res], axis=1), ref, err_msg=n)
    np.testing.assert_array_equal(np.concatenate([r["dW"] for r in res], axis=0), g["dW"])


def test_head_shard_rejects_uneven_groups():
    from non_linear_matrix_persistent_b200 import make_inputs, parallel
    x = make_inputs(W_TP.with_(qk_heads=0, H=3, backward=False))
    with pytest.raises(ValueError):
        parallel.head_shard(x, 0, 2)
    s = parallel.head_shard(make_inputs(W_TP), 1, 2)
    assert s["k"].shape[1] == 1 and s["v"].shape[1] == 2 and s["W"].shape[0] == 2
