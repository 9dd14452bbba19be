"""The bench's N > 1 paths on CPU: two gloo ranks run the host logic that
torchrun drives on GPUs (process group, max-over-ranks timing, per-rank
independent batches or one batch split by KV-head groups, whole-job value).
No GPU and no kernel here."""
import json
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "DBSA_DIST_BACKEND": "gloo"})
    import torch.distributed as tdist
    import bench
    from many_shot_icl_b200 import inputs
    w, r, _ = bench.dist_setup()
    # per-rank device time: the job's time is the slowest rank's
    local_t = 1.0 + 0.5 * r
    t_max = bench.max_over_ranks(local_t, w)
    bench.barrier(w)
    wl = inputs.L31_8B_90K
    sels = inputs.selections(wl, seed_offset=r)     # the bench's per-rank batch
    seeds = [inputs.tensor_seed(wl, 0, role) + 7919 * r for role in range(4)]
    res = {"rank": r, "world": w, "t_max": t_max,
           "value": bench.weak_scaling_value(90000, w, t_max),
           "sel0": [int(x) for x in sels[0]], "seeds": seeds}
    with open(os.path.join(out_dir, "rank%d.json" % r), "w") as f:
        json.dump(res, f)
    tdist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    assert [x["rank"] for x in res] == [0, 1] and all(x["world"] == 2 for x in res)
    # max over ranks on every rank, and the weak-scaling value built from it
    assert all(x["t_max"] == 1.5 for x in res)
    assert all(np.isclose(x["value"], 90000 * 2 / 1.5) for x in res)
    # every rank draws its own independent batch: selections and tensor seeds differ
    assert res[0]["sel0"] != res[1]["sel0"]
    assert not set(res[0]["seeds"]) & set(res[1]["seeds"])
    # each selection is a valid one: sink first, unique blocks
    for x in res:
        assert x["sel0"][0] == 0 and len(set(x["sel0"])) == len(x["sel0"])


def _rank_heads(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "DBSA_DIST_BACKEND": "gloo"})
    import torch
    import torch.distributed as tdist
    import bench
    from many_shot_icl_b200 import inputs
    w, r, _ = bench.dist_setup()
    # one small context of the Llama-3.1-8B head geometry, split by KV heads
    wl_shape = inputs.L31_8B_90K.with_(n_blocks=4, demos_per_block=5, n_queries=3,
                                       query_tokens=4, decode_steps=2)
    wl = bench.Workload(wl_shape, 1, "cpu", rank=r, heads=(r, w))
    kv0, kv1, q0, q1 = wl.heads
    # this rank's slices equal the same slices of the whole batch's tensors
    full_q = inputs.randn((wl.T, 32, 128), inputs.tensor_seed(wl_shape, 0, 0), "bf16")
    full_k = inputs.randn((wl.T, 8, 128), inputs.tensor_seed(wl_shape, 0, 1), "bf16")
    full_kt = inputs.randn((wl.nq, wl.tail_cap, 8, 128), inputs.tensor_seed(wl_shape, 0, 3, 2),
                           "bf16")
    t_max = bench.max_over_ranks(2.0 + r, w)
    res = {"rank": r, "heads": [kv0, kv1, q0, q1],
           "cfg": [wl.cfg.n_q_heads, wl.cfg.n_kv_heads],
           "q_slice": bool(torch.equal(wl.q[0], full_q[:, q0:q1])),
           "k_slice": bool(torch.equal(wl.k[0], full_k[:, kv0:kv1])),
           "kt_slice": bool(torch.equal(wl.kt[0], full_kt[:, :, kv0:kv1])),
           "sel": [[int(x) for x in s_] for s_ in wl.sels],
           "value": bench.strong_scaling_value(wl.T, t_max), "T": wl.T, "t_max": t_max}
    with open(os.path.join(out_dir, "heads%d.json" % r), "w") as f:
        json.dump(res, f)
    tdist.destroy_process_group()


def test_two_gloo_ranks_split_one_batch_by_heads(tmp_path):
    """--shard heads: both ranks hold the same batch (same selections, same
    seeds) and each its own KV-head group with the query heads that read it;
    together they cover every head once.  Attention is independent per head,
    so no collective runs on the data path; the job's value is the batch's
    units over the slowest rank's time (strong scaling)."""
    world, port = 2, _free_port()
    mp.start_processes(_rank_heads, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / ("heads%d.json" % r))) for r in range(world)]
    assert [x["heads"] for x in res] == [[0, 4, 0, 16], [4, 8, 16, 32]]
    assert all(x["cfg"] == [16, 4] for x in res)
    assert all(x["q_slice"] and x["k_slice"] and x["kt_slice"] for x in res)
    assert res[0]["sel"] == res[1]["sel"]
    assert all(np.isclose(x["value"], x["T"] / 3.0) and x["t_max"] == 3.0 for x in res)
