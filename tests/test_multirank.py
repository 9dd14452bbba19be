"""The bench's N > 1 path on CPU: two gloo ranks run the host logic that
torchrun drives on GPUs (process group, max-over-ranks timing, per-rank
independent batches, whole-job value).  No GPU and no kernel here."""
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
