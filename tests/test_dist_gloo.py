"""The multi-rank path of bench.py on CPU, two gloo ranks (torchrun's
layout: one process per rank, rendezvous on 127.0.0.1).  Checked: the
max-over-ranks reduction of the timed milliseconds, the whole-job rate
(weak scaling: all ranks' work at the slowest rank's time), that the ranks'
seeded batches differ, that sharding the batch over ranks leaves every
sample's lengths, flags and block mask as one process computes them over the
whole batch (the path has no cross-sample exchange), and that the reference
arm does its work on rank 0 only, the other ranks exiting 0 silently."""
import contextlib
import datetime
import io
import json
import os
import socket
import types

import numpy as np
import torch.multiprocessing as mp

import workloads as W

WORLD = 2


def _wl():
    return W.Workload("dist", S=2, L=512, b=64, w=1, H=4, d=32, dtype="f32", backward=False,
                      entropy=("uniform", 0.2, 0.6), salt=77)


def _mask_stage(x, wl):
    from oracle import deflate1
    from oracle import flags as ofl
    from oracle import mask as om
    ln = deflate1.block_lengths(x, wl.b)
    fl = ofl.literal_flags(ln, wl.b)
    masks = [[om.block_mask(fl[s], wl.w, c).tolist() for c in range(3)] for s in range(x.shape[0])]
    return ln.tolist(), fl.tolist(), masks


def _worker(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    import bench
    wl = _wl()
    res = {"max": bench.max_over_ranks(1.5 + rank, WORLD, "cpu")}
    res["rate"] = bench.whole_job_rate(WORLD, 1e9, res["max"])
    x = bench.rank_inputs(wl, rank)
    res["x"] = x.tolist()
    res["stage"] = _mask_stage(x, wl)
    buf = io.StringIO()
    if rank != 0:
        with contextlib.redirect_stdout(buf):
            res["ref_rc"] = bench.run_reference(types.SimpleNamespace(steps=1, warmup=0), rank, WORLD)
        res["ref_out"] = buf.getvalue()
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as fh:
        json.dump(res, fh)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks(tmp_path):
    ctx = mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=False,
                             start_method="spawn")
    while not ctx.join(timeout=120):
        pass
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(WORLD)]
    assert r[0]["max"] == r[1]["max"] == 2.5
    assert r[0]["rate"] == r[1]["rate"] == 2 * 1e9 / 2.5e-3
    assert r[0]["x"] != r[1]["x"]                      # per-rank seeded batches
    # sharding leaves every sample as one process computes it over the whole batch
    wl = _wl()
    whole = np.concatenate([np.array(r[i]["x"], dtype=np.uint8) for i in range(WORLD)])
    ln, fl, masks = _mask_stage(whole, wl)
    assert ln == r[0]["stage"][0] + r[1]["stage"][0]
    assert fl == r[0]["stage"][1] + r[1]["stage"][1]
    assert masks == r[0]["stage"][2] + r[1]["stage"][2]
    assert r[1]["ref_rc"] == 0 and r[1]["ref_out"] == ""
