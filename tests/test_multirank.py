"""Data-parallel path on two ranks (gloo, CPU): each rank holds a shard of the calibration
tokens, computes the per-channel absmax on its shard, and bench.combine_statistic (an
all-reduce MAX) must give every rank the absmax of the whole batch; the smoothing factors,
weight codes and per-token codes that follow are then identical on every rank and equal to
the unsharded oracle's."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ln, out_dir):
    import torch.distributed as dist

    import bench
    import oracle as O
    import sq_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = sq_inputs.make_case(96, 256, 64, 21, beta_std=0.0)  # same seed -> same batch on every rank
        shard = c.x[rank::world]                                   # this rank's tokens
        local = O.calib_ln_absmax(shard, c.gamma) if ln else O.calib_absmax(shard, 0)
        ax = torch.from_numpy(local.copy())
        bench.combine_statistic(ax, world)
        ax = ax.numpy()
        aw = O.calib_absmax(c.W, 1)
        s = O.smooth_factors(ax, aw, 0.5)
        wq, sw, gf, _ = O.fold_quant_weights(c.W, s, c.gamma if ln else None)
        xq, sx = O.ln_smooth_quant(shard, gamma_f=gf) if ln else O.ln_smooth_quant(shard, s=s)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), ax=ax, s=s, wq=wq, sw=sw, xq=xq, sx=sx)
    finally:
        dist.destroy_process_group()


def _run(ln, tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, ln, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return [dict(np.load(os.path.join(tmp_path, f"r{r}.npz"))) for r in range(world)]


def _check(ln, tmp_path):
    import oracle as O
    import sq_inputs

    res = _run(ln, tmp_path)
    c = sq_inputs.make_case(96, 256, 64, 21, beta_std=0.0)
    ax = O.calib_ln_absmax(c.x, c.gamma) if ln else O.calib_absmax(c.x, 0)
    s = O.smooth_factors(ax, O.calib_absmax(c.W, 1), 0.5)
    wq, sw, gf, _ = O.fold_quant_weights(c.W, s, c.gamma if ln else None)
    xq, sx = O.ln_smooth_quant(c.x, gamma_f=gf) if ln else O.ln_smooth_quant(c.x, s=s)
    for r, got in enumerate(res):
        assert np.array_equal(got["ax"], ax) and np.array_equal(got["s"], s)
        assert np.array_equal(got["wq"], wq) and np.array_equal(got["sw"], sw)
        assert np.array_equal(got["xq"], xq[r::2]) and np.array_equal(got["sx"], sx[r::2])


def test_two_ranks_plain_calibration(tmp_path):
    _check(False, tmp_path)


def test_two_ranks_layernorm_calibration(tmp_path):
    _check(True, tmp_path)
