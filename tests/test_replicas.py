"""The multi-GPU path (independent replicas, one process per GPU) on CPU ranks:
the same bookkeeping code as bench.py, over gloo with world size 2."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from video_diffusion_transformer_adaln_b200 import replicas, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir, fail_rank):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w, _ = replicas.init("gloo", timeout_s=5)
    res = {"rank": r, "world": w}
    try:
        if rank == fail_rank:
            raise RuntimeError("planted failure on this rank")  # leaves before any collective
        replicas.barrier(w)
        res["max"] = replicas.max_over_ranks(rank + 1.0, w)
        res["sum"] = replicas.sum_over_ranks(rank + 1.0, w)
        res["tput"] = replicas.throughput(100 * (rank + 1), 10.0 * (rank + 1), w)
        res["seed"] = replicas.latent_seed(r)
        wl = synth.WORKLOADS["d256_L512"]
        res["x0"] = int(synth.x_input(wl, res["seed"])[0, 0, 0])
    except Exception as e:  # the surviving rank's collective must end with an error, not hang
        res["error"] = type(e).__name__
    np.save(os.path.join(out_dir, f"r{rank}.npy"), res, allow_pickle=True)


def _run(tmp_path, fail_rank=-1):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, str(tmp_path), fail_rank)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode is not None, "a rank did not finish"
    return [np.load(os.path.join(tmp_path, f"r{r}.npy"), allow_pickle=True).item() for r in range(2)]


def test_two_ranks_reduce_and_draw_independent_latents(tmp_path):
    res = _run(tmp_path)
    for r in res:
        assert "error" not in r, r
        assert r["world"] == 2
        assert r["max"] == 2.0 and r["sum"] == 3.0
        # whole-job tokens/s: all ranks' tokens over the slowest rank's time
        assert r["tput"] == pytest.approx(300 / 0.020)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["x0"] != res[1]["x0"]  # different latents per rank


def test_a_failed_rank_ends_the_others_collective_with_an_error(tmp_path):
    res = _run(tmp_path, fail_rank=1)
    assert res[1]["error"] == "RuntimeError"
    assert "error" in res[0]  # the barrier / reduction times out instead of hanging
