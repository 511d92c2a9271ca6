"""The N-GPU path's host logic on CPU: two gloo ranks (127.0.0.1), each with its
own token batch.  No collective touches the data path, so each rank's codes are
exactly what a single process computes for that rank's batch; the timing
collective is a max over ranks; the job's throughput counts every rank's
tokens over the slowest rank's step."""
import os
import socket

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, multirank

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = inputs.WORKLOADS["c1"]
        X = multirank.rank_activations(w, rank, M=8)
        sign, perm = orc.make_rotation(w.K, w.block, 0)
        q = orc.rotate_quantize(inputs.bf16_to_f32(X), w.a_fmt, w.block, sign, perm, None)
        step_ms = 1.0 + rank                      # this rank's (fake) step time
        worst = multirank.max_over_ranks(dist, step_ms)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), codes=q["codes"], scale=q["scale"], X=X,
                 worst=worst, tok=multirank.aggregate_tokens_per_s(8, world, worst))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # each rank saw the max of the per-rank times and the same job throughput
    for r in res:
        assert float(r["worst"]) == 2.0
        assert float(r["tok"]) == pytest.approx(8 * 2 / 2e-3)
    # distinct batches, and each rank's codes equal a single-process run on its batch
    assert not np.array_equal(res[0]["X"], res[1]["X"])
    w = inputs.WORKLOADS["c1"]
    sign, perm = orc.make_rotation(w.K, w.block, 0)
    for rank, r in enumerate(res):
        X = multirank.rank_activations(w, rank, M=8)
        assert np.array_equal(X, r["X"])
        q = orc.rotate_quantize(inputs.bf16_to_f32(X), w.a_fmt, w.block, sign, perm, None)
        assert np.array_equal(q["codes"], r["codes"])
        assert np.array_equal(np.asarray(q["scale"]), r["scale"])


def test_single_process_helpers():
    assert multirank.max_over_ranks(None, 3.5) == 3.5
    assert multirank.aggregate_tokens_per_s(4096, 4, 0.5) == pytest.approx(4096 * 4 / 0.5e-3)
    assert multirank.rank_token_seed(0) != multirank.rank_token_seed(1)
