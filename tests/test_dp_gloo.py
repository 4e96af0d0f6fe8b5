"""Data-parallel host logic on CPU: two gloo ranks each take their shard of
the rows, compute the LoRA gradients of their shard with the oracle and sum
them with the same all-reduce the GPU benchmark uses; the result equals the
full-batch gradients.  Also the timing reduction (max over ranks)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import oracle
    from lora_fine_tuning_qlora_b200 import dp, inputs
    r, _, w = dp.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    spec = inputs.LayerSpec("dp", M=37, K=48, N=20, r=4, alpha=8.0, act="f32", seed=3)
    d = inputs.layer_inputs(spec)
    Wq, sw = oracle.quantize_weight(d["W"])
    b, e = dp.shard_rows(spec.M, rank, world)
    g = oracle.backward(d["X"][b:e], d["dY"][b:e], Wq, sw, d["A"], d["B"], spec.alpha,
                        want_dx=False)
    flat = torch.from_numpy(np.concatenate([g["dA"].ravel(), g["dB"].ravel(), g["dbias"]]))
    dp.allreduce_grads(flat)
    t = dp.max_over_ranks(float(rank + 1))
    np.save(os.path.join(out_dir, "flat%d.npy" % rank), flat.numpy())
    np.save(os.path.join(out_dir, "t%d.npy" % rank), np.array([t]))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_shard_rows_cover_exactly():
    from lora_fine_tuning_qlora_b200 import dp
    for M in (1, 7, 1024, 1025):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            for a, b in zip(spans, spans[1:]):
                assert a[1] == b[0]
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_gradient_allreduce_matches_full_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import oracle
    from lora_fine_tuning_qlora_b200 import inputs
    spec = inputs.LayerSpec("dp", M=37, K=48, N=20, r=4, alpha=8.0, act="f32", seed=3)
    d = inputs.layer_inputs(spec)
    Wq, sw = oracle.quantize_weight(d["W"])
    g = oracle.backward(d["X"], d["dY"], Wq, sw, d["A"], d["B"], spec.alpha, want_dx=False)
    full = np.concatenate([g["dA"].ravel(), g["dB"].ravel(), g["dbias"]])
    for r in range(world):
        flat = np.load(str(tmp_path / ("flat%d.npy" % r)))
        np.testing.assert_allclose(flat, full, rtol=1e-12, atol=1e-12)
        assert np.load(str(tmp_path / ("t%d.npy" % r)))[0] == world
