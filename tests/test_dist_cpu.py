"""World-size-2 gloo checks of the replica host logic (no GPU): the unit
split partitions the work exactly, the timing reduction takes the maximum,
and two ranks that each run the oracle on their shard of the row blocks
reproduce the single-process result."""
import math
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from block_skipping_softmax_b200.replicas import shard_units


def test_shard_units_partitions():
    for n in (0, 1, 7, 64, 1000):
        for world in (1, 2, 3, 8):
            parts = [list(shard_units(n, r, world)) for r in range(world)]
            flat = [u for p in parts for u in p]
            assert flat == list(range(n))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import oracle
    from block_skipping_softmax_b200 import inputs
    from block_skipping_softmax_b200.replicas import max_over_ranks, shard_units

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = max_over_ranks(float(rank + 1))
        Q, K, V = inputs.prefill_inputs(1, 4, 2, 256, 64, seed=3, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
        units = [(0, h, rb) for h in range(4) for rb in range(4)]
        mine = [units[i] for i in shard_units(len(units), rank, world)]
        r = oracle.prefill(Q, K, V, True, 2.0, 64, 64, units=mine, want_exact=False, nthreads=1)
        np.save(os.path.join(os.environ["BSS_TEST_DIR"], f"O{rank}.npy"), r["O"])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    os.environ["BSS_TEST_DIR"] = str(tmp_path)
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == 2.0 and out[1] == 2.0
    import oracle
    from block_skipping_softmax_b200 import inputs

    Q, K, V = inputs.prefill_inputs(1, 4, 2, 256, 64, seed=3, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    full = oracle.prefill(Q, K, V, True, 2.0, 64, 64, want_exact=False)["O"]
    merged = np.where(np.isnan(np.load(tmp_path / "O0.npy")), np.load(tmp_path / "O1.npy"),
                      np.load(tmp_path / "O0.npy"))
    np.testing.assert_array_equal(merged, full)
