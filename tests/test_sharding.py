"""The multi-GPU split of the forward (one process per GPU, no data-path
collective): contiguous batch slices per rank.  Run here with two and three
gloo processes on CPU; each rank computes its slice with the oracle (the CUDA
path needs a GPU), and the gathered slices must equal the unsplit forward for
every bias kind (the bias is shared over the batch, indexed by head)."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bit_qk_attention_ba_b200.sharding import batch_slice, shard_range  # noqa: E402
from bit_qk_attention_ba_b200.workloads import BIAS_KIND, Workload, make_inputs  # noqa: E402


@pytest.mark.parametrize("n,world", [(5, 2), (4, 8), (12, 3), (0, 2), (7, 7), (1, 4)])
def test_slices_cover_every_unit_once(n, world):
    seen = []
    sizes = []
    prev_hi = 0
    for r in range(world):
        lo, hi = shard_range(n, world, r)
        assert lo == prev_hi and lo <= hi          # contiguous, in rank order
        prev_hi = hi
        seen.extend(range(lo, hi))
        sizes.append(hi - lo)
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_bad_arguments_rejected():
    for args in ((4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            shard_range(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = [
    Workload("sh_dense", 5, 2, 23, 16, dtype="f32", bias="dense", bias_std=0.3),
    Workload("sh_relpos", 3, 2, 12, 8, dtype="f32", bias="relpos2d", grid=(3, 4), bias_std=0.3),
    Workload("sh_cls", 4, 3, 13, 8, dtype="f32", bias="relpos2d_cls", grid=(3, 4), bias_std=0.3),
]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        for w in CASES:
            inp = make_inputs(w)
            gh, gw = w.grid
            mine = {n: batch_slice(inp[n], world, rank) for n in ("q", "k", "v")}
            out = O.forward(mine["q"], mine["k"], mine["v"], BIAS_KIND[w.bias], inp["bias"], inp["ld"], gh, gw,
                            nthreads=1)["out"]
            # gather the slices (test only: the product path has no collective)
            sizes = [shard_range(w.B, world, r)[1] - shard_range(w.B, world, r)[0] for r in range(world)]
            buf = np.zeros((max(sizes),) + out.shape[1:])
            buf[:out.shape[0]] = out
            got = [torch.zeros(buf.shape, dtype=torch.float64) for _ in range(world)]
            dist.all_gather(got, torch.from_numpy(buf))
            if rank == 0:
                full = np.concatenate([g.numpy()[:s] for g, s in zip(got, sizes)])
                ref = O.forward(inp["q"], inp["k"], inp["v"], BIAS_KIND[w.bias], inp["bias"], inp["ld"], gh, gw,
                                nthreads=1)["out"]
                q.put((w.name, float(np.abs(full - ref).max()), full.shape == ref.shape))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sliced_forward_equals_unsplit_forward(world):
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in CASES)
    assert [g[0] for g in got] == sorted(w.name for w in CASES)
    for name, err, same_shape in got:
        assert same_shape and err == 0.0, (name, err)
