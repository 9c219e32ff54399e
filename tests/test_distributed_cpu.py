"""Token-sharded Hessian on CPU ranks (gloo, world size 2): each rank's partial
Hessian of its token share (the oracle stands in for the GPU kernel here), the
all-reduce of scale_calibration_b200.distributed, and the share arithmetic."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from scale_calibration_b200 import distributed as lhd
    dist.init_process_group("gloo", rank=rank, world_size=world)
    counts = [0, 5, 1, 300, 0, 17, 129, 2100]
    layer = synth.make_layer(8, 128, sum(counts), seed=6, n_mats=len(counts), counts=counts)
    t0, t1, loc = lhd.token_shard(layer.n_tok, rank, world, layer.offsets)
    Hl = oracle.hessian(layer.X[t0:t1], c_in=128, offsets=loc).astype(np.float32)

    def add_local(H):
        H += torch.from_numpy(Hl)

    H = torch.zeros(len(counts), 8, 16, 16)
    lhd.sharded_sum(H, add_local)          # from zero
    first = H.numpy().copy()
    lhd.sharded_sum(H, add_local)          # resumed: the same tokens again, entry value counted once
    q.put((rank, first, H.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_allreduce_of_token_shards_gloo_world2():
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    got = [q.get(timeout=300) for _ in ps]
    out = {r: a for r, a, _ in got}
    twice = {r: b for r, _, b in got}
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    counts = [0, 5, 1, 300, 0, 17, 129, 2100]
    layer = synth.make_layer(8, 128, sum(counts), seed=6, n_mats=len(counts), counts=counts)
    Hf = oracle.hessian(layer.X, c_in=128, offsets=layer.offsets)
    for r in (0, 1):
        H = out[r].astype(np.float64)
        assert np.array_equal(out[r], out[0])
        d = np.sqrt(((H - Hf) ** 2).sum(axis=(-1, -2)))
        n = np.sqrt((Hf ** 2).sum(axis=(-1, -2)))
        assert np.all(d <= 1e-6 * np.maximum(n, 1e-30) + (n == 0) * 0)
        assert np.all(H[[0, 4]] == 0)
        H2 = twice[r].astype(np.float64)
        d2 = np.sqrt(((H2 - 2 * Hf) ** 2).sum(axis=(-1, -2)))
        assert np.all(d2 <= 2e-6 * np.maximum(n, 1e-30))


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_token_and_row_shares_partition(world):
    from scale_calibration_b200 import distributed as lhd
    rng = np.random.default_rng(world)
    n = 1001
    off = np.concatenate([[0], np.sort(rng.integers(0, n + 1, 9)), [n]])
    covered = np.zeros(n, int)
    per_group = np.zeros(len(off) - 1, int)
    for r in range(world):
        t0, t1, loc = lhd.token_shard(n, r, world, off)
        covered[t0:t1] += 1
        assert loc[0] >= 0 and loc[-1] <= t1 - t0 and np.all(np.diff(loc) >= 0)
        per_group += np.diff(loc)
        r0, r1 = lhd.row_shard(77, r, world)
        assert 0 <= r0 <= r1 <= 77
    assert np.all(covered == 1)
    assert np.array_equal(per_group, np.diff(off))
    assert sum(lhd.row_shard(77, r, world)[1] - lhd.row_shard(77, r, world)[0] for r in range(world)) == 77
    with pytest.raises(ValueError):
        lhd.token_shard(10, world, world)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("shape", [(1, 4096, 256), (64, 1536, 128), (1, 64, 8), (3, 40, 4)])
def test_sweep_shares_cover_every_block_once(world, shape):
    from scale_calibration_b200 import distributed as lhd
    n_mats, c_out, J = shape
    seen = np.zeros((n_mats, c_out, J), np.int64)
    sizes = []
    for r in range(world):
        kind, lo, hi = lhd.sweep_shard(n_mats, c_out, J, r, world)
        if kind == "mats":
            seen[lo:hi] += 1
            assert n_mats >= world
        elif kind == "cols":
            seen[:, :, lo:hi] += 1
            assert n_mats == 1
        else:
            seen[:, lo:hi] += 1
        sizes.append(int(seen.sum()) - sum(sizes))
    assert np.all(seen == 1)
    unit = {"mats": c_out * J, "cols": c_out, "rows": n_mats * J}[kind]
    assert max(sizes) - min(sizes) <= unit   # shares differ by at most one unit
