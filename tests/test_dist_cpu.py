"""World-size-2 tests of the multi-process plumbing on CPU (gloo): max-over-ranks
timing, token sharding, and the two calibration reductions (amax MAX, Hessian SUM)
checked against the oracle on the unsharded input."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch

    import oracle
    from nvfp4_block_numerics_b200 import dist, inputs

    ws, r, _ = dist.init(backend="gloo", timeout_s=60)
    assert (ws, r) == (world, rank)
    # timing: each rank reports its own device times; everyone gets the maxima
    mx = dist.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank])
    # calibration over token shards
    x = inputs.laplace_bf16(inputs.rng_for(5, "dist", "X"), 301, 64, outlier_channels=(9,), outlier_scale=30)
    r0, r1 = dist.shard_rows(x.shape[0], rank, world)
    xs = np.ascontiguousarray(x[r0:r1])
    amax = torch.tensor([oracle.tensor_amax(xs)[0]], dtype=torch.float32)
    dist.allreduce_amax_(amax)
    H = torch.from_numpy(oracle.hessian_accum(xs))
    dist.allreduce_hessian_(H)
    np.savez(os.path.join(out_dir, f"r{rank}.npz"), mx=np.array(mx), amax=amax.numpy(), H=H.numpy(),
             shard=np.array([r0, r1]))
    dist.finalize()


@pytest.mark.timeout(300)
def test_two_rank_reductions(tmp_path, orc):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    from nvfp4_block_numerics_b200 import inputs

    x = inputs.laplace_bf16(inputs.rng_for(5, "dist", "X"), 301, 64, outlier_channels=(9,), outlier_scale=30)
    H_full = orc.hessian_accum(x)
    amax_full = orc.tensor_amax(x)[0]
    res = [np.load(os.path.join(tmp_path, f"r{r}.npz")) for r in range(world)]
    assert [tuple(r["shard"]) for r in res] == [(0, 151), (151, 301)]
    for r in res:
        assert r["mx"].tolist() == [2.0, 5.0, 0.25]
        assert float(r["amax"][0]) == amax_full
        # sum of the two partial Hessians: the same exact products, summed in another order
        assert np.abs(r["H"] - H_full).max() <= 1e-12 * np.abs(H_full).max()


def test_shard_rows_cover_exactly():
    from nvfp4_block_numerics_b200 import dist

    for n in (0, 1, 7, 16384):
        for w in (1, 2, 3, 8):
            spans = [dist.shard_rows(n, r, w) for r in range(w)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1


def test_single_process_is_a_no_op():
    import torch

    from nvfp4_block_numerics_b200 import dist

    assert not dist.active()
    assert dist.max_over_ranks([3.0, 1.0]) == [3.0, 1.0]
    t = torch.ones(3)
    assert dist.allreduce_hessian_(t) is t and t.sum().item() == 3.0
