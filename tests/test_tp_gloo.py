"""Two gloo ranks on the CPU.
(1) The tensor-parallel shared expert's partial-output contract (TileOPs PR
#778, Partial output contract): every rank computes its shard's partial,
SharedFusedMoE.combine all-reduces the partials and adds the routed output,
and both ranks end with bf16(shared expert + routed).
(2) bench.py's cross-rank steps (barrier, max over ranks, reference arm).
(3) Expert parallelism's all-to-all exchange (ep.TorchDistExchange)."""
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shared_partial_contract_two_ranks(tmp_path):
    from tests._tp_worker import shared_contract_worker
    world = 2
    mp.spawn(shared_contract_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
             join=True)
    outs = [np.load(tmp_path / f"rank{r}.npy") for r in range(world)]
    assert np.array_equal(outs[0], outs[1])


def test_bench_cross_rank_steps_two_ranks(tmp_path):
    """bench.py under two ranks: barrier, max over ranks of the step time, and
    the reference arm returning without work on ranks other than 0."""
    from tests._tp_worker import bench_ranks_worker
    world = 2
    mp.spawn(bench_ranks_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
             join=True)
    vals = [float(np.load(tmp_path / f"bench{r}.npy")[0]) for r in range(world)]
    assert vals == [2.5, 2.5]


def test_ep_exchange_two_ranks(tmp_path):
    """Expert parallelism's all-to-all plumbing (ep.TorchDistExchange) on two
    gloo ranks: uneven and empty splits, and the reverse exchange."""
    from tests._tp_worker import ep_exchange_worker
    world = 2
    mp.spawn(ep_exchange_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
             join=True)
    for r in range(world):
        assert (tmp_path / f"ep{r}.npy").exists()
