"""Tensor-parallel shared expert, partial-output contract (TileOPs PR #778,
Partial output contract), on two gloo ranks on the CPU: every rank computes
its shard's partial, SharedFusedMoE.combine all-reduces the partials and adds
the routed output, and both ranks end with bf16(shared expert + routed)."""
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
