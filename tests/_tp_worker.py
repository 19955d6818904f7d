"""Worker of the world-size-2 gloo run in test_tp_gloo.py (spawned processes
import it by module name)."""
import datetime
import os

import numpy as np
import torch
import torch.distributed as dist


def shared_contract_worker(rank: int, world: int, port: int, result_dir: str) -> None:
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from moe_routed_expert_top_b200.layer import SharedFusedMoE
        from oracle import moe_oracle as O
        rng = np.random.default_rng(5)             # the same inputs on every rank
        T, H, F_s = 6, 16, 16
        bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
        x = bf(rng.standard_normal((T, H)))
        wgu = bf(rng.standard_normal((2 * F_s, H)) * 0.3)
        wd = bf(rng.standard_normal((H, F_s)) * 0.3)
        routed = bf(rng.standard_normal((T, H)))
        # this rank's partial (the GPU path's is checked against the same
        # oracle partial rank by rank); combine all-reduces and adds
        part = torch.from_numpy(O.shared_expert_partial(x, wgu, wd, world, rank)).float()
        out = SharedFusedMoE.combine(part, routed, world_size=world)
        full = O.dense_swiglu_mlp(x, wgu, wd)
        assert np.allclose(part.numpy(), full, rtol=1e-5, atol=1e-5)   # reduced in place
        ref = (torch.from_numpy(full).float() + routed.float()).to(torch.bfloat16).float()
        assert torch.all((out.float() - ref).abs() <= ref.abs() * 2.0 ** -7 + 1e-6)
        np.save(os.path.join(result_dir, f"rank{rank}.npy"), out.float().numpy())
    finally:
        dist.destroy_process_group()


def bench_ranks_worker(rank: int, world: int, port: int, result_dir: str) -> None:
    """bench.py's cross-rank steps on gloo: the barrier, the max over ranks of
    a per-rank time, and the reference arm, which only rank 0 runs."""
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        assert got == 1.5 + (world - 1), got
        if rank > 0:
            os.environ["RANK"] = str(rank)
            assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
        bench.barrier(world)
        np.save(os.path.join(result_dir, f"bench{rank}.npy"), np.array([got]))
    finally:
        dist.destroy_process_group()


def ep_exchange_worker(rank: int, world: int, port: int, result_dir: str) -> None:
    """ep.TorchDistExchange on gloo: counts, uneven row splits (one empty),
    and the reverse exchange bringing every row back to its sender in order."""
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from moe_routed_expert_top_b200.ep import TorchDistExchange
        ex = TorchDistExchange()
        send_counts = torch.tensor([[2, 3], [0, 4]][rank], dtype=torch.int32)
        # row value = 100*source + position in the source's send buffer
        send = torch.stack([torch.full((3,), 100.0 * rank + i) for i in range(int(send_counts.sum()))])
        ss, rs = ex.counts(send_counts)
        assert ss == send_counts.tolist()
        assert rs == [[2, 0], [3, 4]][rank]
        recv = ex.rows(send, ss, rs)
        want = {0: [0, 1], 1: [2, 3, 4, 100, 101, 102, 103]}[rank]
        assert recv[:, 0].tolist() == [float(v) for v in want]
        back = ex.rows(recv * 2, rs, ss)                       # the reverse direction
        assert torch.equal(back, send * 2)
        np.save(os.path.join(result_dir, f"ep{rank}.npy"), back.numpy())
    finally:
        dist.destroy_process_group()
