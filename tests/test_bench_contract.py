"""bench.py's JSON line contract, checked on the CPU through the reference arm
(the oracle on the host cores) on the tiny workload: one line, every key the
contract names, with the reference arm's own values for e2e and cpu_baseline."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_has_the_contract_keys():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["unit"] == "ms/layer" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["ms_per_step"] == d["value"]
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and isinstance(cb["sample"], str) and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_gpus_flag_starts_that_many_ranks():
    """`python bench.py --gpus 2` (no launcher) starts two ranks itself through
    the torch.distributed launcher; rank 0 alone prints the line, and it
    reports n_gpus 2 (the reference arm on the tiny workload, on the CPU)."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--impl", "reference", "--config", "tiny", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, cwd=ROOT,
                       timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"
    assert d["config"]["parallelism"] == "replicas x2"


def test_gpus_flag_must_match_the_launchers_world_size():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "1",
                        "--impl", "reference", "--config", "tiny", "--steps", "1"],
                       capture_output=True, text=True, cwd=ROOT, timeout=600, env=env)
    assert r.returncode != 0
    assert "must agree" in r.stderr


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_work_model_bytes_match_the_workload_sizes():
    """The algorithmic bytes behind every roofline figure, against the sizes the
    workloads fix: x_perm of Qwen3 / DeepSeek-V3 prefill is 134 / 470 MB
    (P x H bf16), Qwen3's touched gate+up weights 805.3 MB, and y leaves the
    down GEMM as f16e (2 bytes per value plus one exponent byte per 128)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from moe_inputs import get_config
    b = _bench_module()
    for name, xperm_mb in (("qwen3_prefill", 134.2), ("dsv3_prefill", 469.8)):
        cfg = get_config(name)
        ids = np.arange(cfg.T * cfg.top_k).reshape(cfg.T, cfg.top_k) % cfg.E  # every expert
        wm = b.work_model(cfg, ids)
        P = cfg.T * cfg.top_k
        assert wm["touched"] == cfg.E
        assert abs(P * cfg.H * 2 / 1e6 - xperm_mb) < 0.1
        w_gu = cfg.E * 2 * cfg.F * cfg.H * 2
        assert wm["gate_up_bytes"] == w_gu + P * cfg.H * 2 + P * cfg.F * 2
        assert wm["down_bytes"] == cfg.E * cfg.H * cfg.F * 2 + P * cfg.F * 2 + P * cfg.H * 2 + P * (cfg.H // 128)
        assert wm["gate_up_flops"] == 4.0 * P * cfg.H * cfg.F
        assert wm["flops"] == 6.0 * P * cfg.H * cfg.F + 6.0 * cfg.T * cfg.H * cfg.F_shared
    cfg = get_config("qwen3_decode")
    ids = np.arange(cfg.T * cfg.top_k).reshape(cfg.T, cfg.top_k) % cfg.E
    assert abs(b.work_model(cfg, ids)["gate_up_bytes"] - 4096 * 2048 * 2 - 4096 * 768 * 2
               - 805.306368e6) < 1
    # FP8 down: e4m3 weights and their 128x128 block scales, e4m3 h
    cfg = get_config("dsv3_decode_fp8")
    ids = np.arange(cfg.T * cfg.top_k).reshape(cfg.T, cfg.top_k) % cfg.E
    wm = b.work_model(cfg, ids)
    P = cfg.T * cfg.top_k
    w_dn = cfg.E * cfg.H * cfg.F + cfg.E * (cfg.H // 128) * (cfg.F // 128) * 4
    assert wm["down_bytes"] == w_dn + P * cfg.F + P * cfg.H * 2 + P * (cfg.H // 128)
