"""Benchmark of the routed-experts forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl b200|reference]

One step = one ``moe_experts_forward`` call (dispatch tables + permute gather,
grouped gate+up GEMM with the SwiGLU(+FP8) epilogue, grouped down GEMM,
weighted unpermute, plus the shared expert where the workload has one) over one
batch of seeded synthetic inputs already resident in HBM. L2 is flushed (a
512 MiB write) before every timed step, outside the timed events. Each rank
runs the same workload on its own GPU (weak scaling; the path needs no
exchange). Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle on the host cores on a bounded
sample of the same workload (there is no installable reference program).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import CONFIGS, get_config, make_hidden, make_logits, make_weights  # noqa: E402

METRIC = "routed-experts fwd ms/layer + TFLOPS, % of B200 roofline (1 GPU)"
# the largest single-GPU workload: DeepSeek-V3-style prefill (T 4096, E 256, k 8,
# H 7168, F 2048, sigmoid routing, routed_scaling_factor 2.5, shared expert 2048)
DEFAULT_CONFIG = "dsv3_prefill"
# TileOPs PR #1580 (H200, bf16) experts-forward times for the same model families
PAGE_MS = {"qwen3_decode": 3.219, "qwen3_prefill": 6.778, "dsv3_decode_fp8": None,
           "dsv3_prefill": 9.465}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def sources_sha256(files) -> str:
    """Hash of the named CUDA source files (paths relative to the package's
    csrc/): a recorded ncu traffic figure is only valid for the exact kernel
    sources it was measured on."""
    import hashlib
    d = os.path.join(ROOT, "moe_routed_expert_top_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(files):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in profiles/roofline_traffic.json for this workload's dominant
    kernel, or None if absent or if any source file of that kernel (listed in
    the record) changed since."""
    p = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(workload)
    if not rec or rec.get("kernel") != kernel or not rec.get("sources"):
        return None
    try:
        if rec.get("source_sha256") != sources_sha256(rec["sources"]):
            return None
    except OSError:
        return None
    return rec.get("traffic_bytes")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------------------
# algorithmic work: FLOPs 6*T*k*H*F (+ 6*T*H*F_s shared); bytes = touched experts'
# weights + hidden in + out + ids/weights; intermediates are implementation traffic
# ---------------------------------------------------------------------------

def work_model(cfg, ids: np.ndarray) -> dict:
    T, H, F, k = cfg.T, cfg.H, cfg.F, cfg.top_k
    P = T * k
    touched = int(np.unique(ids).size)
    flops_routed = 6.0 * P * H * F
    flops_shared = 6.0 * T * H * cfg.F_shared
    w_gu = touched * 2 * F * H * 2
    if cfg.down_fp8:
        w_dn = touched * H * F * 1 + touched * (H // 128) * (F // 128) * 4
    else:
        w_dn = touched * H * F * 2
    w_sh = (3 * H * cfg.F_shared * 2) if cfg.F_shared else 0
    act = T * H * 2 * 2 + P * 8
    total_bytes = w_gu + w_dn + w_sh + act
    # gate+up kernel alone: its weights, its A rows (x_perm), its h output
    gu_bytes = w_gu + P * H * 2 + P * F * (1 if cfg.down_fp8 else 2) + (P * (F // 128) * 4 if cfg.down_fp8 else 0)
    # the down GEMM writes y in the f16e format (fp16 + an int8 per 128 columns),
    # as the forward does on every workload here (its tilings all store f16e)
    y_bytes = P * H * 2 + P * (H // 128)
    dn_bytes = w_dn + P * F * (1 if cfg.down_fp8 else 2) + y_bytes
    return dict(touched=touched, flops=flops_routed + flops_shared, flops_routed=flops_routed,
                bytes=total_bytes, gate_up_bytes=gu_bytes, gate_up_flops=4.0 * P * H * F,
                down_bytes=dn_bytes, down_flops=2.0 * P * H * F)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smmax=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                     hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        pmax = max(r["power"] for r in rows)
        loaded = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smmax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(loaded)}


# ---------------------------------------------------------------------------
# the b200 arm
# ---------------------------------------------------------------------------

def build_layer(cfg, device):
    import moe_routed_expert_top_b200 as M
    from moe_routed_expert_top_b200.layer import RoutedExperts
    w = make_weights(cfg, device)
    layer = RoutedExperts(w["w_gate_up"], w["w_down"], cfg.top_k, cfg.score_fn, cfg.renormalize,
                          cfg.routed_scaling_factor, cfg.down_fp8, w.get("ws_gate_up"),
                          w.get("ws_down"))
    del w
    hidden = make_hidden(cfg, device)
    logits = torch.from_numpy(make_logits(cfg)).to(device)
    ids, weights = layer.route(logits)       # a1 on the GPU (bit-exact with the oracle)
    torch.cuda.synchronize()
    return M, layer, hidden, ids, weights, logits


def time_steps(fn, steps, flush, stream):
    """Per-step CUDA-event times (ms) of fn(), with an L2 flush before each."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def stage_breakdown(M, layer, cfg, hidden, ids, weights, steps, flush):
    """Device time of each stage launched alone through the C entry points on
    the same workspace: tables+gather, gate+up GEMM, down GEMM, (shared), unpermute."""
    prob = layer.problem(cfg.T)
    T = cfg.T
    ws = layer.workspace(T, hidden.device)
    L = M.moe_get_tables_layout(prob)
    dev = hidden.device
    P = L["P"]
    tables = torch.empty(L["total_int32"], dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    x_perm = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=dev)
    if cfg.down_fp8:
        h = torch.empty(P, cfg.F, dtype=torch.uint8, device=dev)
        hs = torch.empty(P, cfg.F // 128, dtype=torch.float32, device=dev)
    else:
        h = torch.empty(P, cfg.F, dtype=torch.bfloat16, device=dev)
        hs = None
    # y as the forward keeps it: f16e (every workload's down tiling stores it)
    f16e = True
    y = torch.empty(P, cfg.H, dtype=torch.float16 if f16e else torch.float32, device=dev)
    y_exp = torch.empty(P, cfg.H // 128, dtype=torch.int8, device=dev) if f16e else None
    out = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
    addend = None
    if cfg.F_shared:
        sh = torch.empty(T, cfg.F_shared, dtype=torch.bfloat16, device=dev)
        addend = torch.empty(T, cfg.H, dtype=torch.float32, device=dev)
    del ws
    stages = {
        "route_permute": lambda: M.moe_route_permute(prob, None, ids, None, hidden, x_perm,
                                                     tables, status),
        "gate_up_gemm": lambda: M.moe_grouped_gemm(
            prob, 0, 2 * cfg.F, cfg.H, x_perm, None, layer.w_gate_up, None, tables,
            M.MOE_EPI_SWIGLU_FP8 if cfg.down_fp8 else M.MOE_EPI_SWIGLU, h, hs, None, status),
        "down_gemm": lambda: M.moe_grouped_gemm(
            prob, 0, cfg.H, cfg.F, h, hs, layer.w_down, layer.w_down_scales, tables,
            M.MOE_EPI_STORE_F16E if f16e else M.MOE_EPI_STORE_F32, y, y_exp, None, status),
    }
    if cfg.F_shared:
        stages["shared_gate_up_gemm"] = lambda: M.moe_grouped_gemm(
            None, T, 2 * cfg.F_shared, cfg.H, hidden, None, layer.ws_gate_up, None, None,
            M.MOE_EPI_SWIGLU, sh, None, None, status)
        stages["shared_down_gemm"] = lambda: M.moe_grouped_gemm(
            None, T, cfg.H, cfg.F_shared, sh, None, layer.ws_down, None, None,
            M.MOE_EPI_STORE_F32, addend, None, None, status)
    if f16e:
        stages["unpermute"] = lambda: M.moe_unpermute_f16e(prob, y, y_exp, tables, weights,
                                                           cfg.routed_scaling_factor, addend, out)
    else:
        stages["unpermute"] = lambda: M.moe_unpermute(prob, y, tables, weights,
                                                      cfg.routed_scaling_factor, addend, out)
    stream = torch.cuda.current_stream()
    res = {}
    for name, fn in stages.items():
        for _ in range(3):
            fn()
        ts = time_steps(fn, steps, flush, stream)
        res[name] = statistics.median(ts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return res


def run_b200(args, cfg, rank, world, device):
    M, layer, hidden, ids, weights, logits = build_layer(cfg, device)
    peaks = load_peaks()
    wm = work_model(cfg, ids.cpu().numpy())
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream()

    def step():
        layer.forward(hidden, ids, weights, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert layer.device_status() == 0, "device status flag set"
    launches_per_step = M.moe_last_launch_count()
    # eager: one C call per step (its launches go out one by one)
    eager = time_steps(step, max(3, min(args.steps, 50)), flush, stream)
    eager_ms = max_over_ranks(sum(eager) / len(eager), world, device)
    timed = step
    if not args.no_graph:
        # the same forward captured once as a CUDA graph and replayed per step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        timed = graph.replay

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else int(os.environ.get("LOCAL_RANK", 0))) as clk:
        t0 = time.perf_counter()
        times = time_steps(timed, args.steps, flush, stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    barrier(world)
    assert layer.device_status() == 0, "device status flag set"
    ms = sum(times) / len(times)
    ms = max_over_ranks(ms, world, device)
    clocks = clk.summary()

    # end to end through the public call with host buffers: every step copies
    # its inputs from pinned host memory and reads its output back.
    hid_h = hidden.cpu().pin_memory()
    ids_h = ids.cpu().pin_memory()
    w_h = weights.cpu().pin_memory()
    out_h = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hid_d = [torch.empty_like(hidden) for _ in range(2)]
    ids_d = [torch.empty_like(ids) for _ in range(2)]
    w_d = [torch.empty_like(weights) for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]

    # (a) serial: copy in, forward, copy out on one stream, L2 flushed per step
    def e2e_step():
        hid_d[0].copy_(hid_h, non_blocking=True)
        ids_d[0].copy_(ids_h, non_blocking=True)
        w_d[0].copy_(w_h, non_blocking=True)
        layer.forward(hid_d[0], ids_d[0], w_d[0], out)
        out_h[0].copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    e2e_times = time_steps(e2e_step, max(3, min(args.steps, 50)), flush, stream)
    e2e_serial_ms = max_over_ranks(sum(e2e_times) / len(e2e_times), world, device)

    # (b) pipelined, as a serving loop runs it: an input-copy stream and an
    # output-copy stream overlap step i+1's inputs and step i-1's output with
    # step i's forward (device inputs and outputs double-buffered; events keep
    # a buffer from being overwritten before its forward, or its read-back, is
    # done). Timed from the first copy to the last read-back with device events.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    # the forward on each buffer pair, captured once as a CUDA graph (as the
    # device-time figure replays it), unless --no-graph
    fwd = [lambda b=b: layer.forward(hid_d[b], ids_d[b], w_d[b], out_d[b]) for b in range(2)]
    if not args.no_graph:
        graphs = []
        for b in range(2):
            hid_d[b].copy_(hidden)
            ids_d[b].copy_(ids)
            w_d[b].copy_(weights)
            fwd[b]()
            torch.cuda.synchronize()
            g_b = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_b):
                fwd[b]()
            graphs.append(g_b)
        torch.cuda.synchronize()
        fwd = [g.replay for g in graphs]

    def run_e2e(n, start=None):
        ev_fw, ev_out = [None, None], [None, None]
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i == 0 and start is not None:
                    s_in.wait_event(start)
                if ev_fw[b] is not None:
                    s_in.wait_event(ev_fw[b])        # forward i-2 has read these inputs
                hid_d[b].copy_(hid_h, non_blocking=True)
                ids_d[b].copy_(ids_h, non_blocking=True)
                w_d[b].copy_(w_h, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if ev_out[b] is not None:
                stream.wait_event(ev_out[b])         # output i-2 has been read back
            fwd[b]()
            ev_fw[b] = torch.cuda.Event()
            ev_fw[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_fw[b])
                out_h[b].copy_(out_d[b], non_blocking=True)
                ev_out[b] = torch.cuda.Event()
                ev_out[b].record(s_out)
        for e in ev_out:
            if e is not None:
                stream.wait_event(e)

    run_e2e(3)
    torch.cuda.synchronize()
    n_e2e = max(3, min(args.steps, 50))
    barrier(world)
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    run_e2e(n_e2e, start=e_start)
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / n_e2e, world, device)
    assert torch.equal(out_h[(n_e2e - 1) & 1], out.cpu()), "end-to-end output differs"

    # stage breakdown and the dominant kernel's roofline
    stages = stage_breakdown(M, layer, cfg, hidden, ids, weights, max(5, min(args.steps, 30)),
                             flush)
    # top-k routing from the router logits (a1), timed on its own: the forward
    # takes the routing as input
    r_ids = torch.empty_like(ids)
    r_w = torch.empty_like(weights)
    prob_r = layer.problem(cfg.T)
    route = lambda: M.moe_route_topk(prob_r, logits, r_ids, r_w)
    for _ in range(3):
        route()
    routing_ms = statistics.median(time_steps(route, max(5, min(args.steps, 30)), flush, stream))
    dom = max(("gate_up_gemm", "down_gemm"), key=lambda s: stages[s])
    dom_bytes = wm["gate_up_bytes"] if dom == "gate_up_gemm" else wm["down_bytes"]
    dom_flops = wm["gate_up_flops"] if dom == "gate_up_gemm" else wm["down_flops"]
    t_dom = stages[dom] * 1e-3
    hbm = peaks["hbm_gbs"]
    bf16 = peaks.get("bf16_tflops", 1590.0)
    t_b = dom_bytes / (hbm * 1e9)
    t_f = dom_flops / (bf16 * 1e12)
    if t_b >= t_f:
        roof = {"bound": "hbm", "achieved": round(dom_bytes / t_dom / 1e9, 1), "peak": hbm,
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": round(dom_flops / t_dom / 1e12, 1), "peak": bf16,
                "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["traffic"] = recorded_traffic(cfg.name, dom)
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"]

    t_s = ms * 1e-3
    t_flop = wm["flops"] / (bf16 * 1e12)
    t_byte = wm["bytes"] / (hbm * 1e9)
    fwd_roof = {"t_flop_us": round(t_flop * 1e6, 1), "t_byte_us": round(t_byte * 1e6, 1),
                "frac": round(max(t_flop, t_byte) / t_s, 4),
                "bound": "hbm" if t_byte >= t_flop else "tensor",
                "algorithmic_bytes": wm["bytes"], "flops": wm["flops"],
                "touched_experts": wm["touched"]}
    tflops = world * wm["flops"] / t_s / 1e12
    h2d = hidden.numel() * 2 + ids.numel() * 4 + weights.numel() * 4
    d2h = out.numel() * 2
    page = PAGE_MS.get(cfg.name)
    line = {
        "metric": METRIC, "value": round(ms, 4), "unit": "ms/layer", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": False, "scaling": "weak",
        "vs_baseline": round(ms / page, 4) if page else None,
        "tflops": round(tflops, 2), "dtype": "bf16+e4m3" if cfg.down_fp8 else "bf16",
        "data": "synthetic",
        "config": config_dict(cfg, world),
        "roofline": roof, "forward_roofline": fwd_roof,
        "stages_ms": {k: round(v, 4) for k, v in stages.items()},
        "routing_ms": round(routing_ms, 4),
        "tflops_routed": round(world * wm["flops_routed"] / t_s / 1e12, 2),
        "launch": "cuda graph replay of moe_experts_forward" if not args.no_graph
                  else "eager moe_experts_forward calls",
        "eager_ms": round(eager_ms, 4),
        "e2e": {"value": round(e2e_ms, 4), "unit": "ms/layer", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "pipelined: every step copies its inputs from pinned host memory and "
                       "reads its output back on copy streams that overlap the neighbouring "
                       "steps' forwards (" + ("eager calls" if args.no_graph else
                                              "a CUDA graph of the forward per buffer") +
                       "); no L2 flush (the weights exceed L2)",
                "serial": round(e2e_serial_ms, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks, "wall_s": round(wall, 3),
    }
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget_s)
    return line


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg / reference arm)
# ---------------------------------------------------------------------------

class OracleRunner:
    """The CPU oracle (as it stands) on the workload.

    Small workloads run whole: ``O.experts_forward`` over every token. Larger
    ones run a sample of experts: routing and the dispatch tables over all T
    tokens, then the oracle's per-expert step (``O.expert_mlp``, which
    ``experts_forward`` runs once per expert on that expert's rows) over ALL
    the rows of S seeded experts out of the ``touched`` ones, its time scaled
    by touched / S; the slot-order weighted sum over the pairs (O(P*H), far
    below 0.1% of the work) is left out of the timing. Expert weights have the
    workload's shapes and distribution (seeded N(0, 0.02) bf16, each drawn when
    first needed and kept; FP8 down weights quantised by the oracle when
    drawn, like the offline preparation the forward takes as given); drawing
    them is not timed."""

    FULL_FLOPS = 5e10   # workloads up to this many routed FLOPs run whole

    def __init__(self, cfg):
        from oracle import moe_oracle as O
        self.O = O
        self.cfg = cfg
        self.threads = torch.get_num_threads()
        try:
            import threadpoolctl
            info = threadpoolctl.threadpool_info()
            self.threads = max([i.get("num_threads", 1) for i in info] + [1])
        except Exception:
            pass
        self.score = O.SOFTMAX if cfg.score_fn == "softmax" else O.SIGMOID
        self.logits = make_logits(cfg)
        self.hidden = make_hidden(cfg, "cpu")
        self.X = O.as_f64(self.hidden)
        ids, _ = O.route_topk(self.logits, cfg.top_k, self.score, cfg.renormalize)
        self.touched = np.unique(ids)
        self.small = 6.0 * cfg.T * cfg.top_k * cfg.H * cfg.F <= self.FULL_FLOPS
        self.cache = {}
        self.shared = {}
        if cfg.F_shared:
            g = torch.Generator().manual_seed(7)
            self.shared = dict(
                ws_gate_up=(torch.randn(2 * cfg.F_shared, cfg.H, generator=g) * 0.02).to(torch.bfloat16),
                ws_down=(torch.randn(cfg.H, cfg.F_shared, generator=g) * 0.02).to(torch.bfloat16))
        # seeded order in which experts enter the sample
        self.order = np.random.default_rng(cfg.seed + 99).permutation(self.touched)

    def _weights(self, e):
        e = int(e)
        if e not in self.cache:
            cfg = self.cfg
            g = torch.Generator().manual_seed(2000 + 977 * e)
            wgu = (torch.randn(2 * cfg.F, cfg.H, generator=g) * 0.02).to(torch.bfloat16)
            wd = (torch.randn(cfg.H, cfg.F, generator=g) * 0.02).to(torch.bfloat16)
            q = s = None
            if cfg.down_fp8:
                w32 = wd.float().numpy()
                parts = [self.O.quant_weight_128x128(w32[i:i + 512])
                         for i in range(0, cfg.H, 512)]
                q = np.concatenate([a for a, _ in parts])
                s = np.concatenate([b for _, b in parts])
            self.cache[e] = (wgu, wd, q, s)
        return self.cache[e]

    def run(self, S: int):
        """(seconds of the whole forward, seconds measured) with S sampled experts
        (all of them on a workload that runs whole)."""
        O, cfg = self.O, self.cfg
        full = S >= len(self.touched)
        experts = self.order if full else self.order[:S]
        for e in experts:
            self._weights(e)                  # drawn before the timed region
        t0 = time.perf_counter()
        ids, w = O.route_topk(self.logits, cfg.top_k, self.score, cfg.renormalize)
        O.dispatch_tables(ids, cfg.E, cfg.padding_M)
        t_route = time.perf_counter() - t0
        if full:
            def loader(name, e):
                wgu, wd, q, s = self.cache[int(e)]
                return {"w_gate_up": wgu, "w_down": wd, "w_down_q": q, "w_down_s": s}[name]
            O.experts_forward(self.hidden, ids, w, None, None, cfg.routed_scaling_factor,
                              fp8=cfg.down_fp8, weight_loader=loader, **self.shared)
            t = time.perf_counter() - t0
            return t, t
        t1 = time.perf_counter()
        flat = ids.reshape(-1)
        for e in experts:
            wgu, wd, q, s = self.cache[int(e)]
            rows = self.X[np.nonzero(flat == e)[0] // cfg.top_k]
            O.expert_mlp(rows, wgu, wd, fp8=cfg.down_fp8, w_down_q_e=q, w_down_s_e=s)
        t_mlp = time.perf_counter() - t1
        t_shared = 0.0
        if cfg.F_shared:
            t2 = time.perf_counter()
            n_sh = max(1, min(cfg.T, 256))
            O.dense_swiglu_mlp(self.X[:n_sh], self.shared["ws_gate_up"], self.shared["ws_down"])
            t_shared = (time.perf_counter() - t2) * cfg.T / n_sh
        measured = time.perf_counter() - t0
        return t_route + t_mlp * len(self.touched) / len(experts) + t_shared, measured

    def pick_sample(self, budget_s: float) -> int:
        """Experts in the sample: doubled from 2 while one run stays under a quarter
        of the budget; all of them (the whole workload) for a small one."""
        if self.small:
            return len(self.touched)
        S = 2
        while S < len(self.touched):
            _, m = self.run(S)
            if m * 2 > budget_s / 2:
                break
            S = min(len(self.touched), S * 2)
        return S

    def describe(self, S: int) -> str:
        cfg = self.cfg
        if S >= len(self.touched):
            return (f"the whole workload: routing, dispatch tables and the per-token oracle "
                    f"forward over all {cfg.T} tokens")
        d = (f"routing + dispatch tables over all {cfg.T} tokens; the oracle's per-expert "
             f"step (expert_mlp) over all rows of {S} seeded experts of the "
             f"{len(self.touched)} touched, time scaled by {len(self.touched)}/{S}")
        if cfg.F_shared:
            d += f"; the shared expert over {min(cfg.T, 256)} tokens, scaled by T/{min(cfg.T, 256)}"
        return d + "; the slot-order weighted sum (O(P*H)) not timed"


def cpu_baseline(cfg, budget_s: float = 20.0) -> dict:
    r = OracleRunner(cfg)
    S = r.pick_sample(budget_s)
    t, m = r.run(S)
    return {"value": round(t * 1e3, 1), "unit": "ms/layer", "cores": int(r.threads),
            "kind": "oracle", "sample": r.describe(S), "sample_s": round(m, 2)}


def config_dict(cfg, world: int) -> dict:
    """The workload as both arms name it."""
    return {"workload": cfg.name, "T": cfg.T, "E": cfg.E, "top_k": cfg.top_k, "H": cfg.H,
            "F": cfg.F, "F_shared": cfg.F_shared, "score_fn": cfg.score_fn,
            "routed_scaling_factor": cfg.routed_scaling_factor, "down_fp8": cfg.down_fp8,
            "l2": "flushed (512 MiB write) before each step",
            "parallelism": f"replicas x{world}"}


def run_reference(args, cfg, world: int) -> dict:
    r = OracleRunner(cfg)
    per_step = min(20.0, 150.0 / max(1, args.steps + args.warmup))
    S = r.pick_sample(per_step)
    times, meas = [], []
    for i in range(args.warmup + args.steps):
        t, m = r.run(S)
        if i >= args.warmup:
            times.append(t * 1e3)
            meas.append(m)
    v = round(statistics.median(times), 1)
    return {"metric": METRIC, "value": v, "unit": "ms/layer", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": config_dict(cfg, world),
            "cpu_baseline": {"value": v, "unit": "ms/layer", "cores": int(r.threads),
                             "kind": "oracle", "sample": r.describe(S),
                             "sample_s": round(statistics.median(meas), 2)},
            "e2e": {"value": v, "unit": "ms/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------
# single-op lines: the training-side FP8 kernels at the shapes of the
# single-kernel benchmark of XTuner PR #2089 (x [131072, 6144] over 256
# experts; gate_up [32768, 4096] and [131072, 8192] over 256 experts)
# ---------------------------------------------------------------------------

OPS = {
    "quant_dual_block": dict(kind="dual", M=131072, K=6144, E=256, per_block=True),
    "quant_dual_tile": dict(kind="dual", M=131072, K=6144, E=256, per_block=False),
    "swiglu_quant_dual_32k": dict(kind="swiglu_dual", M=32768, K=2048, E=0, per_block=True),
    "swiglu_quant_dual_128k": dict(kind="swiglu_dual", M=131072, K=4096, E=256, per_block=True),
    "swiglu_backward_32k": dict(kind="backward", M=32768, K=2048),
    "swiglu_backward_128k": dict(kind="backward", M=131072, K=4096),
}
# the down GEMM with the routing weight folded into its epilogue, then the
# combine, on a whole workload (rows stored bf16 or fp32)
for _w in ("qwen3_decode", "qwen3_prefill", "dsv3_prefill", "dsv3_decode_fp8"):
    for _d in ("bf16", "f32"):
        OPS[f"fold_{_w}_{_d}"] = dict(kind="fold", workload=_w, rows=_d)
# one tensor-parallel rank of the shared expert (moe_shared_expert_forward: the
# rank's F_s / tp columns of the complete weights, fp32 partial output)
OPS["shared_kimi_k2_tp1"] = dict(kind="shared", workload="kimi_k2", tp=1)
OPS["shared_kimi_k2_tp8"] = dict(kind="shared", workload="kimi_k2", tp=8)
OPS["shared_dsv3_prefill_tp1"] = dict(kind="shared", workload="dsv3_prefill", tp=1)
OP_METRIC = "training-FP8 op ms + achieved GB/s, % of B200 HBM roofline (1 GPU)"
SHARED_METRIC = "shared-expert rank partial ms, % of B200 roofline (1 GPU)"
FOLD_METRIC = ("down GEMM with the routing weight folded in + combine, ms per layer, "
               "% of B200 roofline (1 GPU)")


def run_shared(args, device, spec) -> dict:
    """One rank's shared-expert partial on a workload's tokens: the rank reads its
    F_s / tp gate, up and down columns of the complete weights in place."""
    import moe_routed_expert_top_b200 as M
    cfg = get_config(spec["workload"])
    tp = spec["tp"]
    T, H, Fs = cfg.T, cfg.H, cfg.F_shared
    w = make_weights(cfg, device)
    wgu, wd = w["ws_gate_up"], w["ws_down"]
    del w
    hidden = make_hidden(cfg, device)
    out = torch.empty(T, H, dtype=torch.float32, device=device)
    ws = torch.empty(M.moe_shared_workspace_bytes(T, H, Fs, tp), dtype=torch.uint8,
                     device=device)
    fn = lambda: M.moe_shared_expert_forward(T, H, Fs, tp, tp - 1, hidden, wgu, wd, True, out, ws)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "device status flag set"
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = statistics.median(time_steps(fn, args.steps, flush, stream))
    Fp = Fs // tp
    nbytes = 3 * H * Fp * 2 + T * H * 2 + 2 * T * Fp * 2 + T * H * 4
    flops = 6.0 * T * H * Fp
    t_byte = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    tensor = t_flop > t_byte
    achieved = flops / (ms * 1e-3) / 1e12 if tensor else nbytes / (ms * 1e-3) / 1e9
    peak = peaks["bf16_tflops"] if tensor else peaks["hbm_gbs"]
    return {
        "metric": SHARED_METRIC, "op": args.op, "value": round(ms, 4), "unit": "ms",
        "higher_is_better": False, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": cfg.name, "T": T, "H": H, "F_shared": Fs,
                                        "tp_size": tp, "tp_rank": tp - 1,
                                        "l2": "flushed (512 MiB write) before each call"},
        "roofline": {"bound": "tensor" if tensor else "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s" if tensor else "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "algorithmic_bytes": int(nbytes), "flops": flops},
        "timing": "median of per-call CUDA events on the launching stream",
        "clocks": clk.summary(),
    }


def run_fold(args, device, spec) -> dict:
    """Weighted down GEMM + combine on a workload, timed beside the forward's
    own down GEMM (fp32 rows in expert order) + weighted unpermute."""
    cfg = get_config(spec["workload"])
    M, layer, hidden, ids, weights, _ = build_layer(cfg, device)
    peaks = load_peaks()
    wm = work_model(cfg, ids.cpu().numpy())
    prob = layer.problem(cfg.T)
    L = M.moe_get_tables_layout(prob)
    P, H, F, T = L["P"], cfg.H, cfg.F, cfg.T
    tables = torch.empty(L["total_int32"], dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    x_perm = torch.empty(P, H, dtype=torch.bfloat16, device=device)
    M.moe_route_permute(prob, None, ids, None, hidden, x_perm, tables, status)
    if cfg.down_fp8:
        h = torch.empty(P, F, dtype=torch.uint8, device=device)
        hs = torch.empty(P, F // 128, dtype=torch.float32, device=device)
    else:
        h = torch.empty(P, F, dtype=torch.bfloat16, device=device)
        hs = None
    M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, layer.w_gate_up, None, tables,
                       M.MOE_EPI_SWIGLU_FP8 if cfg.down_fp8 else M.MOE_EPI_SWIGLU, h, hs, None,
                       status)
    del x_perm
    f32 = spec["rows"] == "f32"
    y_w = torch.empty(P, H, dtype=torch.float32 if f32 else torch.bfloat16, device=device)
    y = torch.empty(P, H, dtype=torch.float32, device=device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    s = cfg.routed_scaling_factor
    down_w = lambda: M.moe_down_gemm_weighted(prob, H, F, h, hs, layer.w_down,
                                              layer.w_down_scales, tables, weights, s,
                                              M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE,
                                              y_w, status)
    comb = lambda: M.moe_combine(prob, y_w, tables, None, out)
    down = lambda: M.moe_grouped_gemm(prob, 0, H, F, h, hs, layer.w_down, layer.w_down_scales,
                                      tables, M.MOE_EPI_STORE_F32, y, None, None, status)
    unp = lambda: M.moe_unpermute(prob, y, tables, weights, s, None, out)

    def fold():
        down_w()
        comb()

    def plain():
        down()
        unp()

    fns = {"fold": fold, "down_weighted": down_w, "combine": comb, "forward_path": plain,
           "down_f32": down, "unpermute": unp}
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for fn in fns.values():
        for _ in range(args.warmup):
            fn()
    torch.cuda.synchronize()
    res = {}
    with ClockSampler(torch.cuda.current_device()) as clk:
        for name, fn in fns.items():
            res[name] = statistics.median(time_steps(fn, args.steps, flush, stream))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status flag set"
    # the weighted down GEMM: its weights, its A rows (h), its pair-order rows
    rb = 4 if f32 else 2
    dn_bytes = wm["down_bytes"] - P * H * 4 + P * H * rb
    t_s = res["down_weighted"] * 1e-3
    t_byte = dn_bytes / (peaks["hbm_gbs"] * 1e9)
    # FP8 operands: the measured bf16 peak x the nominal fp8/bf16 ratio of 2
    mma_peak = peaks["bf16_tflops"] * (2.0 if cfg.down_fp8 else 1.0)
    t_flop = wm["down_flops"] / (mma_peak * 1e12)
    tensor = t_flop > t_byte
    achieved = (wm["down_flops"] / t_s / 1e12) if tensor else (dn_bytes / t_s / 1e9)
    peak = mma_peak if tensor else peaks["hbm_gbs"]
    return {
        "metric": FOLD_METRIC, "op": args.op, "value": round(res["fold"], 4), "unit": "ms",
        "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
        "dtype": ("e4m3 x e4m3 (block-scaled)" if cfg.down_fp8 else "bf16") +
                 (", fp32 rows" if f32 else ", bf16 rows"),
        "data": "synthetic", "config": {"workload": cfg.name, "rows": spec["rows"], "T": T,
                                        "E": cfg.E, "top_k": cfg.top_k, "H": H, "F": F,
                                        "l2": "flushed (512 MiB write) before each call"},
        "stages_ms": {k: round(v, 4) for k, v in res.items()},
        "roofline": {"bound": "tensor" if tensor else "hbm", "kernel": "down_weighted",
                     "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s" if tensor else "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": None, "algorithmic_bytes": int(dn_bytes),
                     "flops": wm["down_flops"]},
        "timing": "median of per-call CUDA events on the launching stream; forward_path = "
                  "the forward's own down GEMM (fp32 rows, expert order) + unpermute",
        "clocks": clk.summary(),
    }


def run_op(args, device) -> dict:
    import moe_routed_expert_top_b200 as M
    from moe_routed_expert_top_b200 import build
    build.build()
    spec = dict(OPS[args.op])
    if spec["kind"] == "fold":
        return run_fold(args, device, spec)
    if spec["kind"] == "shared":
        return run_shared(args, device, spec)
    if args.override:       # e.g. M=32768: a smaller case of the same op (profiling)
        for item in args.override.split(","):
            key, val = item.split("=", 1)
            if key not in ("M", "K"):
                raise SystemExit(f"--override for --op takes M and K, not {key}")
            spec[key] = int(val)
    kind, Mr, K = spec["kind"], spec["M"], spec["K"]
    E = spec.get("E", 0)
    g = torch.Generator(device=device)
    g.manual_seed(7)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    if kind == "backward":
        gu = (torch.randn(Mr, 2 * K, generator=g, device=device) * 2).to(torch.bfloat16)
        dh = torch.randn(Mr, K, generator=g, device=device).to(torch.bfloat16)
        out = torch.empty(Mr, 2 * K, dtype=torch.bfloat16, device=device)
        fn = lambda: M.moe_swiglu_backward(Mr, K, gu, dh, out)
        nbytes = Mr * 2 * K * 2 + Mr * K * 2 + Mr * 2 * K * 2
        shape = {"gate_up": [Mr, 2 * K]}
    else:
        prob, tables = None, None
        if E:
            # one expert per row, seeded uniform routing; tables from the library
            ids = torch.from_numpy(np.random.default_rng(11).integers(0, E, size=(Mr, 1))
                                   .astype(np.int32)).to(device)
            prob = M.make_problem(T=Mr, H=128, F=128, E=E, top_k=1)
            L = M.moe_get_tables_layout(prob)
            tables = torch.empty(L["total_int32"], dtype=torch.int32, device=device)
            st = torch.zeros(1, dtype=torch.int32, device=device)
            M.moe_route_permute(prob, None, ids, None, None, None, tables, st)
        M_blk = M.moe_dual_blocks(prob, Mr)
        src_cols = 2 * K if kind == "swiglu_dual" else K
        x = torch.randn(Mr, src_cols, generator=g, device=device).to(torch.bfloat16)
        q = torch.empty(Mr, K, dtype=torch.uint8, device=device)
        s = torch.empty(Mr, K // 128, device=device)
        qT = torch.empty(K, 128 * M_blk, dtype=torch.uint8, device=device)
        sT = torch.empty((K // 128, M_blk) if spec["per_block"] else (K, M_blk), device=device)
        mode = M.MOE_TRANS_PER_BLOCK if spec["per_block"] else M.MOE_TRANS_PER_TILE
        if kind == "swiglu_dual":
            fn = lambda: M.moe_swiglu_quant_dual(prob, tables, Mr, K, x, mode, q, s, qT, sT)
        else:
            fn = lambda: M.moe_quant_dual(prob, tables, Mr, K, x, mode, q, s, qT, sT)
        nbytes = (Mr * src_cols * 2 + Mr * K + s.numel() * 4 + qT.numel() + sT.numel() * 4)
        shape = {"x" if kind == "dual" else "gate_up": [Mr, src_cols], "experts": E or 1,
                 "trans": "per_block" if spec["per_block"] else "per_tile",
                 "padded_tokens": 128 * M_blk}
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = time_steps(fn, args.steps, flush, stream)
    ms = statistics.median(times)
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {
        "metric": OP_METRIC, "op": args.op, "value": round(ms, 4), "unit": "ms",
        "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
        "dtype": "bf16 in, e4m3 + fp32 scales out" if kind != "backward" else "bf16",
        "data": "synthetic", "config": {"workload": args.op, **shape,
                                        "l2": "flushed (512 MiB write) before each call"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": None, "algorithmic_bytes": int(nbytes)},
        "timing": "median of per-call CUDA events on the launching stream",
        "clocks": clk.summary(),
    }


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def relaunch_ranks(n: int, argv) -> int:
    """Start n ranks of this same command, one process per GPU, with the
    torch.distributed launcher on this node (127.0.0.1), and return its exit
    status: `python bench.py --gpus N` behaves like the torchrun launch."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    args = list(sys.argv[1:] if argv is None else argv)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *args]
    return subprocess.run(cmd).returncode


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(CONFIGS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager calls instead of a CUDA graph replay of the forward")
    ap.add_argument("--override", default="",
                    help="workload fields to replace, e.g. E=16,T=256 (small profiling cases)")
    ap.add_argument("--op", default=None, choices=list(OPS),
                    help="time one training-side FP8 kernel instead of the forward (1 GPU)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.op is not None:
        torch.cuda.set_device(0)
        print(json.dumps(run_op(args, torch.device("cuda", 0))), flush=True)
        return 0
    cfg = get_config(args.config)
    if args.override:
        kv = dict(item.split("=", 1) for item in args.override.split(","))
        typed = {k: (v.lower() in ("1", "true")) if isinstance(getattr(cfg, k), bool)
                 else type(getattr(cfg, k))(v) for k, v in kv.items()}
        cfg = cfg.replace(name=cfg.name + "[" + args.override + "]", **typed)

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch_ranks(args.gpus, argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started {world} "
                         f"ranks (WORLD_SIZE); they must agree")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, cfg, world)), flush=True)
        return 0

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        from moe_routed_expert_top_b200 import build
        build.build()
        line = run_b200(args, cfg, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
