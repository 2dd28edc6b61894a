"""Benchmark of the sparse+linear attention layer on B200.

One step = one sla_forward of the whole layer (routing, linear state and
aggregation, sparse flash attention with the fused epilogue) over the seeded Wan2.1-1.3B
shaped workload (B=1, H=12, d=128, 32760 tokens padded to 32768, k_h = 5 %,
k_l = 10 %). Inputs are resident in HBM (Q, K, V = 302 MB, larger than the
126 MB L2, so no flush between steps). The timed steps replay a CUDA graph of
one captured sla_forward call; direct-call timing and per-kernel event timing
are reported beside it. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle on a bounded sample

With N > 1 (torchrun) every rank runs its own replica of the layer on its GPU
(weak scaling, no collective); rank 0 prints the line with the max time over
ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402

METRIC = "ms/layer & dense-equiv TFLOP/s, sparse+linear attn N=32K d=128 95% sparse"
UNIT = "dense-equiv TFLOP/s"


# float64 mma.sync (m8n8k4) throughput of this machine's B200, TFLOP/s: a register-only loop of
# independent products on all 148 SMs gave 36.7 / 37.0 / 37.1 at 8 / 16 / 32 warps per SM
# (64 FMA per SM per clock at 1965 MHz). The peak of the pooled-scores stage.
FP64_MMA_TFLOPS = 37.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# algorithmic work per stage (one launch each), for the roofline
# ---------------------------------------------------------------------------

def stage_model(c: wl.LayerConfig) -> dict:
    """Per stage: ("tensor", bf16 FLOP), ("fp64", FLOP) or ("hbm", bytes) of algorithmic work
    per launch."""
    B, H, Hkv, N, Nv, d = c.B, c.H, c.H_kv, c.N, c.N_valid, c.d
    nb = c.nqb
    bf = 2
    m = {}
    m["pool"] = ("hbm", (B * H + B * Hkv) * Nv * d * bf + (B * H + B * Hkv) * nb * d * 8)
    if c.mode == wl.MODE_THREEWAY and nb - c.k_h - c.k_l > 0:
        # phi(Q) (bf16) and, with a gate, g_t (fp32) for the linear branch
        m["pool"] = ("hbm", m["pool"][1] + B * H * Nv * d * bf + (B * H * Nv * 4 if c.has_gate else 0))
    # float64 products q_bar . k_bar on the FP64 tensor path (mma.sync m8n8k4): every (i, j)
    # in three-way mode, the candidates j < i in top-n mode
    pairs = nb * nb if c.mode == wl.MODE_THREEWAY else nb * (nb - 1) // 2
    m["pooled_scores"] = ("fp64", 2.0 * B * H * pairs * d)
    if c.mode == wl.MODE_THREEWAY:
        marg = nb - c.k_h - c.k_l
        m["classify"] = ("hbm", B * H * nb * nb * 8 + B * H * nb * nb * (1 + (2 if marg else 0))
                         + B * H * nb * c.k_h * 4)
        dd = (d * d + d + 127) // 128 * 128
        m["linear_state"] = ("hbm", 2 * B * Hkv * Nv * d * bf + B * Hkv * nb * dd * bf)
        m["linear_aggregate"] = ("tensor", 2.0 * B * H * nb * nb * dd)
        # attended FLOP over critical blocks: QK^T and PV, 2 * 2 * b^2 * d per (row, block)
        m["sparse_flash"] = ("tensor", 4.0 * c.block * c.block * d * B * H * nb * c.k_h)
    else:
        m["select_topn"] = ("hbm", B * H * nb * nb * 8 / 2 + B * Hkv * nb * (c.top_n * 4 + nb))
        # attended (query, key) pairs, upper bound: window tokens plus selected tokens
        # (selected blocks that overlap the window are counted twice)
        pairs = 0.0
        for i in range(nb):
            for r in range(c.block):
                t = i * c.block + r
                pairs += min(c.window, t + 1) + c.block * min(c.top_n, i)
        m["sparse_flash"] = ("tensor", 4.0 * d * B * H * pairs)
        if getattr(c, "nsa_branches", 0):
            # NSA's branches: the selected blocks and the window each alone, and the
            # compressed keys up to the causal limit (c * stride + length - 1 <= t)
            slc = win = cmp_pairs = 0.0
            n_cmp = (Nv - c.cmp_block) // c.cmp_stride + 1 if Nv >= c.cmp_block else 0
            for i in range(nb):
                for r in range(c.block):
                    t = i * c.block + r
                    slc += c.block * min(c.top_n, i)
                    win += min(c.window, t + 1)
                    cmp_pairs += min(n_cmp, max(0, (t - c.cmp_block + 1) // c.cmp_stride + 1))
            kc_bytes = 2 * B * Hkv * n_cmp * d * bf
            del m["sparse_flash"]
            # reads K, V (each token lies in cmp_block / cmp_stride blocks), writes the compressed rows
            m["compress_kv"] = ("hbm", 2 * B * Hkv * Nv * d * bf + kc_bytes)
            m["sparse_flash_cmp"] = ("tensor", 4.0 * d * B * H * cmp_pairs)
            m["sparse_flash_slc"] = ("tensor", 4.0 * d * B * H * slc)
            m["sparse_flash_win"] = ("tensor", 4.0 * d * B * H * win)
            # reads q and the three branch outputs, writes O
            m["branch_combine"] = ("hbm", 5 * B * H * Nv * d * bf)
    return m


def backward_stage_model(c: wl.LayerConfig) -> dict:
    """Per backward stage: ("tensor", FLOP) or ("hbm", bytes) of algorithmic work per launch."""
    B, H, Hkv, N, Nv, d = c.B, c.H, c.H_kv, c.N, c.N_valid, c.d
    nb = c.nqb
    bf = 2
    pairs = c.block * c.block * B * H * nb * c.k_h  # critical (query token, key token) pairs
    lin = nb - c.k_h - c.k_l > 0 or c.linear_all
    dd = (d * d + d + 127) // 128 * 128
    words = (nb + 31) // 32
    if c.mode != wl.MODE_THREEWAY:
        # top-n mode: the attended (query, key) pairs, as counted for the forward pass
        pairs = stage_model(c)["sparse_flash"][1] / (4.0 * d)
        return {"bwd_columns": ("hbm", B * Hkv * nb * c.top_n * 4 + 2 * B * Hkv * nb * words * 4),
                "bwd_delta": ("hbm", 2 * B * H * Nv * d * bf + B * H * N * 4),
                "bwd_flash_dq": ("tensor", 6.0 * d * pairs),
                "bwd_flash_dkdv": ("tensor", 8.0 * d * pairs)}
    m = {"bwd_columns": ("hbm", B * H * nb * c.k_h * 4 + 2 * B * H * nb * words * 4)}
    if lin:
        nqb_pad, nkb_pad = (nb + 127) // 128 * 128, (nb + 63) // 64 * 64
        # reads phi(Q), q, O, dO, S'_i, Z_i (and g_t); writes the fp32 dq part, D_t, [dS'_i | dZ_i]
        m["bwd_linear"] = ("hbm", 4 * B * H * Nv * d * bf + B * H * nb * (d * d * bf + d * 4)
                           + B * H * Nv * 4 * (2 if c.has_gate else 1) + B * H * Nv * d * 4
                           + B * H * nb * dd * bf)
        m["bwd_mask_transpose"] = ("hbm", 2 * B * H * nqb_pad * nkb_pad * 2)
        m["bwd_aggregate_t"] = ("tensor", 2.0 * B * H * nb * nb * dd)  # the forward aggregation, transposed
        # reads K, V, dh'_j, dz_j; writes the fp32 dk and dv parts
        m["bwd_state"] = ("hbm", 2 * B * Hkv * Nv * d * bf + B * Hkv * nb * (d * d * bf + d * 4)
                          + 2 * B * Hkv * Nv * d * 4)
    else:
        m["bwd_delta"] = ("hbm", 2 * B * H * Nv * d * bf + B * H * N * 4)
    # products over the critical tiles: S, dP, dQ (query-stationary) and S^T, dP^T, dV, dK
    m["bwd_flash_dq"] = ("tensor", 6.0 * d * pairs)
    m["bwd_flash_dkdv"] = ("tensor", 8.0 * d * pairs)
    return m


def stage_entries(names, stage_ms, model, peaks):
    out = {}
    for n in names:
        kind, work = model[n]
        t = stage_ms[n] * 1e-3
        if kind == "tensor":
            ach = work / t / 1e12
            out[n] = {"ms": stage_ms[n], "bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                      "frac": ach / peaks["bf16"], "frac_of_sustained": ach / peaks["bf16_sus"], "work": work}
        elif kind == "fp64":
            ach = work / t / 1e12
            out[n] = {"ms": stage_ms[n], "bound": "fp64", "achieved": ach, "unit": "TFLOP/s",
                      "frac": ach / FP64_MMA_TFLOPS, "peak_kind": "fp64 mma.sync, measured", "work": work}
        else:
            ach = work / t / 1e9
            out[n] = {"ms": stage_ms[n], "bound": "hbm", "achieved": ach, "unit": "GB/s",
                      "frac": ach / peaks["hbm"], "work": work}
    return out


def measure_backward(sla, torch, cfg, q, k, v, w_p, w_g, out, ws, steps, warmup, dist, dev, stream, peaks):
    """sla_backward after one sla_forward (whose workspace it reads): per-stage CUDA-event times."""
    gen = torch.Generator().manual_seed(99)
    dout = torch.randn(tuple(out.shape), generator=gen).to(torch.bfloat16).to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dw_p = dw_g = None
    if cfg.has_proj:
        shape = (cfg.H, cfg.d, cfg.d) if cfg.proj_per_head else (cfg.d, cfg.d)
        dw_p = torch.empty(shape, dtype=torch.float32, device=dev)
    if cfg.has_gate:
        dw_g = torch.empty((cfg.H, cfg.d), dtype=torch.float32, device=dev)
    bws = torch.empty(sla.sla_backward_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    sla.sla_forward(q, k, v, w_p, w_g, cfg, out, None, ws)
    names = sla.sla_backward_stage_names(cfg)
    args = (q, k, v, w_p, w_g, cfg, out, dout, dq, dk, dv, dw_p, dw_g, ws, bws)
    for _ in range(warmup):
        sla.sla_backward(*args)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(steps)]
    for e in evs:
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        sla.sla_backward_timed(*args, evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    st, detail = sla.sla_check_device_status(bws)
    if st != 0:
        raise RuntimeError(f"backward device status {st} detail {detail}")
    (ms,) = max_over_ranks(dist, dev, t0.elapsed_time(t1) / steps)
    stage_ms = {n: statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps))
                for i, n in enumerate(names)}
    stages = stage_entries(names, stage_ms, backward_stage_model(cfg), peaks)
    dom = max(names, key=lambda n: stage_ms[n])
    dk_ = stages[dom]
    roof = {"kernel": dom, "bound": dk_["bound"], "achieved": dk_["achieved"], "unit": dk_["unit"],
            "peak": peaks["bf16"] if dk_["bound"] == "tensor" else peaks["hbm"], "frac": dk_["frac"],
            "peak_kind": (f"bf16 burst, {peaks['src']}" if dk_["bound"] == "tensor"
                          else f"HBM copy, {peaks['src']}")}
    del bws, dq, dk, dv, dout
    return {"ms": ms, "dense_equiv_tflops": 2.5 * cfg.dense_flops() / (ms * 1e-3) / 1e12,
            "dense_equiv_note": "2.5 x the dense forward FLOP (the usual backward/forward ratio of attention)",
            "what": "sla_backward: dq, dk, dv, dW_p, dw_g of sum(out * dout), routing held fixed",
            "stages": stages, "roofline": roof, "launches_per_call": len(names) + (2 if cfg.has_proj else 1)}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None):
        self.idx = gpu_index
        self.path = path
        self.proc = None

    def __enter__(self):
        try:
            self.f = open(self.path, "w") if self.path else subprocess.DEVNULL
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
            if self.path:
                self.f.write(out)
                self.f.close()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        load = sorted(sm)[len(sm) // 4:] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(cfg: wl.LayerConfig, x: wl.LayerInputs, units, budget_s: float | None = None):
    """Times the float64 oracle on whole (b, h, query block) units; returns (seconds, units done)."""
    import oracle  # test infrastructure: only this CPU leg of the benchmark uses it

    class Lazy:
        def __init__(self, bits):
            self.bits = bits

        def __getitem__(self, k):
            return wl.bf16_bits_to_f64(self.bits[k])

    t0 = time.perf_counter()
    L = oracle.Layer(cfg, Lazy(x.q), Lazy(x.k), Lazy(x.v), x.f64("w_p"), x.f64("w_g"))
    done = 0
    for (b, h, i) in units:
        L.unit(b, h, i)
        done += 1
        if budget_s is not None and time.perf_counter() - t0 > budget_s:
            break
    return time.perf_counter() - t0, done


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def sample_units(cfg, n, n_heads=2, seed=1234):
    rng = np.random.default_rng(seed)
    heads = rng.permutation(cfg.H)[:max(1, min(cfg.H, n_heads))]
    units = []
    for h in heads:
        for i in rng.permutation(cfg.nqb)[:max(1, n // len(heads))]:
            units.append((0, int(h), int(i)))
    return units


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_linear_sm_b200", "csrc")
    files = {"flash_tc_kernel": ["flash_tc.cu", "tc.cuh", "common.cuh"]}.get(kernel, [])
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    for e in json.load(open(p)):
        if e.get("kernel") == kernel and e.get("workload") == workload and \
                e.get("source_hash") == kernel_source_hash(kernel):
            return e["dram_bytes_per_launch"]
    return None


def route_lists(sla, torch, cfg, q, k, dev):
    """The routing's block lists of the whole layer on the host (three-way: critical lists
    [B, H, nqb, k_h]; top-n: selected lists [B, H_kv, nqb, top_n]); None without lists."""
    topn = cfg.mode == wl.MODE_TOPN_WINDOW
    rows, n = (cfg.H_kv, cfg.top_n) if topn else (cfg.H, cfg.k_h)
    if n == 0:
        return None
    crit = torch.empty((cfg.B, rows, cfg.nqb, n), dtype=torch.int32, device=dev)
    neg = None if topn or cfg.k_l == 0 else torch.empty((cfg.B, cfg.H, cfg.nqb, cfg.k_l), dtype=torch.int32,
                                                        device=dev)
    ws = torch.empty(sla.sla_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    sla.sla_route(q, k, cfg, None, crit, neg, ws)
    st, detail = sla.sla_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"routing device status {st} detail {detail}")
    return crit.cpu().numpy()


def max_over_ranks(dist, device, *vals):
    """The max of each value over all ranks (one all-reduce); the values themselves
    without a process group."""
    if dist is None:
        return [float(v) for v in vals]
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, flop_per_rank, ms_per_step):
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return world * flop_per_rank / (ms_per_step * 1e-3) / 1e12


def units_total(cfg):
    return cfg.B * cfg.H * cfg.nqb


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = wl.generate(cfg)
    units = sample_units(cfg, 8)
    per_step = []
    for s in range(args.warmup + args.steps):
        t, n = oracle_sample(cfg, x, units)
        if s >= args.warmup:
            per_step.append((t, n))
    tsum = sum(t for t, _ in per_step)
    nsum = sum(n for _, n in per_step)
    frac = nsum / units_total(cfg)
    value = frac * cfg.dense_flops() / tsum / 1e12
    full_layer_ms = tsum / frac * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tsum / len(per_step) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "N_valid": cfg.N_valid,
                   "d": cfg.d, "k_h": cfg.k_h, "k_l": cfg.k_l, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{len(units)} (head, query block) units of {units_total(cfg)} per step, "
                                   "full-layer time extrapolated by unit count"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "full_layer_ms_extrapolated": full_layer_ms,
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wan1.3b", choices=list(wl.PRESETS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--clocks-csv", default=None)
    ap.add_argument("--no-backward", action="store_true", help="skip the sla_backward measurement")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="heads: each rank runs its KV groups of one layer (LPT on the routed tiles)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads (H = H_kv; small profiler captures)")
    args = ap.parse_args()
    cfg = wl.preset(args.workload)
    if args.heads > 0:
        cfg = cfg.replace(name=f"{cfg.name}_h{args.heads}", H=args.heads, H_kv=args.heads)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import block_sparse_linear_sm_b200 as sla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    x = wl.generate(cfg)
    dev = torch.device("cuda", local)

    def up(bits):
        return None if bits is None else torch.from_numpy(bits).view(torch.bfloat16).to(dev)

    q, k, v, w_p, w_g = up(x.q), up(x.k), up(x.v), up(x.w_p), up(x.w_g)
    full_cfg, shard_info = cfg, None
    if args.shard == "heads":
        # one layer split over the ranks by KV group: route it whole, estimate each group's
        # work from its routed tiles, balance (LPT), and run this rank's heads
        from block_sparse_linear_sm_b200 import sharding as sh
        costs = sh.unit_costs(cfg, route_lists(sla, torch, cfg, q, k, dev))
        shard = sh.HeadShard(cfg, world, rank, costs)
        if any(not p for p in shard.plan):  # the same plan on every rank: all of them stop here
            raise RuntimeError(f"{world} ranks but only {cfg.H_kv} KV groups to share")
        q, k, v, w_p, w_g = shard.inputs(q, k, v, w_p, w_g)
        cfg = shard.local
        loads = sh.plan_loads(costs, shard.plan)
        shard_info = {"plan": shard.plan, "estimated_loads": loads,
                      "imbalance": max(loads) / (sum(loads) / len(loads)),
                      "what": "KV groups per rank, LPT on the tiles the routing makes the flash kernel run"}
    out = torch.empty(cfg.B, cfg.H, cfg.N, cfg.d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(sla.sla_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    names = sla.sla_stage_names(cfg)
    ns = len(names)

    # warm-up
    for _ in range(args.warmup):
        sla.sla_forward(q, k, v, w_p, w_g, cfg, out, None, ws)
    st, detail = sla.sla_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} detail {detail}")

    # timed region: K steps, per-stage events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clock_path = args.clocks_csv
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local, clock_path) as clk:
        time.sleep(0.3)
        t0.record(stream)
        for s in range(args.steps):
            sla.sla_forward_timed(q, k, v, w_p, w_g, cfg, out, None, ws, evs[s])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = t0.elapsed_time(t1)
    st, detail = sla.sla_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} detail {detail}")
    ms_eager = ms_total / args.steps

    # the same call captured once in a CUDA graph and replayed (how a serving
    # loop launches it): K replays timed with CUDA events, max over ranks
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        sla.sla_forward(q, k, v, w_p, w_g, cfg, out, None, ws, stream=cap)
    cap.synchronize()
    with torch.cuda.graph(graph, stream=cap):
        sla.sla_forward(q, k, v, w_p, w_g, cfg, out, None, ws, stream=cap)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, None) as clk2:
        time.sleep(0.2)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
    barrier()
    st, detail = sla.sla_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} detail {detail}")
    ms_total, ms_eager = max_over_ranks(dist, dev, g0.elapsed_time(g1), ms_eager)
    ms_step = ms_total / args.steps
    # per-replay medians: warm (replays back to back) and cold (a 256 MB buffer,
    # twice the L2, written right before each timed replay)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 10)
    pairs = {"warm": [], "cold": []}
    for kind in ("warm", "cold"):
        for _ in range(reps):
            if kind == "cold":
                flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            graph.replay()
            a1.record(stream)
            pairs[kind].append((a0, a1))
    torch.cuda.synchronize()
    warm_med = statistics.median(a.elapsed_time(b) for a, b in pairs["warm"])
    cold_med = statistics.median(a.elapsed_time(b) for a, b in pairs["cold"])
    warm_med, cold_med = max_over_ranks(dist, dev, warm_med, cold_med)
    del flush, pairs
    del graph
    # token reordering along the Hilbert curve of the video grid (an optional step
    # before the layer): the gather of Q's rows, HBM-bound
    reorder = None
    if cfg.grid is not None:
        order = torch.from_numpy(sla.sla_hilbert_order(*cfg.grid)).to(dev)
        qp = torch.empty_like(q)
        for _ in range(3):
            sla.sla_permute_tokens(q, qp, order)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(args.steps):
            sla.sla_permute_tokens(q, qp, order)
        r1.record(stream)
        torch.cuda.synchronize()
        (r_ms,) = max_over_ranks(dist, dev, r0.elapsed_time(r1) / args.steps)
        moved = 2 * q.numel() * 2 + order.numel() * 4  # read and write Q, read the order
        reorder = {"ms": r_ms, "bound": "hbm", "achieved": moved / (r_ms * 1e-3) / 1e9, "unit": "GB/s",
                   "frac": None,
                   "what": "Q rows gathered into Hilbert-curve order (sla_permute_tokens)"}
        del qp, order
    stage_ms = {n: statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(args.steps))
                for i, n in enumerate(names)}

    # end to end: pinned host inputs -> device, layer, output -> host
    if shard_info is None:
        hq = torch.from_numpy(x.q).view(torch.bfloat16).pin_memory()
        hk = torch.from_numpy(x.k).view(torch.bfloat16).pin_memory()
        hv = torch.from_numpy(x.v).view(torch.bfloat16).pin_memory()
    else:  # this rank's heads
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = hout.numel() * 2
    # the library's host-buffer call: units of whole KV groups, copies in / kernels / copies
    # out on three streams so that they overlap
    n_chunks = max(n for n in range(1, 17) if cfg.H_kv % n == 0)
    arena = torch.empty(sla.sla_forward_host_device_bytes(cfg, n_chunks), dtype=torch.uint8, device=dev)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step():
        sla.sla_forward_host(hq, hk, hv, w_p, w_g, cfg, hout, n_chunks, arena, stream=stream,
                             h2d_stream=s_in, d2h_stream=s_out)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    (e2e_ms,) = max_over_ranks(dist, dev, e0.elapsed_time(e1) / args.e2e_steps)
    st, detail = sla.sla_check_device_status(arena, stream=stream)
    if st != 0:
        raise RuntimeError(f"device status {st} ({detail}) after the end-to-end steps")
    del arena
    barrier()

    peaks = load_peaks()
    backward = None
    if not args.no_backward and not cfg.nsa_branches:  # NSA's branches: forward only
        backward = measure_backward(sla, torch, cfg, q, k, v, w_p, w_g, out, ws, args.steps, args.warmup,
                                    dist, dev, stream, peaks)
        barrier()

    flops = cfg.dense_flops()
    if shard_info is not None:
        # strong scaling: the ranks share one layer's work
        flops = full_cfg.dense_flops() / world
    value = job_throughput(world, flops, ms_step)
    e2e_value = job_throughput(world, flops, e2e_ms)

    if reorder is not None:
        reorder["frac"] = reorder["achieved"] / peaks["hbm"]
    stages = stage_entries(names, stage_ms, stage_model(cfg), peaks)
    dom = max(names, key=lambda n: stage_ms[n])
    kernel_of = {"sparse_flash": "flash_tc_kernel", "sparse_flash_cmp": "flash_tc_kernel",
                 "sparse_flash_slc": "flash_tc_kernel", "sparse_flash_win": "flash_tc_kernel"}
    dk = stages[dom]
    if dk["bound"] == "tensor":
        # The layer's kernels run a few ms at a time at full SM clock (see "clocks"),
        # so the burst GEMM figure is the denominator; the sustained one (taken at
        # the power-capped clock of a seconds-long loop) is given beside it.
        roof = {"kernel": dom, "bound": "tensor", "achieved": dk["achieved"], "peak": peaks["bf16"],
                "unit": "TFLOP/s", "frac": dk["achieved"] / peaks["bf16"],
                "peak_kind": f"bf16 burst, {peaks['src']}",
                "peak_sustained": peaks["bf16_sus"], "frac_of_sustained": dk["achieved"] / peaks["bf16_sus"],
                "traffic": measured_traffic(kernel_of.get(dom, dom), cfg.name),
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"}
    elif dk["bound"] == "fp64":
        roof = {"kernel": dom, "bound": "fp64", "achieved": dk["achieved"], "peak": FP64_MMA_TFLOPS,
                "unit": "TFLOP/s", "frac": dk["frac"], "peak_kind": dk["peak_kind"], "traffic": None}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": dk["achieved"], "peak": peaks["hbm"],
                "unit": "GB/s", "frac": dk["achieved"] / peaks["hbm"],
                "peak_kind": f"HBM copy, {peaks['src']}", "traffic": None}
    if "sparse_flash" in stages and dom != "sparse_flash":
        fk = stages["sparse_flash"]
        roof["flash"] = {"achieved": fk["achieved"], "frac": fk["achieved"] / peaks["bf16"]}

    clocks = clk.summary()
    c2 = clk2.summary()
    if c2.get("sm_mhz") is not None and clocks.get("sm_mhz") is not None:
        clocks["sm_mhz_graph_replays"] = c2["sm_mhz"]
        clocks["reasons"] = sorted(set(clocks["reasons"]) | set(c2["reasons"]))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak" if shard_info is None else "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": full_cfg.name, "B": full_cfg.B, "H": full_cfg.H, "H_kv": full_cfg.H_kv,
                   "N": full_cfg.N, "N_valid": full_cfg.N_valid, "d": full_cfg.d, "k_h": full_cfg.k_h,
                   "k_l": full_cfg.k_l, "has_proj": full_cfg.has_proj, "has_gate": full_cfg.has_gate,
                   "parallelism": f"replicas x{world}" if shard_info is None else f"heads x{world}",
                   "l2": f"inputs (Q,K,V {(cfg.B * (cfg.H + 2 * cfg.H_kv) * cfg.N * cfg.d * 2) / 1e6:.0f} MB) larger "
                         "than the 126 MB L2; no flush"},
        "ms_per_layer": ms_step,
        "per_replay_ms": {"warm_median": warm_med, "cold_median": cold_med, "reps": reps,
                          "cold": "256 MB written before each timed replay (L2 holds none of the layer's data)"},
        "ms_per_step_eager": ms_eager,
        "launch": "CUDA graph replay of one captured sla_forward call (ms_per_step_eager: direct calls)",
        "roofline": roof,
        "head_shard": shard_info,
        "token_reorder": reorder,
        "stages": stages,
        "backward": backward,
        "gpu_launches": ns * args.steps,
        "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                # the inputs' copy rate over the whole step: the call is bound by it when the
                # kernels and the copies out hide behind the copies in
                "h2d_gbs_over_step": h2d / (e2e_ms * 1e-3) / 1e9,
                "api": f"sla_forward_host (pinned host q, k, v and out; {n_chunks} units of whole KV groups "
                       "per batch entry, copies in, kernels and copies out overlapped on three streams)"},
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # about 10-30 s of float64 oracle work on the host cores
        units = sample_units(full_cfg, 512, n_heads=4)
        t, n = oracle_sample(full_cfg, x, units, budget_s=20.0)
        cv = (n / units_total(full_cfg)) * full_cfg.dense_flops() / t / 1e12
        line["cpu_baseline"] = {"value": cv, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                                "sample": f"{n} (head, query block) units of {units_total(full_cfg)} from "
                                          f"4 heads in {t:.1f} s (stops after 20 s); throughput "
                                          f"scaled by unit count"}
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
