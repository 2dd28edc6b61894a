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


# query blocks per step of the reference arm (about 2-4 s of float64 work each)
REF_UNITS = 48


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
    if c.mode == wl.MODE_THREEWAY and (nb - c.k_h - c.k_l > 0 or c.linear_all):
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
    if c.mode != wl.MODE_THREEWAY and getattr(c, "nsa_branches", 0):
        # NSA's branches: pairs per branch as counted for the forward pass; dQ runs all three,
        # the compressed keys' dK / dV their own kernel, the tokens' the selected and window
        fm = stage_model(c)
        pc, ps, pw = (fm[n][1] / (4.0 * d) for n in ("sparse_flash_cmp", "sparse_flash_slc", "sparse_flash_win"))
        n_cmp = (Nv - c.cmp_block) // c.cmp_stride + 1 if Nv >= c.cmp_block else 0
        m = {"bwd_columns": ("hbm", B * Hkv * nb * c.top_n * 4 + 2 * B * Hkv * nb * words * 4),
             # reads q, dO and the three branch outputs and log-sum-exps; writes lse, D, dlogit per branch
             "bwd_nsa_prep": ("hbm", 5 * B * H * Nv * d * bf + 3 * B * H * N * 4
                              + (9 if c.has_gate else 6) * B * H * N * 4),
             "bwd_flash_dq": ("tensor", 6.0 * d * (pc + ps + pw))}
        if n_cmp > 0:
            m["bwd_flash_dkdv_cmp"] = ("tensor", 8.0 * d * pc)
            m["bwd_cmp_reduce"] = ("hbm", 2 * B * Hkv * n_cmp * d * 4)  # the dKc, dVc rows it writes
        m["bwd_flash_dkdv"] = ("tensor", 8.0 * d * (ps + pw))
        return m
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
        shape = (cfg.H, 3, cfg.d) if cfg.nsa_branches else (cfg.H, cfg.d)
        dw_g = torch.empty(shape, dtype=torch.float32, device=dev)
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
    """SM clock and clock-event reasons of one GPU, sampled during a region.

    NVML (nvidia-ml-py) is read from a thread every 20 ms, so even a region of
    a fraction of a second gives tens of samples; without NVML, nvidia-smi -lms 200
    is run in the background. Nothing is set on the GPU: only queries."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index: int, path: str | None, period_s: float = 0.02):
        self.idx = gpu_index
        self.path = path
        self.period = period_s
        self.proc = None
        self.thread = None
        self.samples = []   # (sm_mhz, max_mhz, power_w, reasons bitmask)
        self.lines = []

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.stop = threading.Event()

            def run():
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                while not self.stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), float(mx),
                                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                             int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    self.stop.wait(self.period)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            time.sleep(0.05)
            self.stop.set()
            self.thread.join(timeout=5)
            if self.path:
                with open(self.path, "w") as f:
                    f.write("sm_mhz,max_mhz,power_w,reasons\n")
                    for smp in self.samples:
                        f.write(",".join(str(x) for x in smp) + "\n")
            return
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
                with open(self.path, "w") as f:
                    f.write(out)

    def summary(self) -> dict:
        sm, mx, reasons, power = [], None, set(), []
        if self.samples:
            for clk, m, pw, bits in self.samples:
                sm.append(clk)
                mx = m
                power.append(pw)
                reasons |= {n for n, b in self.REASONS.items() if bits & b}
            src = f"NVML every {self.period * 1e3:.0f} ms"
        else:
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
            src = "nvidia-smi -lms 200"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        load = sorted(sm)[len(sm) // 4:] or sm
        out = {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
               "samples": len(sm), "sm_mhz_min": min(sm), "source": src}
        if power:
            out["power_w_max"] = max(power)
        return out


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

class _LazyBits:
    """Float64 view of bf16 bits, converted slice by slice (full layers do not fit as float64)."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, k):
        return wl.bf16_bits_to_f64(self.bits[k])


def oracle_layer(cfg: wl.LayerConfig, x: wl.LayerInputs):
    import oracle  # test infrastructure: only the CPU legs of the benchmark use it
    return oracle.Layer(cfg, _LazyBits(x.q), _LazyBits(x.k), _LazyBits(x.v), x.f64("w_p"), x.f64("w_g"))


def oracle_sample(cfg: wl.LayerConfig, x: wl.LayerInputs, heads, units_per_head, budget_s=None,
                  seed=1234, layer=None):
    """Times the float64 oracle on a sample of one layer and extrapolates to the whole layer.

    Per sampled head: the head's routing (pooled means, scores, classes; top-n mode: its
    KV group's selection) and linear states are computed first and timed as the head's
    set-up; then units_per_head (b, h, query block) units are timed one by one. The
    full-layer time is B*H (top-n: B*H_kv) set-ups plus B*H*nqb units at the measured
    means. Returns a dict with the extrapolated time and what was sampled."""
    L = layer if layer is not None else oracle_layer(cfg, x)
    rng = np.random.default_rng(seed)
    topn = cfg.mode == wl.MODE_TOPN_WINDOW
    group = cfg.H // cfg.H_kv
    lin = not topn and (cfg.nkb - cfg.k_h - cfg.k_l > 0 or cfg.linear_all)
    t0 = time.perf_counter()
    t_setup = t_units = 0.0
    n_setup = n_units = 0
    for h in heads:
        a = time.perf_counter()
        if topn:
            L.selection(0, h // group)
        else:
            L.classes(0, h)
            if lin:
                L.states(0, h // group)
        t_setup += time.perf_counter() - a
        n_setup += 1
        for i in rng.permutation(cfg.nqb)[:units_per_head]:
            a = time.perf_counter()
            L.unit(0, int(h), int(i))
            t_units += time.perf_counter() - a
            n_units += 1
            if budget_s is not None and time.perf_counter() - t0 > budget_s:
                break
        if budget_s is not None and time.perf_counter() - t0 > budget_s:
            break
    setups = cfg.B * (cfg.H_kv if topn else cfg.H)
    full_s = setups * t_setup / max(n_setup, 1) + units_total(cfg) * t_units / max(n_units, 1)
    return dict(full_layer_s=full_s, seconds=time.perf_counter() - t0, heads=n_setup, units=n_units,
                setup_s_per_head=t_setup / max(n_setup, 1), unit_s=t_units / max(n_units, 1), layer=L)


def _resolves_tie(p, top, rest, rel):
    """Every block of `top` at least as probable as every block of `rest`, up to `rel`."""
    if len(top) == 0 or len(rest) == 0:
        return True
    lo, hi = p[top].min(), p[rest].max()
    return bool(lo >= hi or hi - lo <= rel * max(hi, lo))


def routing_report(cfg, L, mask, heads):
    """The GPU's routing (int8 class mask, [B, H or H_kv, nqb, nkb]) against the oracle's on
    the sampled heads: rows, mismatched rows among those without a near tie, and for the
    near-tie rows how many still match exactly and how many are not a valid resolution of
    the tie (wrong class counts, or a block ranked against the oracle's probabilities by
    more than the tolerance). Runs on the layer the oracle timing of the CPU leg built."""
    import oracle  # test infrastructure: only the CPU legs of the benchmark use it
    rel = oracle.TIE_REL
    rep = dict(rows=0, tie_rows=0, mismatched_rows=0, tie_rows_identical=0, tie_rows_invalid=0)
    if cfg.mode == wl.MODE_THREEWAY:
        for h in heads:
            cls, tie = L.classes(0, h), L.tie_rows(0, h)
            probs = oracle.softmax(L.scores(0, h)) if tie.any() else None
            for i in range(cfg.nqb):
                rep["rows"] += 1
                got = mask[0, h, i]
                if not tie[i]:
                    rep["mismatched_rows"] += int(not np.array_equal(got, cls[i]))
                    continue
                rep["tie_rows"] += 1
                rep["tie_rows_identical"] += int(np.array_equal(got, cls[i]))
                hi_, mid, lo_ = (np.nonzero(got == k)[0] for k in (2, 1, 0))
                ok = (len(hi_) == cfg.k_h and len(lo_) == cfg.k_l
                      and _resolves_tie(probs[i], hi_, np.concatenate([mid, lo_]), rel)
                      and _resolves_tie(probs[i], np.concatenate([hi_, mid]), lo_, rel))
                rep["tie_rows_invalid"] += int(not ok)
    else:
        group = cfg.H // cfg.H_kv
        for hk in sorted({h // group for h in heads}):
            sels, tie = L.selection(0, hk)
            for i in range(cfg.nqb):
                rep["rows"] += 1
                want = np.zeros(cfg.nkb, np.int8)
                want[sels[i]] = 2
                got = mask[0, hk, i]
                if not tie[i]:
                    rep["mismatched_rows"] += int(not np.array_equal(got, want))
                    continue
                rep["tie_rows"] += 1
                rep["tie_rows_identical"] += int(np.array_equal(got, want))
                p = np.zeros(i)
                for h in range(hk * group, (hk + 1) * group):
                    p += oracle.softmax(L.scores(0, h)[i, :i])
                chosen = np.nonzero(got[:i] == 2)[0]
                ok = (not np.any(got[i:] != 0) and len(chosen) == min(cfg.top_n, i)
                      and _resolves_tie(p, chosen, np.setdiff1d(np.arange(i), chosen), rel))
                rep["tie_rows_invalid"] += int(not ok)
    rep["heads"] = [int(h) for h in heads]
    rep["rule"] = ("rows whose k-th and (k+1)-th pooled probabilities (either class boundary; top-n: "
                   "the group sum at position top_n) are within 1e-5 relative are near ties: not "
                   "compared bit for bit, but checked to be a valid resolution of the tie")
    return rep


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def sample_heads(cfg, n, seed=1234):
    rng = np.random.default_rng(seed)
    return sorted(int(h) for h in rng.permutation(cfg.H)[:max(1, min(cfg.H, n))])


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


def linear_branch_cost(cfg, mask):
    """Both ways of forming S_i, Z_i from the routing (int8 classes [B, H, nqb, nkb]):
    the direct sum over the marginal blocks as the aggregation GEMM with the 0/1 marginal
    mask (what runs), and the total minus the critical and negligible blocks. On the
    tensor cores either is a dense GEMM unless whole mask tiles are zero, so the count
    of nonzero 128 x 64 tiles (the aggregation kernel's M x K step) of each mask is the
    cost that could differ; as a gather the complement moves every excluded state."""
    B, H, nqb, nkb = mask.shape
    dd = (cfg.d * cfg.d + cfg.d + 127) // 128 * 128
    marg = mask == 1
    excl = ~marg
    tiles = {"marginal": 0, "excluded": 0, "total": 0}
    for b in range(B):
        for h in range(H):
            for i0 in range(0, nqb, 128):
                for j0 in range(0, nkb, 64):
                    tiles["total"] += 1
                    tiles["marginal"] += bool(marg[b, h, i0:i0 + 128, j0:j0 + 64].any())
                    tiles["excluded"] += bool(excl[b, h, i0:i0 + 128, j0:j0 + 64].any())
    direct = 2.0 * B * H * nqb * nkb * dd
    return {"direct_gemm_flop": direct,
            "complement_gemm_flop": direct * tiles["excluded"] / max(tiles["marginal"], 1),
            "complement_gather_bytes": float(excl.sum()) * dd * 2,
            "nonzero_tiles_128x64": tiles,
            "cheaper_on_tensor_cores": "direct" if tiles["marginal"] <= tiles["excluded"] else "complement",
            "ran": "direct",
            "what": "S_i = sum over marginal j of h_j (GEMM with the marginal mask) against "
                    "S_i = H_total - sum over critical and negligible j of h_j"}


def r_heads(r, heads):
    """The heads whose set-up the oracle sample reached."""
    return heads[:r["heads"]]


def config_keys(cfg, parallelism):
    """The config object of the JSON line (the same keys in both arms)."""
    return {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "H_kv": cfg.H_kv, "N": cfg.N, "N_valid": cfg.N_valid,
            "d": cfg.d, "k_h": cfg.k_h, "k_l": cfg.k_l, "has_proj": cfg.has_proj, "has_gate": cfg.has_gate,
            "parallelism": parallelism}


def run_reference(args, cfg):
    """The oracle arm: each step times the float64 oracle on one sampled head (its set-up and
    REF_UNITS query blocks) and extrapolates to the whole layer like the cpu_baseline leg."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = wl.generate(cfg)
    per_step = []
    heads = sample_heads(cfg, cfg.H, seed=99)
    for s in range(args.warmup + args.steps):
        h = heads[s % len(heads)]
        r = oracle_sample(cfg, x, [h], REF_UNITS, seed=1000 + s)
        r.pop("layer")
        if s >= args.warmup:
            per_step.append(r)
    full_s = statistics.mean(r["full_layer_s"] for r in per_step)
    value = cfg.dense_flops() / full_s / 1e12
    sampled = sum(r["seconds"] for r in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": full_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_keys(cfg, "replicas"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"per step one head's set-up (routing, linear states) and "
                                   f"{min(REF_UNITS, cfg.nqb)} of its {cfg.nqb} query blocks, "
                                   f"{sampled / len(per_step):.1f} s of CPU work "
                                   "per step; ms_per_step is the whole layer extrapolated from the "
                                   "measured set-up and per-unit times"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "sampled_seconds_per_step": sampled / len(per_step),
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
    ap.add_argument("--soak-s", type=float, default=0.3,
                    help="seconds of graph replays right before the timed replays (clock sampling)")
    ap.add_argument("--no-backward", action="store_true", help="skip the sla_backward measurement")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="heads: each rank runs its KV groups of one layer (LPT on the routed tiles)")
    ap.add_argument("--shard-gather", action="store_true",
                    help="with --shard heads: also time steps of the local layer plus all_gather_heads")
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
    full_cfg, shard_info, bshard, full_inputs = cfg, None, None, None
    if args.shard == "heads":
        # one layer split over the ranks by KV group: estimate each group's work from its
        # routed tiles (every rank routes every world-th group; the costs are all-gathered),
        # balance (LPT), and run this rank's heads
        from block_sparse_linear_sm_b200 import sharding as sh

        def route_local(units):
            heads = sh.query_heads(cfg, units)
            return route_lists(sla, torch, sh.local_config(cfg, units), sh.gather_heads(q, heads),
                               sh.gather_heads(k, units), dev)
        if dist is None:
            full_lists = route_lists(sla, torch, cfg, q, k, dev)
            costs = sh.unit_costs(cfg, full_lists)
            pcosts = sh.pair_costs(cfg, full_lists)
        else:
            costs = sh.distributed_costs(cfg, world, rank, route_local, dist)
            pcosts = sh.distributed_pair_costs(cfg, world, rank, route_local, dist)
        # db-SP's block level on the same routing: KV groups cut into runs of query-block
        # pairs (measured after the head-level timing, on the full inputs)
        bshard = sh.BlockShard(cfg, world, rank, pcosts)
        full_inputs = (q, k, v, w_p, w_g)
        shard = sh.HeadShard(cfg, world, rank, costs)
        if any(not p for p in shard.plan):  # the same plan on every rank: all of them stop here
            raise RuntimeError(f"{world} ranks but only {cfg.H_kv} KV groups to share")
        q, k, v, w_p, w_g = shard.inputs(q, k, v, w_p, w_g)
        cfg = shard.local
        loads = sh.plan_loads(costs, shard.plan)
        shard_info = {"plan": shard.plan, "estimated_loads": loads,
                      "imbalance": max(loads) / (sum(loads) / len(loads)),
                      "what": "KV groups per rank, LPT on the tiles the routing makes the flash kernel run; "
                              "each rank routed every world-th group for the estimate"}
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
    with ClockSampler(local, None) as clk:
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
    # A soak of replays back to back (about --soak-s seconds) runs right before the K
    # timed replays, under the same clock sampler: the timed steps run on a GPU at its
    # sustained clock, and the sampler sees tens of samples of that load.
    n_soak = max(1, int(args.soak_s * 1e3 / max(ms_eager, 1e-3))) if args.soak_s > 0 else 0
    s0 = torch.cuda.Event(enable_timing=True)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, clock_path) as clk2:
        time.sleep(0.05)
        s0.record(stream)
        for _ in range(n_soak):
            graph.replay()
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
    barrier()
    soak = None
    if n_soak:
        (soak_ms,) = max_over_ranks(dist, dev, s0.elapsed_time(g0) / n_soak)
        soak = {"replays": n_soak, "ms_per_replay": soak_ms,
                "what": "graph replays back to back right before the timed steps (clocks sampled over both)"}
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
    if shard_info is not None and args.shard_gather and dist is not None:
        # the sharded layer as a caller that needs every head on every rank runs it:
        # the local layer, then the all_gather of the outputs back into head order
        def shard_step():
            sla.sla_forward(q, k, v, w_p, w_g, cfg, out, None, ws)
            return sh.all_gather_heads(out, full_cfg, shard.plan, rank, dist)
        for _ in range(args.warmup):
            shard_step()
        torch.cuda.synchronize()
        barrier()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for _ in range(args.steps):
            shard_step()
        h1.record(stream)
        torch.cuda.synchronize()
        (sg_ms,) = max_over_ranks(dist, dev, h0.elapsed_time(h1) / args.steps)
        shard_info["with_gather_ms_per_step"] = sg_ms
        shard_info["with_gather"] = "eager sla_forward on the local heads + all_gather_heads (NCCL), max over ranks"

    if bshard is not None:
        # the block level: this rank's pieces (KV group, range of query-block pairs) through
        # sla_forward_blocks on the full inputs, max over ranks
        qf, kf, vf, wpf, wgf = full_inputs
        outf = torch.empty(full_cfg.B, full_cfg.H, full_cfg.N, full_cfg.d, dtype=torch.bfloat16, device=dev)
        wss = {}

        def ws_for(lc):
            if lc.name not in wss:
                wss[lc.name] = torch.empty(sla.sla_workspace_bytes(lc), dtype=torch.uint8, device=dev)
            return wss[lc.name]
        for _ in range(args.warmup):
            bshard.run(sla, qf, kf, vf, wpf, wgf, outf, ws_for)
        torch.cuda.synchronize()
        barrier()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            bshard.run(sla, qf, kf, vf, wpf, wgf, outf, ws_for)
        b1.record(stream)
        torch.cuda.synchronize()
        for wsb in wss.values():
            stb, detb = sla.sla_check_device_status(wsb)
            if stb != 0:
                raise RuntimeError(f"device status {stb} ({detb}) in the block-level steps")
        (blk_ms,) = max_over_ranks(dist, dev, b0.elapsed_time(b1) / args.steps)
        bl_loads = sh.block_plan_loads(bshard.costs, bshard.fixed, bshard.plan)
        shard_info["block_level"] = {
            "pieces": [[list(pc) for pc in pcs] for pcs in bshard.plan],
            "estimated_loads": bl_loads, "imbalance": max(bl_loads) / (sum(bl_loads) / len(bl_loads)),
            "ms_per_step": blk_ms,
            "what": "db-SP's block level: (KV group, first pair, end pair) pieces per rank, each run through "
                    "sla_forward_blocks on the full inputs (eager), max over ranks"}
        del outf, wss

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
    if not args.no_backward:
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

    # clocks of the soak and the timed graph replays (the value's region); the eager
    # per-stage steps' own samples are kept beside them
    clocks = clk2.summary()
    c1 = clk.summary()
    if c1.get("sm_mhz") is not None and clocks.get("sm_mhz") is not None:
        clocks["sm_mhz_eager_steps"] = c1["sm_mhz"]
        clocks["reasons"] = sorted(set(clocks["reasons"]) | set(c1["reasons"]))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak" if shard_info is None else "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(config_keys(full_cfg, "replicas" if shard_info is None else f"heads x{world}"),
                       l2=f"inputs (Q,K,V {(cfg.B * (cfg.H + 2 * cfg.H_kv) * cfg.N * cfg.d * 2) / 1e6:.0f} MB) "
                          "larger than the 126 MB L2; no flush"),
        "ms_per_layer": ms_step,
        "per_replay_ms": {"warm_median": warm_med, "cold_median": cold_med, "reps": reps,
                          "cold": "256 MB written before each timed replay (L2 holds none of the layer's data)"},
        "ms_per_step_eager": ms_eager,
        "soak": soak,
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
        heads = sample_heads(full_cfg, 4)
        r = oracle_sample(full_cfg, x, heads, 128, budget_s=20.0)
        cv = full_cfg.dense_flops() / r["full_layer_s"] / 1e12
        line["cpu_baseline"] = {"value": cv, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                                "sample": f"{r['heads']} heads' set-up (routing, linear states) and {r['units']} "
                                          f"of their query blocks in {r['seconds']:.1f} s (stops after 20 s); "
                                          f"the whole layer extrapolated from the measured set-up "
                                          f"({r['setup_s_per_head']:.2f} s per head) and per-unit "
                                          f"({r['unit_s'] * 1e3:.1f} ms) times",
                                "full_layer_s": r["full_layer_s"]}
        # the GPU's routing against the oracle's on the sampled heads (near-tie rows counted)
        rows = full_cfg.H if full_cfg.mode == wl.MODE_THREEWAY else full_cfg.H_kv
        mask = torch.empty((full_cfg.B, rows, full_cfg.nqb, full_cfg.nkb), dtype=torch.int8, device=dev)
        if shard_info is None:
            sla.sla_forward(q, k, v, w_p, w_g, cfg, out, mask, ws)
            st, detail = sla.sla_check_device_status(ws)
            if st != 0:
                raise RuntimeError(f"device status {st} detail {detail}")
            m_host = mask.cpu().numpy()
            line["routing"] = routing_report(full_cfg, r["layer"], m_host, r_heads(r, heads))
            if full_cfg.mode == wl.MODE_THREEWAY:
                line["linear_branch_cost"] = linear_branch_cost(full_cfg, m_host)
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
