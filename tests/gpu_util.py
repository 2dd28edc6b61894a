"""Helpers shared by the GPU parity tests: run the C-ABI layer on seeded inputs
and score it against the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_linear_sm_b200 as sla
from block_sparse_linear_sm_b200 import workloads as wl
import oracle

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev(bits: np.ndarray | None):
    if bits is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class LazyF64:
    """Indexable float64 view of bf16 bit patterns, converted slice by slice on access
    (full-size layers do not fit comfortably in host memory as float64)."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, key):
        return wl.bf16_bits_to_f64(self.bits[key])


class DeviceRun:
    """One sla_forward (and optionally sla_route) of a seeded layer on cuda:0."""

    def __init__(self, cfg: wl.LayerConfig, inputs: wl.LayerInputs | None = None, route=True):
        self.cfg = cfg
        self.x = inputs if inputs is not None else wl.generate(cfg)
        c = cfg
        self.q, self.k, self.v = to_dev(self.x.q), to_dev(self.x.k), to_dev(self.x.v)
        self.w_p, self.w_g = to_dev(self.x.w_p), to_dev(self.x.w_g)
        self.out = torch.empty(c.B, c.H, c.N, c.d, dtype=torch.bfloat16, device="cuda")
        rows = c.H if c.mode == wl.MODE_THREEWAY else c.H_kv
        self.mask = torch.full((c.B, rows, c.nqb, c.nkb), -7, dtype=torch.int8, device="cuda")
        nbytes = sla.sla_workspace_bytes(c)
        assert nbytes > 0
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        sla.sla_forward(self.q, self.k, self.v, self.w_p, self.w_g, c, self.out, self.mask, self.ws)
        st, detail = sla.sla_check_device_status(self.ws)
        assert st == 0, (st, detail)
        self.crit = self.neg = None
        if route:
            n_crit = c.k_h if c.mode == wl.MODE_THREEWAY else c.top_n
            self.crit = torch.full((c.B, rows, c.nqb, max(n_crit, 1)), -9, dtype=torch.int32,
                                   device="cuda")
            self.neg = torch.full((c.B, rows, c.nqb, max(c.k_l, 1)), -9, dtype=torch.int32,
                                  device="cuda")
            self.rmask = torch.full_like(self.mask, -7)
            sla.sla_route(self.q, self.k, c, self.rmask, self.crit if n_crit else None,
                          self.neg if c.k_l and c.mode == wl.MODE_THREEWAY else None, self.ws)
            st, detail = sla.sla_check_device_status(self.ws)
            assert st == 0, (st, detail)
        torch.cuda.synchronize()

    def O(self) -> np.ndarray:
        return bf16_to_f64(self.out)

    def layer(self) -> oracle.Layer:
        x = self.x
        return oracle.Layer(self.cfg, LazyF64(x.q), LazyF64(x.k), LazyF64(x.v), x.f64("w_p"),
                            x.f64("w_g"))


def _resolves_tie(p: np.ndarray, top: np.ndarray, rest: np.ndarray, rel: float) -> bool:
    """True when every block in `top` has a probability at least that of every block in
    `rest`, up to the near-tie tolerance: the set is one valid resolution of the tie."""
    if len(top) == 0 or len(rest) == 0:
        return True
    lo, hi = p[top].min(), p[rest].max()
    return bool(lo >= hi or hi - lo <= rel * max(hi, lo))


def check_routing(run: DeviceRun, L: oracle.Layer) -> dict:
    """Routing against the oracle. Rows without a near tie at a class boundary must match
    bit for bit. Near-tie rows (two pooled probabilities within 1e-5 relative across a
    boundary) admit several correct answers: the GPU's classes must have the right counts
    and order the blocks consistently with the oracle's probabilities up to that tolerance,
    its lists must agree with its own mask; how many of them still match exactly is
    reported. Returns the report."""
    c = run.cfg
    rel = oracle.TIE_REL
    mask = run.mask.cpu().numpy()
    rmask = run.rmask.cpu().numpy() if run.crit is not None else None
    report = dict(rows=0, tie_rows=0, mismatched_rows=0, tie_rows_identical=0, tie_rows_invalid=0)
    if c.mode == wl.MODE_THREEWAY:
        cls, tie = L.route()
        crit = run.crit.cpu().numpy() if c.k_h else None
        neg = run.neg.cpu().numpy() if c.k_l else None
        for b in range(c.B):
            for h in range(c.H):
                probs = oracle.softmax(L.scores(b, h)) if tie[b, h].any() else None
                for i in range(c.nqb):
                    report["rows"] += 1
                    want = cls[b, h, i]
                    got = mask[b, h, i]
                    lists_ok = True
                    if rmask is not None:
                        lists_ok = np.array_equal(rmask[b, h, i], got)
                        if c.k_h:
                            lists_ok &= np.array_equal(crit[b, h, i], np.nonzero(got == 2)[0])
                        if c.k_l:
                            lists_ok &= np.array_equal(neg[b, h, i], np.nonzero(got == 0)[0])
                    if not tie[b, h, i]:
                        report["mismatched_rows"] += int(not (np.array_equal(got, want) and lists_ok))
                        continue
                    report["tie_rows"] += 1
                    report["tie_rows_identical"] += int(np.array_equal(got, want) and lists_ok)
                    p = probs[i]
                    hi_, mid, lo_ = (np.nonzero(got == k)[0] for k in (2, 1, 0))
                    valid = (lists_ok and len(hi_) == c.k_h and len(lo_) == c.k_l
                             and _resolves_tie(p, hi_, np.concatenate([mid, lo_]), rel)
                             and _resolves_tie(p, np.concatenate([hi_, mid]), lo_, rel))
                    report["tie_rows_invalid"] += int(not valid)
    else:
        sels, tie = L.route()
        crit = run.crit.cpu().numpy() if c.top_n else None
        for b in range(c.B):
            for hk in range(c.H_kv):
                group = c.H // c.H_kv
                heads = range(hk * group, (hk + 1) * group)
                for i in range(c.nqb):
                    report["rows"] += 1
                    s = sels[b][hk][i]
                    want = np.zeros(c.nkb, np.int8)
                    want[s] = 2
                    got = mask[b, hk, i]
                    lists_ok = True
                    if rmask is not None:
                        lists_ok = np.array_equal(rmask[b, hk, i], got)
                        if c.top_n:
                            lst = np.full(c.top_n, -1)
                            g = np.nonzero(got == 2)[0]
                            lst[:len(g)] = g[:c.top_n]
                            lists_ok &= len(g) <= c.top_n and np.array_equal(crit[b, hk, i], lst)
                    if not tie[b, hk, i]:
                        report["mismatched_rows"] += int(not (np.array_equal(got, want) and lists_ok))
                        continue
                    report["tie_rows"] += 1
                    report["tie_rows_identical"] += int(np.array_equal(got, want) and lists_ok)
                    # the group's summed probabilities over the past blocks j < i
                    p = np.zeros(i)
                    for h in heads:
                        p += oracle.softmax(L.scores(b, h)[i, :i])
                    chosen = np.nonzero(got[:i] == 2)[0]
                    rest = np.setdiff1d(np.arange(i), chosen)
                    valid = (lists_ok and not np.any(got[i:] != 0) and len(chosen) == min(c.top_n, i)
                             and _resolves_tie(p, chosen, rest, rel))
                    report["tie_rows_invalid"] += int(not valid)
    return report


def unit_errors(run: DeviceRun, L: oracle.Layer, units) -> dict:
    """Max / mean abs error of O over the valid rows of the given (b, h, i) units.

    Rows whose routing is a near tie are scored under the GPU's own routing."""
    c = run.cfg
    mask = run.mask.cpu().numpy()
    errs = []
    for (b, h, i) in units:
        if c.mode == wl.MODE_THREEWAY:
            tie = L.tie_rows(b, h)[i]
            u = L.unit(b, h, i, cls_row=mask[b, h, i] if tie else None)
        else:
            hk = h // (c.H // c.H_kv)
            tie = L.selection(b, hk)[1][i]
            u = L.unit(b, h, i, sel_row=np.nonzero(mask[b, hk, i] == 2)[0] if tie else None)
        nv = max(0, min(c.block, c.N_valid - i * c.block))
        got = bf16_to_f64(run.out[b, h, i * c.block:(i + 1) * c.block])
        if nv < c.block:
            assert np.all(got[nv:] == 0), "padding rows must be zero"
        errs.append(np.abs(got[:nv] - u["O"][:nv]))
    e = np.concatenate(errs)
    return dict(max_abs=float(e.max()), mean_abs=float(e.mean()))


def full_errors(run: DeviceRun, ref: dict) -> dict:
    c = run.cfg
    O = run.O()
    assert np.all(O[:, :, c.N_valid:] == 0)
    e = np.abs(O[:, :, :c.N_valid] - ref["O"][:, :, :c.N_valid])
    return dict(max_abs=float(e.max()), mean_abs=float(e.mean()))
