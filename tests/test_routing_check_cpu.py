"""The GPU tests' routing comparison (gpu_util.check_routing) on the CPU, with the
oracle's own routing standing in for the device's: exact rows count as matches, a
changed row that is not a near tie as a mismatch, and in a planted near-tie row both
resolutions of the tie are valid while a swap across the boundary is not."""
import types

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402
from gpu_util import check_routing  # noqa: E402
from oracle import sla_oracle as oracle  # noqa: E402


def fake_run(c, L):
    """A stand-in for DeviceRun holding the oracle's routing as the 'device' outputs."""
    if c.mode == wl.MODE_THREEWAY:
        mask = np.stack([np.stack([L.classes(b, h) for h in range(c.H)]) for b in range(c.B)])
        crit = np.stack([[[np.nonzero(m == 2)[0] for m in mask[b, h]] for h in range(c.H)] for b in range(c.B)])
        neg = np.stack([[[np.nonzero(m == 0)[0] for m in mask[b, h]] for h in range(c.H)] for b in range(c.B)])
    else:
        sels = [[L.selection(b, hk)[0] for hk in range(c.H_kv)] for b in range(c.B)]
        mask = np.zeros((c.B, c.H_kv, c.nqb, c.nkb), np.int8)
        crit = np.full((c.B, c.H_kv, c.nqb, max(c.top_n, 1)), -1, np.int32)
        for b in range(c.B):
            for hk in range(c.H_kv):
                for i, s in enumerate(sels[b][hk]):
                    mask[b, hk, i, s] = 2
                    crit[b, hk, i, :len(s)] = s
        neg = None
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))
    return types.SimpleNamespace(cfg=c, mask=t(mask), rmask=t(mask.copy()), crit=t(crit), neg=t(neg))


def test_threeway_exact_mismatch_and_planted_tie():
    c = wl.preset("tiny")
    x = wl.generate(c)
    L = oracle.Layer(c, x.f64("q"), x.f64("k"), x.f64("v"), x.f64("w_p"), None)
    rep = check_routing(fake_run(c, L), L)
    assert rep["mismatched_rows"] == 0 and rep["tie_rows_invalid"] == 0
    assert rep["tie_rows_identical"] == rep["tie_rows"]
    # a changed row without a tie is a mismatch
    run = fake_run(c, L)
    ties = L.tie_rows(0, 0)
    i = int(np.nonzero(~ties)[0][0])
    run.mask[0, 0, i] = torch.roll(run.mask[0, 0, i], 1)
    run.rmask[0, 0, i] = run.mask[0, 0, i]
    assert check_routing(run, L)["mismatched_rows"] == 1
    # plant an exact tie across the critical boundary of row (0, 1, i)
    h, i = 1, 2
    s = L.scores(0, h).copy()
    order = np.argsort(-s[i], kind="stable")
    a, b = order[c.k_h - 1], order[c.k_h]
    s[i, b] = s[i, a]
    L._scores[(0, h)] = s
    L._cls.pop((0, h), None)
    run = fake_run(c, L)
    for m in (run.mask, run.rmask):  # the other resolution of the tie
        m[0, h, i, a], m[0, h, i, b] = int(m[0, h, i, b]), int(m[0, h, i, a])
    crit = np.nonzero(run.mask[0, h, i].numpy() == 2)[0]
    run.crit[0, h, i] = torch.from_numpy(crit.astype(np.int32))
    rep = check_routing(run, L)
    assert rep["tie_rows"] >= 1 and rep["tie_rows_invalid"] == 0 and rep["mismatched_rows"] == 0
    assert rep["tie_rows_identical"] == rep["tie_rows"] - 1
    # swapping the best block with the worst in that row is not a valid resolution
    top, last = order[0], order[-1]
    for m in (run.mask, run.rmask):
        m[0, h, i, top], m[0, h, i, last] = int(m[0, h, i, last]), int(m[0, h, i, top])
    run.crit[0, h, i] = torch.from_numpy(np.nonzero(run.mask[0, h, i].numpy() == 2)[0].astype(np.int32))
    run.neg[0, h, i] = torch.from_numpy(np.nonzero(run.mask[0, h, i].numpy() == 0)[0].astype(np.int32))
    assert check_routing(run, L)["tie_rows_invalid"] == 1


def test_topn_exact_and_planted_tie():
    c = wl.small_config(name="topn_small", N=1024, N_valid=1024, d=64, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW,
                        causal=1, top_n=3, window=128, k_h=0, k_l=0, has_proj=0)
    x = wl.generate(c)
    L = oracle.Layer(c, x.f64("q"), x.f64("k"), x.f64("v"), None, None)
    rep = check_routing(fake_run(c, L), L)
    assert rep["mismatched_rows"] == 0 and rep["tie_rows_invalid"] == 0
    # a selection that drops its best block for an unselected one is invalid in a tie row
    # and a mismatch elsewhere
    run = fake_run(c, L)
    i = 10
    sel = np.nonzero(run.mask[0, 0, i].numpy() == 2)[0]
    out = [j for j in range(i) if j not in sel][0]
    run.mask[0, 0, i, sel[0]] = 0
    run.mask[0, 0, i, out] = 2
    run.rmask[0, 0, i] = run.mask[0, 0, i]
    new = np.sort(np.nonzero(run.mask[0, 0, i].numpy() == 2)[0]).astype(np.int32)
    run.crit[0, 0, i, :len(new)] = torch.from_numpy(new)
    rep = check_routing(run, L)
    assert rep["mismatched_rows"] + rep["tie_rows_invalid"] >= 1
