"""The benchmark's algorithmic work per stage (the numerators of its roofline
fractions) against independent counts: closed forms for the three-way layer,
and brute-force counts over the token grid for the top-n mode and NSA's
compressed branch."""
import numpy as np
import pytest

import bench
from block_sparse_linear_sm_b200 import workloads as wl


def test_threeway_flops_are_the_closed_forms():
    c = wl.preset("wan1.3b")
    m = bench.stage_model(c)
    nb = c.N // 64
    assert m["sparse_flash"] == ("tensor", 4.0 * 64 * 64 * c.d * c.B * c.H * nb * c.k_h)
    assert m["pooled_scores"] == ("fp64", 2.0 * c.B * c.H * nb * nb * c.d)
    dd = (c.d * c.d + c.d + 127) // 128 * 128
    assert m["linear_aggregate"] == ("tensor", 2.0 * c.B * c.H * nb * nb * dd)
    # the figures quoted for this workload: 3.35e11 attended FLOP, 8.05e8 FP64 FLOP
    assert abs(m["sparse_flash"][1] - 3.35e11) < 0.01e11
    assert abs(m["pooled_scores"][1] - 8.05e8) < 0.01e8
    b = bench.backward_stage_model(c)
    pairs = 64 * 64 * c.B * c.H * nb * c.k_h
    assert b["bwd_flash_dq"] == ("tensor", 6.0 * c.d * pairs)
    assert b["bwd_flash_dkdv"] == ("tensor", 8.0 * c.d * pairs)


def _topn_pairs_brute(c):
    """Per query token t: min(window, t + 1) window keys plus 64 keys per selected block
    (min(top_n, i) of them), counted on the grid one token at a time."""
    total = 0
    for t in range(c.N):
        i = t // 64
        win = sum(1 for s in range(max(0, t - c.window + 1), t + 1)) if c.window > 0 else 0
        total += win + 64 * min(c.top_n, i)
    return total


@pytest.mark.parametrize("window,top_n", [(100, 3), (0, 2), (512, 0)])
def test_topn_flops_count_window_and_selected_keys(window, top_n):
    c = wl.small_config(N=1024, N_valid=1024, d=64, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW, causal=1,
                        top_n=top_n, window=window, k_h=0, k_l=0, has_proj=0)
    m = bench.stage_model(c)
    assert m["sparse_flash"] == ("tensor", 4.0 * c.d * c.B * c.H * _topn_pairs_brute(c))
    assert m["pooled_scores"] == ("fp64", 2.0 * c.B * c.H * c.d * (c.nqb * (c.nqb - 1) // 2))


def test_nsa_compressed_branch_counts_causal_compressed_keys():
    c = wl.small_config(N=1024, N_valid=1000, d=64, H=2, H_kv=1, mode=wl.MODE_TOPN_WINDOW, causal=1,
                        top_n=2, window=64, k_h=0, k_l=0, has_proj=0, has_gate=1, nsa_branches=1,
                        cmp_block=32, cmp_stride=16)
    m = bench.stage_model(c)
    n_cmp = (c.N_valid - c.cmp_block) // c.cmp_stride + 1
    # brute force: (t, c) pairs with c < n_cmp and c * stride + length - 1 <= t, every padded row
    grid_t = np.arange(c.N)[:, None]
    grid_c = np.arange(n_cmp)[None, :]
    pairs = int(np.sum(grid_c * c.cmp_stride + c.cmp_block - 1 <= grid_t))
    assert m["sparse_flash_cmp"] == ("tensor", 4.0 * c.d * c.B * c.H * pairs)
    slc = sum(64 * min(c.top_n, t // 64) for t in range(c.N))
    win = sum(min(c.window, t + 1) for t in range(c.N))
    assert m["sparse_flash_slc"] == ("tensor", 4.0 * c.d * c.B * c.H * slc)
    assert m["sparse_flash_win"] == ("tensor", 4.0 * c.d * c.B * c.H * win)
    assert "sparse_flash" not in m


def test_routing_report_counts_ties_and_mismatches():
    """bench.routing_report: a mask equal to the oracle's classes has no mismatched row;
    one changed row that is not a near tie is counted once."""
    c = wl.preset("tiny")
    x = wl.generate(c)
    L = bench.oracle_layer(c, x)
    mask = np.stack([L.classes(0, h) for h in range(c.H)])[None]
    rep = bench.routing_report(c, L, mask, [0, 1])
    assert rep["rows"] == c.H * c.nqb and rep["mismatched_rows"] == 0
    ties = L.tie_rows(0, 1)
    i = int(np.nonzero(~ties)[0][0])
    bad = mask.copy()
    bad[0, 1, i] = np.roll(bad[0, 1, i], 1)
    assert bench.routing_report(c, L, bad, [0, 1])["mismatched_rows"] == 1


def test_oracle_sample_extrapolates_set_up_and_units():
    c = wl.preset("tiny")
    x = wl.generate(c)
    r = bench.oracle_sample(c, x, [0, 1], 4)
    assert r["heads"] == 2 and r["units"] == 8
    want = c.B * c.H * r["setup_s_per_head"] + c.B * c.H * c.nqb * r["unit_s"]
    assert abs(r["full_layer_s"] - want) <= 1e-12 * want


def test_routing_report_checks_near_tie_rows():
    """A row with a planted tie at the critical boundary: the oracle's own classes and the
    classes with the two tied blocks swapped are both valid resolutions (one identical, one
    not); swapping a critical block with a negligible one is invalid."""
    c = wl.preset("tiny")
    x = wl.generate(c)
    L = bench.oracle_layer(c, x)
    h, i = 1, 3
    s = L.scores(0, h).copy()
    order = np.argsort(-s[i], kind="stable")
    a, b = order[c.k_h - 1], order[c.k_h]  # last critical, first marginal
    s[i, b] = s[i, a]  # an exact tie across the boundary
    L._scores[(0, h)] = s
    L._cls.pop((0, h), None)
    assert L.tie_rows(0, h)[i]
    mask = np.stack([L.classes(0, g) for g in range(c.H)])[None]
    rep = bench.routing_report(c, L, mask, [h])
    assert rep["tie_rows"] >= 1 and rep["tie_rows_identical"] == rep["tie_rows"]
    assert rep["tie_rows_invalid"] == 0
    swapped = mask.copy()
    swapped[0, h, i, a], swapped[0, h, i, b] = mask[0, h, i, b], mask[0, h, i, a]
    rep = bench.routing_report(c, L, swapped, [h])
    assert rep["tie_rows_identical"] == rep["tie_rows"] - 1 and rep["tie_rows_invalid"] == 0
    assert rep["mismatched_rows"] == 0
    bad = mask.copy()
    top, last = order[0], order[-1]
    bad[0, h, i, top], bad[0, h, i, last] = mask[0, h, i, last], mask[0, h, i, top]
    rep = bench.routing_report(c, L, bad, [h])
    assert rep["tie_rows_invalid"] == 1
