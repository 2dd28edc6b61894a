"""Pins of the float64 oracle against things the pages and the mathematics fix.

Each check compares the oracle with something other than itself:
* torch's own scaled_dot_product_attention (a library routine) when every
  block is critical, or with per-element masks built by brute force;
* closed-form quadratic linear attention when every block is marginal;
* exact zero when every block is negligible;
* hand-derived values and the NSA parameters printed on the pages
  (tests/golden/);
* invariants (constant V, V shifts, token permutations inside a block).
The planted-mistake tests at the end swap a step of the oracle for a plausible
wrong one and check that some pin catches it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import sla_oracle as so

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class Cfg:
    def __init__(self, **kw):
        base = dict(B=1, H=2, H_kv=2, N=256, N_valid=256, d=16, block=32, mode=0, k_h=2, k_l=2,
                    top_n=0, window=0, causal=0, has_proj=1, proj_per_head=0, has_gate=0,
                    smooth_k=0, linear_all=0, cos_filter=0, scale=0.0, cos_theta=0.0)
        base.update(kw)
        self.__dict__.update(base)


def rand_inputs(c, seed=0, v_shift=0.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((c.B, c.H, c.N, c.d))
    k = rng.standard_normal((c.B, c.H_kv, c.N, c.d))
    v = rng.standard_normal((c.B, c.H_kv, c.N, c.d)) + v_shift
    # pad tokens are zero, as the layer receives them
    q[:, :, c.N_valid:] = 0
    k[:, :, c.N_valid:] = 0
    v[:, :, c.N_valid:] = 0
    w_p = rng.normal(0, 1 / math.sqrt(c.d), (c.d, c.d))
    w_g = rng.normal(0, 1 / math.sqrt(c.d), (c.H, c.d))
    if getattr(c, "proj_per_head", 0):
        w_p = rng.normal(0, 1 / math.sqrt(c.d), (c.H, c.d, c.d))
    return q, k, v, w_p, w_g


def wp_of(c, w_p, h):
    return w_p[h] if getattr(c, "proj_per_head", 0) else w_p


def scale_of(c):
    return c.scale if c.scale > 0 else 1 / math.sqrt(c.d)


def sdpa(q, k, v, allow, scale):
    """torch SDPA in float64 with a boolean allow mask; rows with nothing allowed give 0."""
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v))
    A = torch.from_numpy(allow)
    out = F.scaled_dot_product_attention(Q, K, V, attn_mask=A, scale=scale).numpy()
    empty = ~allow.any(axis=-1)
    out = np.where(empty[..., None], 0.0, out)
    return out


def expand_kv(x, group):
    return np.repeat(x, group, axis=1)


# ---------------------------------------------------------------------------
# brute force: classes by counting ranks, outputs through element masks
# ---------------------------------------------------------------------------

def brute_pool(x, n_valid, blk):
    n, d = x.shape
    w = (np.arange(n) < n_valid).astype(np.float64).reshape(n // blk, blk)
    xb = x.reshape(n // blk, blk, d)
    cnt = np.maximum(w.sum(1), 1)
    return (xb * w[..., None]).sum(1) / cnt[:, None]


def brute_rank(s):
    """rank[i, j] = number of blocks that beat j in row i (higher score, or equal score and lower index)."""
    nq, nk = s.shape
    rank = np.zeros((nq, nk), dtype=np.int64)
    for j in range(nk):
        better = (s > s[:, j:j + 1])
        tie_lower = (s == s[:, j:j + 1]) & (np.arange(nk)[None, :] < j)
        rank[:, j] = (better | tie_lower).sum(1)
    return rank


def brute_cos_filter(c, k_head):
    """True for key blocks whose mean pairwise cosine similarity (ordered pairs of valid
    tokens, self-pairs included; Gram matrix of the normalised tokens) is below theta."""
    nb = c.N // c.block
    out = np.zeros(nb, dtype=bool)
    if not getattr(c, "cos_filter", 0):
        return out
    for j in range(nb):
        xs = k_head[j * c.block:min((j + 1) * c.block, c.N_valid)]
        if xs.shape[0] == 0:
            continue
        nrm = np.sqrt((xs * xs).sum(axis=1))
        xn = np.array([x / n if n > 0 else 0 * x for x, n in zip(xs, nrm)])
        out[j] = (xn @ xn.T).mean() < c.cos_theta
    return out


def brute_threeway(c, q, k, v, w_p, w_g):
    g = c.H // c.H_kv
    sc = scale_of(c)
    nb = c.N // c.block
    out = np.zeros((c.B, c.H, c.N, c.d))
    tok_blk = np.arange(c.N) // c.block
    valid = np.arange(c.N) < c.N_valid
    for b in range(c.B):
        for h in range(c.H):
            hk = h // g
            s = brute_pool(q[b, h], c.N_valid, c.block) @ brute_pool(k[b, hk], c.N_valid, c.block).T * sc
            s[:, brute_cos_filter(c, k[b, hk])] = -np.inf
            r = brute_rank(s)
            crit_b = r < c.k_h
            neg_b = r >= nb - c.k_l
            marg_b = ~crit_b & ~neg_b
            if getattr(c, "linear_all", 0):
                marg_b = np.ones_like(crit_b)
            crit = crit_b[tok_blk][:, tok_blk] & valid[None, :]
            marg = marg_b[tok_blk][:, tok_blk] & valid[None, :]
            o_s = sdpa(q[b, h][None], k[b, hk][None], v[b, hk][None], crit[None], sc)[0]
            fq = F.elu(torch.from_numpy(q[b, h])).numpy() + 1
            kk = torch.from_numpy(k[b, hk])
            if getattr(c, "smooth_k", 0):
                kk = kk - kk[:c.N_valid].mean(dim=0, keepdim=True)
            fk = F.elu(kk).numpy() + 1
            a = (fq @ fk.T) * marg
            den = a.sum(1)
            o_l = np.where(den[:, None] > 0, (a @ v[b, hk]) / np.where(den > 0, den, 1)[:, None], 0)
            proj = o_l @ wp_of(c, w_p, h) if c.has_proj else o_l
            gate = torch.sigmoid(torch.from_numpy(q[b, h] @ w_g[h])).numpy() if c.has_gate else 1.0
            o = o_s + (gate[:, None] if c.has_gate else 1.0) * proj
            o[~valid] = 0
            out[b, h] = o
    return out


def brute_topn_window(c, q, k, v):
    g = c.H // c.H_kv
    sc = scale_of(c)
    nb = c.N // c.block
    out = np.zeros((c.B, c.H, c.N, c.d))
    t = np.arange(c.N)
    tok_blk = t // c.block
    valid = t < c.N_valid
    for b in range(c.B):
        for hk in range(c.H_kv):
            heads = range(hk * g, (hk + 1) * g)
            kb = brute_pool(k[b, hk], c.N_valid, c.block)
            S = [brute_pool(q[b, h], c.N_valid, c.block) @ kb.T * sc for h in heads]
            filt = brute_cos_filter(c, k[b, hk])
            for s in S:
                s[:, filt] = -np.inf
            sel = np.zeros((nb, nb), dtype=bool)
            for i in range(1, nb):
                p = np.zeros(i)
                for s in S:
                    row = s[i, :i]
                    if np.isfinite(row).any():  # a head whose candidates are all filtered adds 0
                        p += torch.softmax(torch.from_numpy(row), dim=0).numpy()
                r = brute_rank(p[None, :])[0]
                sel[i, :i] = r < min(c.top_n, i)
            allow = (t[None, :] <= t[:, None]) & valid[None, :] & (
                sel[tok_blk][:, tok_blk] | (t[None, :] > t[:, None] - c.window))
            for h in heads:
                o = sdpa(q[b, h][None], k[b, hk][None], v[b, hk][None], allow[None], sc)[0]
                o[~valid] = 0
                out[b, h] = o
    return out


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def max_err(a, b):
    return float(np.max(np.abs(a - b)))


def pin_all_critical(c, seed=1):
    c.k_h, c.k_l = c.N // c.block, 0
    q, k, v, w_p, w_g = rand_inputs(c, seed)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    allow = np.broadcast_to(np.arange(c.N)[None, :] < c.N_valid, (c.N, c.N))
    ref = sdpa(q, expand_kv(k, c.H // c.H_kv), expand_kv(v, c.H // c.H_kv),
               np.broadcast_to(allow, (c.B, c.H, c.N, c.N)).copy(), scale_of(c))
    ref[:, :, c.N_valid:] = 0
    return max_err(o, ref)


def pin_all_marginal(c, seed=2, v_shift=0.0):
    c.k_h, c.k_l = 0, 0
    q, k, v, w_p, w_g = rand_inputs(c, seed, v_shift)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    g = c.H // c.H_kv
    valid = (np.arange(c.N) < c.N_valid).astype(np.float64)
    ref = np.zeros_like(o)
    for b in range(c.B):
        for h in range(c.H):
            fq = F.elu(torch.from_numpy(q[b, h])) + 1
            fk = (F.elu(torch.from_numpy(k[b, h // g])) + 1) * torch.from_numpy(valid)[:, None]
            a = fq @ fk.T                                   # quadratic form, N x N
            ol = (a @ torch.from_numpy(v[b, h // g])) / a.sum(1, keepdim=True)
            if c.has_proj:
                ol = ol @ torch.from_numpy(wp_of(c, w_p, h))
            if c.has_gate:
                ol = torch.sigmoid(torch.from_numpy(q[b, h]) @ torch.from_numpy(w_g[h]))[:, None] * ol
            ref[b, h] = ol.numpy()
    ref[:, :, c.N_valid:] = 0
    return max_err(o, ref)


def pin_brute_threeway(c, seed=3):
    q, k, v, w_p, w_g = rand_inputs(c, seed)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    return max_err(o, brute_threeway(c, q, k, v, w_p, w_g))


def pin_brute_topn(c, seed=4):
    q, k, v, w_p, w_g = rand_inputs(c, seed)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    return max_err(o, brute_topn_window(c, q, k, v))


@pytest.mark.parametrize("kw", [dict(), dict(N_valid=250), dict(H=4, H_kv=2, N_valid=241),
                                dict(block=64, d=32, scale=0.3)])
def test_all_critical_is_dense_attention(kw):
    assert pin_all_critical(Cfg(**kw)) < 1e-12


@pytest.mark.parametrize("kw", [dict(has_proj=0), dict(N_valid=250), dict(has_gate=1),
                                dict(H=4, H_kv=1, N_valid=200, has_gate=1)])
def test_all_marginal_is_closed_form_linear_attention(kw):
    assert pin_all_marginal(Cfg(**kw)) < 1e-12


def test_all_marginal_with_shifted_values():
    assert pin_all_marginal(Cfg(has_proj=0), v_shift=3.0) < 1e-12


@pytest.mark.parametrize("kw", [dict(), dict(has_gate=1, N_valid=230)])
def test_all_negligible_is_zero(kw):
    c = Cfg(**kw)
    c.k_h, c.k_l = 0, c.N // c.block
    q, k, v, w_p, w_g = rand_inputs(c, 5)
    o = oracle.forward(c, q, k, v, w_p, w_g)
    assert np.all(o["O"] == 0) and np.all(o["O_s"] == 0) and np.all(o["O_l"] == 0)


@pytest.mark.parametrize("kw", [dict(), dict(k_h=3, k_l=0, has_gate=1), dict(k_h=0, k_l=5),
                                dict(k_h=1, k_l=6, N_valid=250, has_gate=1),
                                dict(H=4, H_kv=2, k_h=2, k_l=3, N_valid=237),
                                dict(k_h=8, k_l=0), dict(has_proj=0, k_h=4, k_l=1),
                                dict(k_h=3, k_l=3, N_valid=225)])
def test_threeway_matches_elementwise_brute_force(kw):
    assert pin_brute_threeway(Cfg(**kw)) < 1e-11


@pytest.mark.parametrize("kw", [dict(H=4, H_kv=2, mode=1, top_n=3, window=80, causal=1),
                                dict(H=2, H_kv=1, mode=1, top_n=2, window=32, causal=1, N_valid=250),
                                dict(H=4, H_kv=1, mode=1, top_n=20, window=1, causal=1),
                                dict(H=2, H_kv=2, mode=1, top_n=4, window=0, causal=1)])
def test_topn_window_matches_elementwise_brute_force(kw):
    assert pin_brute_topn(Cfg(**kw)) < 1e-11


def test_golden_pooled_route_example():
    g = json.load(open(os.path.join(GOLDEN, "pooled_route_example.json")))
    c = Cfg(H=1, H_kv=1, N=8, N_valid=8, d=4, block=2, k_h=g["k_h"], k_l=g["k_l"], has_proj=1)
    a = np.array([math.log(4), math.log(2), 0.0, 0.0])
    q = np.zeros((1, 1, 8, 4)); k = np.zeros((1, 1, 8, 4)); v = np.zeros((1, 1, 8, 4))
    q[0, 0, 0:2] = np.array(g["q_block0"], float)
    for j in range(4):
        k[0, 0, 2 * j] = [a[j] - 1, 1, 0, 0]
        k[0, 0, 2 * j + 1] = [a[j] + 1, -1, 0, 0]
    v[0, 0, 0:2] = g["v_block0"]
    v[0, 0, 2:4] = g["v_block1"]
    v[0, 0, 4:] = [[-9.0, 9.0, -9.0, 9.0]] * 4        # negligible blocks never reach O
    w_p = 0.5 * np.eye(4)
    L = oracle.Layer(c, q, k, v, w_p, None)
    p0 = oracle.softmax(L.scores(0, 0)[0])
    np.testing.assert_allclose(p0, g["expected_p_row0"], rtol=0, atol=1e-12)
    assert L.classes(0, 0)[0].tolist() == g["expected_classes_row0"]
    assert bool(L.tie_rows(0, 0)[0]) == g["expected_tie_row0_kl2"]
    c1 = Cfg(H=1, H_kv=1, N=8, N_valid=8, d=4, block=2, k_h=1, k_l=1)
    assert bool(oracle.Layer(c1, q, k, v).tie_rows(0, 0)[0]) == g["expected_tie_row0_kl1"]
    o = L.unit(0, 0, 0)["O"]
    np.testing.assert_allclose(o, [g["expected_O_row_no_gate"]] * 2, atol=1e-12)
    cg = Cfg(H=1, H_kv=1, N=8, N_valid=8, d=4, block=2, k_h=1, k_l=2, has_gate=1)
    og = oracle.Layer(cg, q, k, v, w_p, np.zeros((1, 4))).unit(0, 0, 0)["O"]
    np.testing.assert_allclose(og, [g["expected_O_row_gate0"]] * 2, atol=1e-12)


def test_golden_nsa_selected_tokens():
    """Q = 0 makes every pooled score equal, so the selection is the 16 lowest past blocks.
    A late query then attends 16 x 64 selected tokens plus its 512-token window."""
    g = json.load(open(os.path.join(GOLDEN, "nsa_selected_branch.json")))
    blk, n_sel, w = g["selected_block"], g["selected_blocks"], g["window"]
    nb = 40
    c = Cfg(H=2, H_kv=1, N=nb * blk, N_valid=nb * blk, d=8, block=blk, mode=1, top_n=n_sel,
            window=w, causal=1, has_proj=0)
    rng = np.random.default_rng(11)
    q = np.zeros((1, 2, c.N, 8))
    k = rng.standard_normal((1, 1, c.N, 8))
    v = rng.standard_normal((1, 1, c.N, 8))
    L = oracle.Layer(c, q, k, v)
    sels, _ = L.route()
    i = nb - 1
    assert sels[0][0][i].tolist() == list(range(n_sel))
    assert len(sels[0][0][i]) * blk == g["selected_tokens"]
    o = L.unit(0, 0, i)["O"]
    for r in (0, 31, 63):
        t = i * blk + r
        att = np.concatenate([np.arange(n_sel * blk), np.arange(t - w + 1, t + 1)])
        assert att.size == g["selected_tokens"] + g["window"]
        np.testing.assert_allclose(o[r], v[0, 0, att].mean(0), atol=1e-12)


def test_constant_values_give_constant_branches():
    c = Cfg(k_h=2, k_l=3, has_gate=1, N_valid=250)
    q, k, v, w_p, w_g = rand_inputs(c, 6)
    cv = np.linspace(-1, 2, c.d)
    v[:] = cv
    v[:, :, c.N_valid:] = 0
    r = oracle.forward(c, q, k, v, w_p, w_g)
    val = slice(0, c.N_valid)
    np.testing.assert_allclose(r["O_s"][:, :, val], np.broadcast_to(cv, r["O_s"][:, :, val].shape), atol=1e-12)
    np.testing.assert_allclose(r["O_l"][:, :, val], np.broadcast_to(cv, r["O_l"][:, :, val].shape), atol=1e-12)


def test_value_shift_moves_both_branches():
    c = Cfg(k_h=2, k_l=2, N_valid=240)
    q, k, v, w_p, w_g = rand_inputs(c, 7)
    v2 = v.copy()
    v2[:, :, :c.N_valid] += 3.0
    a = oracle.forward(c, q, k, v, w_p, w_g)
    b = oracle.forward(c, q, k, v2, w_p, w_g)
    val = slice(0, c.N_valid)
    np.testing.assert_allclose(b["O_s"][:, :, val] - a["O_s"][:, :, val], 3.0, atol=1e-11)
    np.testing.assert_allclose(b["O_l"][:, :, val] - a["O_l"][:, :, val], 3.0, atol=1e-11)


def test_token_permutation_inside_blocks():
    c = Cfg(k_h=2, k_l=2, has_gate=1)
    q, k, v, w_p, w_g = rand_inputs(c, 8)
    rng = np.random.default_rng(9)
    perm = np.concatenate([j * c.block + rng.permutation(c.block) for j in range(c.N // c.block)])
    a = oracle.Layer(c, q, k, v, w_p, w_g)
    b = oracle.Layer(c, q[:, :, perm], k[:, :, perm], v[:, :, perm], w_p, w_g)
    for h in range(c.H):
        assert np.array_equal(a.classes(0, h), b.classes(0, h))
    np.testing.assert_allclose(a.forward()["O"][:, :, perm], b.forward()["O"], atol=1e-11)


def test_positive_query_scale_keeps_threeway_classes():
    c = Cfg(k_h=3, k_l=2)
    q, k, v, w_p, w_g = rand_inputs(c, 10)
    a = oracle.Layer(c, q, k, v)
    b = oracle.Layer(c, 2.5 * q, k, v)
    for h in range(c.H):
        assert np.array_equal(a.classes(0, h), b.classes(0, h))


# ---------------------------------------------------------------------------
# planted mistakes: each plausible slip in the oracle must fail some pin
# ---------------------------------------------------------------------------

def _fails_some_pin(monkeypatch, name, fn, pins):
    monkeypatch.setattr(so, name, fn)
    errs = [p() for p in pins]
    return max(errs) > 1e-6


PINS = [lambda: pin_all_critical(Cfg(N_valid=250)),
        lambda: pin_all_marginal(Cfg(N_valid=250, has_gate=1)),
        lambda: pin_brute_threeway(Cfg(k_h=2, k_l=3, has_gate=1, N_valid=250)),
        lambda: pin_brute_threeway(Cfg(k_h=3, k_l=3, N_valid=225)),
        lambda: pin_brute_topn(Cfg(H=4, H_kv=2, mode=1, top_n=3, window=80, causal=1)),
        lambda: pin_brute_topn(Cfg(H=2, H_kv=1, mode=1, top_n=2, window=40, causal=1, N_valid=225))]


def test_planted_phi_without_offset_is_caught(monkeypatch):
    assert _fails_some_pin(monkeypatch, "phi",
                           lambda x: np.where(x > 0, x, np.exp(np.minimum(x, 0)) - 1) + 0.5, PINS)


def test_planted_ascending_order_is_caught(monkeypatch):
    assert _fails_some_pin(monkeypatch, "block_order",
                           lambda s: np.argsort(s, kind="stable"), PINS)


def test_planted_transposed_projection_is_caught(monkeypatch):
    def bad_combine(o_s, o_l, q_rows, w_p, w_g_head):
        proj = o_l @ w_p.T if w_p is not None else o_l
        g = so.sigmoid(q_rows @ w_g_head) if w_g_head is not None else np.ones(q_rows.shape[0])
        return o_s + g[:, None] * proj
    assert _fails_some_pin(monkeypatch, "combine", bad_combine, PINS)


def test_planted_pooling_over_padding_is_caught(monkeypatch):
    def bad_pool(x, n_valid, block):
        n, d = x.shape
        return x.reshape(n // block, block, d).mean(axis=1)
    assert _fails_some_pin(monkeypatch, "pool_blocks", bad_pool, PINS)


def test_planted_state_over_padding_is_caught(monkeypatch):
    orig = so.linear_states

    def bad_states(k, v, n_valid, block, k_offset=None):
        return orig(k, v, k.shape[0], block, k_offset)
    assert _fails_some_pin(monkeypatch, "linear_states", bad_states, PINS)


def test_planted_unscaled_attention_is_caught(monkeypatch):
    orig = so.softmax_attention

    def bad_attn(q_rows, keys, vals, scale, allow=None):
        return orig(q_rows, keys, vals, 1.0, allow)
    assert _fails_some_pin(monkeypatch, "softmax_attention", bad_attn, PINS)


def test_planted_window_off_by_one_is_caught(monkeypatch):
    orig_unit = so.Layer.unit

    def bad_unit(self, b, h, i, cls_row=None, sel_row=None):
        self.c.window += 1
        try:
            return orig_unit(self, b, h, i, cls_row, sel_row)
        finally:
            self.c.window -= 1
    monkeypatch.setattr(so.Layer, "unit", bad_unit)
    assert pin_brute_topn(Cfg(H=4, H_kv=2, mode=1, top_n=3, window=80, causal=1)) > 1e-6


# ---------------------------------------------------------------------------
# projection per query head (w_p [H, d, d]; the scope table's boundary sketch
# allows W_p shared or per head)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kw", [dict(), dict(N_valid=250, has_gate=1), dict(H=3, H_kv=3, k_h=1, k_l=3)])
def test_per_head_projection_matches_brute_force(kw):
    assert pin_brute_threeway(Cfg(proj_per_head=1, **kw)) < 1e-12


def test_per_head_projection_all_marginal_closed_form():
    assert pin_all_marginal(Cfg(proj_per_head=1, H=3, H_kv=3, has_gate=1)) < 1e-12


def test_per_head_projection_with_equal_matrices_is_the_shared_one():
    c = Cfg(N_valid=250)
    q, k, v, w_p, w_g = rand_inputs(c, 11)
    shared = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    c2 = Cfg(N_valid=250, proj_per_head=1)
    per_head = oracle.forward(c2, q, k, v, np.stack([w_p] * c2.H), w_g)["O"]
    assert np.array_equal(shared, per_head)
    # distinct matrices per head change only the heads whose matrix changed
    w3 = np.stack([w_p, 2.0 * w_p])
    o3 = oracle.forward(c2, q, k, v, w3, w_g)["O"]
    assert np.array_equal(o3[:, 0], shared[:, 0]) and not np.allclose(o3[:, 1], shared[:, 1])


# ---------------------------------------------------------------------------
# options from the SLA critique page's notes on the open-source code:
# smooth-K (zero-mean K) and the linear branch over all tokens
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kw", [dict(smooth_k=1), dict(linear_all=1), dict(smooth_k=1, linear_all=1),
                                dict(smooth_k=1, linear_all=1, N_valid=241, H=4, H_kv=2, has_gate=1),
                                dict(linear_all=1, k_h=0, k_l=8)])
def test_options_match_brute_force(kw):
    assert pin_brute_threeway(Cfg(**kw)) < 1e-12


def test_smooth_k_changes_only_the_linear_branch():
    """K - m shifts every pooled score and attention logit of a row by q . m, so the classes
    and O_s are those without smooth-K; only phi(K) in the linear branch changes."""
    c0, c1 = Cfg(N_valid=250), Cfg(N_valid=250, smooth_k=1)
    q, k, v, w_p, w_g = rand_inputs(c0, 21)
    k = k + 0.7  # a key mean far from zero
    k[:, :, c0.N_valid:] = 0
    r0 = oracle.forward(c0, q, k, v, w_p, w_g)
    r1 = oracle.forward(c1, q, k, v, w_p, w_g)
    L0, L1 = so.Layer(c0, q, k, v, w_p, w_g), so.Layer(c1, q, k, v, w_p, w_g)
    for h in range(c0.H):
        assert np.array_equal(L0.classes(0, h), L1.classes(0, h))
    assert max_err(r0["O_s"], r1["O_s"]) < 1e-12
    assert max_err(r0["O_l"], r1["O_l"]) > 1e-3


def test_smooth_k_is_a_no_op_for_zero_mean_keys():
    c0, c1 = Cfg(N_valid=250), Cfg(N_valid=250, smooth_k=1)
    q, k, v, w_p, w_g = rand_inputs(c0, 22)
    k[:, :, :c0.N_valid] -= k[:, :, :c0.N_valid].mean(axis=2, keepdims=True)
    o0 = oracle.forward(c0, q, k, v, w_p, w_g)["O"]
    o1 = oracle.forward(c1, q, k, v, w_p, w_g)["O"]
    assert max_err(o0, o1) < 1e-12


def test_linear_all_with_every_block_negligible_is_linear_attention():
    """No critical block and the linear branch over all tokens: O is plain kernelised linear
    attention over every valid token (closed form)."""
    c = Cfg(N_valid=250, k_h=0, k_l=8, linear_all=1, has_gate=1)
    q, k, v, w_p, w_g = rand_inputs(c, 23)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    ref = np.zeros_like(o)
    valid = (np.arange(c.N) < c.N_valid).astype(np.float64)
    for h in range(c.H):
        fq = F.elu(torch.from_numpy(q[0, h])) + 1
        fk = (F.elu(torch.from_numpy(k[0, h])) + 1) * torch.from_numpy(valid)[:, None]
        a = fq @ fk.T
        ol = (a @ torch.from_numpy(v[0, h])) / a.sum(1, keepdim=True) @ torch.from_numpy(w_p)
        g = torch.sigmoid(torch.from_numpy(q[0, h]) @ torch.from_numpy(w_g[h]))[:, None]
        ref[0, h] = (g * ol).numpy()
    ref[:, :, c.N_valid:] = 0
    assert max_err(o, ref) < 1e-12


def test_planted_smooth_k_with_the_padded_mean_is_caught(monkeypatch):
    """A key mean taken over the padded length instead of the valid tokens fails a pin."""
    def bad_mean(k, n_valid):
        return k.mean(axis=0)
    monkeypatch.setattr(so, "key_mean", bad_mean)
    assert pin_brute_threeway(Cfg(smooth_k=1, N_valid=241)) > 1e-6


# ---------------------------------------------------------------------------
# token reordering along a Hilbert curve (SpargeAttn token-reorder note)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_hilbert_curve_visits_every_cell_with_unit_steps(bits):
    side = 1 << bits
    pts = {}
    for x in range(side):
        for y in range(side):
            for z in range(side):
                pts[so.hilbert_key3(x, y, z, bits)] = (x, y, z)
    assert sorted(pts) == list(range(side ** 3))       # a bijection onto [0, side^3)
    assert pts[0] == (0, 0, 0)
    steps = [np.abs(np.subtract(pts[k + 1], pts[k])).sum() for k in range(side ** 3 - 1)]
    assert all(st == 1 for st in steps)                 # consecutive cells are grid neighbours


def test_hilbert_order_is_a_permutation_of_a_ragged_grid():
    order = so.hilbert_order(3, 5, 7)
    assert sorted(order.tolist()) == list(range(105))
    # on a power-of-two cube the order walks the curve: unit steps in (t, h, w)
    o = so.hilbert_order(4, 4, 4)
    coords = np.stack(np.unravel_index(o, (4, 4, 4)), axis=1)
    assert np.all(np.abs(np.diff(coords, axis=0)).sum(axis=1) == 1)


def test_permute_tokens_round_trip():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 3, 70, 4))
    order = so.hilbert_order(2, 5, 6)                    # 60 grid tokens, 10 padding rows
    y = so.permute_tokens(x, order)
    assert np.array_equal(y[:, :, 60:], x[:, :, 60:])
    assert np.array_equal(y[:, :, 7], x[:, :, order[7]])
    assert np.array_equal(so.permute_tokens(y, order, inverse=True), x)


def test_hilbert_order_raises_block_similarity_of_a_smooth_field():
    """The reorder note's claim on a smooth field over a (t, h, w) grid: tokens that share
    a block become more alike (mean in-block cosine similarity)."""
    rng = np.random.default_rng(7)
    t, h, w = 6, 10, 16
    tt, hh, ww = np.meshgrid(np.arange(t), np.arange(h), np.arange(w), indexing="ij")
    coords = np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1).astype(np.float64)
    om = rng.normal(0, 0.3, (32, 3))
    field = np.cos(coords @ om.T + rng.uniform(0, 6.28, 32)) @ rng.standard_normal((32, 16))
    raster = so.block_cos_sim(field, 16)
    curve = so.block_cos_sim(field[so.hilbert_order(t, h, w)], 16)
    assert curve > raster + 0.1


# ---------------------------------------------------------------------------
# SpargeAttn key-block similarity filter (S_hat[i, j] = -inf when CosSim(K_j) < theta)
# ---------------------------------------------------------------------------

def _block_keys(c, seed, spread):
    """Keys whose blocks differ in self-similarity: block j shares a direction with weight
    spread[j] (1 = identical tokens, 0 = independent)."""
    rng = np.random.default_rng(seed)
    q, k, v, w_p, w_g = rand_inputs(c, seed)
    for j in range(c.N // c.block):
        lo, hi = j * c.block, (j + 1) * c.block
        base = rng.standard_normal((c.B, c.H_kv, 1, c.d))
        k[:, :, lo:hi] = spread[j] * base + (1 - spread[j]) * k[:, :, lo:hi]
    k[:, :, c.N_valid:] = 0
    return q, k, v, w_p, w_g


@pytest.mark.parametrize("kw", [dict(), dict(N_valid=241), dict(H=4, H_kv=2, has_gate=1, linear_all=1)])
def test_cos_filter_matches_brute_force(kw):
    c = Cfg(cos_filter=1, cos_theta=0.3, **kw)
    spread = np.linspace(0.0, 0.9, c.N // c.block)
    q, k, v, w_p, w_g = _block_keys(c, 31, spread)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    assert max_err(o, brute_threeway(c, q, k, v, w_p, w_g)) < 1e-12
    # some blocks are filtered and some are not
    sims = so.block_cos_sims(k[0, 0], c.N_valid, c.block)
    assert (sims < c.cos_theta).any() and (sims >= c.cos_theta).any()


def test_cos_filter_in_top_n_mode_matches_brute_force():
    c = Cfg(mode=1, causal=1, H=4, H_kv=2, has_proj=0, top_n=3, window=40, k_h=0, k_l=0,
            cos_filter=1, cos_theta=0.3)
    spread = np.linspace(0.0, 0.9, c.N // c.block)
    q, k, v, w_p, w_g = _block_keys(c, 32, spread)
    o = oracle.forward(c, q, k, v, w_p, w_g)["O"]
    assert max_err(o, brute_topn_window(c, q, k, v)) < 1e-12


def test_cos_filter_extremes():
    """theta below every CosSim (>= 0) filters nothing; theta above every CosSim (<= 1)
    filters every block, and the classes then follow the block index."""
    c0 = Cfg(N_valid=250)
    q, k, v, w_p, w_g = rand_inputs(c0, 33)
    ref = oracle.forward(c0, q, k, v, w_p, w_g)["O"]
    none = oracle.forward(Cfg(N_valid=250, cos_filter=1, cos_theta=-0.5), q, k, v, w_p, w_g)["O"]
    assert np.array_equal(ref, none)
    c2 = Cfg(N_valid=250, cos_filter=1, cos_theta=1.5)
    L = so.Layer(c2, q, k, v, w_p, w_g)
    cls = L.classes(0, 0)
    nb = c2.N // c2.block
    assert np.all(cls[:, :c2.k_h] == so.CRITICAL) and np.all(cls[:, nb - c2.k_l:] == so.NEGLIGIBLE)


def test_block_cos_sims_closed_forms():
    """Identical tokens give 1; two opposite tokens give 0; orthogonal unit tokens give 1/n."""
    x = np.zeros((8, 4))
    x[:4] = [1.0, 2.0, 0.0, -1.0]
    x[4] = [1.0, 0, 0, 0]
    x[5] = [-1.0, 0, 0, 0]
    x[6:8] = np.eye(4)[:2]
    sims = so.block_cos_sims(x, 8, 4)
    assert abs(sims[0] - 1.0) < 1e-15
    # block 1: e1, -e1, e1', e2 -> sum = (1, 1, 0, 0), |sum|^2 = 2, / 16
    assert abs(sims[1] - 2.0 / 16.0) < 1e-15


# ---------------------------------------------------------------------------
# NSA's three branches (top-n mode option)
# ---------------------------------------------------------------------------

def nsa_cfg(**kw):
    base = dict(mode=1, causal=1, top_n=2, window=40, k_h=0, k_l=0, has_proj=0, has_gate=0, nsa_branches=1,
                cmp_block=8, cmp_stride=4, N=256, N_valid=256, H=4, H_kv=2, d=16, block=32)
    base.update(kw)
    return Cfg(**base)


def nsa_brute(c, q, k, v, w_g, sels):
    """Element-mask brute force of the three branches: compressed keys through an explicit
    pooling matrix, every branch by torch SDPA with its boolean mask."""
    N, bl, nv = c.N, c.block, c.N_valid
    n_c = (nv - c.cmp_block) // c.cmp_stride + 1 if nv >= c.cmp_block else 0
    P = np.zeros((n_c, N))
    for cc in range(n_c):
        P[cc, cc * c.cmp_stride:cc * c.cmp_stride + c.cmp_block] = 1.0 / c.cmp_block
    t = np.arange(N)[:, None]
    s = np.arange(N)[None, :]
    out = np.zeros((c.B, c.H, N, c.d))
    for b in range(c.B):
        for h in range(c.H):
            hk = h // (c.H // c.H_kv)
            selm = np.zeros((c.N // bl, c.N // bl), bool)
            for i, row in enumerate(sels[b][hk]):
                selm[i, np.asarray(row, dtype=np.int64)] = True
            ok = (s <= t) & (s < nv)
            m_slc = ok & selm[t // bl, s // bl]
            m_win = ok & (s > t - c.window)
            m_cmp = np.arange(n_c)[None, :] * c.cmp_stride + c.cmp_block - 1 <= t
            Q, K, V = q[b, h], k[b, hk], v[b, hk]
            o_slc = sdpa(Q, K, V, m_slc, scale_of(c))
            o_win = sdpa(Q, K, V, m_win, scale_of(c))
            o_cmp = sdpa(Q, P @ K, P @ V, m_cmp, scale_of(c)) if n_c else np.zeros_like(Q)
            g = 1 / (1 + np.exp(-(Q @ w_g[h].T))) if c.has_gate else np.ones((N, 3))
            o = g[:, :1] * o_cmp + g[:, 1:2] * o_slc + g[:, 2:3] * o_win
            o[nv:] = 0
            out[b, h] = o
    return out


@pytest.mark.parametrize("kw", [dict(), dict(has_gate=1), dict(N_valid=241, has_gate=1),
                                dict(cmp_block=32, cmp_stride=16, window=0, top_n=3),
                                dict(top_n=0, window=64, cmp_block=16, cmp_stride=16)])
def test_nsa_branches_match_elementwise_brute_force(kw):
    c = nsa_cfg(**kw)
    q, k, v, _, _ = rand_inputs(c, seed=31)
    w_g = np.random.default_rng(32).normal(0, 0.5, (c.H, 3, c.d))
    L = so.Layer(c, q, k, v, None, w_g)
    sels = L.route()[0]
    got = L.forward()["O"]
    want = nsa_brute(c, q, k, v, w_g, sels)
    assert np.abs(got - want).max() <= 1e-10


def test_nsa_compressed_branch_with_unit_blocks_is_causal_attention():
    """cmp_block = cmp_stride = 1: every token is its own compressed block, so the
    compressed branch is dense causal attention (torch SDPA, causal mask)."""
    c = nsa_cfg(top_n=0, window=0, cmp_block=1, cmp_stride=1, N_valid=250)
    q, k, v, _, _ = rand_inputs(c, seed=33)
    got = so.Layer(c, q, k, v).forward()["O"]
    for h in range(c.H):
        hk = h // (c.H // c.H_kv)
        Q, K, V = (torch.from_numpy(np.ascontiguousarray(a[0, x][:c.N_valid])) for a, x in
                   ((q, h), (k, hk), (v, hk)))
        want = F.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=scale_of(c)).numpy()
        assert np.abs(got[0, h, :c.N_valid] - want).max() <= 1e-12


def test_nsa_zero_gates_halve_the_branch_sum():
    c = nsa_cfg(has_gate=1)
    q, k, v, _, _ = rand_inputs(c, seed=34)
    half = so.Layer(c, q, k, v, None, np.zeros((c.H, 3, c.d))).forward()["O"]
    c1 = nsa_cfg(has_gate=0)
    full = so.Layer(c1, q, k, v).forward()["O"]
    assert np.abs(half - 0.5 * full).max() <= 1e-12


def test_compress_kv_means_and_ragged_tail():
    x = np.arange(20.0).reshape(10, 2)
    got = so.compress_kv(x, 9, 4, 2)  # blocks of 4 at stride 2 inside the 9 valid tokens
    assert got.shape == (3, 2)
    np.testing.assert_allclose(got[:, 0], [3.0, 7.0, 11.0])  # means of rows 0-3, 2-5, 4-7 (column 0 = 2 t)
    assert so.compress_kv(x, 3, 4, 2).shape == (0, 2)
