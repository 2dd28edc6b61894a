"""Pins of the float64 gradient oracle (oracle/sla_grad.py).

The gradient oracle restates the layer in float64 PyTorch and lets autograd
differentiate it. It is pinned against things other than itself:
* its forward values equal ``sla_oracle``'s forward pass (the pinned oracle);
* its gradients equal central finite differences of ``sla_oracle``'s forward
  pass (routing held fixed), one random direction per input;
* with every block critical they equal the textbook gradients of dense softmax
  attention (dV = P^T dO, dS = P * (dP - rowsum(dO * O)), dQ = dS K s, dK = dS^T Q s);
* with every block negligible they are zero.
Planted mistakes (a gradient that ignores the gate; NSA's compressed keys taken as
constants) fail the finite-difference pin.
The block-by-block chain rule (``block_grads``, used on sampled blocks of
full-size layers) is pinned against autograd on every block of small layers.
"""
import math

import numpy as np
import pytest
import torch

from oracle import sla_grad as sg
from oracle import sla_oracle as so


class Cfg:
    def __init__(self, **kw):
        base = dict(B=1, H=2, H_kv=2, N=128, N_valid=128, d=8, block=32, mode=0, k_h=1, k_l=1,
                    top_n=0, window=0, causal=0, has_proj=1, proj_per_head=0, has_gate=1,
                    smooth_k=0, linear_all=0, cos_filter=0, scale=0.0, cos_theta=0.0)
        base.update(kw)
        self.__dict__.update(base)


def inputs(c, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((c.B, c.H, c.N, c.d))
    k = rng.standard_normal((c.B, c.H_kv, c.N, c.d))
    v = rng.standard_normal((c.B, c.H_kv, c.N, c.d))
    for x in (q, k, v):
        x[:, :, c.N_valid:] = 0  # padding tokens are zero
    shape_p = (c.H, c.d, c.d) if c.proj_per_head else (c.d, c.d)
    w_p = rng.normal(0, 1 / math.sqrt(c.d), shape_p)
    w_g = rng.normal(0, 1 / math.sqrt(c.d), (c.H, 3, c.d) if getattr(c, "nsa_branches", 0) else (c.H, c.d))
    d_out = rng.standard_normal((c.B, c.H, c.N, c.d))
    return q, k, v, w_p, w_g, d_out


def oracle_loss(c, q, k, v, w_p, w_g, d_out, classes):
    """sum(O * d_out) from sla_oracle's own forward pass, with the routing given."""
    layer = so.Layer(c, q, k, v, w_p, w_g)
    total = 0.0
    for b in range(c.B):
        for h in range(c.H):
            for i in range(c.N // c.block):
                if c.mode == 0:
                    o = layer.unit(b, h, i, cls_row=classes[b, h, i])["O"]
                else:
                    o = layer.unit(b, h, i, sel_row=classes[b][h // (c.H // c.H_kv)][i])["O"]
                total += float((o * d_out[b, h, i * c.block:(i + 1) * c.block]).sum())
    return total


CASES = {
    "proj_gate": {},
    "ragged": dict(N_valid=117),
    "gqa": dict(H=4, H_kv=2),
    "per_head_proj": dict(proj_per_head=1),
    "smooth_k": dict(smooth_k=1),
    "linear_all": dict(linear_all=1, k_l=2),
    "plain": dict(has_proj=0, has_gate=0),
    "all_marginal": dict(k_h=0, k_l=0),
    "topn_window_gqa": dict(mode=1, causal=1, top_n=1, window=40, k_h=0, k_l=0, has_proj=0, has_gate=0,
                            H=4, H_kv=2),
    "topn_ragged": dict(mode=1, causal=1, top_n=2, window=20, k_h=0, k_l=0, has_proj=0, has_gate=0,
                        N=160, N_valid=150),
    # NSA's three branches: compressed blocks overlapping (length 16, stride 8), gates, GQA
    "nsa_gates_gqa": dict(mode=1, causal=1, top_n=1, window=40, k_h=0, k_l=0, has_proj=0, has_gate=1,
                          H=4, H_kv=2, nsa_branches=1, cmp_block=16, cmp_stride=8),
    # ragged tail (the last compressed block ends before it), no gates, length 24 / stride 20
    "nsa_ragged": dict(mode=1, causal=1, top_n=2, window=20, k_h=0, k_l=0, has_proj=0, has_gate=0,
                       N=160, N_valid=150, nsa_branches=1, cmp_block=24, cmp_stride=20),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_restated_forward_matches_the_oracle(name):
    c = Cfg(**CASES[name])
    q, k, v, w_p, w_g, _ = inputs(c, seed=11)
    ref = so.forward(c, q, k, v, w_p, w_g)["O"]
    T = lambda a: torch.from_numpy(a)
    got = sg.layer_forward_torch(c, T(q), T(k), T(v), T(w_p) if c.has_proj else None,
                                 T(w_g) if c.has_gate else None).numpy()
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def _fd_check(c, grads_fn, seed=5, eps=1e-6, rel=1e-6):
    q, k, v, w_p, w_g, d_out = inputs(c, seed=seed)
    classes = so.Layer(c, q, k, v, w_p, w_g).route()[0]
    g = grads_fn(c, q, k, v, w_p, w_g, d_out, classes)
    rng = np.random.default_rng(seed + 100)
    names = ["q", "k", "v"] + (["w_p"] if c.has_proj and c.mode == 0 else []) + \
        (["w_g"] if c.has_gate and (c.mode == 0 or getattr(c, "nsa_branches", 0)) else [])
    worst = {}
    for name in names:
        args = dict(q=q, k=k, v=v, w_p=w_p, w_g=w_g)
        delta = rng.standard_normal(args[name].shape)
        if name in ("q", "k", "v"):
            delta[:, :, c.N_valid:] = 0
        plus = dict(args)
        minus = dict(args)
        plus[name] = args[name] + eps * delta
        minus[name] = args[name] - eps * delta
        fd = (oracle_loss(c, d_out=d_out, classes=classes, **plus) -
              oracle_loss(c, d_out=d_out, classes=classes, **minus)) / (2 * eps)
        an = float((g["d" + name] * delta).sum())
        worst[name] = abs(fd - an) / max(1e-3, abs(fd))
    return worst


@pytest.mark.parametrize("name", sorted(CASES))
def test_gradients_match_finite_differences_of_the_oracle(name):
    c = Cfg(**CASES[name])
    worst = _fd_check(c, lambda c, *a: sg.layer_grads(c, *a[:6], classes=a[6]))
    assert all(e < 1e-6 for e in worst.values()), worst


def test_all_critical_gradients_are_dense_attention_gradients():
    c = Cfg(k_h=4, k_l=0, has_proj=1, has_gate=1, N_valid=117)
    q, k, v, w_p, w_g, d_out = inputs(c, seed=3)
    g = sg.layer_grads(c, q, k, v, w_p, w_g, d_out)
    s = 1 / math.sqrt(c.d)
    nv = c.N_valid
    for h in range(c.H):
        Q, K, V, dO = q[0, h, :nv], k[0, h, :nv], v[0, h, :nv], d_out[0, h, :nv]
        S = Q @ K.T * s
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        O = P @ V
        dV = P.T @ dO
        dP = dO @ V.T
        dS = P * (dP - (dO * O).sum(axis=1, keepdims=True))
        np.testing.assert_allclose(g["dq"][0, h, :nv], dS @ K * s, atol=1e-12)
        np.testing.assert_allclose(g["dk"][0, h, :nv], dS.T @ Q * s, atol=1e-12)
        np.testing.assert_allclose(g["dv"][0, h, :nv], dV, atol=1e-12)
        assert np.all(g["dq"][0, h, nv:] == 0) and np.all(g["dk"][0, h, nv:] == 0)
    # no linear branch: the projection and the gate get no gradient
    assert np.all(g["dw_p"] == 0) and np.all(g["dw_g"] == 0)


def test_all_negligible_gradients_are_zero():
    c = Cfg(k_h=0, k_l=4)
    q, k, v, w_p, w_g, d_out = inputs(c, seed=4)
    g = sg.layer_grads(c, q, k, v, w_p, w_g, d_out)
    for key in ("dq", "dk", "dv", "dw_p", "dw_g"):
        assert np.all(g[key] == 0), key


def test_planted_gate_without_gradient_is_caught(monkeypatch):
    c = Cfg(**CASES["proj_gate"])
    real = torch.sigmoid
    monkeypatch.setattr(sg.torch, "sigmoid", lambda x: real(x).detach())
    worst = _fd_check(c, lambda c, *a: sg.layer_grads(c, *a[:6], classes=a[6]))
    assert max(worst.values()) > 1e-3


def test_planted_compressed_branch_without_key_gradient_is_caught(monkeypatch):
    """NSA: a gradient that treats the compressed keys and values as constants (no path
    back through the block means to K and V) fails the finite-difference pin on dk / dv."""
    c = Cfg(**CASES["nsa_gates_gqa"])
    real = sg._masked_softmax_attention

    def planted(q, k, v, allow, scale):
        if k.shape[0] != c.N:  # the compressed branch: n_c block means instead of N tokens
            k, v = k.detach(), v.detach()
        return real(q, k, v, allow, scale)

    monkeypatch.setattr(sg, "_masked_softmax_attention", planted)
    worst = _fd_check(c, lambda c, *a: sg.layer_grads(c, *a[:6], classes=a[6]))
    assert worst["k"] > 1e-3 and worst["v"] > 1e-3, worst
    assert worst["q"] < 1e-6, worst


BLOCK_CASES = {
    "proj_gate": dict(N=256, N_valid=250, k_h=2, k_l=2),
    "gqa": dict(H=4, H_kv=2, N=256, k_h=2, k_l=1),
    "per_head_proj": dict(proj_per_head=1, N=256, k_h=2, k_l=2),
    "linear_all": dict(linear_all=1, N=256, k_h=2, k_l=3),
    "plain": dict(has_proj=0, has_gate=0, N=256, N_valid=230, k_h=3, k_l=1),
    "all_critical": dict(N=256, k_h=8, k_l=0),
    "smooth_k": dict(smooth_k=1, N=256, N_valid=241, k_h=2, k_l=2),
    "smooth_k_linear_all_gqa": dict(smooth_k=1, linear_all=1, H=4, H_kv=2, N=256, k_h=2, k_l=1),
    "topn_window_gqa": dict(mode=1, causal=1, top_n=2, window=40, k_h=0, k_l=0, has_proj=0, has_gate=0,
                            H=4, H_kv=2, N=256, N_valid=250),
    "nsa_gates_gqa": dict(mode=1, causal=1, top_n=2, window=40, k_h=0, k_l=0, has_proj=0, has_gate=1,
                          nsa_branches=1, cmp_block=16, cmp_stride=8, H=4, H_kv=2, N=256, N_valid=256),
    "nsa_ragged_no_gates": dict(mode=1, causal=1, top_n=1, window=24, k_h=0, k_l=0, has_proj=0, has_gate=0,
                                nsa_branches=1, cmp_block=32, cmp_stride=16, H=3, H_kv=1, N=320, N_valid=301),
}


@pytest.mark.parametrize("name", sorted(BLOCK_CASES))
def test_block_grads_equal_autograd(name):
    """The block-by-block chain rule (used at full size on sampled blocks) equals autograd."""
    c = Cfg(**BLOCK_CASES[name])
    q, k, v, w_p, w_g, d_out = inputs(c, seed=21)
    classes = so.Layer(c, q, k, v, w_p, w_g).route()[0]
    ref = sg.layer_grads(c, q, k, v, w_p, w_g, d_out, classes=classes)
    nb = c.N // c.block
    for b in range(c.B):
        got = sg.block_grads(c, q, k, v, w_p, w_g, d_out, classes, b, range(nb), range(nb))
        scale = lambda a: max(1e-12, float(np.abs(a).max()))
        for (h, i), rows in got["dq"].items():
            want = ref["dq"][b, h, i * c.block:(i + 1) * c.block]
            assert np.abs(rows - want).max() <= 1e-10 * scale(ref["dq"]), (name, "dq", h, i)
        for key in ("dk", "dv"):
            for (hk, j), rows in got[key].items():
                want = ref[key][b, hk, j * c.block:(j + 1) * c.block]
                assert np.abs(rows - want).max() <= 1e-10 * scale(ref[key]), (name, key, hk, j)
        if c.has_proj and c.mode == 0:
            assert np.abs(got["dw_p"] - ref["dw_p"]).max() <= 1e-10 * scale(ref["dw_p"])
        if c.has_gate and (c.mode == 0 or c.nsa_branches):
            assert len(got["dw_g"]) == c.H
            for h, row in got["dw_g"].items():
                assert np.abs(row - ref["dw_g"][h]).max() <= 1e-10 * scale(ref["dw_g"])
