"""Float64 gradients of the three-way sparse+linear attention layer.

TEST INFRASTRUCTURE, like ``sla_oracle``: a plain, slow statement of what the
layer's backward pass computes, used only to check the CUDA path. It shares no
code with that path. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.

What it follows. The pages ask for fine-tuning with the layer in place (SLA
analysis page, arXiv 2509.24006: the model is fine-tuned for a few steps with
SLA; SALAD summary: the gated branches are trained on a small set of videos),
so the layer needs gradients with respect to Q, K, V, the projection W_p and
the gate vectors w_g. The pages print no backward pass. The gradient is read
as the plain derivative of the forward pass with the routing held fixed: the
block classes are a piecewise-constant function of the pooled scores, so they
contribute no gradient and are taken as given.

The layer is restated here in float64 PyTorch, element by element on the
N x N token grid (tiny and small shapes only):

* O_s: softmax attention of each valid query row over the valid key tokens of
  its critical blocks; a row with none gives 0.
* O_l: linear attention over the valid key tokens of the marginal blocks (or of
  every block with linear_all), phi = elu + 1, K shifted by the mean valid key
  with smooth-K: O_l = (phi(Q) phi(K)^T . M) V / rowsum(phi(Q) phi(K)^T . M);
  a row with no such token gives 0.
* O = O_s + g * (O_l W_p), g = sigmoid(q . w_g[h]); padding rows are 0.

``torch.autograd`` then differentiates L = sum(O * dO). The restatement is
pinned against ``sla_oracle`` (the same forward values) and its gradients
against central finite differences of ``sla_oracle``'s own forward pass.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import sla_oracle as so


def _phi(x: torch.Tensor) -> torch.Tensor:
    return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))


def _token_mask(block_mask: np.ndarray, block: int, n_valid: int) -> torch.Tensor:
    """[nqb, nkb] bool block mask -> [N, N] bool token mask, keys past n_valid dropped."""
    m = np.repeat(np.repeat(block_mask, block, axis=0), block, axis=1)
    m[:, n_valid:] = False
    return torch.from_numpy(m)


def _masked_softmax_attention(q, k, v, allow, scale):
    s = (q @ k.T) * scale
    m = torch.where(allow, s, torch.full_like(s, -1e300)).amax(dim=1, keepdim=True).detach()
    m = torch.where(torch.isfinite(m) & (m > -1e299), m, torch.zeros_like(m))
    # disallowed entries are moved to the row max first: exp of them stays finite, so
    # the masked branch contributes exact zeros to the gradient
    e = torch.where(allow, torch.exp(torch.where(allow, s, m) - m), torch.zeros_like(s))
    den = e.sum(dim=1, keepdim=True)
    return torch.where(den > 0, (e @ v) / torch.where(den > 0, den, torch.ones_like(den)),
                       torch.zeros_like(q[:, :v.shape[1]]))


def layer_forward_torch(cfg, q, k, v, w_p=None, w_g=None, classes: Optional[np.ndarray] = None):
    """Three-way layer output O [B, H, N, d] (float64 torch, differentiable in every input).

    ``classes`` [B, H, nqb, nkb] fixes the routing (default: ``sla_oracle``'s own).
    """
    c = so.OracleCfg.of(cfg)
    assert c.mode == 0, "gradients are stated for the three-way mode"
    if classes is None:
        layer = so.Layer(cfg, q.detach().numpy(), k.detach().numpy(), v.detach().numpy(),
                         None if w_p is None else w_p.detach().numpy(),
                         None if w_g is None else w_g.detach().numpy())
        classes = layer.route()[0]
    nb, bl, nv = c.nb, c.block, c.N_valid
    valid_kb = np.arange(nb) * bl < nv
    out = []
    for b in range(c.B):
        heads = []
        for h in range(c.H):
            hk = h // c.group
            cls = classes[b, h]
            crit = _token_mask(cls == so.CRITICAL, bl, nv)
            if c.linear_all:
                marg_b = np.broadcast_to(valid_kb[None, :], cls.shape).copy()
            else:
                marg_b = cls == so.MARGINAL
            marg = _token_mask(marg_b, bl, nv)
            qh, kh, vh = q[b, h], k[b, hk], v[b, hk]
            o_s = _masked_softmax_attention(qh, kh, vh, crit, c.sm_scale)
            kl = kh
            if c.smooth_k:
                kl = kh - kh[:nv].mean(dim=0, keepdim=True)
            a = (_phi(qh) @ _phi(kl).T) * marg
            den = a.sum(dim=1, keepdim=True)
            o_l = torch.where(den > 0, (a @ vh) / torch.where(den > 0, den, torch.ones_like(den)),
                              torch.zeros_like(qh))
            if c.has_proj and w_p is not None:
                o_l = o_l @ (w_p[h] if c.proj_per_head else w_p)
            if c.has_gate and w_g is not None:
                o_l = torch.sigmoid(qh @ w_g[h])[:, None] * o_l
            o = o_s + o_l
            row_ok = (torch.arange(c.N) < nv)[:, None]
            heads.append(torch.where(row_ok, o, torch.zeros_like(o)))
        out.append(torch.stack(heads))
    return torch.stack(out)


def layer_grads(cfg, q: np.ndarray, k: np.ndarray, v: np.ndarray, w_p: Optional[np.ndarray],
                w_g: Optional[np.ndarray], d_out: np.ndarray,
                classes: Optional[np.ndarray] = None) -> Dict[str, Optional[np.ndarray]]:
    """Gradients of L = sum(O * d_out) with the routing held fixed (float64 NumPy in and out).

    Returns dq, dk, dv ([B, H(_kv), N, d]), dw_p (shape of w_p or None), dw_g
    ([H, d] or None) and O.
    """
    c = so.OracleCfg.of(cfg)
    t = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tq, tk, tv = t(q), t(k), t(v)
    twp = t(w_p) if c.has_proj else None
    twg = t(w_g) if c.has_gate else None
    if classes is None:
        classes = so.Layer(cfg, q, k, v, w_p, w_g).route()[0]
    o = layer_forward_torch(cfg, tq, tk, tv, twp, twg, classes)
    loss = (o * torch.from_numpy(np.asarray(d_out, dtype=np.float64))).sum()
    loss.backward()
    # an input with no path to the loss (e.g. no linear branch) has a zero gradient
    g = lambda x: None if x is None else (x.grad if x.grad is not None else torch.zeros_like(x)).detach().numpy().copy()
    return dict(dq=g(tq), dk=g(tk), dv=g(tv), dw_p=g(twp), dw_g=g(twg), O=o.detach().numpy())
