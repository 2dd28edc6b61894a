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
* Top-n mode: O = O_s under the element mask (selected blocks or window,
  causal). With NSA's branches (sparse attention survey, section 2, NSA's three
  parallel branches): O = sum_b g_b o_b over the compressed branch (attention
  over the block means of cmp_block tokens at cmp_stride, C = A K and A V with
  A the averaging matrix, causal at the block's last token), the selected
  branch and the window branch, each its own softmax, g_b = sigmoid(q .
  w_g[h][b]) or 1.

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


def _topn_allow(c, sel_rows, part: str = "union") -> torch.Tensor:
    """[N, N] bool, top-n mode: query t attends key s when s <= t, s is valid, and s's
    block is selected for t's block or s > t - window (``part`` "union"); NSA's selected
    branch keeps only the first condition ("sel"), its window branch only the second
    ("win")."""
    N, bl, nv = c.N, c.block, c.N_valid
    selm = np.zeros((c.nb, c.nb), dtype=bool)
    for i, row in enumerate(sel_rows):
        selm[i, np.asarray(row, dtype=np.int64)] = True
    t = np.arange(N)[:, None]
    s = np.arange(N)[None, :]
    in_sel = selm[t // bl, s // bl]
    in_win = (s > t - c.window) if c.window > 0 else np.zeros((N, N), dtype=bool)
    allowed = {"union": in_sel | in_win, "sel": in_sel, "win": in_win}[part]
    return torch.from_numpy((s <= t) & (s < nv) & allowed)


def _compression(c):
    """NSA's compressed branch as a linear map: the [n_c, N] matrix whose row c averages
    tokens c*stride .. c*stride + length - 1 (compressed blocks of valid tokens only), and
    the [N, n_c] causal mask (query t attends block c when c*stride + length - 1 <= t)."""
    length, stride, nv = c.cmp_block, c.cmp_stride, c.N_valid
    n_c = (nv - length) // stride + 1 if nv >= length else 0
    m = np.zeros((n_c, c.N))
    for j in range(n_c):
        m[j, j * stride:j * stride + length] = 1.0 / length
    t = np.arange(c.N)[:, None]
    allow = np.arange(n_c)[None, :] * stride + length - 1 <= t
    return torch.from_numpy(m), torch.from_numpy(allow)


def _nsa_head(c, qh, kh, vh, sel_rows, w_g_head):
    """NSA's three branches for one query head: compressed, selected and window attention,
    each its own softmax, summed with the gates sigmoid(q . w_g[h][b]) (1 without gates)."""
    mc, allow_c = _compression(c)
    if mc.shape[0] > 0:
        o_cmp = _masked_softmax_attention(qh, mc @ kh, mc @ vh, allow_c, c.sm_scale)
    else:
        o_cmp = torch.zeros_like(qh)
    o_slc = _masked_softmax_attention(qh, kh, vh, _topn_allow(c, sel_rows, "sel"), c.sm_scale)
    o_win = _masked_softmax_attention(qh, kh, vh, _topn_allow(c, sel_rows, "win"), c.sm_scale)
    if w_g_head is not None:
        g = torch.sigmoid(qh @ w_g_head.T)  # [N, 3]: compressed, selected, window
        return g[:, 0:1] * o_cmp + g[:, 1:2] * o_slc + g[:, 2:3] * o_win
    return o_cmp + o_slc + o_win


def layer_forward_torch(cfg, q, k, v, w_p=None, w_g=None, classes=None):
    """Layer output O [B, H, N, d] (float64 torch, differentiable in every input).

    ``classes`` fixes the routing (default: ``sla_oracle``'s own): the three-way
    classes [B, H, nqb, nkb], or in the top-n mode the selected lists
    [B][H_kv][nqb] (the top-n mode has no linear branch: O = O_s, or with NSA's
    branches the gated sum of the compressed, selected and window attentions).
    """
    c = so.OracleCfg.of(cfg)
    if classes is None:
        layer = so.Layer(cfg, q.detach().numpy(), k.detach().numpy(), v.detach().numpy(),
                         None if w_p is None else w_p.detach().numpy(),
                         None if w_g is None else w_g.detach().numpy())
        classes = layer.route()[0]
    if c.mode != 0:
        out = []
        for b in range(c.B):
            heads = []
            for h in range(c.H):
                hk = h // c.group
                if c.nsa_branches:
                    o = _nsa_head(c, q[b, h], k[b, hk], v[b, hk], classes[b][hk],
                                  w_g[h] if c.has_gate and w_g is not None else None)
                else:
                    o = _masked_softmax_attention(q[b, h], k[b, hk], v[b, hk],
                                                  _topn_allow(c, classes[b][hk]), c.sm_scale)
                row_ok = (torch.arange(c.N) < c.N_valid)[:, None]
                heads.append(torch.where(row_ok, o, torch.zeros_like(o)))
            out.append(torch.stack(heads))
        return torch.stack(out)
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
                classes=None) -> Dict[str, Optional[np.ndarray]]:
    """Gradients of L = sum(O * d_out) with the routing held fixed (float64 NumPy in and out).
    ``classes``: as for ``layer_forward_torch``.

    Returns dq, dk, dv ([B, H(_kv), N, d]), dw_p (shape of w_p or None), dw_g
    ([H, d]; [H, 3, d] with NSA's branches; or None) and O.
    """
    c = so.OracleCfg.of(cfg)
    t = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tq, tk, tv = t(q), t(k), t(v)
    twp = t(w_p) if c.has_proj and c.mode == 0 else None
    twg = t(w_g) if c.has_gate and (c.mode == 0 or c.nsa_branches) else None
    if classes is None:
        classes = so.Layer(cfg, q, k, v, w_p, w_g).route()[0]
    o = layer_forward_torch(cfg, tq, tk, tv, twp, twg, classes)
    loss = (o * torch.from_numpy(np.asarray(d_out, dtype=np.float64))).sum()
    loss.backward()
    # an input with no path to the loss (e.g. no linear branch) has a zero gradient
    g = lambda x: None if x is None else (x.grad if x.grad is not None else torch.zeros_like(x)).detach().numpy().copy()
    return dict(dq=g(tq), dk=g(tk), dv=g(tv), dw_p=g(twp), dw_g=g(twg), O=o.detach().numpy())


# ---------------------------------------------------------------------------
# the same gradients block by block (full-size layers, sampled blocks)
# ---------------------------------------------------------------------------

def _dphi(x: np.ndarray) -> np.ndarray:
    """phi'(x) for phi = elu + 1: 1 for x > 0, e^x otherwise."""
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def block_grads(cfg, q, k, v, w_p, w_g, d_out, classes, b: int, q_blocks, k_blocks, heads=None):
    """Exact float64 gradients on chosen blocks, by the chain rule written out per block.

    An independent statement of what ``layer_grads`` computes by autograd, for
    layers too large for the token grid. For batch b it returns
      dq[(h, i)]  rows of query block i of head h        (every h in ``heads``)
      dk[(hk, j)], dv[(hk, j)]  rows of key block j of KV head hk, summed over the
                  query heads of its group that are in ``heads``
      dw_p        the contribution of ``heads`` to dW_p (shape of w_p), dw_g[h] rows.
    Steps (routing fixed; phi = elu + 1; s = softmax scale):
      sparse  per query block i over its critical tokens C_i: P = softmax(s Q_i K_C^T),
              O_s = P V_C, dP = dO_i V_C^T, D = rowsum(dO_i * O_s), dS = P * (dP - D);
              dq += s dS K_C, dK_C += s dS^T Q_i, dV_C += P^T dO_i
      linear  S_i = sum_{j in M_i} phi(K_j)^T V_j, Z_i likewise, O_l = phi(q) S_i / den,
              den = phi(q) . Z_i; u = O_l W_p, du = g dO, dO_l = du W_p^T;
              dq += (dO_l S_i^T - (dO_l . O_l) Z_i) / den * phi'(q);
              dS_i = sum_t phi(q_t)^T dO_l,t / den_t, dZ_i = -sum_t phi(q_t) (dO_l,t . O_l,t) / den_t;
              dh_j = sum_{i: j in M_i} dS_i, dz_j likewise;
              dV_j += phi(K_j) dh_j, dK_j += (V_j dh_j^T + dz_j) * phi'(K_j); dW_p += O_l^T du
              (smooth-K: K_j - m in phi and phi', and every valid row of dK also gets
              -1/N_valid times the sum over the head's valid tokens of that linear term)
      gate    g = sigmoid(q . w_g[h]), dlogit = (dO . u) g (1 - g): dq += dlogit w_g[h],
              dw_g[h] += sum_t dlogit q_t
    Padding rows (index >= N_valid) contribute nothing and get zero rows.
    """
    c = so.OracleCfg.of(cfg)
    if c.mode != 0 and c.nsa_branches:
        return _block_grads_nsa(c, q, k, v, w_g if c.has_gate else None, d_out, classes, b, q_blocks, k_blocks,
                                heads)
    if c.mode != 0:
        return _block_grads_topn(c, q, k, v, d_out, classes, b, q_blocks, k_blocks, heads)
    nb, bl, nv, d, s = c.nb, c.block, c.N_valid, c.d, c.sm_scale
    heads = list(range(c.H)) if heads is None else list(heads)
    q_blocks, k_blocks = list(q_blocks), list(k_blocks)
    out = dict(dq={}, dk={}, dv={}, dw_g={},
               dw_p=None if not c.has_proj else np.zeros(np.shape(w_p)))
    valid_kb = np.arange(nb) * bl < nv
    rows_of = lambda i: slice(i * bl, min((i + 1) * bl, nv))
    for h in heads:
        hk = h // c.group
        Q = np.asarray(q[b, h], dtype=np.float64)
        K = np.asarray(k[b, hk], dtype=np.float64)
        V = np.asarray(v[b, hk], dtype=np.float64)
        dO = np.asarray(d_out[b, h], dtype=np.float64).copy()
        dO[nv:] = 0.0
        cls = classes[b, h]
        wp = None
        if c.has_proj:
            wp = np.asarray(w_p[h] if c.proj_per_head else w_p, dtype=np.float64)
        # ---- linear branch, every query block (dk / dv of any key block need all of them)
        marg = (np.broadcast_to(valid_kb[None, :], cls.shape) if c.linear_all else cls == so.MARGINAL)
        Mf = marg.astype(np.float64)
        # smooth-K: the linear branch sees K minus the mean valid key
        koff = so.key_mean(K, nv) if c.smooth_k else np.zeros(d)
        Kl = K - koff[None, :]
        hs, zs = so.linear_states(K, V, nv, bl, koff if c.smooth_k else None)
        S = (Mf @ hs.reshape(nb, d * d)).reshape(nb, d, d)
        Z = Mf @ zs
        phq = so.phi(Q)
        phq[nv:] = 0.0
        den = np.zeros(c.N)
        Ol = np.zeros((c.N, d))
        for i in range(nb):
            r = rows_of(i)
            if r.start >= r.stop:
                continue
            den[r] = phq[r] @ Z[i]
            num = phq[r] @ S[i]
            Ol[r] = np.where(den[r, None] > 0, num / np.where(den[r, None] > 0, den[r, None], 1.0), 0.0)
        u = Ol @ wp if wp is not None else Ol
        g = so.sigmoid(Q @ np.asarray(w_g[h], dtype=np.float64)) if c.has_gate else np.ones(c.N)
        g[nv:] = 0.0
        du = g[:, None] * dO
        dOl = du @ wp.T if wp is not None else du
        if wp is not None:
            if c.proj_per_head:
                out["dw_p"][h] += Ol.T @ du
            else:
                out["dw_p"] += Ol.T @ du
        dlogit = np.zeros(c.N)
        if c.has_gate:
            dlogit = (dO * u).sum(axis=1) * g * (1.0 - g)
            dlogit[nv:] = 0.0
            out["dw_g"][h] = dlogit @ Q
        inv = np.where(den > 0, 1.0 / np.where(den > 0, den, 1.0), 0.0)
        cdot = (dOl * Ol).sum(axis=1) * inv  # (dO_l . O_l) / den
        dS = np.zeros((nb, d, d))
        dZ = np.zeros((nb, d))
        for i in range(nb):
            r = rows_of(i)
            if r.start >= r.stop:
                continue
            dS[i] = phq[r].T @ (dOl[r] * inv[r, None])
            dZ[i] = -(phq[r] * cdot[r, None]).sum(axis=0)

        # ---- sparse branch per query block (cached: dk / dv revisit blocks)
        cache = {}

        def sparse(i):
            if i not in cache:
                r = rows_of(i)
                crit = np.nonzero(cls[i] == so.CRITICAL)[0]
                toks = np.concatenate([np.arange(j * bl, min((j + 1) * bl, nv)) for j in crit]) \
                    if crit.size else np.zeros(0, np.int64)
                if toks.size == 0 or r.start >= r.stop:
                    cache[i] = (toks, None, None)
                else:
                    x = Q[r] @ K[toks].T * s
                    P = np.exp(x - x.max(axis=1, keepdims=True))
                    P /= P.sum(axis=1, keepdims=True)
                    Os = P @ V[toks]
                    dP = dO[r] @ V[toks].T
                    dSm = P * (dP - (dO[r] * Os).sum(axis=1, keepdims=True))
                    cache[i] = (toks, P, dSm)
            return cache[i]

        for i in q_blocks:
            r = rows_of(i)
            g_rows = np.zeros((bl, d))
            n = r.stop - r.start
            if n > 0:
                toks, P, dSm = sparse(i)
                dq = np.zeros((n, d))
                if P is not None:
                    dq += s * dSm @ K[toks]
                dphi = (dOl[r] @ S[i].T - (dOl[r] * Ol[r]).sum(axis=1, keepdims=True) * Z[i][None, :]) \
                    * inv[r, None]
                dq += dphi * _dphi(Q[r])
                if c.has_gate:
                    dq += dlogit[r, None] * np.asarray(w_g[h], dtype=np.float64)[None, :]
                g_rows[:n] = dq
            out["dq"][(h, i)] = g_rows
        # smooth-K: dk_t = dkl_t - mean over the valid tokens of dkl (dkl = gradient through k - m)
        kmean_grad = np.zeros(d)
        if c.smooth_k:
            dH = (Mf.T @ dS.reshape(nb, d * d)).reshape(nb, d, d)
            dZk = Mf.T @ dZ
            for j in range(nb):
                rk = rows_of(j)
                if rk.start >= rk.stop:
                    continue
                dkl = (V[rk] @ dH[j].T + dZk[j][None, :]) * _dphi(Kl[rk])
                kmean_grad += dkl.sum(axis=0)
            kmean_grad /= nv
        for j in k_blocks:
            rk = rows_of(j)
            nk = rk.stop - rk.start
            dk = out["dk"].setdefault((hk, j), np.zeros((bl, d)))
            dv = out["dv"].setdefault((hk, j), np.zeros((bl, d)))
            if nk == 0:
                continue
            for i in np.nonzero(cls[:, j] == so.CRITICAL)[0]:
                toks, P, dSm = sparse(i)
                if P is None:
                    continue
                sel = (toks >= rk.start) & (toks < rk.stop)
                r = rows_of(i)
                dv[:nk] += P[:, sel].T @ dO[r]
                dk[:nk] += s * dSm[:, sel].T @ Q[r]
            dh = Mf[:, j] @ dS.reshape(nb, d * d)
            dz = Mf[:, j] @ dZ
            dh = dh.reshape(d, d)
            phk = so.phi(Kl[rk])
            dv[:nk] += phk @ dh
            dk[:nk] += (V[rk] @ dh.T + dz[None, :]) * _dphi(Kl[rk]) - kmean_grad[None, :]
    return out


def _block_grads_topn(c, q, k, v, d_out, sels, b, q_blocks, k_blocks, heads=None):
    """Top-n mode of ``block_grads`` (sparse branch only). Query block i attends the
    tokens of its candidate blocks (selected blocks of its KV group and the blocks the
    causal window reaches) under the element mask s <= t, s valid, (block(s) selected
    or s > t - window); then P, dP, dS and the three products as in the three-way mode."""
    nb, bl, nv, d, s = c.nb, c.block, c.N_valid, c.d, c.sm_scale
    heads = list(range(c.H)) if heads is None else list(heads)
    out = dict(dq={}, dk={}, dv={}, dw_g={}, dw_p=None)
    rows_of = lambda i: slice(i * bl, min((i + 1) * bl, nv))

    def cand_blocks(sel, i):
        first = max(0, (i * bl - c.window + 1) // bl) if c.window > 0 else i + 1
        return sorted(set(int(j) for j in sel) | set(range(first, i + 1)))

    for h in heads:
        hk = h // c.group
        Q = np.asarray(q[b, h], dtype=np.float64)
        K = np.asarray(k[b, hk], dtype=np.float64)
        V = np.asarray(v[b, hk], dtype=np.float64)
        dO = np.asarray(d_out[b, h], dtype=np.float64).copy()
        dO[nv:] = 0.0
        sel_rows = sels[b][hk]
        cache = {}

        def sparse(i):
            if i not in cache:
                r = rows_of(i)
                blocks = cand_blocks(sel_rows[i], i)
                toks = np.concatenate([np.arange(j * bl, min((j + 1) * bl, nv)) for j in blocks]) \
                    if blocks else np.zeros(0, np.int64)
                if toks.size == 0 or r.start >= r.stop:
                    cache[i] = (toks, None, None)
                else:
                    t = np.arange(r.start, r.stop)[:, None]
                    sj = toks[None, :]
                    in_sel = np.isin(sj // bl, np.asarray(sel_rows[i], dtype=np.int64))
                    in_win = (sj > t - c.window) if c.window > 0 else np.zeros_like(in_sel)
                    allow = (sj <= t) & (in_sel | in_win)
                    x = np.where(allow, Q[r] @ K[toks].T * s, -np.inf)
                    m = x.max(axis=1, keepdims=True)
                    m = np.where(np.isfinite(m), m, 0.0)
                    P = np.where(allow, np.exp(x - m), 0.0)
                    den = P.sum(axis=1, keepdims=True)
                    P = np.where(den > 0, P / np.where(den > 0, den, 1.0), 0.0)
                    Os = P @ V[toks]
                    dP = dO[r] @ V[toks].T
                    dSm = P * (dP - (dO[r] * Os).sum(axis=1, keepdims=True))
                    cache[i] = (toks, P, dSm)
            return cache[i]

        for i in q_blocks:
            r = rows_of(i)
            g_rows = np.zeros((bl, d))
            n = r.stop - r.start
            if n > 0:
                toks, P, dSm = sparse(i)
                if P is not None:
                    g_rows[:n] = s * dSm @ K[toks]
            out["dq"][(h, i)] = g_rows
        for j in k_blocks:
            rk = rows_of(j)
            nk = rk.stop - rk.start
            dk = out["dk"].setdefault((hk, j), np.zeros((bl, d)))
            dv = out["dv"].setdefault((hk, j), np.zeros((bl, d)))
            if nk == 0:
                continue
            for i in range(j, nb):
                if j not in cand_blocks(sel_rows[i], i):
                    continue
                toks, P, dSm = sparse(i)
                if P is None:
                    continue
                selc = (toks >= rk.start) & (toks < rk.stop)
                r = rows_of(i)
                dv[:nk] += P[:, selc].T @ dO[r]
                dk[:nk] += s * dSm[:, selc].T @ Q[r]
    return out


def _softmax_rows(x: np.ndarray, allow: np.ndarray) -> np.ndarray:
    """Row softmax of x over the allowed entries (rows with none give 0)."""
    x = np.where(allow, x, -np.inf)
    m = x.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(allow, np.exp(x - m), 0.0)
    den = e.sum(axis=1, keepdims=True)
    return np.where(den > 0, e / np.where(den > 0, den, 1.0), 0.0)


def _block_grads_nsa(c, q, k, v, w_g, d_out, sels, b, q_blocks, k_blocks, heads=None):
    """NSA's three branches (top-n mode with nsa_branches) block by block. Per query head h
    and valid row t: o_b = softmax attention of branch b (compressed keys and values A K,
    A V with t attending block c when c * stride + length - 1 <= t; the selected blocks of
    t's block; the window t - window < s <= t), O = sum_b g_b o_b, g_b = sigmoid(q_t .
    w_g[h][b]) (1 without gates). With dO_b = g_b dO: D_b = dO_b . o_b, dP_b = dO_b V_b^T,
    dS_b = P_b (dP_b - D_b); dq += s dS_b K_b + sum_b dlogit_b w_g[h][b] with dlogit_b =
    (dO . o_b) g_b (1 - g_b); dK_b += s dS_b^T q, dV_b += P_b^T dO_b; the compressed keys'
    and values' gradients go back to each token of their block with weight 1 / length.
    The compressed branch runs over every valid row of each head (a compressed key's
    gradient gathers from every later query). dk, dv sum over the KV group's heads in
    ``heads``; dw_g[h] (all three rows) for every head in ``heads``."""
    nb, bl, nv, d, s = c.nb, c.block, c.N_valid, c.d, c.sm_scale
    length, stride = c.cmp_block, c.cmp_stride
    n_c = (nv - length) // stride + 1 if nv >= length else 0
    heads = list(range(c.H)) if heads is None else list(heads)
    q_blocks, k_blocks = list(q_blocks), list(k_blocks)
    out = dict(dq={}, dk={}, dv={}, dw_g={}, dw_p=None)
    rows_of = lambda i: slice(i * bl, min((i + 1) * bl, nv))
    clast = np.arange(n_c) * stride + length - 1  # query t attends block c when clast[c] <= t
    for hk in sorted({h // c.group for h in heads}):
        K = np.asarray(k[b, hk], dtype=np.float64)
        V = np.asarray(v[b, hk], dtype=np.float64)
        Kc = np.stack([K[j * stride:j * stride + length].mean(axis=0) for j in range(n_c)]) if n_c else np.zeros((0, d))
        Vc = np.stack([V[j * stride:j * stride + length].mean(axis=0) for j in range(n_c)]) if n_c else np.zeros((0, d))
        sel_rows = sels[b][hk]
        dKc, dVc = np.zeros((n_c, d)), np.zeros((n_c, d))
        dk = {j: np.zeros((bl, d)) for j in k_blocks}
        dv = {j: np.zeros((bl, d)) for j in k_blocks}
        for h in [x for x in heads if x // c.group == hk]:
            Q = np.asarray(q[b, h], dtype=np.float64)
            dO = np.asarray(d_out[b, h], dtype=np.float64).copy()
            dO[nv:] = 0.0
            if w_g is not None:
                g = so.sigmoid(Q @ np.asarray(w_g[h], dtype=np.float64).T)  # [N, 3]
            else:
                g = np.ones((c.N, 3))
            dlogit = np.zeros((c.N, 3))
            dq_cmp = {}
            # ---- compressed branch over every valid row
            for r0 in range(0, nv, 4096):
                r1 = min(nv, r0 + 4096)
                t = np.arange(r0, r1)
                if n_c == 0:
                    continue
                allow = clast[None, :] <= t[:, None]
                P = _softmax_rows(Q[r0:r1] @ Kc.T * s, allow)
                oc = P @ Vc
                dOc = g[r0:r1, 0:1] * dO[r0:r1]
                dS = P * (dOc @ Vc.T - (dOc * oc).sum(axis=1, keepdims=True))
                dKc += s * dS.T @ Q[r0:r1]
                dVc += P.T @ dOc
                dlogit[r0:r1, 0] = (dO[r0:r1] * oc).sum(axis=1)
                for i in q_blocks:
                    r = rows_of(i)
                    lo, hi = max(r.start, r0), min(r.stop, r1)
                    if lo < hi:
                        dq_cmp.setdefault(i, np.zeros((bl, d)))[lo - r.start:hi - r.start] = \
                            s * dS[lo - r0:hi - r0] @ Kc

            # ---- selected and window branches of query block i
            def branch(i, kind):
                r = rows_of(i)
                t = np.arange(r.start, r.stop)[:, None]
                if kind == "sel":
                    blocks = sorted(int(j) for j in sel_rows[i])
                else:
                    first = max(0, (i * bl - c.window + 1) // bl) if c.window > 0 else i + 1
                    blocks = list(range(first, i + 1))
                toks = np.concatenate([np.arange(j * bl, min((j + 1) * bl, nv)) for j in blocks]) \
                    if blocks else np.zeros(0, np.int64)
                if toks.size == 0 or r.start >= r.stop:
                    return toks, None, None, None
                sj = toks[None, :]
                allow = (sj <= t) & ((sj > t - c.window) if kind == "win" else True)
                P = _softmax_rows(Q[r] @ K[toks].T * s, allow)
                ob = P @ V[toks]
                gb = g[r, 1 if kind == "sel" else 2][:, None]
                dOb = gb * dO[r]
                dS = P * (dOb @ V[toks].T - (dOb * ob).sum(axis=1, keepdims=True))
                return toks, P, dS, (ob, dOb)

            for i in range(nb):
                r = rows_of(i)
                if r.start >= r.stop:
                    continue
                for col, kind in ((1, "sel"), (2, "win")):
                    toks, P, dS, extra = branch(i, kind)
                    if P is None:
                        continue
                    ob, dOb = extra
                    dlogit[r, col] = (dO[r] * ob).sum(axis=1)
                    n = r.stop - r.start
                    if i in q_blocks:
                        dq_cmp.setdefault(i, np.zeros((bl, d)))[:n] += s * dS @ K[toks]
                    for j in k_blocks:
                        rk = slice(j * bl, min((j + 1) * bl, nv))
                        nk = rk.stop - rk.start
                        selc = (toks >= rk.start) & (toks < rk.stop)
                        if nk <= 0 or not selc.any():
                            continue
                        dv[j][:nk] += P[:, selc].T @ dOb
                        dk[j][:nk] += s * dS[:, selc].T @ Q[r]
            dlogit = dlogit * g * (1.0 - g) if w_g is not None else np.zeros_like(dlogit)
            dlogit[nv:] = 0.0
            for i in q_blocks:
                r = rows_of(i)
                rows = dq_cmp.get(i, np.zeros((bl, d))).copy()
                n = max(0, r.stop - r.start)
                if w_g is not None and n > 0:
                    rows[:n] += dlogit[r] @ np.asarray(w_g[h], dtype=np.float64)
                out["dq"][(h, i)] = rows
            if w_g is not None:
                out["dw_g"][h] = dlogit.T @ Q
        # ---- the compressed keys' and values' gradients back to their tokens
        for j in k_blocks:
            for x in range(bl):
                tok = j * bl + x
                if tok >= nv:
                    continue
                cs = [cc for cc in range(n_c) if cc * stride <= tok <= cc * stride + length - 1]
                for cc in cs:
                    dk[j][x] += dKc[cc] / length
                    dv[j][x] += dVc[cc] / length
            out["dk"][(hk, j)] = dk[j]
            out["dv"][(hk, j)] = dv[j]
    return out
