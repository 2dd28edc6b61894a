"""Float64 CPU oracle of the block-routed sparse+linear attention layer.

TEST INFRASTRUCTURE. This module is the plain, slow statement of what the layer
computes, written from the pages' description and used only to check the CUDA
path. It shares no code with that path and imports nothing from it. Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import it. The product never routes through it.

Everything is float64 NumPy. Inputs arrive as float64 arrays holding the exact
values of the bf16 inputs. One unit of work is one (batch, head, query block).

What each step follows (page title, section):

* Block pooling: SLA analysis (arXiv 2509.24006), paragraph on compressed
  attention prediction - mean pooling reduces the N x N map to an (N/b)^2
  block problem; 2025 sparse-attention review, section 11 (SpargeAttn),
  prediction algorithm - q_i = mean(Q_i), k_j = mean(K_j).
* Pooled scores: same SpargeAttn passage - S_hat[i] = q_i k^T,
  P_hat[i] = Softmax(S_hat[i]); scaled by 1/sqrt(d) as for attention logits.
* Three-way classification: SLA analysis, core-innovation paragraph
  (critical / marginal / negligible per Q-K block pair) and the SLA2 remark
  (block-level TopK / BottomK); 2025 review, section 10 (SLA).
* Top-n selection with a window: 2025 review, section 4 (MoBA: block
  representative, Q times compressed K, top-K); sparse attention survey,
  section 2 (NSA selected branch, block 64, n = 16; window w = 512).
* Sparse exact attention: 2025 review, section 2.3 (NSA operator design:
  fixed-size indexed KV blocks, outer loop over queries); softmax attention
  restricted to the critical blocks.
* Linear attention on marginal blocks: SLA analysis, comparison table
  (linear attention at O(N d^2)) and core-innovation paragraph; the kernel
  map phi = elu + 1 (the pages leave phi open).
* Combine: SLA analysis, Proj paragraph - O = O^s + Proj(O^l); SALAD summary,
  method details - an input-dependent gate balances the two branches.
* Key-block similarity filter: 2025 review, section 11 (SpargeAttn), prediction
  algorithm - s_kj = CosSim(K_j) and S_hat[i, j] = -inf when s_kj < theta.
  CosSim is read as the mean cosine similarity over all ordered pairs of the
  block's valid tokens, self-pairs included: |sum_t k_t / |k_t||^2 / n^2 (a
  zero token counts as the zero vector). Filtered blocks rank below every
  other block (equal scores: lower index first) and get probability 0 in the
  top-n softmax; a row whose candidates are all filtered has all
  probabilities 0.
* NSA's three branches (top-n mode option): sparse attention survey, section 2
  (NSA: a compressed branch over coarse blocks of 32 tokens at stride 16, the
  selected branch and the sliding window, in parallel); each branch is its own
  softmax and the branches are summed with per-head gates g = sigmoid(q . w_g)
  (one gate vector per branch; g = 1 without a gate). The compression is read
  as the mean of each compressed block, and a query attends the compressed
  blocks that lie entirely in its past.
* Token reordering: 2025 review, section 11 (SpargeAttn), the token-reorder
  note - ordering tokens along a Hilbert curve raises the similarity of the
  tokens that share a block. The curve is the 3-D Hilbert curve over the
  (t, h, w) grid, computed with Skilling's axes-to-transpose method ("Programming
  the Hilbert curve", AIP Conf. Proc. 707, 2004); tokens are ordered by their
  key on the smallest power-of-two cube holding the grid.
* Options from the SLA critique page's notes on the open-source code: smooth-K
  (K made zero-mean; here: minus the mean of the head's valid key tokens,
  which only changes phi(K) since softmax rows and pooled rankings shift by a
  per-row constant) and the linear branch over all tokens instead of the
  marginal blocks only.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

CRITICAL = 2
MARGINAL = 1
NEGLIGIBLE = 0

TIE_REL = 1e-5


# ---------------------------------------------------------------------------
# elementary steps
# ---------------------------------------------------------------------------

def phi(x: np.ndarray) -> np.ndarray:
    """Feature map of the linear branch: elu(x) + 1 (x + 1 for x > 0, e^x otherwise)."""
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def pool_blocks(x: np.ndarray, n_valid: int, block: int) -> np.ndarray:
    """Mean of the valid tokens of each block: x [N, d] -> [N/block, d].

    A block with no valid token pools to zero.
    """
    n, d = x.shape
    nb = n // block
    out = np.zeros((nb, d))
    for j in range(nb):
        lo = j * block
        hi = min(lo + block, n_valid)
        if hi > lo:
            out[j] = x[lo:hi].sum(axis=0) / (hi - lo)
    return out


def pooled_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """s_ij = (qbar_i . kbar_j) * scale."""
    return (qbar @ kbar.T) * scale


def softmax(s: np.ndarray) -> np.ndarray:
    """Row softmax (max-subtracted); a row of -inf only gives zeros."""
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    tot = e.sum(axis=-1, keepdims=True)
    return np.where(tot > 0, e / np.where(tot > 0, tot, 1.0), 0.0)


def block_cos_sims(x: np.ndarray, n_valid: int, block: int) -> np.ndarray:
    """CosSim of every block: |sum_t x_t / |x_t||^2 / n^2 over its n valid tokens (0 if none)."""
    nb = x.shape[0] // block
    out = np.zeros(nb)
    for j in range(nb):
        lo, hi = j * block, min((j + 1) * block, n_valid)
        if hi <= lo:
            continue
        xs = x[lo:hi]
        nrm = np.linalg.norm(xs, axis=1)
        unit = xs / np.where(nrm > 0, nrm, 1.0)[:, None]
        acc = unit.sum(axis=0)
        out[j] = float(acc @ acc) / float((hi - lo) ** 2)
    return out


def block_order(score_row: np.ndarray) -> np.ndarray:
    """Indices sorted by score descending; equal scores keep the lower index first."""
    return np.argsort(-score_row, kind="stable")


def classify_threeway(scores: np.ndarray, k_h: int, k_l: int) -> np.ndarray:
    """Per row: the k_h best blocks are critical, the k_l worst negligible, the rest marginal."""
    nqb, nkb = scores.shape
    assert 0 <= k_h and 0 <= k_l and k_h + k_l <= nkb
    cls = np.full((nqb, nkb), MARGINAL, dtype=np.int8)
    for i in range(nqb):
        o = block_order(scores[i])
        cls[i, o[:k_h]] = CRITICAL
        if k_l > 0:
            cls[i, o[nkb - k_l:]] = NEGLIGIBLE
    return cls


def threeway_tie_rows(scores: np.ndarray, k_h: int, k_l: int, rel: float = TIE_REL) -> np.ndarray:
    """Rows whose class boundary separates two pooled probabilities within ``rel``.

    The boundaries are between sorted positions k_h-1 / k_h and nkb-k_l-1 / nkb-k_l;
    probabilities are the row softmax of the pooled scores.
    """
    nqb, nkb = scores.shape
    p = softmax(scores)
    tie = np.zeros(nqb, dtype=bool)
    for i in range(nqb):
        o = block_order(scores[i])
        for pos in (k_h, nkb - k_l):
            if 0 < pos < nkb:
                a, b = p[i, o[pos - 1]], p[i, o[pos]]
                if abs(a - b) <= rel * max(a, b):
                    tie[i] = True
    return tie


def select_topn(group_scores: Sequence[np.ndarray], top_n: int, rel: float = TIE_REL):
    """Top-n past blocks per query block, shared by the query heads of one KV group.

    For query block i the candidates are the blocks j < i. Each head's pooled
    scores over the candidates go through a softmax; the group sums the
    probabilities and keeps the min(top_n, i) largest (lower index first on
    equal sums). Returns (ascending selected lists, tie flags).
    """
    nqb, nkb = group_scores[0].shape
    sel: List[np.ndarray] = []
    tie = np.zeros(nqb, dtype=bool)
    for i in range(nqb):
        if i == 0:
            sel.append(np.zeros(0, dtype=np.int64))
            continue
        p = np.zeros(i)
        for s in group_scores:
            p += softmax(s[i, :i])
        o = block_order(p)
        n = min(top_n, i)
        sel.append(np.sort(o[:n]))
        if n < i:
            a, b = p[o[n - 1]], p[o[n]]
            tie[i] = abs(a - b) <= rel * max(a, b)
    return sel, tie


def softmax_attention(q_rows: np.ndarray, keys: np.ndarray, vals: np.ndarray, scale: float,
                      allow: Optional[np.ndarray] = None) -> np.ndarray:
    """Exact softmax attention of q_rows over (keys, vals); rows with no allowed key give 0."""
    m = q_rows.shape[0]
    out = np.zeros((m, vals.shape[1]))
    if keys.shape[0] == 0:
        return out
    s = (q_rows @ keys.T) * scale
    if allow is not None:
        s = np.where(allow, s, -np.inf)
    for r in range(m):
        row = s[r]
        if not np.isfinite(row).any():
            continue
        w = np.exp(row - row[np.isfinite(row)].max())
        out[r] = (w @ vals) / w.sum()
    return out


def key_mean(k: np.ndarray, n_valid: int) -> np.ndarray:
    """Mean of the valid key tokens of one head (the smooth-K offset)."""
    return k[:n_valid].mean(axis=0) if n_valid > 0 else np.zeros(k.shape[1])


def linear_states(k: np.ndarray, v: np.ndarray, n_valid: int, block: int,
                  k_offset: Optional[np.ndarray] = None):
    """Per key block j: h_j = phi(K_j - m)^T V_j (d x d) and z_j = sum_t phi(k_t - m), valid
    tokens only; m = k_offset (smooth-K) or 0."""
    n, d = k.shape
    if k_offset is not None:
        k = k - k_offset[None, :]
    nb = n // block
    h = np.zeros((nb, d, v.shape[1]))
    z = np.zeros((nb, d))
    for j in range(nb):
        lo = j * block
        hi = min(lo + block, n_valid)
        if hi <= lo:
            continue
        fk = phi(k[lo:hi])
        h[j] = fk.T @ v[lo:hi]
        z[j] = fk.sum(axis=0)
    return h, z


def linear_attention(q_rows: np.ndarray, s_state: np.ndarray, z_state: np.ndarray) -> np.ndarray:
    """O_l[t] = phi(q_t) S / (phi(q_t) . Z)."""
    fq = phi(q_rows)
    return (fq @ s_state) / (fq @ z_state)[:, None]


def compress_kv(x: np.ndarray, n_valid: int, length: int, stride: int) -> np.ndarray:
    """NSA compressed branch, token compression: compressed block c covers tokens
    c*stride .. c*stride + length - 1 and exists while that range holds valid tokens only;
    its key (value) is the mean of those tokens (the pages give no compression function;
    the mean is the parameter-free reading, as for the pooled routing)."""
    n_c = (n_valid - length) // stride + 1 if n_valid >= length else 0
    out = np.zeros((n_c, x.shape[1]))
    for c in range(n_c):
        out[c] = x[c * stride:c * stride + length].mean(axis=0)
    return out


def combine(o_s: np.ndarray, o_l: np.ndarray, q_rows: np.ndarray,
            w_p: Optional[np.ndarray], w_g_head: Optional[np.ndarray]) -> np.ndarray:
    """O = O_s + g * (O_l W_p); W_p = I without projection, g = 1 without gate."""
    proj = o_l @ w_p if w_p is not None else o_l
    g = sigmoid(q_rows @ w_g_head) if w_g_head is not None else np.ones(q_rows.shape[0])
    return o_s + g[:, None] * proj


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------

@dataclass
class OracleCfg:
    B: int
    H: int
    H_kv: int
    N: int
    N_valid: int
    d: int
    block: int = 64
    mode: int = 0
    k_h: int = 0
    k_l: int = 0
    top_n: int = 0
    window: int = 0
    causal: int = 0
    has_proj: int = 1
    proj_per_head: int = 0
    has_gate: int = 0
    smooth_k: int = 0    # linear branch on K minus the head's mean valid key
    linear_all: int = 0  # linear branch over every valid key block, not only the marginal ones
    cos_filter: int = 0  # pooled scores of key blocks with CosSim < cos_theta become -inf
    scale: float = 0.0
    cos_theta: float = 0.0
    nsa_branches: int = 0  # top-n mode: compressed, selected and window branches, each its own softmax
    cmp_block: int = 32    # compressed branch: tokens per compressed block ...
    cmp_stride: int = 16   # ... and the stride between compressed blocks

    OPTIONAL = ("proj_per_head", "smooth_k", "linear_all", "cos_filter", "cos_theta", "nsa_branches",
                "cmp_block", "cmp_stride")
    DEFAULTS = {"cmp_block": 32, "cmp_stride": 16}

    @classmethod
    def of(cls, c) -> "OracleCfg":
        return cls(**{f: getattr(c, f, cls.DEFAULTS.get(f, 0)) if f in cls.OPTIONAL else getattr(c, f)
                      for f in cls.__dataclass_fields__})

    @property
    def nb(self) -> int:
        return self.N // self.block

    @property
    def sm_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.H // self.H_kv


class Layer:
    """One layer's inputs (float64) with per-head caches of pooled means, classes and states."""

    def __init__(self, cfg, q, k, v, w_p=None, w_g=None):
        self.c = OracleCfg.of(cfg)
        c = self.c
        assert c.N % c.block == 0 and c.H % c.H_kv == 0
        self.q, self.k, self.v = q, k, v
        # W_p: one d x d matrix shared by the heads, or one per query head ([H, d, d])
        self.w_p = w_p if c.has_proj else None
        if self.w_p is not None:
            assert self.w_p.shape == ((c.H, c.d, c.d) if c.proj_per_head else (c.d, c.d))
        # w_g: [H, d] gate vectors; with NSA's branches [H, 3, d] (compressed, selected, window)
        self.w_g = w_g if c.has_gate else None
        self._kbar: Dict[Tuple[int, int], np.ndarray] = {}
        self._scores: Dict[Tuple[int, int], np.ndarray] = {}
        self._cls: Dict[Tuple[int, int], np.ndarray] = {}
        self._sel: Dict[Tuple[int, int], tuple] = {}
        self._states: Dict[Tuple[int, int], tuple] = {}

    # -- routing ------------------------------------------------------------
    def kbar(self, b, hk):
        key = (b, hk)
        if key not in self._kbar:
            self._kbar[key] = pool_blocks(self.k[b, hk], self.c.N_valid, self.c.block)
        return self._kbar[key]

    def scores(self, b, h):
        key = (b, h)
        if key not in self._scores:
            c = self.c
            qbar = pool_blocks(self.q[b, h], c.N_valid, c.block)
            s = pooled_scores(qbar, self.kbar(b, h // c.group), c.sm_scale)
            if c.cos_filter:
                # key blocks whose tokens are not alike are not represented by their mean
                sim = block_cos_sims(self.k[b, h // c.group], c.N_valid, c.block)
                s[:, sim < c.cos_theta] = -np.inf
            self._scores[key] = s
        return self._scores[key]

    def classes(self, b, h):
        """Mode A: int8 [nqb, nkb] of CRITICAL / MARGINAL / NEGLIGIBLE."""
        key = (b, h)
        if key not in self._cls:
            self._cls[key] = classify_threeway(self.scores(b, h), self.c.k_h, self.c.k_l)
        return self._cls[key]

    def tie_rows(self, b, h):
        return threeway_tie_rows(self.scores(b, h), self.c.k_h, self.c.k_l)

    def selection(self, b, hk):
        """Mode B: (list of ascending selected blocks per query block, tie flags)."""
        key = (b, hk)
        if key not in self._sel:
            c = self.c
            heads = range(hk * c.group, (hk + 1) * c.group)
            self._sel[key] = select_topn([self.scores(b, h) for h in heads], c.top_n)
        return self._sel[key]

    def states(self, b, hk):
        key = (b, hk)
        if key not in self._states:
            c = self.c
            off = key_mean(self.k[b, hk], c.N_valid) if c.smooth_k else None
            self._states[key] = linear_states(self.k[b, hk], self.v[b, hk], c.N_valid, c.block, off)
        return self._states[key]

    # -- one unit -----------------------------------------------------------
    def _tokens_of(self, blocks: Iterable[int]) -> np.ndarray:
        c = self.c
        toks = [np.arange(j * c.block, min((j + 1) * c.block, c.N_valid)) for j in blocks]
        toks = [t for t in toks if t.size]
        return np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)

    def unit(self, b: int, h: int, i: int, cls_row: Optional[np.ndarray] = None,
             sel_row: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
        """Outputs of query block i of head h: dict with O, O_s, O_l (each [block, d]).

        ``cls_row`` / ``sel_row`` override the oracle's own routing for this row
        (used to score outputs under another router's classes).
        Rows of padding tokens are zero.
        """
        c = self.c
        hk = h // c.group
        lo, hi = i * c.block, (i + 1) * c.block
        nv = max(0, min(hi, c.N_valid) - lo)
        d = c.d
        O = np.zeros((c.block, d))
        O_s = np.zeros((c.block, d))
        O_l = np.zeros((c.block, d))
        if nv == 0:
            return dict(O=O, O_s=O_s, O_l=O_l)
        qr = self.q[b, h, lo:lo + nv]
        K, V = self.k[b, hk], self.v[b, hk]
        if c.mode == 0:
            row = self.classes(b, h)[i] if cls_row is None else cls_row
            crit = self._tokens_of(np.nonzero(row == CRITICAL)[0])
            o_s = softmax_attention(qr, K[crit], V[crit], c.sm_scale)
            # the linear branch covers the marginal blocks, or every block holding a
            # valid token with linear_all
            marg = (np.arange(c.nb)[np.arange(c.nb) * c.block < c.N_valid] if c.linear_all
                    else np.nonzero(row == MARGINAL)[0])
            if marg.size:
                hs, zs = self.states(b, hk)
                o_l = linear_attention(qr, hs[marg].sum(axis=0), zs[marg].sum(axis=0))
            else:
                o_l = np.zeros_like(qr)
            w_g = self.w_g[h] if self.w_g is not None else None
            w_p = self.w_p[h] if self.w_p is not None and c.proj_per_head else self.w_p
            o = combine(o_s, o_l, qr, w_p, w_g)
        else:
            sel = self.selection(b, hk)[0][i] if sel_row is None else sel_row
            # candidate tokens: selected blocks plus the blocks the window can reach
            first_win = max(0, (lo - c.window + 1) // c.block) if c.window > 0 else i + 1
            blocks = sorted(set(int(j) for j in sel) | set(range(first_win, i + 1)))
            cand = self._tokens_of(blocks)
            t = np.arange(lo, lo + nv)[:, None]
            s = cand[None, :]
            in_sel = np.isin(s // c.block, np.asarray(sel, dtype=np.int64))
            in_win = (s > t - c.window) if c.window > 0 else np.zeros_like(in_sel)
            if not c.nsa_branches:
                # one softmax over selected blocks and window together
                allow = (s <= t) & (in_sel | in_win)
                o_s = softmax_attention(qr, K[cand], V[cand], c.sm_scale, allow)
                o = o_s
            else:
                # NSA's three branches, each its own softmax, combined with per-head gates
                o_slc = softmax_attention(qr, K[cand], V[cand], c.sm_scale, (s <= t) & in_sel)
                o_win = softmax_attention(qr, K[cand], V[cand], c.sm_scale, (s <= t) & in_win)
                Kc, Vc = self.compressed(b, hk)
                cidx = np.arange(Kc.shape[0])[None, :]
                o_cmp = softmax_attention(qr, Kc, Vc, c.sm_scale,
                                          cidx * c.cmp_stride + c.cmp_block - 1 <= t)
                g = (sigmoid(qr @ self.w_g[h].T) if self.w_g is not None else np.ones((nv, 3)))
                o = g[:, 0:1] * o_cmp + g[:, 1:2] * o_slc + g[:, 2:3] * o_win
                o_s = o
            o_l = np.zeros_like(qr)
        O[:nv], O_s[:nv], O_l[:nv] = o, o_s, o_l
        return dict(O=O, O_s=O_s, O_l=O_l)

    def compressed(self, b, hk):
        """NSA compressed keys and values of KV head hk (cached)."""
        key = ("cmp", b, hk)
        if key not in self._states:
            c = self.c
            self._states[key] = (compress_kv(self.k[b, hk], c.N_valid, c.cmp_block, c.cmp_stride),
                                 compress_kv(self.v[b, hk], c.N_valid, c.cmp_block, c.cmp_stride))
        return self._states[key]

    # -- whole layer ----------------------------------------------------------
    def forward(self) -> Dict[str, np.ndarray]:
        c = self.c
        out = {k: np.zeros((c.B, c.H, c.N, c.d)) for k in ("O", "O_s", "O_l")}
        for b in range(c.B):
            for h in range(c.H):
                for i in range(c.nb):
                    u = self.unit(b, h, i)
                    for k in out:
                        out[k][b, h, i * c.block:(i + 1) * c.block] = u[k]
        return out

    def route(self):
        """Mode A: classes [B, H, nqb, nkb] and tie flags [B, H, nqb].
        Mode B: selected lists [B][H_kv][nqb] and tie flags [B, H_kv, nqb]."""
        c = self.c
        if c.mode == 0:
            cls = np.stack([np.stack([self.classes(b, h) for h in range(c.H)]) for b in range(c.B)])
            tie = np.stack([np.stack([self.tie_rows(b, h) for h in range(c.H)]) for b in range(c.B)])
            return cls, tie
        sels = [[self.selection(b, hk)[0] for hk in range(c.H_kv)] for b in range(c.B)]
        tie = np.stack([np.stack([self.selection(b, hk)[1] for hk in range(c.H_kv)])
                        for b in range(c.B)])
        return sels, tie


def forward(cfg, q, k, v, w_p=None, w_g=None) -> Dict[str, np.ndarray]:
    """Whole-layer outputs O, O_s, O_l as float64 [B, H, N, d]."""
    return Layer(cfg, q, k, v, w_p, w_g).forward()


# ---------------------------------------------------------------------------
# token reordering along a Hilbert curve (SpargeAttn token-reorder note)
# ---------------------------------------------------------------------------

def hilbert_key3(x: int, y: int, z: int, bits: int) -> int:
    """Index of grid point (x, y, z) along the 3-D Hilbert curve of side 2**bits.

    Skilling's method: undo the excess work level by level (invert or exchange
    low bits against the first axis), Gray-encode across the axes, then read
    the transposed index out bit by bit, first axis most significant.
    """
    X = [int(x), int(y), int(z)]
    top = 1 << (bits - 1)
    q = top
    while q > 1:
        low = q - 1
        for i in range(3):
            if X[i] & q:
                X[0] ^= low
            else:
                swap = (X[0] ^ X[i]) & low
                X[0] ^= swap
                X[i] ^= swap
        q >>= 1
    for i in range(1, 3):
        X[i] ^= X[i - 1]
    flip = 0
    q = top
    while q > 1:
        if X[2] & q:
            flip ^= q - 1
        q >>= 1
    for i in range(3):
        X[i] ^= flip
    key = 0
    for b in range(bits - 1, -1, -1):
        for i in range(3):
            key = (key << 1) | ((X[i] >> b) & 1)
    return key


def hilbert_order(t: int, h: int, w: int) -> np.ndarray:
    """order[n'] = raster index (t-major, then h, then w) of the n'-th token along the curve."""
    bits = max(1, int(max(t, h, w) - 1).bit_length())
    keys = np.array([hilbert_key3(a, b, c, bits) for a in range(t) for b in range(h) for c in range(w)],
                    dtype=np.int64)
    return np.argsort(keys, kind="stable").astype(np.int32)


def permute_tokens(x: np.ndarray, order: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Gather y[..., n', :] = x[..., order[n'], :] (inverse: the scatter back); tokens past
    len(order) stay where they are."""
    y = x.copy()
    n = len(order)
    if inverse:
        y[..., order, :] = x[..., :n, :]
    else:
        y[..., :n, :] = x[..., order, :]
    return y


def block_cos_sim(x: np.ndarray, block: int) -> float:
    """Mean over blocks of the mean pairwise cosine similarity of a block's tokens
    (the SpargeAttn CosSim of a block), full blocks only."""
    n = x.shape[0] // block * block
    xn = x[:n] / np.linalg.norm(x[:n], axis=1, keepdims=True)
    s = xn.reshape(-1, block, x.shape[1]).sum(axis=1)
    return float(np.mean((s * s).sum(axis=1) / block ** 2))
