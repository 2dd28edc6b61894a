"""Head-sharded multi-GPU layer with load balancing on the routed work.

Sparse attention survey, db-SP note: when a dynamic block mask is spread over
several GPUs, splitting the tokens (or the heads) evenly does not split the
sparse work evenly, so the partition should balance the effective blocks each
device executes (db-SP partitions at the head level and the block level).

This module does the head level. The unit is a KV group: a KV head and the
query heads that read it, since they share K, V and (top-n mode) the selection.
Each unit's cost is estimated from the routing as the 64-key tiles the sparse
flash kernel executes for it (pairs of query blocks share one merged block
list) plus the linear branch's fixed per-head work; units go to ranks by
longest-processing-time-first (LPT). The costs need the routing of every group:
each rank routes only every world-th group (distributed_costs) and the ranks
share the costs with one small all_gather, so no rank routes the whole layer.
Each rank then gathers its heads into
contiguous local tensors, runs the whole layer on them through the C ABI, and
the outputs can be all-gathered back into head order. Nothing here computes
any part of the layer: the layer runs in the CUDA kernels of libsla.so.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np

from . import workloads as wl


def unit_costs(cfg: wl.LayerConfig, crit: Optional[np.ndarray] = None) -> np.ndarray:
    """Estimated work per KV group, in 64 x 64 flash tiles (float64 [H_kv]).

    ``crit``: the routing's block lists as host int32, three-way mode [B, H, nqb, k_h]
    (critical blocks), top-n mode [B, H_kv, nqb, top_n] (selected, -1 padded). Without
    routing every unit costs the same.
    """
    c = cfg
    group = c.H // c.H_kv
    if crit is None:
        return np.ones(c.H_kv)
    nqb = c.nqb
    cost = np.zeros(c.H_kv)
    if c.mode == wl.MODE_THREEWAY:
        for b in range(c.B):
            for h in range(c.H):
                tiles = 0
                for p in range(0, nqb, 2):
                    rows = crit[b, h, p:p + 2].reshape(-1)
                    tiles += np.unique(rows[rows >= 0]).size  # merged list of the pair
                # the linear branch's per-head work, as tiles of the same FLOP: state and
                # aggregation ~ 2 * nqb * nkb * d^2 against 4 * 64^2 * d per tile
                marg = nqb - c.k_h - c.k_l > 0 or c.linear_all
                lin = (2.0 * nqb * c.nkb * c.d * c.d) / (4.0 * 64 * 64 * c.d) if marg else 0.0
                cost[h // group] += tiles + lin
    else:
        wb = (c.window + 62) // 64 + 1 if c.window > 0 else 0  # blocks the window reaches
        for b in range(c.B):
            for hk in range(c.H_kv):
                tiles = 0
                for i in range(nqb):
                    sel = crit[b, hk, i]
                    tiles += np.unique(sel[sel >= 0]).size + min(wb, i + 1)
                cost[hk] += tiles * group  # every query head of the group runs the tiles
    return cost


def probe_units(cfg: wl.LayerConfig, world: int, rank: int) -> List[int]:
    """The KV groups whose routing this rank computes for the cost estimate: every
    world-th group from this rank's index, so the ranks split the routing work evenly."""
    return list(range(rank, cfg.H_kv, world))


def unit_costs_of(cfg: wl.LayerConfig, units: Sequence[int], crit_local: Optional[np.ndarray]) -> np.ndarray:
    """Costs of the given KV groups from the routing of the layer restricted to them
    (``crit_local``: the lists of local_config(cfg, units), or None)."""
    if not units:
        return np.zeros(0)
    return unit_costs(local_config(cfg, units), crit_local)


def distributed_costs(cfg: wl.LayerConfig, world: int, rank: int, route_local, dist) -> np.ndarray:
    """Every KV group's cost on every rank, with each rank routing only its probe groups.

    ``route_local(units)`` routes the layer restricted to ``units`` (local_config) and
    returns its host lists as unit_costs expects them (or None without lists). The costs
    are exchanged with one all_gather of a padded float64 vector, so every rank ends with
    the same vector and computes the same plan."""
    import torch

    mine = probe_units(cfg, world, rank)
    local = unit_costs_of(cfg, mine, route_local(mine) if mine else None)
    width = (cfg.H_kv + world - 1) // world
    buf = torch.zeros(width, dtype=torch.float64)
    buf[:len(local)] = torch.from_numpy(np.asarray(local, dtype=np.float64))
    backend = dist.get_backend() if hasattr(dist, "get_backend") else "gloo"
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    buf = buf.to(dev)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    costs = np.zeros(cfg.H_kv)
    for r, part in enumerate(parts):
        units = probe_units(cfg, world, r)
        costs[units] = part.cpu().numpy()[:len(units)]
    return costs


def balance(costs: Sequence[float], world: int) -> List[List[int]]:
    """LPT assignment: units by decreasing cost, each to the least-loaded rank (ties: the
    lower unit index first, then the lower rank). Deterministic, so every rank computes
    the same plan. Returns the ascending unit lists of the ranks."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda u: (-float(costs[u]), u))
    loads = [0.0] * world
    plan: List[List[int]] = [[] for _ in range(world)]
    for u in order:
        r = min(range(world), key=lambda x: (loads[x], x))
        plan[r].append(u)
        loads[r] += float(costs[u])
    return [sorted(p) for p in plan]


def plan_loads(costs: Sequence[float], plan: List[List[int]]) -> List[float]:
    return [float(sum(costs[u] for u in p)) for p in plan]


def query_heads(cfg: wl.LayerConfig, units: Sequence[int]) -> List[int]:
    """The query heads of the given KV groups, in order."""
    group = cfg.H // cfg.H_kv
    return [u * group + g for u in units for g in range(group)]


def local_config(cfg: wl.LayerConfig, units: Sequence[int]) -> wl.LayerConfig:
    """The layer restricted to the given KV groups (same sequence, routing and options)."""
    group = cfg.H // cfg.H_kv
    return cfg.replace(name=f"{cfg.name}_heads{len(units) * group}", H=len(units) * group, H_kv=len(units))


def gather_heads(x, heads: Sequence[int]):
    """Contiguous copy of heads ``heads`` (dimension 1) of a [B, H, ...] tensor."""
    import torch

    idx = torch.as_tensor(list(heads), dtype=torch.long, device=x.device)
    return torch.index_select(x, 1, idx).contiguous()


def all_gather_heads(local_out, cfg: wl.LayerConfig, plan: List[List[int]], rank: int, dist):
    """Every rank's local output [B, H_local, N, d] back into the full [B, H, N, d], in head
    order, on every rank (one all_gather of equally padded blocks)."""
    import torch

    group = cfg.H // cfg.H_kv
    max_heads = max(len(p) for p in plan) * group
    B, hl, N, d = local_out.shape
    pad = torch.zeros((B, max_heads, N, d), dtype=local_out.dtype, device=local_out.device)
    pad[:, :hl] = local_out
    parts = [torch.empty_like(pad) for _ in plan]
    dist.all_gather(parts, pad)
    full = torch.empty((B, cfg.H, N, d), dtype=local_out.dtype, device=local_out.device)
    for r, units in enumerate(plan):
        heads = query_heads(cfg, units)
        if heads:
            full[:, heads] = parts[r][:, :len(heads)]
    return full


class HeadShard:
    """This rank's share of a head-sharded layer: its KV groups, the local configuration,
    and the layer run on its gathered heads through the C ABI."""

    def __init__(self, cfg: wl.LayerConfig, world: int, rank: int, costs: Optional[np.ndarray] = None):
        self.cfg = cfg
        self.costs = unit_costs(cfg) if costs is None else np.asarray(costs, dtype=np.float64)
        self.plan = balance(self.costs, world)
        self.units = self.plan[rank]
        self.heads = query_heads(cfg, self.units)
        self.local = local_config(cfg, self.units) if self.units else None

    def inputs(self, q, k, v, w_p=None, w_g=None):
        """Local q, k, v (and per-head parameters) for this rank's heads."""
        import torch

        c = self.cfg
        lq, lk, lv = gather_heads(q, self.heads), gather_heads(k, self.units), gather_heads(v, self.units)
        lwp = w_p
        if w_p is not None and c.proj_per_head:
            lwp = torch.index_select(w_p, 0, torch.as_tensor(self.heads, device=w_p.device)).contiguous()
        lwg = None
        if w_g is not None:
            lwg = torch.index_select(w_g, 0, torch.as_tensor(self.heads, device=w_g.device)).contiguous()
        return lq, lk, lv, lwp, lwg


# ---------------------------------------------------------------------------
# block level (db-SP's second level): KV groups split into ranges of query blocks
# ---------------------------------------------------------------------------

def pair_costs(cfg: wl.LayerConfig, crit: Optional[np.ndarray] = None) -> np.ndarray:
    """Estimated work per (KV group, pair of query blocks), in 64 x 64 flash tiles (float64
    [H_kv, npairs]): the pair's merged block list for every head of the group (top-n mode:
    its selected blocks and the window's blocks) plus, with a linear branch, the
    aggregation rows of the pair. ``crit`` as for unit_costs; without it every pair costs
    the same."""
    c = cfg
    group = c.H // c.H_kv
    npairs = (c.nqb + 1) // 2
    if crit is None:
        return np.ones((c.H_kv, npairs))
    cost = np.zeros((c.H_kv, npairs))
    if c.mode == wl.MODE_THREEWAY:
        marg = c.nqb - c.k_h - c.k_l > 0 or c.linear_all
        # aggregation of one query block row: 2 * nkb * (d^2 + d) against 4 * 64^2 * d per tile
        agg = (2.0 * c.nkb * c.d * c.d) / (4.0 * 64 * 64 * c.d) if marg else 0.0
        for b in range(c.B):
            for h in range(c.H):
                for p in range(npairs):
                    rows = crit[b, h, 2 * p:2 * p + 2].reshape(-1)
                    n_rows = min(2, c.nqb - 2 * p)
                    cost[h // group, p] += np.unique(rows[rows >= 0]).size + agg * n_rows
    else:
        wb = (c.window + 62) // 64 + 1 if c.window > 0 else 0
        for b in range(c.B):
            for hk in range(c.H_kv):
                for i in range(c.nqb):
                    sel = crit[b, hk, i]
                    cost[hk, i // 2] += (np.unique(sel[sel >= 0]).size + min(wb, i + 1)) * group
    return cost


def distributed_pair_costs(cfg: wl.LayerConfig, world: int, rank: int, route_local, dist) -> np.ndarray:
    """pair_costs of the whole layer on every rank, each rank routing only its probe
    groups (as distributed_costs does for the head level): one all_gather of a padded
    float64 [ceil(H_kv / world), npairs] block per rank."""
    import torch

    npairs = (cfg.nqb + 1) // 2
    mine = probe_units(cfg, world, rank)
    local = pair_costs(local_config(cfg, mine), route_local(mine)) if mine else np.zeros((0, npairs))
    width = (cfg.H_kv + world - 1) // world
    buf = torch.zeros((width, npairs), dtype=torch.float64)
    if len(mine):
        buf[:len(mine)] = torch.from_numpy(np.asarray(local, dtype=np.float64))
    backend = dist.get_backend() if hasattr(dist, "get_backend") else "gloo"
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    buf = buf.to(dev)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    costs = np.zeros((cfg.H_kv, npairs))
    for r, part in enumerate(parts):
        units = probe_units(cfg, world, r)
        costs[units] = part.cpu().numpy()[:len(units)]
    return costs


def fixed_costs(cfg: wl.LayerConfig, costs: np.ndarray, share: float = 0.5) -> np.ndarray:
    """Work of a KV group that every call holding any of its query blocks repeats (routing,
    key pooling, linear states), as ``share`` of the group's mean per-head flash work. With
    the Wan-1.3B layer the router and the state kernels take about half the flash kernel's
    time (0.15 + 0.11 against 0.46 ms)."""
    group = cfg.H // cfg.H_kv
    return np.full(cfg.H_kv, share * float(np.mean(costs.sum(axis=1))) / group * group)


def block_plan(costs: np.ndarray, fixed: np.ndarray, world: int) -> List[List[tuple]]:
    """Pieces (KV group, first pair, end pair) of every rank: the (group, pair) units in
    group-major order cut into world contiguous runs of about equal work, so a rank holds
    at most two partial groups. A run ends inside a group when the next pair would take
    the rank past its share; every rank that holds part of a group pays the group's fixed
    work, and the share counts the fixed work of the world - 1 cuts. Deterministic: every
    rank computes the same plan. Returns, per rank, a list of (unit, p0, p1), p0 < p1."""
    if world < 1:
        raise ValueError("world must be >= 1")
    n_units, npairs = costs.shape
    mean_fixed = float(np.mean(fixed)) if n_units else 0.0
    target = (float(costs.sum()) + float(fixed.sum()) + (world - 1) * mean_fixed) / world
    plan: List[List[tuple]] = [[] for _ in range(world)]
    r, load = 0, 0.0
    for u in range(n_units):
        p = 0
        while p < npairs:
            load += float(fixed[u])  # this rank starts on (part of) group u
            q = p
            while q < npairs and (r == world - 1 or q == p or load + float(costs[u, q]) <= target):
                load += float(costs[u, q])
                q += 1
            plan[r].append((u, p, q))
            if r < world - 1 and (q < npairs or load >= target):  # this rank's share is used up
                r, load = r + 1, 0.0
            p = q
    return plan


def block_plan_loads(costs: np.ndarray, fixed: np.ndarray, plan: List[List[tuple]]) -> List[float]:
    """Work of each rank under a block plan: its pairs plus the fixed work of each group it
    touches."""
    out = []
    for pieces in plan:
        units = {u for u, _, _ in pieces}
        out.append(float(sum(costs[u, p0:p1].sum() for u, p0, p1 in pieces) + sum(fixed[u] for u in units)))
    return out


class BlockShard:
    """This rank's share of a block-split layer: for every piece (KV group, pairs p0..p1)
    it runs the layer on the group's heads through sla_forward_blocks, which writes the
    output rows of query blocks 2 p0 .. 2 p1 - 1."""

    def __init__(self, cfg: wl.LayerConfig, world: int, rank: int, costs: Optional[np.ndarray] = None,
                 fixed: Optional[np.ndarray] = None):
        self.cfg = cfg
        self.costs = pair_costs(cfg) if costs is None else np.asarray(costs, dtype=np.float64)
        self.fixed = fixed_costs(cfg, self.costs) if fixed is None else np.asarray(fixed, dtype=np.float64)
        self.plan = block_plan(self.costs, self.fixed, world)
        self.pieces = self.plan[rank]

    def calls(self) -> List[tuple]:
        """The sla_forward_blocks calls that run this rank's pieces: (first group, end group,
        first query block, end query block). Consecutive pieces that each cover a whole group
        merge into one call over the range of groups; a partial piece is a call of its own."""
        c = self.cfg
        npairs = (c.nqb + 1) // 2
        out: List[tuple] = []
        for u, p0, p1 in self.pieces:
            qb0, qb1 = 2 * p0, min(2 * p1, c.nqb)
            whole = p0 == 0 and p1 == npairs
            if whole and out and out[-1][1] == u and out[-1][2] == 0 and out[-1][3] == c.nqb:
                out[-1] = (out[-1][0], u + 1, 0, c.nqb)
            else:
                out.append((u, u + 1, qb0, qb1))
        return out

    def run(self, sla, q, k, v, w_p, w_g, out, ws_for, stream=None):
        """Runs this rank's pieces; ``out`` [B, H, N, d] receives their rows (the others
        are not written). ``ws_for(local_cfg)`` returns a workspace for that config. The
        heads of a range of groups are a slice of dimension 1, a view without a copy when
        B = 1; otherwise they are copied to a contiguous buffer (and the rows back)."""
        c = self.cfg
        group = c.H // c.H_kv
        for u0, u1, qb0, qb1 in self.calls():
            h0, h1 = u0 * group, u1 * group
            lc = local_config(c, list(range(u0, u1)))
            lq, lk, lv = (x[:, a:b].contiguous() for x, a, b in ((q, h0, h1), (k, u0, u1), (v, u0, u1)))
            lwp = w_p
            if w_p is not None and c.proj_per_head:
                lwp = w_p[h0:h1].contiguous()
            lwg = None if w_g is None else w_g[h0:h1].contiguous()
            lout = out[:, h0:h1]
            local = lout if lout.is_contiguous() else lout.contiguous()
            sla.sla_forward_blocks(lq, lk, lv, lwp, lwg, lc, qb0, qb1, local, None, ws_for(lc), stream)
            if local is not lout:
                lout[:, :, qb0 * 64:qb1 * 64] = local[:, :, qb0 * 64:qb1 * 64]
