"""Multi-rank host logic of bench.py on the CPU: two gloo ranks.

The layer runs as independent replicas (one per GPU, no collective on the data
path); what is shared between ranks is the timing: every rank's step time is
reduced with a max, and the whole-job throughput counts every rank's work over
the slowest rank's time. The reference arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports step times (r + 1, 5 - r) ms: the job sees the slowest rank's
        got = bench.max_over_ranks(dist, torch.device("cpu"), rank + 1.0, 5.0 - rank)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == [2.0, 5.0] and res[1] == [2.0, 5.0]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench

    # 2 ranks x 1e12 FLOP each in 1000 ms (the slowest rank) = 2 TFLOP/s
    assert bench.job_throughput(2, 1e12, 1000.0) == pytest.approx(2.0)
    assert bench.job_throughput(1, 6.594e12, 0.87) == pytest.approx(6.594e12 / 0.87e-3 / 1e12)
    assert bench.max_over_ranks(None, None, 1.5, 2) == [1.5, 2.0]


@pytest.mark.timeout(120)
def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=110)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


# ---------------------------------------------------------------------------
# head-sharded layer: planning and the all-gather back into head order
# ---------------------------------------------------------------------------

def test_balance_is_deterministic_and_covers_every_unit():
    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh

    costs = [5.0, 1.0, 4.0, 4.0, 3.0, 2.0, 2.0, 1.0, 6.0, 3.0, 1.0, 1.0]
    for world in (1, 2, 3, 5, 8, 12, 16):
        plan = sh.balance(costs, world)
        assert plan == sh.balance(costs, world)
        assert sorted(u for p in plan for u in p) == list(range(len(costs)))
        loads = sh.plan_loads(costs, plan)
        # LPT bound: the largest load is at most the mean plus the largest single cost
        assert max(loads) <= sum(costs) / world + max(costs) + 1e-9
    # uneven costs: LPT beats assigning units round-robin
    assert max(sh.plan_loads(costs, sh.balance(costs, 4))) == 9.0
    rr = [[u for u in range(12) if u % 4 == r] for r in range(4)]
    assert max(sh.plan_loads(costs, rr)) > 9.0


def test_unit_costs_count_the_merged_tiles():
    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    c = wl.small_config(N=256, N_valid=256, H=2, H_kv=1, k_h=2, k_l=2, has_proj=1)  # 4 blocks, no marginal
    crit = np.zeros((1, 2, 4, 2), np.int32)
    crit[0, 0] = [[0, 1], [0, 1], [2, 3], [0, 3]]  # pairs: {0,1} -> 2 tiles, {0,2,3} -> 3
    crit[0, 1] = [[0, 1], [2, 3], [0, 1], [0, 1]]  # {0,1,2,3} -> 4, {0,1} -> 2
    assert sh.unit_costs(c, crit).tolist() == [2 + 3 + 4 + 2]
    assert sh.unit_costs(c).tolist() == [1.0]


def _shard_rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = wl.small_config(N=128, N_valid=128, H=6, H_kv=3, d=8)
        shard = sh.HeadShard(cfg, world, rank, costs=np.array([3.0, 1.0, 2.0]))
        x = torch.arange(cfg.B * cfg.H * cfg.N * cfg.d, dtype=torch.float32).reshape(cfg.B, cfg.H, cfg.N, cfg.d)
        kv = torch.arange(cfg.B * cfg.H_kv * cfg.N * cfg.d, dtype=torch.float32).reshape(
            cfg.B, cfg.H_kv, cfg.N, cfg.d)
        lq, lk, lv, _, _ = shard.inputs(x, kv, kv)
        # stand-in for the layer's output: a function of each local row that remembers its head
        local_out = lq * 2 + 1
        full = sh.all_gather_heads(local_out, cfg, shard.plan, rank, dist)
        ok = bool(torch.equal(full, x * 2 + 1)) and lk.shape[1] == len(shard.units)
        dist.barrier()
        q.put((rank, (shard.plan, ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_head_sharded_gather_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # costs [3, 1, 2]: rank 0 takes unit 0, rank 1 units 1 and 2; both ranks agree
    assert res[0][0] == res[1][0] == [[0], [1, 2]]
    assert res[0][1] and res[1][1]


def _fake_routing(cfg):
    """Deterministic critical lists [B, H, nqb, k_h] for a small layer (a stand-in for the
    routing the GPU computes; only the cost estimate reads them)."""
    rng = np.random.default_rng(5)
    crit = np.zeros((cfg.B, cfg.H, cfg.nqb, cfg.k_h), np.int32)
    for b in range(cfg.B):
        for h in range(cfg.H):
            for i in range(cfg.nqb):
                crit[b, h, i] = np.sort(rng.choice(cfg.nkb, cfg.k_h, replace=False))
    return crit


def _costs_rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = wl.small_config(N=1024, N_valid=1000, H=10, H_kv=5, k_h=3, k_l=2)
        full = _fake_routing(cfg)
        group = cfg.H // cfg.H_kv
        routed = []

        def route_local(units):
            routed.extend(units)
            heads = [u * group + g for u in units for g in range(group)]
            return full[:, heads]
        costs = sh.distributed_costs(cfg, world, rank, route_local, dist)
        q.put((rank, (costs.tolist(), sorted(routed))))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_distributed_costs_route_a_share_and_agree_two_gloo_ranks():
    """Each rank routes only every second KV group; after the all_gather both ranks hold
    the cost vector of the whole layer, equal to the single-process estimate."""
    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_costs_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = wl.small_config(N=1024, N_valid=1000, H=10, H_kv=5, k_h=3, k_l=2)
    want = sh.unit_costs(cfg, _fake_routing(cfg)).tolist()
    assert res[0][0] == res[1][0] == want
    assert res[0][1] == [0, 2, 4] and res[1][1] == [1, 3]


def test_block_plan_covers_every_pair_once_and_balances():
    """db-SP's block level: the (KV group, pair) units cut into contiguous runs. Every unit
    lands on exactly one rank, a rank's pieces are contiguous in group-major order, at most
    two of them are partial groups, and each rank's load stays within one group's fixed
    work plus one pair of the equal share; the plan is the same on every call."""
    from block_sparse_linear_sm_b200 import sharding as sh
    rng = np.random.default_rng(5)
    for world in (1, 2, 3, 7, 12, 20):
        costs = rng.uniform(0.5, 4.0, (6, 40))
        costs[2] *= 4  # one heavy group
        fixed = np.full(6, 30.0)
        plan = sh.block_plan(costs, fixed, world)
        assert plan == sh.block_plan(costs, fixed, world)
        cover = np.zeros(costs.shape, dtype=int)
        flat = []
        for pieces in plan:
            partial = sum(1 for u, p0, p1 in pieces if p0 > 0 or p1 < costs.shape[1])
            assert partial <= 2
            for u, p0, p1 in pieces:
                assert 0 <= p0 < p1 <= costs.shape[1]
                cover[u, p0:p1] += 1
                flat.append((u, p0, p1))
        assert np.all(cover == 1)
        # contiguous in group-major order across ranks
        order = [(u, p) for u, p0, p1 in flat for p in range(p0, p1)]
        assert order == [(u, p) for u in range(costs.shape[0]) for p in range(costs.shape[1])]
        loads = sh.block_plan_loads(costs, fixed, plan)
        share = (costs.sum() + fixed.sum() + (world - 1) * fixed.mean()) / world
        assert max(loads[:-1] or [0]) <= share + fixed.max() + costs.max() + 1e-9
        if world > 1:
            head = sh.plan_loads(costs.sum(1) + fixed, sh.balance(costs.sum(1) + fixed, world))
            assert max(loads) <= max(head) + fixed.max() + costs.max() + 1e-9


def test_pair_costs_sum_to_the_unit_costs():
    """The per-pair work of the block level adds up to the per-group work of the head
    level (the same merged-list tiles, the linear branch spread over the query blocks)."""
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl
    from oracle import sla_oracle as oracle
    for kw in (dict(N=1216, N_valid=1200, d=64, H=4, H_kv=2, k_h=3, k_l=4, has_gate=1),
               dict(N=1024, N_valid=1024, d=64, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW, causal=1, top_n=3,
                    window=128, k_h=0, k_l=0, has_proj=0)):
        c = wl.small_config(**kw)
        x = wl.generate(c)
        L = oracle.Layer(c, x.f64("q"), x.f64("k"), x.f64("v"), x.f64("w_p"), None)
        if c.mode == wl.MODE_THREEWAY:
            crit = np.stack([[[np.nonzero(row == 2)[0] for row in L.classes(0, h)] for h in range(c.H)]])
        else:
            crit = np.full((1, c.H_kv, c.nqb, c.top_n), -1)
            for hk in range(c.H_kv):
                for i, s in enumerate(L.selection(0, hk)[0]):
                    crit[0, hk, i, :len(s)] = s
        pc = sh.pair_costs(c, crit)
        assert pc.shape == (c.H_kv, (c.nqb + 1) // 2)
        np.testing.assert_allclose(pc.sum(axis=1), sh.unit_costs(c, crit), rtol=1e-12)


def test_block_shard_calls_merge_whole_groups_and_cover_every_row():
    """BlockShard's calls: consecutive whole groups run as one sla_forward_blocks call over
    a range of heads, a partial group as a call over its query blocks; run on two ranks
    with a stand-in for the library (it copies its q rows of the given query blocks into
    out) writes every output row exactly once, from the right heads, through views when
    B = 1."""
    import torch

    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    cfg = wl.small_config(N=1024, N_valid=1000, H=10, H_kv=5, k_h=3, k_l=2)
    npairs = (cfg.nqb + 1) // 2
    costs, fixed = np.ones((cfg.H_kv, npairs)), np.zeros(cfg.H_kv)
    shards = [sh.BlockShard(cfg, 2, r, costs, fixed) for r in range(2)]
    assert shards[0].calls() == [(0, 2, 0, cfg.nqb), (2, 3, 0, 8)]
    assert shards[1].calls() == [(2, 3, 8, cfg.nqb), (3, 5, 0, cfg.nqb)]

    q = torch.arange(cfg.B * cfg.H * cfg.N * 2, dtype=torch.float32).view(cfg.B, cfg.H, cfg.N, 2)
    kv = torch.zeros(cfg.B, cfg.H_kv, cfg.N, 2)
    out = torch.full_like(q, -1.0)
    writes = torch.zeros(cfg.B, cfg.H, cfg.N, dtype=torch.int32)
    seen = []

    class FakeLib:
        @staticmethod
        def sla_forward_blocks(lq, lk, lv, lwp, lwg, lc, qb0, qb1, lout, mask, ws, stream):
            assert lq.shape[1] == lc.H and lk.shape[1] == lc.H_kv and lout.shape == lq.shape
            seen.append((lc.H, qb0, qb1, lq.untyped_storage().data_ptr() == q.untyped_storage().data_ptr()))
            lout[:, :, qb0 * 64:qb1 * 64] = lq[:, :, qb0 * 64:qb1 * 64]

    base = out.untyped_storage().data_ptr()
    for r, shard in enumerate(shards):
        before = out.clone()
        shard.run(FakeLib, q, kv, kv, None, None, out, lambda lc: None)
        writes += (out != before).any(-1).int()
    assert torch.equal(out, q)
    assert int(writes.max()) == 1 and int(writes.min()) >= 0
    assert out.untyped_storage().data_ptr() == base
    assert [s[:3] for s in seen] == [(4, 0, cfg.nqb), (2, 0, 8), (2, 8, cfg.nqb), (4, 0, cfg.nqb)]
    assert all(s[3] for s in seen)  # B = 1: the heads are views of q, not copies


def _block_rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = wl.small_config(N=1024, N_valid=1000, H=10, H_kv=5, k_h=3, k_l=2)
        full = _fake_routing(cfg)
        group = cfg.H // cfg.H_kv
        routed = []

        def route_local(units):
            routed.extend(units)
            heads = [u * group + g for u in units for g in range(group)]
            return full[:, heads]
        costs = sh.distributed_pair_costs(cfg, world, rank, route_local, dist)
        shard = sh.BlockShard(cfg, world, rank, costs)
        q.put((rank, (costs.tolist(), sorted(routed), shard.plan, shard.pieces)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_block_level_costs_and_plan_agree_two_gloo_ranks():
    """The block level across two gloo ranks: each routes every second KV group, the
    all_gather gives both the whole layer's per-pair costs (equal to the single-process
    estimate), both compute the same plan, and each takes its own pieces of it."""
    sys.path.insert(0, ROOT)
    from block_sparse_linear_sm_b200 import sharding as sh
    from block_sparse_linear_sm_b200 import workloads as wl

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_block_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = wl.small_config(N=1024, N_valid=1000, H=10, H_kv=5, k_h=3, k_l=2)
    want = sh.pair_costs(cfg, _fake_routing(cfg))
    for r in (0, 1):
        np.testing.assert_allclose(np.array(res[r][0]), want, rtol=1e-12)
    assert res[0][1] == [0, 2, 4] and res[1][1] == [1, 3]
    assert res[0][2] == res[1][2]
    assert res[0][3] == res[0][2][0] and res[1][3] == res[1][2][1]
