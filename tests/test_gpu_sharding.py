"""Head-sharded layer on one GPU: every rank's share run in turn and put back in head
order equals the whole layer bit for bit (each stage works per head, or per KV group,
so a layer restricted to some heads computes exactly their rows), and matches the
float64 oracle on sampled units of every head. The ranks run one after another on
one device; none waits for another."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_linear_sm_b200 as sla  # noqa: E402
from block_sparse_linear_sm_b200 import sharding as sh  # noqa: E402
from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU runs deselect these anyway
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_util import MAX_ABS, MEAN_ABS, DeviceRun, unit_errors  # noqa: E402


CASES = [
    dict(name="threeway_gate", N=2048, N_valid=2001, d=128, H=6, H_kv=6, k_h=4, k_l=6, has_gate=1),
    dict(name="threeway_gqa", N=1536, N_valid=1536, d=64, H=8, H_kv=4, k_h=3, k_l=2, has_gate=1),
    dict(name="per_head_proj", N=1024, N_valid=1000, d=128, H=5, H_kv=5, k_h=2, k_l=3, proj_per_head=1),
    dict(name="topn_gqa", N=2048, N_valid=2048, d=128, H=8, H_kv=4, mode=wl.MODE_TOPN_WINDOW, causal=1,
         top_n=4, window=256, k_h=0, k_l=0, has_proj=0),
]


@pytest.mark.parametrize("kw", CASES, ids=[c["name"] for c in CASES])
@pytest.mark.parametrize("world", [2, 3])
def test_head_shards_reassemble_the_whole_layer(kw, world):
    cfg = wl.small_config(**kw)
    run = DeviceRun(cfg, route=True)
    crit = run.crit.cpu().numpy() if (cfg.k_h if cfg.mode == wl.MODE_THREEWAY else cfg.top_n) else None
    costs = sh.unit_costs(cfg, crit)
    full = torch.empty_like(run.out)
    for r in range(world):
        shard = sh.HeadShard(cfg, world, r, costs)
        if not shard.units:
            continue
        q, k, v, w_p, w_g = shard.inputs(run.q, run.k, run.v, run.w_p, run.w_g)
        lc = shard.local
        out = torch.empty(lc.B, lc.H, lc.N, lc.d, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(sla.sla_workspace_bytes(lc), dtype=torch.uint8, device="cuda")
        sla.sla_forward(q, k, v, w_p, w_g, lc, out, None, ws)
        assert sla.sla_check_device_status(ws) == (0, 0)
        full[:, shard.heads] = out
    assert torch.equal(full, run.out)
    # the reassembled shards against the float64 oracle on sampled units of every head
    L = run.layer()
    run.out = full
    rng = np.random.default_rng(world)
    units = [(0, h, int(i)) for h in range(cfg.H) for i in rng.choice(cfg.nqb, 2, replace=False)]
    err = unit_errors(run, L, units)
    assert err["max_abs"] <= MAX_ABS and err["mean_abs"] <= MEAN_ABS, err


BLOCK_CASES = CASES + [
    dict(name="threeway_odd_blocks", N=1216, N_valid=1200, d=128, H=3, H_kv=3, k_h=3, k_l=4, has_gate=1),
    dict(name="nsa_branches", N=2048, N_valid=2000, d=64, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW, causal=1,
         top_n=3, window=128, k_h=0, k_l=0, has_proj=0, nsa_branches=1, cmp_block=32, cmp_stride=16, has_gate=1),
]


@pytest.mark.parametrize("kw", BLOCK_CASES, ids=[c["name"] for c in BLOCK_CASES])
@pytest.mark.parametrize("world", [3, 5])
def test_block_split_reassembles_the_whole_layer(kw, world):
    """db-SP's block level: each rank runs its pieces (KV group, range of query-block
    pairs) through sla_forward_blocks into one output buffer; together they write every
    row exactly as the whole-layer sla_forward does, bit for bit."""
    cfg = wl.small_config(**kw)
    run = DeviceRun(cfg, route=True)
    crit = run.crit.cpu().numpy() if (cfg.k_h if cfg.mode == wl.MODE_THREEWAY else cfg.top_n) else None
    costs = sh.pair_costs(cfg, crit)
    full = torch.full_like(run.out, float("nan"))
    wss = {}

    def ws_for(lc):
        if lc.name not in wss:
            wss[lc.name] = torch.empty(sla.sla_workspace_bytes(lc), dtype=torch.uint8, device="cuda")
        return wss[lc.name]

    split_groups = 0
    for r in range(world):
        shard = sh.BlockShard(cfg, world, r, costs)
        split_groups += sum(1 for u, p0, p1 in shard.pieces if p0 > 0 or p1 < costs.shape[1])
        shard.run(sla, run.q, run.k, run.v, run.w_p, run.w_g, full, ws_for)
        for ws in wss.values():
            assert sla.sla_check_device_status(ws) == (0, 0)
    assert split_groups > 0, "the plan split no group: the test would not exercise the block level"
    assert torch.equal(full, run.out)


def test_block_range_rejects_bad_ranges():
    cfg = wl.small_config(N=1024, N_valid=1000, d=64, H=2, H_kv=2, k_h=2, k_l=2)
    run = DeviceRun(cfg, route=False)
    for qb0, qb1 in ((1, 4), (0, 0), (4, 2), (0, 17), (2, 5), (-2, 4)):
        with pytest.raises(RuntimeError):
            sla.sla_forward_blocks(run.q, run.k, run.v, run.w_p, run.w_g, cfg, qb0, qb1, run.out, None, run.ws)
