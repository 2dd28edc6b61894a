"""The layer on host buffers (sla_forward_host) against the device call.

Each head of the layer is computed independently of the others, so the
pipelined host call, which runs the layer as units of whole KV groups, must
give the same bits as one sla_forward call on device copies of the same
inputs. Checked for one unit per batch entry and for one unit per KV group,
for three-way layers (GQA, batch 2, per-head projection) and NSA's branches,
twice back to back on one arena, and at the Wan2.1-1.3B shape the bench uses.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_linear_sm_b200 as sla  # noqa: E402
from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU runs deselect these anyway
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_util import DeviceRun  # noqa: E402


def host(bits: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).pin_memory()


def host_call(run: DeviceRun, n_chunks: int, repeats: int = 1):
    c = run.cfg
    hq, hk, hv = host(run.x.q), host(run.x.k), host(run.x.v)
    hout = torch.full(tuple(run.out.shape), float("nan"), dtype=torch.bfloat16).pin_memory()
    nbytes = sla.sla_forward_host_device_bytes(c, n_chunks)
    assert nbytes > 0
    dev = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s, s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(repeats):
        sla.sla_forward_host(hq, hk, hv, run.w_p, run.w_g, c, hout, n_chunks, dev, stream=s,
                             h2d_stream=s_in, d2h_stream=s_out)
    st, detail = sla.sla_check_device_status(dev, stream=s)  # synchronises s: out is on the host
    assert st == 0, (st, detail)
    return hout


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


CASES = [
    dict(name="gqa_batch2_d128", B=2, N=1024, N_valid=1000, d=128, H=4, H_kv=2, k_h=3, k_l=4, has_gate=1),
    dict(name="per_head_proj_d64", N=1024, N_valid=1024, d=64, H=3, H_kv=3, k_h=2, k_l=3, proj_per_head=1,
         has_gate=1),
    dict(name="nsa_branches_d128", N=1024, N_valid=1024, d=128, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW, causal=1,
         top_n=2, window=128, k_h=0, k_l=0, has_proj=0, has_gate=1, nsa_branches=1),
]


@pytest.mark.parametrize("per_group", [False, True], ids=["one_unit", "unit_per_kv_group"])
@pytest.mark.parametrize("kw", CASES, ids=[c["name"] for c in CASES])
def test_host_call_equals_the_device_call(kw, per_group):
    cfg = wl.small_config(**kw)
    run = DeviceRun(cfg, route=False)
    n = cfg.H_kv if per_group else 1
    hout = host_call(run, n, repeats=2)
    assert same_bits(hout, run.out.cpu())


def test_bench_shape_host_call():
    cfg = wl.preset("wan1.3b")
    run = DeviceRun(cfg, route=False)
    hout = host_call(run, cfg.H_kv)
    assert same_bits(hout, run.out.cpu())
