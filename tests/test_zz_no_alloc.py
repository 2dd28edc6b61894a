"""sla_route_noalloc against sla_route.

sla_route_noalloc serves callers that cannot allocate device memory for a
workspace (plugin hosts that pass only inputs and outputs, code under another
framework's memory pool, loops where cudaMalloc would synchronise the device).
Its scratch is a static device array inside the library; these tests check that
its routing equals the workspace-based entry point's on two calls in a row (the
array keeps the previous call's contents), and that a configuration too large
for the array is refused. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_linear_sm_b200 as sla  # noqa: E402
from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _noalloc():
    fn = sla.lib().sla_route_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, P, ctypes.POINTER(sla.sla_config), P, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _noalloc_status():
    fn = sla.lib().sla_route_noalloc_status
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)]
    fn.restype = ctypes.c_int
    return fn


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def _outputs(cfg):
    rows = cfg.H if cfg.mode == wl.MODE_THREEWAY else cfg.H_kv
    n_crit = cfg.k_h if cfg.mode == wl.MODE_THREEWAY else cfg.top_n
    mask = torch.full((cfg.B, rows, cfg.nqb, cfg.nkb), -7, dtype=torch.int8, device="cuda")
    crit = torch.full((cfg.B, rows, cfg.nqb, max(n_crit, 1)), -9, dtype=torch.int32, device="cuda")
    neg = torch.full((cfg.B, rows, cfg.nqb, max(cfg.k_l, 1)), -9, dtype=torch.int32, device="cuda")
    return mask, crit, neg


CASES = [wl.preset("tiny"), wl.preset("wan1.3b"),
         # the key-block filter's flags also live in the static array (after the scores)
         wl.preset("wan1.3b_cosfilter"),
         wl.small_config(name="cosfilter_small", H=4, H_kv=2, N=1024, N_valid=1000, d=64, k_h=3, k_l=4,
                         cos_filter=1, cos_theta=1.0 / 64),  # i.i.d. blocks: about half filtered
         wl.small_config(name="topn", mode=wl.MODE_TOPN_WINDOW, H=8, H_kv=2, N=2048, N_valid=2000,
                         d=128, top_n=4, window=200, causal=1, has_proj=0, generator="block_shift")]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_route_matches_workspace_route(cfg):
    x = wl.generate(cfg)
    q, k = _dev(x.q), _dev(x.k)
    c = sla.make_config(cfg)
    threeway = cfg.mode == wl.MODE_THREEWAY
    ref = _outputs(cfg)
    ws = torch.empty(sla.sla_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    sla.sla_route(q, k, cfg, ref[0], ref[1] if (cfg.k_h if threeway else cfg.top_n) else None,
                  ref[2] if threeway and cfg.k_l else None, ws)
    torch.cuda.synchronize()
    fn = _noalloc()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        got = _outputs(cfg)
        st = fn(q.data_ptr(), k.data_ptr(), ctypes.byref(c), got[0].data_ptr(),
                got[1].data_ptr() if (cfg.k_h if threeway else cfg.top_n) else None,
                got[2].data_ptr() if threeway and cfg.k_l else None, stream)
        assert st == sla.SLA_OK, sla.status_string(st)
        detail = ctypes.c_int32(-1)
        dst = _noalloc_status()(stream, ctypes.byref(detail))
        assert dst == sla.SLA_OK and detail.value == 0, (sla.status_string(dst), detail.value)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b), f"call {call}: routing differs from sla_route"


def test_noalloc_route_refuses_configs_beyond_its_scratch():
    cfg = wl.preset("nsa_causal")  # 537 MB of pooled scores, more than the static array
    c = sla.make_config(cfg)
    st = _noalloc()(16, 16, ctypes.byref(c), None, 16, None, None)
    assert st == sla.SLA_ERR_WORKSPACE
