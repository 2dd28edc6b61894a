"""Host-only checks of the C-ABI library: it loads without a GPU, exports every
function include/sla.h declares, and rejects bad arguments before launching
anything (no compute call is made here)."""
import ctypes
import os
import re

import numpy as np

import pytest

import block_sparse_linear_sm_b200 as sla
from block_sparse_linear_sm_b200 import workloads as wl


def declared_functions():
    src = open(sla.HEADER_PATH).read()
    return sorted(set(re.findall(r"^SLA_API\s+[\w\s\*]+?\b(sla_\w+)\s*\(", src, re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("sla_route", "sla_forward", "sla_workspace_bytes", "sla_status_string",
                 "sla_check_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol():
    L = sla.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_config_struct_layout_matches_header():
    src = open(sla.HEADER_PATH).read()
    body = src[src.index("typedef struct {"):src.index("} sla_config;")]
    fields = re.findall(r"^\s*(?:int32_t|float)\s+(\w+);", body, re.M)
    assert fields == [f for f, _ in sla.sla_config._fields_]
    assert ctypes.sizeof(sla.sla_config) == 4 * len(fields)


@pytest.mark.parametrize("name", wl.PRESETS)
def test_presets_are_valid(name):
    c = wl.preset(name)
    assert sla.sla_validate_config(c) == sla.SLA_OK
    assert sla.sla_workspace_bytes(c) > 0
    assert sla.sla_num_stages(c) == len(sla.sla_stage_names(c)) > 0


BAD = [
    (dict(block=32), sla.SLA_ERR_UNSUPPORTED),
    (dict(d=96), sla.SLA_ERR_UNSUPPORTED),
    (dict(N=1000, N_valid=1000), sla.SLA_ERR_INVALID_ARG),
    (dict(N_valid=1025), sla.SLA_ERR_INVALID_ARG),
    (dict(N_valid=960), sla.SLA_ERR_INVALID_ARG),
    (dict(H=3, H_kv=2), sla.SLA_ERR_INVALID_ARG),
    (dict(k_h=10, k_l=7), sla.SLA_ERR_INVALID_ARG),
    (dict(k_h=-1), sla.SLA_ERR_INVALID_ARG),
    (dict(causal=1), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=1, causal=0), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=1, causal=1, top_n=65, has_proj=0), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=1, causal=1, top_n=4, has_proj=1), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=7), sla.SLA_ERR_INVALID_ARG),
    (dict(proj_per_head=2), sla.SLA_ERR_INVALID_ARG),
    (dict(smooth_k=2), sla.SLA_ERR_INVALID_ARG),
    (dict(cos_filter=3), sla.SLA_ERR_INVALID_ARG),
    (dict(cos_filter=1, cos_theta=float("nan")), sla.SLA_ERR_INVALID_ARG),
    (dict(linear_all=-1), sla.SLA_ERR_INVALID_ARG),
    (dict(mode=1, causal=1, top_n=4, has_proj=0, smooth_k=1), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=1, causal=1, top_n=4, has_proj=0, linear_all=1), sla.SLA_ERR_UNSUPPORTED),
    (dict(proj_per_head=1, has_proj=0), sla.SLA_ERR_UNSUPPORTED),
    (dict(proj_per_head=1, H=4, H_kv=2), sla.SLA_ERR_UNSUPPORTED),
    (dict(mode=1, causal=1, top_n=4, has_proj=0, proj_per_head=1), sla.SLA_ERR_UNSUPPORTED),
    (dict(scale=-1.0), sla.SLA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), sla.SLA_ERR_INVALID_ARG),
    # empty problems are rejected, not treated as no-ops
    (dict(B=0), sla.SLA_ERR_INVALID_ARG),
    (dict(H=0, H_kv=0), sla.SLA_ERR_INVALID_ARG),
    (dict(N=0, N_valid=0), sla.SLA_ERR_INVALID_ARG),
    (dict(N_valid=0, N=64, k_h=1, k_l=0), sla.SLA_ERR_INVALID_ARG),
    # one key block past the routing sort's limit of 4096
    (dict(N=4097 * 64, N_valid=4097 * 64, k_h=4, k_l=4), sla.SLA_ERR_UNSUPPORTED),
]


def test_largest_block_count_is_accepted():
    """N = 4096 blocks of 64 (262144 tokens) is the largest supported length."""
    c = wl.small_config(N=4096 * 64, N_valid=4096 * 64 - 5, k_h=40, k_l=400)
    assert sla.sla_validate_config(c) == sla.SLA_OK
    assert sla.sla_workspace_bytes(c) > 0


@pytest.mark.parametrize("kw,code", BAD)
def test_invalid_configs_are_rejected(kw, code):
    base = dict(N=1024, N_valid=1024)
    base.update(kw)
    c = wl.small_config(**base)
    assert sla.sla_validate_config(c) == code
    assert sla.sla_workspace_bytes(c) == 0
    assert sla.sla_num_stages(c) == -1


def _call_forward(cfg, q=16, k=16, v=16, w_p=16, w_g=16, out=16, ws=256, ws_bytes=None):
    c = sla.make_config(cfg)
    if ws_bytes is None:
        ws_bytes = sla.sla_workspace_bytes(cfg)
    return sla.lib().sla_forward(q, k, v, w_p, w_g, ctypes.byref(c), out, None, ws, ws_bytes, None)


def test_forward_rejects_bad_pointers_before_launch():
    cfg = wl.small_config(N=1024, N_valid=1024, has_gate=1)
    # fake (never dereferenced) addresses: every case fails validation on the host
    assert _call_forward(cfg, q=None) == sla.SLA_ERR_INVALID_ARG
    assert _call_forward(cfg, out=None) == sla.SLA_ERR_INVALID_ARG
    assert _call_forward(cfg, q=24) == sla.SLA_ERR_INVALID_ARG          # misaligned
    assert _call_forward(cfg, w_p=None) == sla.SLA_ERR_INVALID_ARG      # has_proj
    assert _call_forward(cfg, w_g=None) == sla.SLA_ERR_INVALID_ARG      # has_gate
    assert _call_forward(cfg, ws=None) == sla.SLA_ERR_WORKSPACE
    assert _call_forward(cfg, ws=128) == sla.SLA_ERR_WORKSPACE          # misaligned
    assert _call_forward(cfg, ws_bytes=sla.sla_workspace_bytes(cfg) - 1) == sla.SLA_ERR_WORKSPACE
    bad = wl.small_config(N=1024, N_valid=1024, d=80)
    assert _call_forward(bad) == sla.SLA_ERR_UNSUPPORTED


def _call_forward_host(cfg, n_chunks=2, q=16, k=16, v=16, w_p=16, w_g=16, out=16, dev=256, dev_bytes=None):
    c = sla.make_config(cfg)
    if dev_bytes is None:
        dev_bytes = sla.sla_forward_host_device_bytes(cfg, n_chunks)
    return sla.lib().sla_forward_host(q, k, v, w_p, w_g, ctypes.byref(c), out, n_chunks, dev, dev_bytes,
                                      None, None, None)


def test_forward_host_rejects_bad_arguments_before_any_copy():
    cfg = wl.small_config(N=1024, N_valid=1024, H=4, H_kv=2, has_gate=1)
    # fake (never dereferenced) addresses: every case fails validation on the host
    assert _call_forward_host(cfg, n_chunks=0) == sla.SLA_ERR_INVALID_ARG
    assert _call_forward_host(cfg, n_chunks=3) == sla.SLA_ERR_INVALID_ARG   # does not divide H_kv
    assert _call_forward_host(cfg, q=None) == sla.SLA_ERR_INVALID_ARG
    assert _call_forward_host(cfg, out=None) == sla.SLA_ERR_INVALID_ARG
    assert _call_forward_host(cfg, v=40) == sla.SLA_ERR_INVALID_ARG        # misaligned
    assert _call_forward_host(cfg, w_p=None) == sla.SLA_ERR_INVALID_ARG    # has_proj
    assert _call_forward_host(cfg, w_g=None) == sla.SLA_ERR_INVALID_ARG    # has_gate
    assert _call_forward_host(cfg, dev=None) == sla.SLA_ERR_WORKSPACE
    assert _call_forward_host(cfg, dev=128) == sla.SLA_ERR_WORKSPACE       # misaligned
    need = sla.sla_forward_host_device_bytes(cfg, 2)
    assert _call_forward_host(cfg, dev_bytes=need - 1) == sla.SLA_ERR_WORKSPACE
    assert _call_forward_host(wl.small_config(N=1024, N_valid=1024, d=80)) == sla.SLA_ERR_UNSUPPORTED


def test_forward_host_arena_holds_io_and_one_workspace_per_unit():
    cfg = wl.small_config(B=2, N=1024, N_valid=1000, H=4, H_kv=2, has_gate=1)
    assert sla.sla_forward_host_device_bytes(cfg, 0) == 0
    assert sla.sla_forward_host_device_bytes(cfg, 3) == 0
    io = (2 * cfg.B * cfg.H + 2 * cfg.B * cfg.H_kv) * cfg.N * cfg.d * 2
    for n in (1, 2):
        unit = cfg.replace(B=1, H=cfg.H // n, H_kv=cfg.H_kv // n)
        ws = sla.sla_workspace_bytes(unit)
        total = sla.sla_forward_host_device_bytes(cfg, n)
        assert io + cfg.B * n * ws <= total <= io + cfg.B * n * ws + 256 * (6 + cfg.B * n)


def test_route_rejects_missing_lists():
    cfg = wl.small_config(N=1024, N_valid=1024, k_h=3, k_l=2)
    c = sla.make_config(cfg)
    nb = sla.sla_workspace_bytes(cfg)
    L = sla.lib()
    assert L.sla_route(16, 16, ctypes.byref(c), None, None, 16, 256, nb, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_route(16, 16, ctypes.byref(c), None, 16, None, 256, nb, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_route(16, 16, ctypes.byref(c), None, 16, 16, 256, 0, None) == sla.SLA_ERR_WORKSPACE


def test_timed_forward_checks_event_count():
    cfg = wl.small_config(N=1024, N_valid=1024)
    c = sla.make_config(cfg)
    L = sla.lib()
    evs = (ctypes.c_void_p * 2)(1, 2)
    r = L.sla_forward_timed(16, 16, 16, 16, None, ctypes.byref(c), 16, None, 256,
                            sla.sla_workspace_bytes(cfg), None, evs, 2)
    assert r == sla.SLA_ERR_INVALID_ARG
    assert L.sla_forward_timed(16, 16, 16, 16, None, ctypes.byref(c), 16, None, 256,
                               sla.sla_workspace_bytes(cfg), None, None, 0) == sla.SLA_ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert sla.status_string(s)
    assert "unknown" in sla.status_string(99)
    assert sla.sla_version().count(".") == 2


def test_workspace_grows_with_the_problem():
    a = wl.small_config(N=1024, N_valid=1024)
    b = wl.small_config(N=2048, N_valid=2048)
    assert sla.sla_workspace_bytes(b) > sla.sla_workspace_bytes(a)
    assert sla.sla_workspace_bytes(a) % 256 == 0


def test_per_head_projection_is_accepted_with_one_kv_head_per_query_head():
    c = wl.small_config(N=1024, N_valid=1000, H=4, H_kv=4, proj_per_head=1)
    assert sla.sla_validate_config(c) == sla.SLA_OK
    assert sla.sla_workspace_bytes(c) == sla.sla_workspace_bytes(wl.small_config(N=1024, N_valid=1000, H=4, H_kv=4))


def test_selftest_rejects_bad_arguments_before_launch():
    L = sla.lib()
    assert L.sla_selftest_wait_timeout(None, 4096, 1_000_000, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_selftest_wait_timeout(256 + 16, 4096, 1_000_000, None) == sla.SLA_ERR_INVALID_ARG  # misaligned
    assert L.sla_selftest_wait_timeout(256, 128, 1_000_000, None) == sla.SLA_ERR_INVALID_ARG       # too small
    assert L.sla_selftest_wait_timeout(256, 4096, 10, None) == sla.SLA_ERR_INVALID_ARG             # limit too short
    assert L.sla_selftest_wait_timeout(256, 4096, 5_000_000_000, None) == sla.SLA_ERR_INVALID_ARG  # too long


def test_linear_all_keeps_the_linear_stages_without_marginal_blocks():
    # k_h + k_l = nb leaves no marginal block; with linear_all the linear branch still runs
    c0 = wl.small_config(N=1024, N_valid=1024, k_h=8, k_l=8)
    c1 = wl.small_config(N=1024, N_valid=1024, k_h=8, k_l=8, linear_all=1)
    assert "linear_state" not in sla.sla_stage_names(c0)
    assert "linear_state" in sla.sla_stage_names(c1) and "linear_aggregate" in sla.sla_stage_names(c1)
    assert sla.sla_workspace_bytes(c1) > sla.sla_workspace_bytes(c0)


@pytest.mark.parametrize("grid", [(1, 1, 1), (2, 3, 4), (4, 4, 4), (5, 7, 3), (21, 30, 52)])
def test_hilbert_order_matches_the_oracle(grid):
    from oracle import sla_oracle as so
    got = sla.sla_hilbert_order(*grid)
    assert np.array_equal(got, so.hilbert_order(*grid))


def test_reorder_entry_points_reject_bad_arguments():
    L = sla.lib()
    out = (ctypes.c_int32 * 8)()
    assert L.sla_hilbert_order(0, 2, 2, out) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_hilbert_order(2, 2, 2, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_hilbert_order(2048, 2048, 2048, out) == sla.SLA_ERR_INVALID_ARG  # > 2^30 tokens
    # x == y, misaligned, d not a multiple of 8, n_order > n_tok
    assert L.sla_permute_tokens(256, 256, 256, 4, 1, 4, 8, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_permute_tokens(256, 512 + 4, 256, 4, 1, 4, 8, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_permute_tokens(256, 512, 256, 4, 1, 4, 12, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_permute_tokens(256, 512, 256, 5, 1, 4, 8, 0, None) == sla.SLA_ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# backward entry points (host checks only: every call below fails validation)
# ---------------------------------------------------------------------------

def _call_backward(cfg, ptr=16, ws=256, bws=256, ws_bytes=None, bws_bytes=None, **over):
    c = sla.make_config(cfg)
    if ws_bytes is None:
        ws_bytes = sla.sla_workspace_bytes(cfg)
    if bws_bytes is None:
        bws_bytes = sla.sla_backward_workspace_bytes(cfg)
    a = dict(q=ptr, k=ptr, v=ptr, w_p=ptr, w_g=ptr, out=ptr, dout=ptr, dq=ptr, dk=ptr, dv=ptr, dw_p=ptr,
             dw_g=ptr)
    a.update(over)
    return sla.lib().sla_backward(a["q"], a["k"], a["v"], a["w_p"], a["w_g"], ctypes.byref(c), a["out"],
                                  a["dout"], a["dq"], a["dk"], a["dv"], a["dw_p"], a["dw_g"], ws, ws_bytes,
                                  bws, bws_bytes, None)


def test_backward_scope():
    three = wl.small_config(N=1024, N_valid=1000, has_gate=1)
    assert sla.sla_backward_workspace_bytes(three) > 0
    assert sla.sla_backward_stage_names(three) == [
        "bwd_columns", "bwd_linear", "bwd_mask_transpose", "bwd_aggregate_t", "bwd_state", "bwd_flash_dq",
        "bwd_flash_dkdv"]
    # no marginal block: D_t straight from the output
    no_lin = wl.small_config(N=1024, N_valid=1024, k_h=8, k_l=8)
    assert sla.sla_backward_stage_names(no_lin) == ["bwd_columns", "bwd_delta", "bwd_flash_dq", "bwd_flash_dkdv"]
    assert sla.sla_backward_workspace_bytes(wl.small_config(N=1024, N_valid=1024, smooth_k=1)) > 0
    # top-n mode: the sparse branch only
    topn = wl.preset("nsa_causal")
    assert sla.sla_backward_workspace_bytes(topn) > 0
    assert sla.sla_backward_stage_names(topn) == ["bwd_columns", "bwd_delta", "bwd_flash_dq", "bwd_flash_dkdv"]
    # NSA's three branches: the compressed keys' gradients come before the token dK / dV
    nsa = wl.preset("nsa_branches")
    assert sla.sla_backward_workspace_bytes(nsa) > 0
    assert sla.sla_backward_stage_names(nsa) == [
        "bwd_columns", "bwd_nsa_prep", "bwd_flash_dq", "bwd_flash_dkdv_cmp", "bwd_cmp_reduce", "bwd_flash_dkdv"]
    # no compressed block (fewer valid tokens than one compressed block): no compressed stages
    short = wl.small_config(name="nsa_short", N=64, N_valid=20, d=64, H=2, H_kv=1, mode=wl.MODE_TOPN_WINDOW, causal=1,
                            top_n=2, window=16, k_h=0, k_l=0, has_proj=0, nsa_branches=1, cmp_block=32,
                            cmp_stride=16)
    assert sla.sla_backward_stage_names(short) == ["bwd_columns", "bwd_nsa_prep", "bwd_flash_dq", "bwd_flash_dkdv"]
    bad = wl.small_config(N=1024, N_valid=1024, d=80)
    assert sla.sla_backward_workspace_bytes(bad) == 0 and sla.sla_backward_num_stages(bad) == -1
    assert _call_backward(bad) == sla.SLA_ERR_UNSUPPORTED


def test_backward_rejects_bad_arguments_before_launch():
    cfg = wl.small_config(N=1024, N_valid=1000, has_gate=1)
    for name in ("q", "k", "v", "out", "dout", "dq", "dk", "dv", "w_p", "w_g", "dw_p", "dw_g"):
        assert _call_backward(cfg, **{name: None}) == sla.SLA_ERR_INVALID_ARG, name
        assert _call_backward(cfg, **{name: 24}) == sla.SLA_ERR_INVALID_ARG, name  # misaligned
    assert _call_backward(cfg, ws=None) == sla.SLA_ERR_WORKSPACE
    assert _call_backward(cfg, ws_bytes=sla.sla_workspace_bytes(cfg) - 1) == sla.SLA_ERR_WORKSPACE
    assert _call_backward(cfg, bws=None) == sla.SLA_ERR_WORKSPACE
    assert _call_backward(cfg, bws=128) == sla.SLA_ERR_WORKSPACE
    assert _call_backward(cfg, bws_bytes=sla.sla_backward_workspace_bytes(cfg) - 1) == sla.SLA_ERR_WORKSPACE
    # without projection and gate their gradients may be NULL; a short scratch still stops the call
    plain = wl.small_config(N=1024, N_valid=1000, has_proj=0, has_gate=0)
    assert _call_backward(plain, w_p=None, w_g=None, dw_p=None, dw_g=None, bws_bytes=0) == sla.SLA_ERR_WORKSPACE
    c = sla.make_config(cfg)
    evs = (ctypes.c_void_p * 2)(1, 2)
    r = sla.lib().sla_backward_timed(16, 16, 16, 16, 16, ctypes.byref(c), 16, 16, 16, 16, 16, 16, 16, 256,
                                     sla.sla_workspace_bytes(cfg), 256, sla.sla_backward_workspace_bytes(cfg),
                                     None, evs, 2)
    assert r == sla.SLA_ERR_INVALID_ARG


def test_backward_scratch_grows_with_the_problem():
    small = wl.small_config(N=1024, N_valid=1024, has_gate=1)
    big = wl.small_config(N=4096, N_valid=4096, has_gate=1)
    assert sla.sla_backward_workspace_bytes(big) > 2 * sla.sla_backward_workspace_bytes(small)


def test_nsa_branches_configuration():
    c = wl.preset("nsa_branches")
    assert sla.sla_validate_config(c) == sla.SLA_OK
    assert sla.sla_stage_names(c) == ["pool", "pooled_scores", "select_topn", "compress_kv", "sparse_flash_cmp",
                                      "sparse_flash_slc", "sparse_flash_win"]
    # the three branch outputs and the compressed keys add to the workspace
    assert sla.sla_workspace_bytes(c) > sla.sla_workspace_bytes(wl.preset("nsa_causal"))
    # the gates belong to NSA's branches; no branches in the three-way mode
    assert sla.sla_backward_workspace_bytes(c) > sla.sla_backward_workspace_bytes(wl.preset("nsa_causal"))
    assert sla.sla_validate_config(wl.preset("nsa_causal").replace(has_gate=1)) == sla.SLA_ERR_UNSUPPORTED
    assert sla.sla_validate_config(wl.preset("wan1.3b").replace(nsa_branches=1)) == sla.SLA_ERR_UNSUPPORTED
    assert sla.sla_validate_config(c.replace(cmp_stride=0)) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_validate_config(c.replace(nsa_branches=2)) == sla.SLA_ERR_INVALID_ARG


def test_noalloc_entry_points_reject_bad_arguments_without_a_device():
    """sla_route_noalloc checks its arguments before it looks for a device; its status
    reader needs a device and reports a CUDA error where there is none."""
    c = sla.make_config(wl.preset("tiny"))
    L = sla.lib()
    assert L.sla_route_noalloc(None, 16, ctypes.byref(c), None, 16, 16, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_route_noalloc(16, 16, ctypes.byref(c), None, None, 16, None) == sla.SLA_ERR_INVALID_ARG
    assert L.sla_route_noalloc(8, 16, ctypes.byref(c), None, 16, 16, None) == sla.SLA_ERR_INVALID_ARG
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if not has_gpu:
        detail = ctypes.c_int32(0)
        assert L.sla_route_noalloc_status(None, ctypes.byref(detail)) == sla.SLA_ERR_CUDA


def test_forward_blocks_rejects_bad_ranges_before_launch():
    """sla_forward_blocks: the query-block range starts on a pair, is not empty and stays
    inside the layer (an odd end only at the last block); checked before any launch."""
    c = sla.make_config(wl.small_config(N=1216, N_valid=1200, d=64))  # 19 query blocks
    L = sla.lib()
    ws = 256
    nbytes = sla.sla_workspace_bytes(wl.small_config(N=1216, N_valid=1200, d=64))
    for qb0, qb1 in ((1, 4), (0, 0), (4, 2), (0, 20), (2, 5), (-2, 4)):
        assert L.sla_forward_blocks(16, 16, 16, 16, 16, ctypes.byref(c), qb0, qb1, 16, None, ws, nbytes,
                                    None) == sla.SLA_ERR_INVALID_ARG, (qb0, qb1)
