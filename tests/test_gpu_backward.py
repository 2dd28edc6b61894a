"""GPU parity of the backward pass (sla_backward) against the float64 gradient oracle.

Each case runs sla_forward and then sla_backward through the C ABI on seeded
bf16 inputs and a seeded bf16 dO. It compares dq, dk, dv, dW_p and dw_g element
by element with oracle/sla_grad.py, which gets the same bf16 values and the
GPU's own routing classes. Bar: relative Frobenius error <= 2e-2 per tensor.
The arithmetic rounds P, dS, phi(K), the states and the outputs to bf16 (about
4e-3 each), so a dropped term or a wrong index shows up as an O(1) error.
The all-critical cases check the sparse branch alone, the all-marginal ones
the linear branch, the projection and the gate alone. Full-size layers (the
bench's shapes) are compared on sampled query and key blocks of every head, and
on dW_p and dw_g in full, against the oracle's block-by-block statement.

Every tensor also has an element-wise bar: max |got - ref| <= 2e-2 * max |ref|
(the "<name>_elem" entries). A gradient element sums many terms that carry the
same few bf16 roundings, so its error is about 4.5e-3 of the spread of the
values, like the Frobenius ratio; the bar is four times that. A few wrong rows
(a mis-indexed key block or KV group) give errors of the size of the values
themselves and fail it even where the Frobenius ratio of a large tensor would
not notice them.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_linear_sm_b200 as sla  # noqa: E402
from block_sparse_linear_sm_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU runs deselect these anyway
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_util import DeviceRun, bf16_to_f64, to_dev  # noqa: E402
from oracle import sla_grad  # noqa: E402

REL = 2e-2   # relative Frobenius error per tensor, and max |err| / max |ref| per tensor


def elem_ratio(pairs):
    """max |got - ref| over max |ref| across (got, ref) pairs (max |got| when ref is 0)."""
    err = max(float(np.max(np.abs(g - r))) for g, r in pairs)
    top = max(float(np.max(np.abs(r))) for _, r in pairs)
    return err / top if top > 0 else err


def d_out_bits(c, seed):
    rng = np.random.default_rng(seed)
    return wl.to_bf16_bits(rng.standard_normal((c.B, c.H, c.N, c.d)))


def topn_selection(run):
    """The GPU's own top-n selection as lists [B][H_kv][nqb] (from its routing mask)."""
    m = run.mask.cpu().numpy()
    return [[[np.nonzero(m[b, hk, i] == 2)[0] for i in range(m.shape[2])] for hk in range(m.shape[1])]
            for b in range(m.shape[0])]


def run_backward(cfg, seed=3, v_shift=0.0, keep=None):
    """Relative Frobenius error per gradient tensor; ``keep`` (a dict) receives the GPU's
    gradients ("got") and the oracle's ("ref")."""
    x = wl.generate(cfg, v_shift=v_shift)
    run = DeviceRun(cfg, x, route=False)
    c = cfg
    dob = d_out_bits(c, seed)
    dout = to_dev(dob)
    dq, dk, dv = torch.empty_like(run.q), torch.empty_like(run.k), torch.empty_like(run.v)
    dw_p = dw_g = None
    if c.has_proj:
        shape = (c.H, c.d, c.d) if c.proj_per_head else (c.d, c.d)
        dw_p = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    if c.has_gate:
        shape = (c.H, 3, c.d) if c.nsa_branches else (c.H, c.d)
        dw_g = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    nbytes = sla.sla_backward_workspace_bytes(c)
    assert nbytes > 0
    bws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    sla.sla_backward(run.q, run.k, run.v, run.w_p, run.w_g, c, run.out, dout, dq, dk, dv, dw_p, dw_g,
                     run.ws, bws)
    st, detail = sla.sla_check_device_status(bws)
    assert st == 0, (st, detail)
    classes = run.mask.cpu().numpy() if c.mode == wl.MODE_THREEWAY else topn_selection(run)
    ref = sla_grad.layer_grads(c, x.f64("q"), x.f64("k"), x.f64("v"),
                               x.f64("w_p") if c.has_proj else None,
                               x.f64("w_g") if c.has_gate else None,
                               wl.bf16_bits_to_f64(dob), classes=classes)
    got = dict(dq=bf16_to_f64(dq), dk=bf16_to_f64(dk), dv=bf16_to_f64(dv))
    if dw_p is not None:
        got["dw_p"] = dw_p.double().cpu().numpy()
    if dw_g is not None:
        got["dw_g"] = dw_g.double().cpu().numpy()
    errs = {}
    for key, g in got.items():
        r = ref[key]
        assert np.all(np.isfinite(g)), key
        nr = np.linalg.norm(r)
        errs[key] = float(np.linalg.norm(g - r) / nr) if nr > 0 else float(np.abs(g).max())
        errs[key + "_elem"] = elem_ratio([(g, r)])
    # padding rows of the gradients are zero
    for key in ("dq", "dk", "dv"):
        assert np.all(got[key][:, :, c.N_valid:] == 0), key
    if keep is not None:
        keep.update(got=got, ref=ref, x=x, dout=wl.bf16_bits_to_f64(dob))
    return errs


def small(**kw):
    return wl.small_config(**kw)


NSA = dict(mode=wl.MODE_TOPN_WINDOW, causal=1, k_h=0, k_l=0, has_proj=0, nsa_branches=1)


CASES = [
    dict(name="all_crit_d64", N=768, N_valid=763, d=64, k_h=12, k_l=0),
    dict(name="all_crit_gqa_d128", N=1024, N_valid=1024, d=128, H=4, H_kv=2, k_h=16, k_l=0),
    dict(name="all_marg_d64", N=1024, N_valid=1000, d=64, k_h=0, k_l=0, has_gate=1),
    dict(name="all_marg_per_head_d128", N=1024, N_valid=1024, d=128, H=2, H_kv=2, k_h=0, k_l=0,
         proj_per_head=1, has_gate=1),
    dict(name="mixed_d64", N=1024, N_valid=1024, d=64, k_h=4, k_l=4, has_gate=1),
    dict(name="mixed_ragged_d128", N=2048, N_valid=2001, d=128, H=4, H_kv=4, k_h=5, k_l=7, has_gate=1),
    dict(name="mixed_gqa_d128", N=1536, N_valid=1473, d=128, H=4, H_kv=2, k_h=3, k_l=2, has_gate=1),
    dict(name="no_proj_d128", N=1024, N_valid=1000, d=128, k_h=2, k_l=2, has_proj=0),
    dict(name="linear_all_d64", N=1024, N_valid=1000, d=64, k_h=3, k_l=4, linear_all=1),
    dict(name="odd_blocks_d128", N=1216, N_valid=1200, d=128, k_h=3, k_l=4, has_gate=1),
    dict(name="batch2_d64", B=2, N=640, N_valid=600, d=64, H=2, H_kv=1, k_h=2, k_l=1, has_gate=1),
    dict(name="single_block_d128", N=64, N_valid=50, d=128, k_h=1, k_l=0),
    dict(name="many_tiles_d128", N=4096, N_valid=4096, d=128, H=2, H_kv=2, k_h=16, k_l=16, has_gate=1),
    dict(name="smooth_k_d128", N=1536, N_valid=1500, d=128, H=4, H_kv=4, k_h=3, k_l=4, smooth_k=1, has_gate=1),
    dict(name="smooth_k_d64", N=1024, N_valid=1000, d=64, k_h=2, k_l=3, smooth_k=1),
    dict(name="smooth_linear_all_gqa", N=1536, N_valid=1473, d=128, H=4, H_kv=2, k_h=3, k_l=2, smooth_k=1,
         linear_all=1, has_gate=1),
    # top-n + window mode (causal, GQA, shared selections): the sparse branch only
    dict(name="topn_gqa_d128", N=2048, N_valid=2048, d=128, H=4, H_kv=2, mode=wl.MODE_TOPN_WINDOW, causal=1,
         top_n=4, window=256, k_h=0, k_l=0, has_proj=0),
    dict(name="topn_odd_group_ragged_d64", N=1536, N_valid=1500, d=64, H=3, H_kv=1, mode=wl.MODE_TOPN_WINDOW,
         causal=1, top_n=3, window=100, k_h=0, k_l=0, has_proj=0),
    dict(name="topn_no_window_d128", N=1024, N_valid=1024, d=128, H=2, H_kv=2, mode=wl.MODE_TOPN_WINDOW,
         causal=1, top_n=2, window=0, k_h=0, k_l=0, has_proj=0),
    dict(name="topn_window_only_d64", N=1024, N_valid=1000, d=64, H=4, H_kv=1, mode=wl.MODE_TOPN_WINDOW,
         causal=1, top_n=0, window=192, k_h=0, k_l=0, has_proj=0),
    # NSA's three branches (compressed, selected, window; gated or summed): the gradient runs
    # back through each branch's own softmax, the gates, and the block means of the
    # compressed keys and values to every token they average
    dict(name="nsa_gqa_gates_d128", N=2048, N_valid=2048, d=128, H=4, H_kv=2, top_n=4, window=256,
         cmp_block=32, cmp_stride=16, has_gate=1, **NSA),
    dict(name="nsa_odd_group_ragged_d64", N=1536, N_valid=1500, d=64, H=3, H_kv=1, top_n=3, window=100,
         cmp_block=32, cmp_stride=16, has_gate=0, **NSA),
    dict(name="nsa_unit_cmp_d128", N=1024, N_valid=1000, d=128, H=2, H_kv=2, top_n=2, window=64,
         cmp_block=1, cmp_stride=1, has_gate=1, **NSA),
    dict(name="nsa_wide_blocks_no_window_d64", N=2048, N_valid=2048, d=64, H=4, H_kv=1, top_n=2, window=0,
         cmp_block=64, cmp_stride=48, has_gate=1, **NSA),
    dict(name="nsa_many_cmp_tiles_d128", N=4096, N_valid=4033, d=128, H=2, H_kv=1, top_n=3, window=128,
         cmp_block=32, cmp_stride=16, has_gate=1, **NSA),
]


@pytest.mark.parametrize("kw", CASES, ids=[c["name"] for c in CASES])
def test_backward_matches_gradient_oracle(kw):
    errs = run_backward(small(**kw))
    print(kw["name"], errs)
    assert all(e <= REL for e in errs.values()), errs


def test_backward_linear_branch_with_shifted_values():
    """All blocks marginal, V + 3: the linear branch's output is O(1) and dominates dV."""
    errs = run_backward(small(name="marg_shift", N=1024, N_valid=1024, d=128, k_h=0, k_l=0, has_gate=1),
                        v_shift=3.0)
    assert all(e <= REL for e in errs.values()), errs


def test_backward_smooth_k_mean_term():
    """All blocks marginal with smooth-K. The linear branch's dk is G - colsum(G) / N_valid
    (G: the gradient with respect to k - m), so its column sum over the valid rows is exactly
    0. The mean term is only about 1 % of dk, below the per-tensor bar, so it is checked
    through that column sum: the GPU's must be far below colsum(G), the value it would have
    without the term."""
    c = small(name="smooth_all_marg", N=1024, N_valid=1000, d=64, k_h=0, k_l=0, smooth_k=1, has_gate=1)
    keep = {}
    errs = run_backward(c, keep=keep)
    assert all(e <= REL for e in errs.values()), errs
    nv = c.N_valid
    x = keep["x"]
    k = x.f64("k")
    k_c = k.copy()
    k_c[:, :, :nv] -= k[:, :, :nv].mean(axis=2, keepdims=True)
    # G from the oracle on the centred keys with smooth-K off (the routing is unchanged)
    g = sla_grad.layer_grads(c.replace(smooth_k=0), x.f64("q"), k_c, x.f64("v"), x.f64("w_p"),
                             x.f64("w_g"), keep["dout"])["dk"]
    col_g = g[:, :, :nv].sum(axis=2)
    col_ref = keep["ref"]["dk"][:, :, :nv].sum(axis=2)
    col_got = keep["got"]["dk"][:, :, :nv].sum(axis=2)
    assert np.linalg.norm(col_ref) <= 1e-9 * np.linalg.norm(col_g)
    ratio = np.linalg.norm(col_got - col_ref) / np.linalg.norm(col_g)
    print("smooth-K column-sum ratio", ratio)
    assert ratio <= 0.1, ratio


def test_backward_all_negligible_is_zero():
    c = small(name="all_neg", N=512, N_valid=512, d=64, k_h=0, k_l=8, has_gate=1)
    x = wl.generate(c)
    run = DeviceRun(c, x, route=False)
    dout = to_dev(d_out_bits(c, 5))
    dq, dk, dv = torch.full_like(run.q, 7), torch.full_like(run.k, 7), torch.full_like(run.v, 7)
    dw_p = torch.full((c.d, c.d), 7.0, device="cuda")
    dw_g = torch.full((c.H, c.d), 7.0, device="cuda")
    bws = torch.empty(sla.sla_backward_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    sla.sla_backward(run.q, run.k, run.v, run.w_p, run.w_g, c, run.out, dout, dq, dk, dv, dw_p, dw_g,
                     run.ws, bws)
    assert sla.sla_check_device_status(bws) == (0, 0)
    for t in (dq, dk, dv, dw_p, dw_g):
        assert torch.count_nonzero(t).item() == 0


# ---------------------------------------------------------------------------
# full-size layers: sampled blocks of every head against the block-wise oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["wan1.3b", "salad", "wan1.3b_cosfilter", "wan1.3b_opensource"])
def test_full_size_backward_on_sampled_blocks(name):
    """The bench's layer shapes (one sla_forward + sla_backward call, as bench.py times them).
    dq on three query blocks and dk, dv on three key blocks of every head (first, middle,
    last: the ragged tail included), dW_p and dw_g in full, against oracle block_grads."""
    from gpu_util import LazyF64

    cfg = wl.preset(name)
    x = wl.generate(cfg)
    run = DeviceRun(cfg, x, route=False)
    c = cfg
    dob = d_out_bits(c, 17)
    dout = to_dev(dob)
    dq, dk, dv = torch.empty_like(run.q), torch.empty_like(run.k), torch.empty_like(run.v)
    dw_p = torch.empty((c.d, c.d), dtype=torch.float32, device="cuda") if c.has_proj else None
    dw_g = torch.empty((c.H, c.d), dtype=torch.float32, device="cuda") if c.has_gate else None
    bws = torch.empty(sla.sla_backward_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    sla.sla_backward(run.q, run.k, run.v, run.w_p, run.w_g, c, run.out, dout, dq, dk, dv, dw_p, dw_g,
                     run.ws, bws)
    assert sla.sla_check_device_status(bws) == (0, 0)
    nb = c.nqb
    qb, kb = [0, nb // 2, nb - 1], [0, nb // 2 + 1, nb - 1]
    classes = run.mask.cpu().numpy()
    ref = sla_grad.block_grads(c, LazyF64(x.q), LazyF64(x.k), LazyF64(x.v),
                               x.f64("w_p") if c.has_proj else None, x.f64("w_g") if c.has_gate else None,
                               LazyF64(dob), classes, 0, qb, kb)
    bl = c.block

    def rel(pairs):
        num = sum(float(np.sum((g - r) ** 2)) for g, r in pairs)
        den = sum(float(np.sum(r ** 2)) for _, r in pairs)
        return (num / den) ** 0.5

    dq_h = lambda h, i: bf16_to_f64(dq[0, h, i * bl:(i + 1) * bl])
    pairs = {"dq": [(dq_h(h, i), r) for (h, i), r in ref["dq"].items()]}
    for key, t in (("dk", dk), ("dv", dv)):
        pairs[key] = [(bf16_to_f64(t[0, hk, j * bl:(j + 1) * bl]), r) for (hk, j), r in ref[key].items()]
    if c.has_proj:
        pairs["dw_p"] = [(dw_p.double().cpu().numpy(), ref["dw_p"])]
    if c.has_gate:
        g = dw_g.double().cpu().numpy()
        pairs["dw_g"] = [(g[h], r) for h, r in ref["dw_g"].items()]
    errs = {}
    for key, pr in pairs.items():
        errs[key] = rel(pr)
        errs[key + "_elem"] = elem_ratio(pr)
    print(name, errs)
    assert all(e <= REL for e in errs.values()), errs


def test_full_size_topn_backward_on_sampled_blocks():
    """The NSA-shaped top-n layer (H=64, H_kv=4, N=65536, top 16, window 512): dq on four query
    blocks of the 16 heads of KV group 0, dk and dv on three key blocks of KV head 0 (complete:
    they sum over exactly those heads), against oracle block_grads."""
    from gpu_util import LazyF64

    c = wl.preset("nsa_causal")
    x = wl.generate(c)
    run = DeviceRun(c, x, route=False)
    dob = d_out_bits(c, 19)
    dout = to_dev(dob)
    dq, dk, dv = torch.empty_like(run.q), torch.empty_like(run.k), torch.empty_like(run.v)
    bws = torch.empty(sla.sla_backward_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    sla.sla_backward(run.q, run.k, run.v, None, None, c, run.out, dout, dq, dk, dv, None, None, run.ws, bws)
    assert sla.sla_check_device_status(bws) == (0, 0)
    nb, bl = c.nqb, c.block
    qb, kb = [1, 17, nb // 2, nb - 1], [0, nb // 2 + 1, nb - 1]
    ref = sla_grad.block_grads(c, LazyF64(x.q), LazyF64(x.k), LazyF64(x.v), None, None, LazyF64(dob),
                               topn_selection(run), 0, qb, kb, heads=range(c.H // c.H_kv))

    def rel(pairs):
        num = sum(float(np.sum((g - r) ** 2)) for g, r in pairs)
        den = sum(float(np.sum(r ** 2)) for _, r in pairs)
        return (num / den) ** 0.5

    pairs = {"dq": [(bf16_to_f64(dq[0, h, i * bl:(i + 1) * bl]), r) for (h, i), r in ref["dq"].items()]}
    for key, t in (("dk", dk), ("dv", dv)):
        pairs[key] = [(bf16_to_f64(t[0, hk, j * bl:(j + 1) * bl]), r) for (hk, j), r in ref[key].items()]
    errs = {}
    for key, pr in pairs.items():
        errs[key] = rel(pr)
        errs[key + "_elem"] = elem_ratio(pr)
    print("nsa_causal", errs)
    assert all(e <= REL for e in errs.values()), errs


def test_full_length_nsa_branches_backward_on_sampled_blocks():
    """NSA's three branches at the preset's full sequence length (N = 65536, d = 128, top 16,
    window 512, compressed blocks of 32 at stride 16, gates), one KV group of four query heads:
    dq on four query blocks of every head, dk and dv on three key blocks of the KV head
    (complete: they sum over the group's heads) and dw_g in full, against the oracle's
    block-by-block statement of the three branches."""
    from gpu_util import LazyF64

    c = wl.preset("nsa_branches").replace(name="nsa_branches_group4", H=4, H_kv=1)
    x = wl.generate(c)
    run = DeviceRun(c, x, route=False)
    dob = d_out_bits(c, 23)
    dout = to_dev(dob)
    dq, dk, dv = torch.empty_like(run.q), torch.empty_like(run.k), torch.empty_like(run.v)
    dw_g = torch.full((c.H, 3, c.d), float("nan"), dtype=torch.float32, device="cuda")
    bws = torch.empty(sla.sla_backward_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    sla.sla_backward(run.q, run.k, run.v, None, run.w_g, c, run.out, dout, dq, dk, dv, None, dw_g, run.ws, bws)
    assert sla.sla_check_device_status(bws) == (0, 0)
    nb, bl = c.nqb, c.block
    qb, kb = [1, 17, nb // 2, nb - 1], [0, nb // 2 + 1, nb - 1]
    ref = sla_grad.block_grads(c, LazyF64(x.q), LazyF64(x.k), LazyF64(x.v), None, x.f64("w_g"), LazyF64(dob),
                               topn_selection(run), 0, qb, kb)

    def rel(pairs):
        num = sum(float(np.sum((g - r) ** 2)) for g, r in pairs)
        den = sum(float(np.sum(r ** 2)) for _, r in pairs)
        return (num / den) ** 0.5

    pairs = {"dq": [(bf16_to_f64(dq[0, h, i * bl:(i + 1) * bl]), r) for (h, i), r in ref["dq"].items()]}
    for key, t in (("dk", dk), ("dv", dv)):
        pairs[key] = [(bf16_to_f64(t[0, hk, j * bl:(j + 1) * bl]), r) for (hk, j), r in ref[key].items()]
    g = dw_g.double().cpu().numpy()
    pairs["dw_g"] = [(g[h], r) for h, r in ref["dw_g"].items()]
    errs = {}
    for key, pr in pairs.items():
        errs[key] = rel(pr)
        errs[key + "_elem"] = elem_ratio(pr)
    print("nsa_branches_group4", errs)
    assert all(e <= REL for e in errs.values()), errs
