"""Token reordering on the GPU: the gather / scatter kernel against a NumPy gather
(bit-exact) with the Hilbert order of the Wan2.1-1.3B grid."""
import numpy as np
import pytest
import torch

import block_sparse_linear_sm_b200 as sla
from block_sparse_linear_sm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_permute_tokens_is_the_gather_and_its_inverse(d):
    cfg = wl.preset("wan1.3b")
    order = sla.sla_hilbert_order(*cfg.grid)                    # 32760 grid tokens
    rows, n_tok = 3, cfg.N                                       # 8 padding rows stay in place
    rng = np.random.default_rng(3)
    bits = wl.to_bf16_bits(rng.standard_normal((rows, n_tok, d)))
    x = torch.from_numpy(bits).view(torch.bfloat16).cuda()
    y = torch.empty_like(x)
    z = torch.empty_like(x)
    od = torch.from_numpy(order).cuda()
    sla.sla_permute_tokens(x, y, od)
    sla.sla_permute_tokens(y, z, od, inverse=True)
    torch.cuda.synchronize()
    want = bits.copy()
    want[:, :len(order)] = bits[:, order]
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want)
    assert torch.equal(z.view(torch.int16), x.view(torch.int16))
