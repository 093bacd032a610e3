"""The two shardings of the multi-GPU layer prune, checked on one GPU with the ranks'
shares run one after another (no rank waits on another): the Hessians of token shards sum
to the whole layer's H, and prunes of row slices against one H reproduce, bit for bit,
the rows of the whole-layer prune wherever rows are independent."""
import numpy as np
import pytest

import synth
from tests import _parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.integration]


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def test_token_shards_sum_to_the_layer_hessian():
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    from post_weight_pruning_b200 import sharded
    wl = synth.custom(8, 384, 3000, dtype="bf16", outlier_frac=0.02, outlier_scale=50.0)
    _, Xt = P.torch_inputs(synth.make_W(wl), synth.make_X_tokens(wl), "bf16")
    H = pwp.hessian_accumulate(Xt)
    world = 3
    Hs = torch.zeros_like(H)
    for r in range(world):
        t0, t1 = sharded.token_range(wl.n, world, r)
        Hs += sharded.hessian_sharded(Xt[t0:t1].contiguous())   # no process group: one rank's share
    torch.cuda.synchronize()
    d = torch.sqrt(torch.diagonal(H))
    assert float(((Hs - H).abs() / torch.outer(d, d)).max()) < 3e-5     # each side within 1e-5 of fp64


@pytest.mark.parametrize("method,pattern,nm,sparsity", [
    ("thanos", "nm", (2, 4), 0.5), ("sparsegpt", "nm", (4, 8), 0.5), ("thanos", "nm", (4, 8), 0.5),
    ("wanda", "unstructured", (2, 4), 0.5), ("magnitude", "nm", (2, 4), 0.5),
])
def test_row_slices_reproduce_the_layer(method, pattern, nm, sparsity):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    from post_weight_pruning_b200 import sharded
    c, b = 300, 256                                     # slices of 100 rows: ragged 128-row tiles
    wl = synth.custom(c, b, 1024, dtype="bf16", outlier_frac=0.02, outlier_scale=20.0)
    Wt, Xt = P.torch_inputs(synth.make_W(wl), synth.make_X_tokens(wl), "bf16")
    H = pwp.hessian_accumulate(Xt)
    kw = dict(method=method, pattern=pattern, nm=nm, sparsity=sparsity, block=128, damp=0.01)
    W_full, m_full, st_full = pwp.prune_layer(Wt, H=H.clone(), **kw)
    W_parts, m_parts, pruned = [], [], 0
    for r in range(3):
        r0, r1 = sharded.row_range(c, 3, r)
        Wp, mp_, stp = sharded.prune_rows(Wt[r0:r1].contiguous(), H.clone(), **kw)
        W_parts.append(Wp)
        m_parts.append(mp_)
        pruned += stp.pruned
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(m_parts), m_full)
    assert torch.equal(torch.cat(W_parts), W_full)
    assert pruned == st_full.pruned
    if pattern == "nm":
        n_keep, m = nm
        mk = m_full.cpu().numpy().astype(bool)
        assert np.all(mk.reshape(c, -1, m).sum(axis=2) == m - n_keep)
