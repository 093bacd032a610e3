"""Parity at the full sizes of the benchmark workloads (4096x4096 at 50% unstructured,
11008x4096 at 2:4, 4096x11008 at 4:8; n = 16384 or 32768 bf16 tokens), in the
configuration bench.py times.  Checked: properties that hold at any size (removed weights
exactly 0, the exact removal count or every N:M group keeping n); sampled entries of H
against fp64 dot products of the activation columns; and the first block's selection
against the oracle, which at that point depends only on W and the column norms
(tests/_fullsize.py), except within 2e-5 (relative) of the selection boundary."""
import numpy as np
import pytest

import synth
from tests import _fullsize as F
from tests import _parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.fullsize]

TIE_TOL = 2e-5


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("name", ["q_proj4096x4096", "up_proj11008x4096_2of4", "down_proj4096x11008_4of8"])
def test_full_size_workload(name):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.workload(name)
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    Wt, Xt = P.torch_inputs(W, X, wl.dtype)
    g = F.column_norms_sq(X, wl.dtype)

    # sampled entries of H = 2 X X^T (diagonal ones included)
    H = pwp.hessian_accumulate(Xt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(77)
    ii = rng.integers(0, wl.b, 48)
    jj = rng.integers(0, wl.b, 48)
    ii = np.concatenate([ii, ii[:16]])
    jj = np.concatenate([jj, ii[:16]])
    Hs = H[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].cpu().numpy().astype(np.float64)
    del H
    ref = 2.0 * np.einsum("tk,tk->k", synth.to_f64(X[:, ii], wl.dtype), synth.to_f64(X[:, jj], wl.dtype))
    scale = 2.0 * np.sqrt(g[ii] * g[jj])
    assert np.max(np.abs(Hs - ref) / scale) < 1e-4

    # the prune
    nm = wl.nm if wl.pattern == "nm" else (0, 0)
    W_hat, mask, st = pwp.prune_layer(Wt, X=Xt, method="thanos", pattern=wl.pattern, nm=nm, sparsity=wl.sparsity,
                                      block=wl.block, damp=wl.damp)
    torch.cuda.synchronize()
    assert st.status == 0
    assert bool(torch.all(W_hat[mask.bool()] == 0).item())
    m = mask.cpu().numpy().astype(bool)
    c, b = m.shape
    if wl.pattern == "unstructured":
        want = int(np.floor(float(np.float32(wl.sparsity)) * c * b))
        assert int(m.sum()) == st.pruned == st.target == want
    else:
        n_keep, mm = nm
        assert np.all(m.reshape(c, -1, mm).sum(axis=2) == mm - n_keep)
        assert st.pruned == st.target == int(m.sum())

    # the first block's decisions
    W64 = synth.to_f64(W, wl.dtype)
    m0, decided = F.block0_expected(W64, g, pattern=wl.pattern, nm=nm, sparsity=wl.sparsity, block=wl.block,
                                    tol=TIE_TOL)
    B = min(wl.block, b)
    assert decided.mean() > 0.99
    assert np.array_equal(m[:, :B][decided], m0[decided])
