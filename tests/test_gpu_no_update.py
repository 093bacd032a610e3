"""GPU parity of the no-update baselines (Wanda, magnitude) against the fp64 oracle:
per-row quota or N:M groups, kept weights bit-exact, removed weights exactly 0, exact
counts.  Magnitude scores are exact on both sides, so its masks must match exactly;
Wanda's fp32 scores may differ from the oracle's fp64 ones only at near-ties of a row's
(or group's) threshold."""
import numpy as np
import pytest

import oracle
import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu

# score ties within 1e-6 relative: the stated bar for mask disagreements
TIE_TOL = 1e-6


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _run(W, X, dtype, method, pattern, nm, s, via):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    Wt, Xt = P.torch_inputs(W, X, dtype)
    if via == "x":
        W_hat, mask, st = pwp.prune_layer(Wt, X=Xt, method=method, pattern=pattern, nm=nm, sparsity=s)
    else:
        H = pwp.hessian_accumulate(Xt)
        H0 = H.clone()
        W_hat, mask, st = pwp.prune_layer(Wt, H=H if method == "wanda" else None, method=method,
                                          pattern=pattern, nm=nm, sparsity=s)
        if method == "wanda":
            assert torch.equal(H, H0)          # Wanda only reads the diagonal
    torch.cuda.synchronize()
    return W_hat.cpu().numpy(), mask.cpu().numpy().astype(bool), st


def _check(W, X, dtype, method, pattern, nm, s, via):
    W64 = synth.to_f64(W, dtype)
    X64 = synth.to_f64(X, dtype)
    W_hat, mask, st = _run(W, X, dtype, method, pattern, nm, s, via)
    orc = oracle.prune_no_update(W64, Xt=X64, sparsity=float(np.float32(s)), pattern=pattern, nm=nm,
                                 method=method)
    assert st.status == 0
    assert st.pruned == st.target == orc["target"] == int(mask.sum())
    assert np.all(W_hat[mask] == 0.0)
    assert np.array_equal(W_hat[~mask], W64[~mask].astype(np.float32))     # no update, bit-exact
    if pattern == "unstructured":
        assert np.all(mask.sum(axis=1) == orc["mask"].sum(axis=1))
    else:
        n_keep, m = nm
        assert np.all(mask.reshape(mask.shape[0], -1, m).sum(axis=2) == m - n_keep)
    dis = np.argwhere(mask != orc["mask"])
    if method == "magnitude":
        assert len(dis) == 0
        return
    S, Mo = orc["S"], orc["mask"]
    for k, q in dis:
        if pattern == "unstructured":
            ref = S[k][Mo[k]].max()
        else:
            m = nm[1]
            g0 = (q // m) * m
            ref = S[k, g0:g0 + m][Mo[k, g0:g0 + m]].max()
        assert abs(S[k, q] - ref) <= TIE_TOL * max(ref, 1e-300), (k, q, S[k, q], ref)


@pytest.mark.parametrize("method", ["wanda", "magnitude"])
@pytest.mark.parametrize("pattern,nm,s", [("unstructured", (0, 0), 0.5), ("unstructured", (0, 0), 0.37),
                                          ("nm", (2, 4), 0.5), ("nm", (4, 8), 0.5)])
@pytest.mark.parametrize("via", ["x", "h"])
def test_no_update_matches_oracle(method, pattern, nm, s, via):
    wl = synth.custom(96, 520, 300, dtype="bf16", outlier_frac=0.02, outlier_scale=20.0, sparsity=s, seed=5)
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    _check(W, X, "bf16", method, pattern, nm, s, via)


@pytest.mark.parametrize("c,b,n,dtype,s", [(7, 11008, 64, "fp32", 0.5),     # an 11008-wide row (down_proj)
                                           (33, 250, 40, "fp32", 0.9),
                                           (5, 3, 8, "fp32", 0.34),         # quota 1 of 3
                                           (16, 64, 32, "bf16", 0.0)])      # nothing removed
def test_no_update_shapes(c, b, n, dtype, s):
    wl = synth.custom(c, b, n, dtype=dtype, sparsity=s, seed=c + b)
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    for method in ("wanda", "magnitude"):
        _check(W, X, dtype, method, "unstructured", (0, 0), s, "x")


def test_no_update_exact_ties_take_lower_columns():
    """Weights on a 1/64 grid: whole rows of equal |W|; the per-row cut falls inside a tie
    group and both sides take its lower columns."""
    wl = synth.custom(40, 300, 64, dtype="fp32", sparsity=0.5, seed=9)
    W = (np.round(synth.make_W(wl).astype(np.float64) * 64.0) / 64.0).astype(np.float32)
    rng = np.random.default_rng(9)
    X = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=(64, 300))
    for method in ("magnitude", "wanda"):
        W_hat, mask, st = _run(W, X, "fp32", method, "unstructured", (0, 0), 0.5, "x")
        orc = oracle.prune_no_update(W.astype(np.float64), Xt=X.astype(np.float64), sparsity=0.5,
                                     method=method)
        assert np.array_equal(mask, orc["mask"])
