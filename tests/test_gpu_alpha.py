"""GPU parity of the alpha variant (outlier rows kept dense; "Pruning LLMs with Thanos",
section "Thanos versus SparseGPT on LLaMA-3 8B"): the rows the library keeps are the
oracle's outlier rows, they come back bit-for-bit with an empty mask, and the other rows
match the oracle's prune of those rows as a layer of their own under the usual bars."""
import numpy as np
import pytest

import oracle
import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu

TIE_TOL = 1e-6


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("c,b,n,B,dtype,method,pattern,nm,alpha", [
    (40, 64, 128, 16, "fp32", "thanos", "unstructured", (0, 0), 0.1),
    (40, 64, 128, 16, "fp32", "thanos", "nm", (2, 4), 0.1),
    (64, 128, 256, 32, "bf16", "thanos", "nm", (4, 8), 0.1),
    (50, 96, 160, 32, "fp32", "sparsegpt", "unstructured", (0, 0), 0.25),
])
def test_alpha_variant_matches_oracle(c, b, n, B, dtype, method, pattern, nm, alpha):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.custom(c, b, n, dtype=dtype, outlier_frac=0.05, outlier_scale=10.0, pattern=pattern, nm=nm,
                      sparsity=0.5, block=B, name="alpha_layer")
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    Wt, Xt = P.torch_inputs(W, X, dtype)
    W_hat_t, mask_t, st = pwp.prune_layer(Wt, X=Xt, method=method, pattern=pattern, nm=nm, sparsity=0.5, block=B,
                                          damp=0.01, alpha=alpha)
    torch.cuda.synchronize()
    W_hat = W_hat_t.cpu().numpy().astype(np.float64)
    mask = mask_t.cpu().numpy().astype(bool)
    W64, X64 = synth.to_f64(W, dtype), synth.to_f64(X, dtype)
    orc = oracle.prune_layer_alpha(W64, Xt=X64, alpha=alpha, sparsity=float(np.float32(0.5)), pattern=pattern, nm=nm,
                                   block=B, damp=0.01, method=method)
    out = orc["outliers"]
    assert int(out.sum()) == int(np.floor(alpha * c))
    # the outlier rows: unchanged, nothing removed
    assert np.array_equal(W_hat[out], W64[out]) and not mask[out].any()
    # the other rows: the oracle's prune of them as a layer of their own
    keep = ~out
    inner = orc["inner"]
    res = P.compare(W[keep], dtype, (W_hat[keep], mask[keep], st), inner, pattern=pattern, nm=nm, block=B,
                    tie_tol=TIE_TOL)
    assert res["status"] == 0 and res["zeros_exact"], res
    assert res["n_mask"] == inner["pruned"] == st.pruned == st.target, res
    assert res["agree"] >= P.MASK_AGREE and res["n_dis_not_tie"] == 0, res
    assert res["w_rel"] <= P.W_REL_TOL, res
    lg = oracle.recon_loss(W64, W_hat, oracle.gram(X64))
    assert abs(lg - orc["loss"]) <= P.LOSS_REL_TOL * orc["loss"], (lg, orc["loss"])
