"""The bounded device-side waits give up cleanly.  With the wait limit at 0 every
ordinary mbarrier wait of the tensor-core kernels runs out at its first poll (copies and
MMAs already in flight are still waited for before a CTA leaves), so the call must end
with PWP_ETIMEOUT recorded in the device stats and the site of the kernel that gave up,
and no fault.  After the limit is restored, the next call on the same stream must match
the oracle again.  No GPU fault, trap or endless wait is involved: a wait that runs out is
the designed way out of these kernels."""
import numpy as np
import pytest

import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu

PWP_ETIMEOUT = 5
SITE_HESSIAN, SITE_STREAM = 6, 7


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _layer():
    wl = synth.custom(256, 512, 1024, dtype="bf16", outlier_frac=0.02, outlier_scale=20.0, block=128,
                      name="timeout_layer")
    return wl, synth.make_W(wl), synth.make_X_tokens(wl)


def _expect_correct(W, X, wl):
    kw = dict(method="thanos", pattern="unstructured", nm=(0, 0), block=wl.block, sparsity=wl.sparsity,
              damp=wl.damp)
    gpu = P.run_gpu(W, X, wl.dtype, **kw)
    orc = P.run_oracle(W, X, wl.dtype, **kw)
    res = P.compare(W, wl.dtype, gpu, orc, pattern="unstructured", nm=(0, 0), block=wl.block, tie_tol=1e-6)
    assert res["status"] == 0 and res["zeros_exact"], res
    assert res["n_mask"] == orc["pruned"] == res["stats_pruned"], res
    assert res["n_dis_not_tie"] == 0 and res["w_rel"] <= P.W_REL_TOL, res


def test_hessian_wait_that_runs_out_reports_timeout():
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl, W, X = _layer()
    Wt, Xt = P.torch_inputs(W, X, wl.dtype)
    prev = pwp.set_wait_limit(0)
    try:
        _, _, st_t = pwp.prune_layer(Wt, X=Xt, sparsity=0.5, block=128, check=False)
        torch.cuda.synchronize()
    finally:
        pwp.set_wait_limit(prev)
    st = pwp.read_stats(st_t)
    assert st.status == PWP_ETIMEOUT and st.status_site == SITE_HESSIAN, (st.status, st.status_site)
    _expect_correct(W, X, wl)


def test_tensor_core_update_wait_that_runs_out_reports_timeout():
    """H is built with the default limit; the prune then times out in its first tensor-core
    update (the factor's trailing update runs on the same kernel)."""
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl, W, X = _layer()
    Wt, Xt = P.torch_inputs(W, X, wl.dtype)
    H = pwp.hessian_accumulate(Xt)
    prev = pwp.set_wait_limit(0)
    try:
        _, _, st_t = pwp.prune_layer(Wt, H=H, sparsity=0.5, block=128, check=False)
        torch.cuda.synchronize()
    finally:
        pwp.set_wait_limit(prev)
    st = pwp.read_stats(st_t)
    assert st.status == PWP_ETIMEOUT and st.status_site == SITE_STREAM, (st.status, st.status_site)
    _expect_correct(W, X, wl)
    # the same stream and library state once more, with H rebuilt: still correct
    H2 = pwp.hessian_accumulate(Xt)
    W_hat, mask, st2 = pwp.prune_layer(Wt, H=H2, sparsity=0.5, block=128)
    torch.cuda.synchronize()
    assert st2.status == 0 and int(mask.sum().item()) == int(np.floor(0.5 * 256 * 512))
