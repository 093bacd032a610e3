"""The stepwise sweep on the GPU (pwp_sweep_step): one rank reproduces pwp_prune_layer,
and row slices pruned as several ranks under one global budget -- ranks emulated in this
process, one after another on one stream, their buffers summed and gathered by the host
(no kernel waits on another) -- reproduce the whole-layer prune and the oracle."""
import numpy as np
import pytest

import oracle
import synth
from post_weight_pruning_b200 import sharded
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _ranks(Wt, H, world, **kw):
    import post_weight_pruning_b200 as pwp
    c = Wt.shape[0]
    sweeps = []
    for r in range(world):
        r0, r1 = sharded.row_range(c, world, r)
        sweeps.append(pwp.Sweep(Wt[r0:r1].contiguous(), H.clone(), c, world, r, **kw))
    sharded.global_sweep(sweeps, sharded.LocalComm())
    outs = [sw.result() for sw in sweeps]
    W_hat = np.concatenate([o[0].cpu().numpy() for o in outs])
    mask = np.concatenate([o[1].cpu().numpy().astype(bool) for o in outs])
    return W_hat, mask, sum(o[2].pruned for o in outs)


@pytest.mark.parametrize("c,b,n,B,dtype,method", [
    (96, 256, 512, 32, "fp32", "thanos"),
    (256, 512, 1024, 128, "bf16", "thanos"),
    (100, 200, 300, 48, "fp32", "sparsegpt"),
])
def test_sweep_ranks_reproduce_the_whole_layer(c, b, n, B, dtype, method):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.custom(c, b, n, dtype=dtype, outlier_frac=0.02, outlier_scale=20.0, block=B, name="sweep_layer")
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    Wt, Xt = P.torch_inputs(W, X, dtype)
    H = pwp.hessian_accumulate(Xt)
    kw = dict(method=method, sparsity=0.5, block=B, damp=0.01)
    W1, m1, st1 = pwp.prune_layer(Wt, H=H.clone(), **kw)
    torch.cuda.synchronize()
    W1, m1 = W1.cpu().numpy(), m1.cpu().numpy().astype(bool)
    for world in (1, 2, 3):
        Wg, mg, pruned = _ranks(Wt, H, world, **kw)
        torch.cuda.synchronize()
        assert pruned == st1.pruned == st1.target, world
        assert np.array_equal(mg, m1), world
        assert np.array_equal(Wg, W1), world


def test_sweep_ranks_split_tied_thresholds_like_the_oracle():
    """Weights on a 1/64 grid and +-1 activations: the first block's threshold cuts through
    large groups of equal scores held by different ranks; (column, row) order with lower
    ranks' rows first gives the oracle's mask."""
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    rng = np.random.default_rng(11)
    c, b, n = 90, 64, 128
    W = (np.round(rng.normal(0, 0.02, size=(c, b)) * 64) / 64).astype(np.float32)
    X = rng.choice([-1.0, 1.0], size=(n, b)).astype(np.float32)
    Wt, Xt = torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda()
    H = pwp.hessian_accumulate(Xt)
    Wg, mg, pruned = _ranks(Wt, H, 3, method="thanos", sparsity=0.33, block=32, damp=0.01)
    orc = oracle.prune_layer(W.astype(np.float64), Xt=X.astype(np.float64), sparsity=float(np.float32(0.33)),
                             block=32, damp=0.01)
    assert (orc["dscore"][:, :32] == orc["blocks"][0]["t_last"]).sum() > 20
    assert pruned == orc["zstar"]
    assert np.array_equal(mg[:, :32], orc["mask"][:, :32])
    assert float(np.linalg.norm(Wg - orc["W"]) / np.linalg.norm(orc["W"])) <= P.W_REL_TOL
