"""The host entry point (pwp_prune_layer_host, prune_layer_host in the binding) on the GPU:
W and X come from pinned host memory, X in row chunks folded into H as they land, and the
finished column blocks return during the sweep.  Its results must equal, bit for bit, the
device entry point given the same H: built in the same row chunks (eight for n >= 8192,
else one), since fp32 sums in another grouping round differently.  The device entry point
itself is held to the oracle by the parity tests."""
import numpy as np
import pytest

import synth
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _pinned(t):
    return t.cpu().contiguous().pin_memory()


def _chunked_h(pwp, Xd):
    """H the way the host entry point builds it: eight row chunks when n >= 8192."""
    n = Xd.shape[0]
    nch = 8 if n >= 8192 else 1
    rows = -(-n // nch)
    H = None
    for r0 in range(0, n, rows):
        H = pwp.hessian_accumulate(Xd[r0:r0 + rows], H, beta=1 if r0 > 0 else 0)
    return H


def _both(c, b, n, dtype, seed, **kw):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.custom(c, b, n, dtype=dtype, sparsity=kw.get("sparsity", 0.5), seed=seed)
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    Wd, Xd = P.torch_inputs(W, X, dtype)
    W_h, m_h, st_h = pwp.prune_layer_host(_pinned(Wd), _pinned(Xd), **kw)
    torch.cuda.synchronize()
    if kw.get("method", "thanos") in ("wanda", "magnitude"):
        W_d, m_d, st_d = pwp.prune_layer(Wd, X=Xd, **kw)
    else:
        W_d, m_d, st_d = pwp.prune_layer(Wd, H=_chunked_h(pwp, Xd), **kw)
    torch.cuda.synchronize()
    sh = pwp.read_stats(st_h)
    assert sh.status == 0 and sh.pruned == sh.target == st_d.target
    assert torch.equal(m_h, m_d.cpu())
    assert torch.equal(W_h, W_d.cpu())
    return W_h, m_h, sh


@pytest.mark.parametrize("method", ["thanos", "sparsegpt"])
@pytest.mark.parametrize("pattern,nm", [("unstructured", (2, 4)), ("nm", (2, 4))])
@pytest.mark.parametrize("n", [600, 9000])
def test_host_entry_equals_device_entry(method, pattern, nm, n):
    _both(256, 384 + 64, n, "bf16", 11 + n, method=method, pattern=pattern, nm=nm, block=128)


def test_host_entry_fp32_ragged_blocks():
    # b not a multiple of the block: the last column block returned is narrow
    _both(100, 300, 700, "fp32", 5, method="thanos", block=64)


@pytest.mark.parametrize("method", ["wanda", "magnitude"])
def test_host_entry_no_update(method):
    _both(96, 256, 9000, "bf16", 3, method=method)


def test_host_entry_outlier_rows():
    # alpha > 0: the outlier rows are scattered back at the end, one copy of the whole result
    W_h, m_h, _ = _both(200, 256, 640, "bf16", 8, method="thanos", alpha=0.1, block=64)
    assert int(m_h.sum()) > 0


def test_host_entry_rejects_pageable_buffers():
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    W = torch.zeros(8, 16)
    X = torch.zeros(4, 16).pin_memory()
    with pytest.raises(ValueError):
        pwp.prune_layer_host(W, X)


@pytest.mark.parametrize("kw", [dict(method="thanos"), dict(method="sparsegpt", pattern="nm", nm=(2, 4)),
                                dict(method="wanda"), dict(method="thanos", alpha=0.1, block=64)])
def test_layers_entry_equals_one_layer_calls(kw):
    """pwp_prune_layers_host (double-buffered transfers across layers) gives every layer
    what pwp_prune_layer_host gives it alone, bit for bit."""
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    Ws, Xs = [], []
    for seed in range(3):
        wl = synth.custom(128, 256, 9000, dtype="bf16", sparsity=0.5, seed=40 + seed)
        W, X = synth.make_W(wl), synth.make_X_tokens(wl)
        Wd, Xd = P.torch_inputs(W, X, "bf16")
        Ws.append(_pinned(Wd))
        Xs.append(_pinned(Xd))
    W_l, m_l, st_l = pwp.prune_layers_host(Ws, Xs, **kw)
    torch.cuda.synchronize()
    recs = pwp.read_stats_list(st_l)
    for i in range(3):
        W_1, m_1, st_1 = pwp.prune_layer_host(Ws[i], Xs[i], **kw)
        torch.cuda.synchronize()
        s1 = pwp.read_stats(st_1)
        assert recs[i].status == 0 and recs[i].pruned == recs[i].target == s1.target
        assert torch.equal(m_l[i], m_1)
        assert torch.equal(W_l[i], W_1)


def test_layers_entry_rejects_mixed_shapes():
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    W = [torch.zeros(8, 16).pin_memory(), torch.zeros(8, 32).pin_memory()]
    X = [torch.zeros(4, 16).pin_memory(), torch.zeros(4, 32).pin_memory()]
    with pytest.raises(ValueError):
        pwp.prune_layers_host(W, X)
