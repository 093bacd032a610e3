"""pwp_prune_layer_noalloc, the prune entry point for callers that cannot hand the
library a workspace (an operator inside a runtime that only passes it its input and
output buffers, or a process whose device memory belongs to a framework allocator).

It takes its scratch from one static device array inside the library.  Here it is
called through the C ABI twice in a row on the same inputs -- the second call finds
the first call's leftovers in that shared array -- and both results must match the
regular workspace entry point, pwp_prune_layer, within the parity tolerances the
other GPU tests use.  The file name sorts after the other plain parity files, so a run
that stops at the first failure has already run them."""
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

W_REL_TOL = 1e-3
MASK_AGREE = 0.9999


def _setup():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_pruning_b200 as pwp
    L = pwp.lib()
    f = L.pwp_prune_layer_noalloc
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.POINTER(pwp.Config), ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return torch, pwp, f


def _inputs(torch, pwp, wl):
    W, X = synth.make_W(wl), synth.make_X_tokens(wl)
    if wl.dtype == "bf16":
        Wt, Xt = pwp.from_bf16_bits(W), pwp.from_bf16_bits(X)
    else:
        Wt, Xt = torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda()
    H = pwp.hessian_accumulate(Xt)
    torch.cuda.synchronize()
    return Wt, H


@pytest.mark.parametrize("wl,kw", [
    (synth.workload("layer128x256_fp32"), dict(method="thanos", pattern="unstructured")),
    (synth.custom(256, 512, 1024, dtype="bf16", outlier_frac=0.005, outlier_scale=50.0, block=128),
     dict(method="thanos", pattern="nm", nm=(2, 4))),
    (synth.custom(96, 200, 320, dtype="fp32", block=48, sparsity=0.37),
     dict(method="sparsegpt", pattern="unstructured")),
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(wl, kw):
    torch, pwp, f = _setup()
    Wt, H = _inputs(torch, pwp, wl)
    c, b = Wt.shape
    args = dict(sparsity=wl.sparsity, block=wl.block, damp=wl.damp, **kw)
    W_ref, M_ref, st_ref = pwp.prune_layer(Wt, H=H.clone(), **args)
    torch.cuda.synchronize()
    cfg = pwp.config(**{k: v for k, v in args.items()})
    wcode = pwp.BF16 if Wt.dtype == torch.bfloat16 else pwp.FP32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        Hc = H.clone()
        W_out = torch.full((c, b), float("nan"), dtype=torch.float32, device="cuda")
        mask = torch.full((c, b), 7, dtype=torch.uint8, device="cuda")
        stats = pwp.new_stats()
        rc = f(ctypes.byref(cfg), ctypes.c_void_p(Wt.data_ptr()), wcode, c, b, ctypes.c_void_p(Hc.data_ptr()),
               ctypes.c_void_p(W_out.data_ptr()), ctypes.c_void_p(mask.data_ptr()),
               ctypes.c_void_p(stats.data_ptr()), stream)
        assert rc == 0, pwp.status_string(rc)
        torch.cuda.synchronize()
        st = pwp.read_stats(stats)
        assert st.status == 0 and st.pruned == st_ref.pruned == st.target
        Wn, Mn = W_out.cpu().numpy().astype(np.float64), mask.cpu().numpy()
        Wr, Mr = W_ref.cpu().numpy().astype(np.float64), M_ref.cpu().numpy()
        assert set(np.unique(Mn).tolist()) <= {0, 1}
        assert np.mean(Mn == Mr) >= MASK_AGREE, call
        assert np.linalg.norm(Wn - Wr) / np.linalg.norm(Wr) <= W_REL_TOL, call
        assert np.all(Wn[Mn == 1] == 0.0)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    torch, pwp, f = _setup()
    cfg = pwp.config(pattern="nm", nm=(4, 8), block=128)
    need = pwp.workspace_bytes(cfg, 4096, 11008)
    assert need > 16 * 1024 * 1024
    fake = ctypes.c_void_p(1 << 20)
    rc = f(ctypes.byref(cfg), fake, pwp.BF16, 4096, 11008, fake, fake, fake, fake, None)
    assert rc == 3   # PWP_EWORKSPACE, nothing enqueued
