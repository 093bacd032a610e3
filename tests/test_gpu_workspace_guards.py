"""No write outside the caller's buffers: every buffer the library writes (W_out, the
mask, H, the workspace, the stats word) is a window into a larger allocation whose
margins hold a guard pattern; after the call the margins must be unchanged and the
results must equal those of a call on plain buffers, bit for bit."""
import ctypes

import numpy as np
import pytest

import synth
from tests import _parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.integration]

GUARD = 4096                       # guard elements on each side (a multiple of 256 bytes)
F32_FILL = 0x7FC0DEAD              # a NaN pattern no kernel writes
U8_FILL = 0xA5


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _window(shape, dtype):
    torch = _torch()
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    if dtype == torch.float32:
        buf.view(torch.int32).fill_(F32_FILL)
    else:
        buf.fill_(U8_FILL)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _margins_intact(buf, n):
    torch = _torch()
    raw = buf.view(torch.int32) if buf.dtype == torch.float32 else buf
    fill = F32_FILL if buf.dtype == torch.float32 else U8_FILL
    return bool(torch.all(raw[:GUARD] == fill).item()) and bool(torch.all(raw[GUARD + n:] == fill).item())


@pytest.mark.parametrize("c,b,n,B,dtype,method,pattern,nm", [
    (70, 256, 300, 128, "fp32", "thanos", "unstructured", (0, 0)),      # tensor-core update
    (37, 200, 300, 48, "bf16", "thanos", "nm", (2, 4)),                 # ragged last block
    (24, 150, 200, 32, "fp32", "sparsegpt", "unstructured", (0, 0)),    # CUDA-core fallbacks
    (40, 128, 256, 64, "bf16", "sparsegpt", "nm", (4, 8)),
    (33, 96, 64, 128, "bf16", "wanda", "unstructured", (0, 0)),
    (9, 64, 16, 128, "fp32", "magnitude", "nm", (2, 4)),
])
def test_writes_stay_inside_the_buffers(c, b, n, B, dtype, method, pattern, nm):
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    wl = synth.custom(c, b, n, dtype=dtype, outlier_frac=0.02, outlier_scale=20.0, block=B, seed=c * b)
    Wt, Xt = P.torch_inputs(synth.make_W(wl), synth.make_X_tokens(wl), dtype)
    kw = dict(method=method, pattern=pattern, nm=nm, sparsity=0.5, block=B, damp=0.01)
    second_order = method in ("thanos", "sparsegpt")

    ref_H = torch.empty((b, b), dtype=torch.float32, device="cuda") if second_order else None
    W_ref, m_ref, _ = pwp.prune_layer(Wt, X=Xt, H=ref_H, **kw)

    Wb, W_out = _window((c, b), torch.float32)
    Mb, mask = _window((c, b), torch.uint8)
    Hb, H = _window((b, b), torch.float32) if second_order else (None, None)
    nws = pwp.workspace_bytes(pwp.config(**kw), c, b)
    Sb, ws_t = _window((nws,), torch.uint8)
    nst = ctypes.sizeof(pwp.Stats)
    Tb, stats = _window((nst,), torch.uint8)
    stats.zero_()
    W_hat, m, st = pwp.prune_layer(Wt, X=Xt, H=H, W_out=W_out, mask=mask, workspace=pwp.Workspace(ws_t, nws),
                                   stats=stats, **kw)
    torch.cuda.synchronize()
    assert st.status == 0
    assert _margins_intact(Wb, c * b) and _margins_intact(Mb, c * b)
    assert _margins_intact(Sb, nws) and _margins_intact(Tb, nst)
    if second_order:
        assert _margins_intact(Hb, b * b)
    assert torch.equal(W_hat.view(torch.int32), W_ref.view(torch.int32))
    assert torch.equal(m, m_ref)


def test_hessian_writes_only_h():
    torch = _torch()
    import post_weight_pruning_b200 as pwp
    for dtype, b, n in (("bf16", 200, 700), ("fp32", 130, 90)):
        wl = synth.custom(4, b, n, dtype=dtype, seed=b)
        _, Xt = P.torch_inputs(synth.make_W(wl), synth.make_X_tokens(wl), dtype)
        Hb, H = _window((b, b), torch.float32)
        pwp.hessian_accumulate(Xt, H)
        torch.cuda.synchronize()
        assert _margins_intact(Hb, b * b)
        assert torch.equal(H, pwp.hessian_accumulate(Xt))
