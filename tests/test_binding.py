"""Argument checks of the Python binding (CPU): the kernels see only pointers and the
sizes passed beside them, so a tensor of the wrong shape, element type or device must be
refused before any call into the library."""
import pytest

torch = pytest.importorskip("torch")

import post_weight_pruning_b200 as pwp  # noqa: E402


def _prune(**kw):
    W = kw.pop("W", torch.zeros(8, 16, dtype=torch.bfloat16))
    return pwp.prune_layer(W, **kw)


@pytest.mark.parametrize("kw, err", [
    (dict(H=torch.zeros(16, 8)), ValueError),                         # H not [b, b]
    (dict(H=torch.zeros(16, 16, dtype=torch.float64)), TypeError),    # H not fp32
    (dict(H=torch.zeros(16, 16, dtype=torch.bfloat16)), TypeError),
    (dict(X=torch.zeros(32, 12, dtype=torch.bfloat16)), ValueError),  # X width != b
    (dict(X=torch.zeros(32, 16, dtype=torch.float16)), TypeError),    # X element type
    (dict(X=torch.zeros(32, 16, 1)), ValueError),                     # X not 2-D
    (dict(H=torch.zeros(16, 16), W_out=torch.zeros(8, 16, dtype=torch.bfloat16)), TypeError),
    (dict(H=torch.zeros(16, 16), W_out=torch.zeros(16, 8)), ValueError),
    (dict(H=torch.zeros(16, 16), mask=torch.zeros(8, 16, dtype=torch.bool)), TypeError),
    (dict(H=torch.zeros(16, 16), mask=torch.zeros(8, 8, dtype=torch.uint8)), ValueError),
    (dict(H=torch.zeros(16, 16), stats=torch.zeros(8, dtype=torch.uint8)), ValueError),
    (dict(W=torch.zeros(8, 16, dtype=torch.int8), H=torch.zeros(16, 16)), TypeError),
    (dict(W=torch.zeros(8, 16, 2), H=torch.zeros(16, 16)), ValueError),
])
def test_prune_layer_refuses_mismatched_buffers(kw, err):
    with pytest.raises(err):
        _prune(**kw)


def test_prune_layer_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        _prune(H=torch.zeros(16, 16))


def test_prune_layer_refuses_short_workspace_claim():
    ws = pwp.Workspace(torch.zeros(64, dtype=torch.uint8), 65)
    with pytest.raises(ValueError, match="workspace"):
        _prune(H=torch.zeros(16, 16), workspace=ws)


def test_hessian_and_factor_refuse_mismatched_buffers():
    with pytest.raises(ValueError):
        pwp.hessian_accumulate(torch.zeros(32, 16, dtype=torch.bfloat16), H=torch.zeros(16, 15))
    with pytest.raises(TypeError):
        pwp.hessian_accumulate(torch.zeros(32, 16, dtype=torch.float16))
    with pytest.raises(ValueError):
        pwp.damp_factor(torch.zeros(16, 15))
    with pytest.raises(TypeError):
        pwp.damp_factor(torch.zeros(16, 16, dtype=torch.float64))


def test_pack_24_refuses_mismatched_buffers():
    with pytest.raises(TypeError):
        pwp.pack_24(torch.zeros(4, 8, dtype=torch.bfloat16), torch.zeros(4, 8, dtype=torch.uint8))
    with pytest.raises(ValueError):
        pwp.pack_24(torch.zeros(4, 8), torch.zeros(4, 4, dtype=torch.uint8))
    with pytest.raises(TypeError):
        pwp.pack_24(torch.zeros(4, 8), torch.zeros(4, 8, dtype=torch.bool))
