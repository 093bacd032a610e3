"""C-ABI checks that need no GPU: the library loads, exports every entry point that
include/pwp.h declares, and rejects bad arguments on the host before launching."""
import ctypes
import os
import re

import pytest

import post_weight_pruning_b200 as pwp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pwp_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = pwp.lib()
    names = _declared()
    assert {"pwp_prune_layer", "pwp_prune_layer_x", "pwp_hessian_accumulate",
            "pwp_workspace_bytes", "pwp_status_string"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for s in range(7):
        assert pwp.status_string(s)
    assert pwp.status_string(99) == "unknown status"


@pytest.mark.parametrize("kw", [
    dict(sparsity=1.0), dict(sparsity=-0.1), dict(block=0), dict(block=129),
    dict(pattern="nm", nm=(2, 3)), dict(pattern="nm", nm=(4, 4)), dict(pattern="nm", nm=(0, 4)),
    dict(pattern="nm", nm=(2, 4), block=6), dict(damp=-1.0), dict(method=7), dict(alpha=1.0), dict(alpha=-0.1),
    dict(method="wanda", alpha=0.1),
])
def test_invalid_configs_have_no_workspace(kw):
    cfg = pwp.config(**kw)
    assert pwp.workspace_bytes(cfg, 64, 64) == 0


def test_workspace_grows_with_shape_and_is_256_aligned():
    cfg = pwp.config(block=128)
    a = pwp.workspace_bytes(cfg, 128, 256)
    b = pwp.workspace_bytes(cfg, 4096, 4096)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    assert pwp.workspace_bytes(pwp.config(pattern="nm", nm=(2, 4)), 64, 66) == 0   # b % m != 0


def test_argument_errors_return_before_any_launch():
    L = pwp.lib()
    cfg = pwp.config()
    vp = ctypes.c_void_p
    # null pointers -> EINVAL
    assert L.pwp_prune_layer(ctypes.byref(cfg), None, 0, 16, 16, None, None, None, None, 0, None, None) == 1
    # too-small workspace -> EWORKSPACE (pointers are never dereferenced on the host)
    fake = vp(1 << 20)
    assert L.pwp_prune_layer(ctypes.byref(cfg), fake, 0, 16, 16, fake, fake, fake, fake, 10, fake, None) == 3
    # misaligned workspace
    n = pwp.workspace_bytes(cfg, 16, 16)
    assert L.pwp_prune_layer(ctypes.byref(cfg), fake, 0, 16, 16, fake, fake, fake, vp((1 << 20) + 8), n,
                             fake, None) == 3
    # bad dtype / beta / shape
    assert L.pwp_hessian_accumulate(fake, 7, 10, 16, fake, 0, None) == 1
    assert L.pwp_hessian_accumulate(fake, 0, 10, 16, fake, 2, None) == 1
    assert L.pwp_hessian_accumulate(fake, 0, 10, 0, fake, 0, None) == 1
    assert L.pwp_damp_factor(fake, 16, 0.01, fake, None, 0, fake, None) == 3
    assert L.pwp_prune_layer_x(ctypes.byref(cfg), fake, 0, 16, 16, fake, 0, -1, fake, fake, fake, fake, n,
                               fake, None) == 1
    # the host entry point: null host buffers, a negative n, then a short workspace
    a = [fake] * 8
    assert L.pwp_prune_layer_host(ctypes.byref(cfg), None, 0, 16, 16, fake, 0, 10, *a[:7], fake, n, fake,
                                  None) == 1
    assert L.pwp_prune_layer_host(ctypes.byref(cfg), fake, 0, 16, 16, fake, 0, -1, *a[:7], fake, n, fake,
                                  None) == 1
    assert L.pwp_prune_layer_host(ctypes.byref(cfg), fake, 0, 16, 16, fake, 0, 10, *a[:7], fake, 10, fake,
                                  None) == 3
    # the multi-layer host entry point: null arrays, a negative count, then short device scratch
    arr = (vp * 2)(fake, fake)
    nb = L.pwp_layers_host_bytes(ctypes.byref(cfg), 16, 16, 10, 0, 0)
    assert nb > 0 and nb % 256 == 0
    assert L.pwp_prune_layers_host(ctypes.byref(cfg), 2, None, 0, 16, 16, arr, 0, 10, arr, arr, fake, nb, fake,
                                   None) == 1
    assert L.pwp_prune_layers_host(ctypes.byref(cfg), -1, arr, 0, 16, 16, arr, 0, 10, arr, arr, fake, nb, fake,
                                   None) == 1
    assert L.pwp_prune_layers_host(ctypes.byref(cfg), 2, arr, 0, 16, 16, arr, 0, 10, arr, arr, fake, nb - 256, fake,
                                   None) == 3
    assert L.pwp_layers_host_bytes(ctypes.byref(cfg), 16, 16, -1, 0, 0) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(pwp, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(pwp, "_lib", None)
    with pytest.raises(ImportError):
        pwp.lib()


def test_no_update_methods_validation():
    """Wanda and magnitude ignore block and damp, still check the pattern, and take H only
    where they need it (magnitude never; Wanda through pwp_prune_layer)."""
    L = pwp.lib()
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    for method in ("wanda", "magnitude"):
        cfg = pwp.config(method=method, block=1000, damp=-1.0)          # ignored fields
        n = pwp.workspace_bytes(cfg, 16, 64)
        assert n > 0 and n % 256 == 0
        assert pwp.workspace_bytes(pwp.config(method=method, pattern="nm", nm=(2, 4)), 16, 66) == 0
        assert pwp.workspace_bytes(pwp.config(method=method, sparsity=1.0), 16, 64) == 0
        # too-small workspace still wins over everything after the argument checks
        assert L.pwp_prune_layer(ctypes.byref(cfg), fake, 0, 16, 64, fake, fake, fake, fake, 10, fake, None) == 3
    # Wanda through pwp_prune_layer needs H; magnitude does not (it fails on the workspace)
    cfg = pwp.config(method="wanda")
    assert L.pwp_prune_layer(ctypes.byref(cfg), fake, 0, 16, 64, None, fake, fake, fake, 10, fake, None) == 1
    cfg = pwp.config(method="magnitude")
    assert L.pwp_prune_layer(ctypes.byref(cfg), fake, 0, 16, 64, None, fake, fake, fake, 10, fake, None) == 3
    bad = pwp.config(method=4)
    assert pwp.workspace_bytes(bad, 16, 64) == 0


def test_pack24_argument_errors():
    L = pwp.lib()
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    assert L.pwp_pack_24(None, fake, 4, 8, fake, fake, fake, None) == 1
    assert L.pwp_pack_24(fake, fake, 4, 6, fake, fake, fake, None) == 1            # b % 4 != 0
    assert L.pwp_pack_24(fake, fake, 0, 8, fake, fake, fake, None) == 1            # c < 1
    assert L.pwp_pack_24(vp((1 << 20) + 4), fake, 4, 8, fake, fake, fake, None) == 1   # W-hat not 16-byte aligned
    assert L.pwp_pack_24(fake, vp((1 << 20) + 2), 4, 8, fake, fake, fake, None) == 1   # mask not 4-byte aligned


@pytest.mark.parametrize("c,b,B,method,mib", [
    (4096, 4096, 128, "thanos", 281.8), (4096, 4096, 128, "sparsegpt", 109.1), (4096, 4096, 128, "wanda", 1.0),
    (4096, 4096, 128, "magnitude", 1.0), (256, 512, 128, "thanos", 10.2), (1024, 1024, 64, "thanos", 12.6),
    (1024, 1024, 128, "thanos", 33.5),
])
def test_workspace_sizes_match_the_documented_figures(c, b, B, method, mib):
    import post_weight_pruning_b200 as pwp
    n = pwp.workspace_bytes(pwp.config(method=method, block=B), c, b)
    assert round(n / 2**20, 1) == mib
    # the no-workspace entry point takes every shape whose workspace fits its 16 MiB array
    assert (n <= 16 * 2**20) == (mib <= 16.0)


def test_wait_limit_setter_returns_the_previous_limit_and_restores_the_default():
    default = 1 << 26
    assert pwp.set_wait_limit(-1) == default          # untouched so far in this process
    assert pwp.set_wait_limit(0) == default
    assert pwp.set_wait_limit(12345) == 0
    assert pwp.set_wait_limit(-5) == 12345
    assert pwp.set_wait_limit(-1) == default


def test_alpha_workspace_holds_the_compact_layer():
    """With alpha > 0 the workspace holds the prune of the c - floor(alpha c) kept rows plus
    their compact copy (fp32 weights and mask) and the per-row scores, flags and positions."""
    base = pwp.workspace_bytes(pwp.config(block=32), 36, 64)
    got = pwp.workspace_bytes(pwp.config(block=32, alpha=0.1), 40, 64)   # floor(4.0) = 4 outlier rows
    al = lambda x: (x + 255) // 256 * 256
    assert got == al(base) + al(36 * 64 * 4) + al(36 * 64) + al(40 * 8) + 2 * al(40 * 4)
    # alpha too small to keep a row: the plain workspace
    assert pwp.workspace_bytes(pwp.config(block=32, alpha=0.01), 40, 64) == pwp.workspace_bytes(pwp.config(block=32), 40, 64)
