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


class _FakeLib:
    """Stands in for libpwp.so so that the marshalling runs on the CPU: records the
    arguments of each entry point and reports success."""

    def __init__(self, ws_bytes=4096):
        self.ws_bytes = ws_bytes
        self.calls = {}
        self.log = []

    def pwp_workspace_bytes(self, cfg, c, b):
        return self.ws_bytes

    def _record(name):
        def f(self, *a):
            self.calls[name] = a
            self.log.append((name, a))
            return 0
        return f

    pwp_prune_layer = _record("pwp_prune_layer")
    pwp_prune_layer_x = _record("pwp_prune_layer_x")
    pwp_pack_24 = _record("pwp_pack_24")
    pwp_hessian_accumulate = _record("pwp_hessian_accumulate")


@pytest.fixture
def fake(monkeypatch):
    import ctypes
    f = _FakeLib()
    monkeypatch.setattr(pwp, "lib", lambda: f)
    monkeypatch.setattr(pwp, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(pwp, "_stream_ptr", lambda stream=None: ctypes.c_void_p(0))
    return f


def _ptr(v):
    return v.value if hasattr(v, "value") else v


def test_prune_layer_x_marshalling(fake):
    c, b, n = 6, 32, 40
    W = torch.zeros(c, b, dtype=torch.bfloat16)
    X = torch.zeros(n, b, dtype=torch.float32)
    W_hat, mask, st = pwp.prune_layer(W, X=X, method="thanos", pattern="nm", nm=(2, 4), block=16, damp=0.05)
    a = fake.calls["pwp_prune_layer_x"]
    cfg = a[0]._obj
    assert (cfg.method, cfg.pattern, cfg.nm_n, cfg.nm_m, cfg.block) == (pwp.THANOS, pwp.NM, 2, 4, 16)
    assert cfg.damp == pytest.approx(0.05)
    assert _ptr(a[1]) == W.data_ptr() and a[2] == pwp.BF16 and (a[3], a[4]) == (c, b)
    assert _ptr(a[5]) == X.data_ptr() and a[6] == pwp.FP32 and a[7] == n
    assert _ptr(a[8]) not in (None, 0)                      # an H scratch was allocated
    assert _ptr(a[9]) == W_hat.data_ptr() and _ptr(a[10]) == mask.data_ptr()
    assert a[12] == fake.ws_bytes
    assert W_hat.shape == (c, b) and W_hat.dtype == torch.float32
    assert mask.shape == (c, b) and mask.dtype == torch.uint8
    assert st.status == 0


def test_prune_layer_no_update_passes_no_h(fake):
    W = torch.zeros(4, 16, dtype=torch.float32)
    X = torch.zeros(8, 16, dtype=torch.bfloat16)
    pwp.prune_layer(W, X=X, method="wanda", sparsity=0.25)
    a = fake.calls["pwp_prune_layer_x"]
    assert a[0]._obj.method == pwp.WANDA
    assert _ptr(a[8]) in (None, 0)
    pwp.prune_layer(W, method="magnitude", check=False)
    a = fake.calls["pwp_prune_layer"]
    assert a[0]._obj.method == pwp.MAGNITUDE and _ptr(a[5]) in (None, 0)


def test_prune_layer_with_h_and_caller_buffers(fake):
    c, b = 5, 24
    W = torch.zeros(c, b)
    H = torch.zeros(b, b)
    W_out = torch.zeros(c, b)
    mask = torch.zeros(c, b, dtype=torch.uint8)
    ws = pwp.Workspace(torch.zeros(4096, dtype=torch.uint8), 4096)
    stats = pwp.new_stats("cpu")
    r = pwp.prune_layer(W, H=H, W_out=W_out, mask=mask, workspace=ws, stats=stats, check=False)
    assert r[0] is W_out and r[1] is mask and r[2] is stats
    a = fake.calls["pwp_prune_layer"]
    assert _ptr(a[5]) == H.data_ptr() and _ptr(a[8]) == ws.ws.data_ptr() and a[9] == 4096
    assert _ptr(a[10]) == stats.data_ptr()


def test_pack_24_marshalling(fake):
    c, b = 3, 100
    values, meta, st = pwp.pack_24(torch.zeros(c, b), torch.zeros(c, b, dtype=torch.uint8))
    a = fake.calls["pwp_pack_24"]
    assert (a[2], a[3]) == (c, b)
    assert values.shape == (c, b // 2) and values.dtype == torch.int16
    assert meta.shape == (c, 4) and meta.dtype == torch.int32        # ceil(25 groups / 8)
    assert _ptr(a[4]) == values.data_ptr() and _ptr(a[5]) == meta.data_ptr()


def test_prune_block_builds_one_h_per_input(fake):
    b1, b2, n = 16, 24, 32
    weights = {"q": torch.zeros(8, b1), "k": torch.zeros(4, b1), "o": torch.zeros(6, b1),
               "down": torch.zeros(5, b2)}
    acts = {"attn_in": torch.zeros(n, b1, dtype=torch.bfloat16), "o_in": torch.zeros(n, b1),
            "down_in": torch.zeros(n, b2, dtype=torch.bfloat16)}
    feeds = {"q": "attn_in", "k": "attn_in", "o": "o_in", "down": "down_in"}
    out = pwp.prune_block(weights, acts, feeds, method="thanos", sparsity=0.5, block=8)
    assert set(out) == set(weights)
    hess = [a for name, a in fake.log if name == "pwp_hessian_accumulate"]
    prunes = [a for name, a in fake.log if name == "pwp_prune_layer"]
    assert [_ptr(a[0]) for a in hess] == [acts[k].data_ptr() for k in ("attn_in", "o_in", "down_in")]
    assert [(a[3], a[4]) for a in prunes] == [(8, b1), (4, b1), (6, b1), (5, b2)]
    h_ptr = [_ptr(a[4]) for a in hess]                  # where each H was built
    # q gets a copy of the attention input's H, k (its last reader) the H itself
    assert _ptr(prunes[0][5]) != h_ptr[0] and _ptr(prunes[1][5]) == h_ptr[0]
    assert _ptr(prunes[2][5]) == h_ptr[1] and _ptr(prunes[3][5]) == h_ptr[2]


def test_prune_block_wanda_needs_no_h(fake):
    weights = {"gate": torch.zeros(8, 16), "up": torch.zeros(8, 16)}
    acts = {"mlp_in": torch.zeros(32, 16, dtype=torch.bfloat16)}
    pwp.prune_block(weights, acts, {"gate": "mlp_in", "up": "mlp_in"}, method="wanda")
    assert not [1 for name, _ in fake.log if name == "pwp_hessian_accumulate"]
    xs = [a for name, a in fake.log if name == "pwp_prune_layer_x"]
    assert len(xs) == 2 and all(_ptr(a[5]) == acts["mlp_in"].data_ptr() for a in xs)


def test_prune_block_checks_its_wiring(fake):
    with pytest.raises(ValueError, match="no input"):
        pwp.prune_block({"q": torch.zeros(4, 16)}, {"attn_in": torch.zeros(8, 16)}, {})
    with pytest.raises(ValueError, match="does not match"):
        pwp.prune_block({"q": torch.zeros(4, 16)}, {"a": torch.zeros(8, 12)}, {"q": "a"})


class _StreamCtx:
    """Stands in for torch.cuda.stream(s): records which stream is current."""
    current = []

    def __init__(self, s):
        self.s = s

    def __enter__(self):
        _StreamCtx.current.append(self.s)

    def __exit__(self, *exc):
        _StreamCtx.current.pop()


@pytest.fixture
def fake_streams(fake, monkeypatch):
    """The fake library, each entry point also noting the current stream at its call."""
    monkeypatch.setattr(pwp, "_stream_ctx", _StreamCtx)
    seen = []
    for name in ("pwp_prune_layer", "pwp_prune_layer_x", "pwp_pack_24", "pwp_hessian_accumulate"):
        inner = getattr(fake, name)

        def f(*a, _inner=inner, _name=name):
            seen.append((_name, _StreamCtx.current[-1] if _StreamCtx.current else None))
            return _inner(*a)
        monkeypatch.setattr(fake, name, f)
    return seen


def test_calls_given_a_stream_run_with_it_current(fake_streams):
    """With a caller's stream, the call's allocations, copies and host reads happen with that
    stream current (positional or keyword); without one, nothing changes torch's stream."""
    s = object()
    W = torch.zeros(4, 16)
    X = torch.zeros(8, 16, dtype=torch.bfloat16)
    pwp.prune_layer(W, X=X, stream=s)
    pwp.hessian_accumulate(X, None, 0, s)
    pwp.pack_24(torch.zeros(2, 8), torch.zeros(2, 8, dtype=torch.uint8), stream=s)
    pwp.prune_block({"q": W}, {"a": X}, {"q": "a"}, stream=s, method="thanos")
    assert [x[1] for x in fake_streams] == [s] * len(fake_streams) and len(fake_streams) == 5
    fake_streams.clear()
    pwp.prune_layer(W, X=X)
    pwp.hessian_accumulate(X)
    assert [x[1] for x in fake_streams] == [None, None]
    assert not _StreamCtx.current
