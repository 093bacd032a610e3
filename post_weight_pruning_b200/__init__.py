"""Python binding of libpwp (B200 layer-reconstruction pruning).

Argument marshalling only: every step of the prune runs in the CUDA kernels of
libpwp.so, reached through its C ABI (include/pwp.h).  PyTorch provides device
memory and the current stream.  There is no CPU fallback: if the library is
missing, loading it raises.

Names mirror the C entry points: ``hessian_accumulate``, ``damp_factor``,
``prune_layer`` (H given or built from X), ``workspace_bytes``, plus
``prune_layer_host`` for a call that starts and ends in host memory.
"""
from __future__ import annotations

import ctypes
import functools
import inspect
import os
from dataclasses import dataclass

import numpy as np

__all__ = [
    "lib", "Config", "Stats", "THANOS", "SPARSEGPT", "WANDA", "MAGNITUDE", "UNSTRUCTURED", "NM", "BF16", "FP32",
    "PwpError", "config", "workspace_bytes", "hessian_accumulate", "damp_factor", "prune_layer",
    "prune_layer_host", "prune_block", "pack_24", "status_string", "set_wait_limit", "Sweep", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpwp.so")

THANOS, SPARSEGPT, WANDA, MAGNITUDE = 0, 1, 2, 3
METHODS = {"thanos": THANOS, "sparsegpt": SPARSEGPT, "wanda": WANDA, "magnitude": MAGNITUDE}
UNSTRUCTURED, NM = 0, 1
BF16, FP32 = 0, 1


class Config(ctypes.Structure):
    _fields_ = [("method", ctypes.c_int32), ("pattern", ctypes.c_int32), ("nm_n", ctypes.c_int32),
                ("nm_m", ctypes.c_int32), ("sparsity", ctypes.c_float), ("block", ctypes.c_int32),
                ("damp", ctypes.c_float), ("alpha", ctypes.c_float)]


class Stats(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int32), ("status_site", ctypes.c_int32),
                ("pruned", ctypes.c_int64), ("target", ctypes.c_int64), ("lam", ctypes.c_float),
                ("shortfall", ctypes.c_int32), ("reread_blocks", ctypes.c_int32),
                ("tie_blocks", ctypes.c_int32), ("reserved", ctypes.c_int32 * 4)]


class SweepArgs(ctypes.Structure):
    _fields_ = [("cfg", ctypes.POINTER(Config)), ("W", ctypes.c_void_p), ("wtype", ctypes.c_int32),
                ("c", ctypes.c_int32), ("b", ctypes.c_int32), ("c_total", ctypes.c_int64), ("H", ctypes.c_void_p),
                ("W_out", ctypes.c_void_p), ("mask", ctypes.c_void_p), ("ws", ctypes.c_void_p),
                ("ws_bytes", ctypes.c_size_t), ("stats", ctypes.c_void_p), ("ties_all", ctypes.c_void_p),
                ("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("stream", ctypes.c_void_p)]


class PwpError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None
_vp, _sz, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_SIGS = {
    "pwp_workspace_bytes": (_sz, [ctypes.POINTER(Config), _i32, _i32]),
    "pwp_factor_workspace_bytes": (_sz, [_i32]),
    "pwp_hessian_accumulate": (_i32, [_vp, _i32, _i64, _i32, _vp, _i32, _vp]),
    "pwp_damp_factor": (_i32, [_vp, _i32, _f32, _vp, _vp, _sz, _vp, _vp]),
    "pwp_prune_layer": (_i32, [ctypes.POINTER(Config), _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz,
                               _vp, _vp]),
    "pwp_prune_layer_x": (_i32, [ctypes.POINTER(Config), _vp, _i32, _i32, _i32, _vp, _i32, _i64, _vp,
                                 _vp, _vp, _vp, _sz, _vp, _vp]),
    "pwp_prune_layer_host": (_i32, [ctypes.POINTER(Config), _vp, _i32, _i32, _i32, _vp, _i32, _i64, _vp, _vp,
                                    _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "pwp_layers_host_bytes": (_sz, [ctypes.POINTER(Config), _i32, _i32, _i64, _i32, _i32]),
    "pwp_prune_layers_host": (_i32, [ctypes.POINTER(Config), _i32, _vp, _i32, _i32, _i32, _vp, _i32, _i64, _vp,
                                     _vp, _vp, _sz, _vp, _vp]),
    "pwp_pack_24": (_i32, [_vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "pwp_status_string": (ctypes.c_char_p, [_i32]),
    "pwp_sweep_step": (_i32, [ctypes.POINTER(SweepArgs), _i32, _i32]),
    "pwp_sweep_buffers": (_i32, [ctypes.POINTER(SweepArgs), ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(_i64),
                                 ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(_i64),
                                 ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(_i64)]),
    "pwp_set_wait_limit": (_i64, [_i64]),
    "pwp_version": (_i32, []),
}


def lib():
    """Load libpwp.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libpwp.so not built ({LIB_PATH}); run python -m post_weight_pruning_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s) -> str:
    return lib().pwp_status_string(int(s)).decode()


def set_wait_limit(polls: int) -> int:
    """Polls every bounded device-side wait of the tensor-core kernels makes before it
    gives up with PWP_ETIMEOUT (negative: the default, 2^26).  Returns the previous limit."""
    return int(lib().pwp_set_wait_limit(int(polls)))


def _check(status, where):
    if status != 0:
        raise PwpError(status, where)


def config(method="thanos", pattern="unstructured", nm=(2, 4), sparsity=0.5, block=128, damp=0.01,
           alpha=0.0) -> Config:
    m = METHODS[method] if isinstance(method, str) else int(method)
    if isinstance(pattern, str):
        p = {"unstructured": UNSTRUCTURED, "nm": NM}[pattern]
    else:
        p = int(pattern)
    n_keep, m_grp = nm if p == NM else (0, 0)
    return Config(m, p, int(n_keep), int(m_grp), float(sparsity), int(block), float(damp), float(alpha))


def workspace_bytes(cfg: Config, c: int, b: int) -> int:
    return int(lib().pwp_workspace_bytes(ctypes.byref(cfg), int(c), int(b)))


# ------------------------------------------------------------------- torch helpers

def _torch():
    import torch
    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _stream_ctx(stream):
    return _torch().cuda.stream(stream)


def _on_stream(fn):
    """Run a binding call with the caller's stream, when one is given, as torch's current
    stream: the device memory the call allocates then belongs to that stream (the caching
    allocator hands it out again only in that stream's order, after the call's kernels),
    and the call's own copies and host reads of results are ordered after its kernels."""
    params = list(inspect.signature(fn).parameters.values())
    # where a positional stream argument would sit (None: keyword-only)
    pos = next((i for i, p in enumerate(params) if p.name == "stream" and p.kind == p.POSITIONAL_OR_KEYWORD), None)

    @functools.wraps(fn)
    def wrapped(*a, **kw):
        stream = kw.get("stream")
        if stream is None and pos is not None and len(a) > pos:
            stream = a[pos]
        if stream is None:
            return fn(*a, **kw)
        with _stream_ctx(stream):
            return fn(*a, **kw)
    return wrapped


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if dev is not None and t.device != dev:
            raise ValueError(f"tensors on different devices ({dev}, {t.device})")
        dev = t.device


def _expect(t, name, shape, dtypes):
    """The kernels see only a pointer and the sizes passed beside it, so a tensor whose
    shape or element type differs from them would be read or written out of bounds:
    reject it here."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {[str(d) for d in dtypes]}")


def new_stats(device="cuda"):
    torch = _torch()
    return torch.zeros(ctypes.sizeof(Stats), dtype=torch.uint8, device=device)


def read_stats(stats_t) -> Stats:
    raw = stats_t.cpu().numpy().tobytes()
    return Stats.from_buffer_copy(raw)


@_on_stream
def hessian_accumulate(X, H=None, beta=0, stream=None):
    """H := beta*H + 2 X X^T for token-major X ([n, b], bf16 or fp32 CUDA tensor)."""
    torch = _torch()
    if X.dim() != 2:
        raise ValueError(f"X: expected [n, b], got shape {tuple(X.shape)}")
    n, b = X.shape
    _expect(X, "X", (n, b), (torch.bfloat16, torch.float32))
    _expect(H, "H", (b, b), (torch.float32,))
    _need_cuda(X, H)
    if H is None:
        H = torch.empty((b, b), dtype=torch.float32, device=X.device)
    st = lib().pwp_hessian_accumulate(_vp(X.data_ptr()), _dtype_code(X), int(n), int(b), _vp(H.data_ptr()),
                                      int(beta), _stream_ptr(stream))
    _check(st, "pwp_hessian_accumulate")
    return H


@_on_stream
def damp_factor(H, damp=0.01, stream=None):
    """In place: upper triangle of H becomes U with (H + lambda I)^-1 = U^T U.
    Returns (g_diag, stats tensor)."""
    torch = _torch()
    b = H.shape[0]
    _expect(H, "H", (b, b), (torch.float32,))
    _need_cuda(H)
    g = torch.empty(b, dtype=torch.float32, device=H.device)
    nws = int(lib().pwp_factor_workspace_bytes(int(b)))
    ws = torch.empty(nws, dtype=torch.uint8, device=H.device)
    stats = new_stats(H.device)
    st = lib().pwp_damp_factor(_vp(H.data_ptr()), int(b), float(damp), _vp(g.data_ptr()), _vp(ws.data_ptr()),
                               nws, _vp(stats.data_ptr()), _stream_ptr(stream))
    _check(st, "pwp_damp_factor")
    return g, stats


@dataclass
class Workspace:
    ws: object
    nbytes: int


def make_workspace(cfg: Config, c, b, device="cuda") -> Workspace:
    torch = _torch()
    n = workspace_bytes(cfg, c, b)
    if n == 0:
        raise PwpError(1, "pwp_workspace_bytes")
    return Workspace(torch.empty(n, dtype=torch.uint8, device=device), n)


@_on_stream
def prune_layer(W, *, H=None, X=None, sparsity=0.5, pattern="unstructured", nm=(2, 4), block=128,
                damp=0.01, method="thanos", alpha=0.0, W_out=None, mask=None, workspace=None, stats=None,
                stream=None, check=True):
    """Prune one layer on the GPU.

    W: [c, b] bf16/fp32 CUDA tensor.  Give either H (undamped 2XX^T, fp32 [b, b],
    DESTROYED by thanos/sparsegpt: holds U afterwards; wanda reads its diagonal) or X
    (token-major [n, b] activations; for thanos/sparsegpt an H scratch is allocated
    unless H is also passed).  method "magnitude" needs neither.  Returns (W_hat fp32,
    mask uint8, Stats) -- with check=False the stats tensor is returned unread and
    nothing syncs."""
    torch = _torch()
    if W.dim() != 2:
        raise ValueError(f"W: expected [c, b], got shape {tuple(W.shape)}")
    c, b = W.shape
    _expect(W, "W", (c, b), (torch.bfloat16, torch.float32))
    _expect(H, "H", (b, b), (torch.float32,))
    if X is not None:
        if X.dim() != 2:
            raise ValueError(f"X: expected [n, b], got shape {tuple(X.shape)}")
        _expect(X, "X", (X.shape[0], b), (torch.bfloat16, torch.float32))
    _expect(W_out, "W_out", (c, b), (torch.float32,))
    _expect(mask, "mask", (c, b), (torch.uint8,))
    _expect(stats, "stats", (ctypes.sizeof(Stats),), (torch.uint8,))
    if workspace is not None and workspace.nbytes > workspace.ws.numel() * workspace.ws.element_size():
        raise ValueError(f"workspace: {workspace.nbytes} bytes claimed, tensor holds "
                         f"{workspace.ws.numel() * workspace.ws.element_size()}")
    _need_cuda(W, H, X, W_out, mask, stats, workspace.ws if workspace is not None else None)
    cfg = config(method, pattern, nm, sparsity, block, damp, alpha)
    if workspace is None:
        workspace = make_workspace(cfg, c, b, W.device)
    if W_out is None:
        W_out = torch.empty((c, b), dtype=torch.float32, device=W.device)
    if mask is None:
        mask = torch.empty((c, b), dtype=torch.uint8, device=W.device)
    if stats is None:
        stats = new_stats(W.device)
    L = lib()
    no_update = cfg.method in (WANDA, MAGNITUDE)
    if X is not None:
        if H is None and not no_update:
            H = torch.empty((b, b), dtype=torch.float32, device=W.device)
        st = L.pwp_prune_layer_x(ctypes.byref(cfg), _vp(W.data_ptr()), _dtype_code(W), int(c), int(b),
                                 _vp(X.data_ptr()), _dtype_code(X), int(X.shape[0]),
                                 _vp(H.data_ptr() if H is not None else 0),
                                 _vp(W_out.data_ptr()), _vp(mask.data_ptr()), _vp(workspace.ws.data_ptr()),
                                 workspace.nbytes, _vp(stats.data_ptr()), _stream_ptr(stream))
        where = "pwp_prune_layer_x"
    else:
        if H is None and cfg.method != MAGNITUDE:
            raise ValueError("give H or X")
        st = L.pwp_prune_layer(ctypes.byref(cfg), _vp(W.data_ptr()), _dtype_code(W), int(c), int(b),
                               _vp(H.data_ptr() if H is not None else 0), _vp(W_out.data_ptr()),
                               _vp(mask.data_ptr()),
                               _vp(workspace.ws.data_ptr()), workspace.nbytes, _vp(stats.data_ptr()),
                               _stream_ptr(stream))
        where = "pwp_prune_layer"
    _check(st, where)
    if not check:
        return W_out, mask, stats
    s = read_stats(stats)
    if s.status != 0:
        raise PwpError(s.status, where + " (device)")
    return W_out, mask, s


@_on_stream
def prune_block(weights, activations, feeds, *, stream=None, check=True, **cfg):
    """Prune the linear layers of one transformer block.  Thanos / SparseGPT: one H per
    distinct input, built once on the tensor cores and shared by every layer that reads
    that input (q, k and v read the attention input; gate and up the MLP input).  Wanda /
    magnitude: no H.

    weights: {layer: W [c, b]}; activations: {input: X [n, b]} (token-major);
    feeds: {layer: input}; cfg: as for ``prune_layer`` (method, pattern, sparsity, ...).
    Returns {layer: (W_hat, mask, Stats)} (the unread stats tensor with check=False)."""
    for layer, W in weights.items():
        if layer not in feeds or feeds[layer] not in activations:
            raise ValueError(f"layer {layer!r}: no input given")
        if W.dim() != 2 or activations[feeds[layer]].shape[-1] != W.shape[1]:
            raise ValueError(f"layer {layer!r}: W {tuple(W.shape)} does not match its input "
                             f"{tuple(activations[feeds[layer]].shape)}")
    method = cfg.get("method", "thanos")
    m = METHODS[method] if isinstance(method, str) else int(method)
    out = {}
    for inp, X in activations.items():
        users = [layer for layer in weights if feeds[layer] == inp]
        if not users:
            continue
        if m in (WANDA, MAGNITUDE):
            # no Hessian: Wanda takes the feature norms straight from X
            for layer in users:
                out[layer] = prune_layer(weights[layer], X=X, stream=stream, check=check, **cfg)
            continue
        H = hessian_accumulate(X, stream=stream)
        for i, layer in enumerate(users):
            # the prune overwrites its H with the factor: every reader of the input but
            # the last gets a copy
            Hl = H if i == len(users) - 1 else H.clone()
            out[layer] = prune_layer(weights[layer], H=Hl, stream=stream, check=check, **cfg)
        del H
    return out


class Sweep:
    """One rank's rows of a layer pruned with the unstructured budget counted over every
    rank's rows, step by step (pwp_sweep_step): ``sharded.global_sweep`` drives the block
    loop and combines ``level1`` and ``level2`` (summed) and ``ties`` (gathered into
    ``ties_all``) over ranks between the steps.

    W_local: [c, b] bf16/fp32 CUDA tensor (this rank's rows, in rank order), H: the layer's
    undamped fp32 [b, b] H (the same on every rank; destroyed), c_total: every rank's rows."""
    STEPS = {"setup": 0, "score": 1, "pick_bin": 2, "reread": 3, "pick_key": 4, "count_ties": 5, "cut_ties": 6,
             "solve": 7, "finish": 8}

    @_on_stream
    def __init__(self, W_local, H, c_total, world=1, rank=0, *, method="thanos", sparsity=0.5, block=128,
                 damp=0.01, stream=None):
        torch = _torch()
        if W_local.dim() != 2:
            raise ValueError(f"W: expected [c, b], got shape {tuple(W_local.shape)}")
        c, b = W_local.shape
        _expect(W_local, "W", (c, b), (torch.bfloat16, torch.float32))
        _expect(H, "H", (b, b), (torch.float32,))
        _need_cuda(W_local, H)
        self.cfg = config(method, "unstructured", (0, 0), sparsity, block, damp)
        self.c, self.b, self.world, self.rank = int(c), int(b), int(world), int(rank)
        self.nblk = (b + int(block) - 1) // int(block)
        dev = W_local.device
        self.W, self.H = W_local, H
        self.W_out = torch.empty((c, b), dtype=torch.float32, device=dev)
        self.mask = torch.empty((c, b), dtype=torch.uint8, device=dev)
        self.ws = make_workspace(self.cfg, c, b, dev)
        self.stats = new_stats(dev)
        self.ties_all = torch.zeros((world, 128), dtype=torch.int32, device=dev)
        self.stream = stream
        self.args = SweepArgs(ctypes.pointer(self.cfg), W_local.data_ptr(), _dtype_code(W_local), c, b, int(c_total),
                              H.data_ptr(), self.W_out.data_ptr(), self.mask.data_ptr(), self.ws.ws.data_ptr(),
                              self.ws.nbytes, self.stats.data_ptr(), self.ties_all.data_ptr(), self.world, self.rank,
                              _stream_ptr(stream).value)
        p = [ctypes.c_void_p() for _ in range(3)]
        n = [_i64() for _ in range(3)]
        _check(lib().pwp_sweep_buffers(ctypes.byref(self.args), ctypes.byref(p[0]), ctypes.byref(n[0]),
                                       ctypes.byref(p[1]), ctypes.byref(n[1]), ctypes.byref(p[2]), ctypes.byref(n[2])),
               "pwp_sweep_buffers")
        base = self.ws.ws.data_ptr()

        def view(ptr, count):
            off = ptr.value - base
            return self.ws.ws[off: off + 4 * count.value].view(torch.int32)
        self.level1, self.level2, self.ties = view(p[0], n[0]), view(p[1], n[1]), view(p[2], n[2])

    def step(self, name, t=0):
        _check(lib().pwp_sweep_step(ctypes.byref(self.args), self.STEPS[name], int(t)), f"pwp_sweep_step({name})")

    def result(self, check=True):
        """(W_hat fp32 [c, b], mask uint8 [c, b], Stats of this rank: pruned = its removals)."""
        if not check:
            return self.W_out, self.mask, self.stats
        if self.stream is None:
            s = read_stats(self.stats)
        else:
            with _stream_ctx(self.stream):   # the read follows the steps on their stream
                s = read_stats(self.stats)
        if s.status != 0:
            raise PwpError(s.status, "pwp_sweep_step (device)")
        return self.W_out, self.mask, s


@_on_stream
def pack_24(W_hat, mask, *, stream=None, check=True):
    """Compressed 2:4 storage of a pruned layer (pwp_pack_24).  W_hat: fp32 [c, b] and
    mask: uint8 [c, b] CUDA tensors with exactly two kept entries in every aligned group
    of four.  Returns (values: int16 [c, b/2] holding bfloat16 bit patterns, meta: int32
    [c, ceil(b/32)] holding the 4-bit position fields, Stats or the unread stats tensor)."""
    torch = _torch()
    if W_hat.dim() != 2:
        raise ValueError(f"W_hat: expected [c, b], got shape {tuple(W_hat.shape)}")
    c, b = W_hat.shape
    _expect(W_hat, "W_hat", (c, b), (torch.float32,))
    _expect(mask, "mask", (c, b), (torch.uint8,))
    _need_cuda(W_hat, mask)
    values = torch.empty((c, b // 2), dtype=torch.int16, device=W_hat.device)
    meta = torch.empty((c, (b // 4 + 7) // 8), dtype=torch.int32, device=W_hat.device)
    stats = new_stats(W_hat.device)
    st = lib().pwp_pack_24(_vp(W_hat.data_ptr()), _vp(mask.data_ptr()), int(c), int(b), _vp(values.data_ptr()),
                           _vp(meta.data_ptr()), _vp(stats.data_ptr()), _stream_ptr(stream))
    _check(st, "pwp_pack_24")
    if not check:
        return values, meta, stats
    s = read_stats(stats)
    if s.status != 0:
        raise PwpError(s.status, "pwp_pack_24 (device)")
    return values, meta, s


@_on_stream
def prune_layer_host(W_host, X_host, *, out_W=None, out_mask=None, device="cuda", stream=None, **kw):
    """End-to-end call from host memory (pwp_prune_layer_host): W ([c, b]) and X ([n, b]),
    bf16/fp32 pinned torch CPU tensors, go to the device on a copy stream of the call's own
    -- X in chunks folded into H as they land, W while H is factored -- and the finished
    column blocks of W_hat and the mask come back into pinned host tensors during the sweep.
    Keyword arguments as prune_layer (method, sparsity, pattern, nm, block, damp, alpha).
    Returns (W_hat, mask, stats tensor); nothing syncs: synchronise the stream (the current
    one by default) before reading them."""
    torch = _torch()
    if W_host.dim() != 2 or X_host.dim() != 2 or X_host.shape[1] != W_host.shape[1]:
        raise ValueError(f"W [c, b] and X [n, b] expected, got {tuple(W_host.shape)} and {tuple(X_host.shape)}")
    c, b = W_host.shape
    n = X_host.shape[0]
    for name, t in (("W_host", W_host), ("X_host", X_host)):
        if t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{name}: a contiguous pinned CPU tensor is required")
        if t.dtype not in (torch.bfloat16, torch.float32):
            raise ValueError(f"{name}: bf16 or fp32 expected, got {t.dtype}")
    if out_W is None:
        out_W = torch.empty((c, b), dtype=torch.float32, pin_memory=True)
    if out_mask is None:
        out_mask = torch.empty((c, b), dtype=torch.uint8, pin_memory=True)
    for name, t, dt in (("out_W", out_W, torch.float32), ("out_mask", out_mask, torch.uint8)):
        if t.shape != (c, b) or t.dtype != dt or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{name}: a contiguous pinned CPU tensor [{c}, {b}] of {dt} is required")
    cfg = config(kw.pop("method", "thanos"), kw.pop("pattern", "unstructured"), kw.pop("nm", (2, 4)),
                 kw.pop("sparsity", 0.5), kw.pop("block", 128), kw.pop("damp", 0.01), kw.pop("alpha", 0.0))
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    dev = torch.device(device)
    W_dev = torch.empty((c, b), dtype=W_host.dtype, device=dev)
    X_dev = torch.empty((n, b), dtype=X_host.dtype, device=dev)
    no_update = cfg.method in (WANDA, MAGNITUDE)
    H_dev = None if no_update else torch.empty((b, b), dtype=torch.float32, device=dev)
    W_out = torch.empty((c, b), dtype=torch.float32, device=dev)
    mask = torch.empty((c, b), dtype=torch.uint8, device=dev)
    workspace = make_workspace(cfg, c, b, dev)
    stats = new_stats(dev)
    st = lib().pwp_prune_layer_host(ctypes.byref(cfg), _vp(W_host.data_ptr()), _dtype_code(W_host), int(c), int(b),
                                    _vp(X_host.data_ptr()), _dtype_code(X_host), int(n), _vp(W_dev.data_ptr()),
                                    _vp(X_dev.data_ptr()), _vp(H_dev.data_ptr() if H_dev is not None else 0),
                                    _vp(W_out.data_ptr()), _vp(mask.data_ptr()), _vp(out_W.data_ptr()),
                                    _vp(out_mask.data_ptr()), _vp(workspace.ws.data_ptr()), workspace.nbytes,
                                    _vp(stats.data_ptr()), _stream_ptr(stream))
    _check(st, "pwp_prune_layer_host")
    return out_W, out_mask, stats


@_on_stream
def prune_layers_host(Ws_host, Xs_host, *, out_Ws=None, out_masks=None, device="cuda", stream=None, **kw):
    """A sequence of same-shaped layers from pinned host memory (pwp_prune_layers_host):
    layer i+1's transfers overlap layer i's work and layer i's results come back while
    layer i+1 is pruned.  Ws_host[i] ([c, b]) and Xs_host[i] ([n, b]) are pinned CPU tensors
    of one dtype each (bf16 or fp32); keyword arguments as prune_layer.  Returns (W_hats,
    masks, stats tensor of len(Ws_host) records); nothing syncs: synchronise the stream (the
    current one by default) before reading them."""
    torch = _torch()
    nl = len(Ws_host)
    if len(Xs_host) != nl:
        raise ValueError("one X per W expected")
    if nl == 0:
        return [], [], new_stats(device)
    c, b = Ws_host[0].shape
    n = Xs_host[0].shape[0]
    for name, ts, shape in (("W", Ws_host, (c, b)), ("X", Xs_host, (n, b))):
        for t in ts:
            if (tuple(t.shape) != shape or t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous()
                    or t.dtype != ts[0].dtype or t.dtype not in (torch.bfloat16, torch.float32)):
                raise ValueError(f"{name}: contiguous pinned CPU tensors of one shape {shape} and dtype "
                                 f"(bf16 or fp32) expected")
    if out_Ws is None:
        out_Ws = [torch.empty((c, b), dtype=torch.float32, pin_memory=True) for _ in range(nl)]
    if out_masks is None:
        out_masks = [torch.empty((c, b), dtype=torch.uint8, pin_memory=True) for _ in range(nl)]
    for name, ts, dt in (("out_Ws", out_Ws, torch.float32), ("out_masks", out_masks, torch.uint8)):
        if len(ts) != nl or any(t.shape != (c, b) or t.dtype != dt or not t.is_pinned() or not t.is_contiguous()
                                for t in ts):
            raise ValueError(f"{name}: {nl} contiguous pinned CPU tensors [{c}, {b}] of {dt} expected")
    cfg = config(kw.pop("method", "thanos"), kw.pop("pattern", "unstructured"), kw.pop("nm", (2, 4)),
                 kw.pop("sparsity", 0.5), kw.pop("block", 128), kw.pop("damp", 0.01), kw.pop("alpha", 0.0))
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    L = lib()
    wt, xt = _dtype_code(Ws_host[0]), _dtype_code(Xs_host[0])
    nbytes = int(L.pwp_layers_host_bytes(ctypes.byref(cfg), int(c), int(b), int(n), wt, xt))
    if nbytes == 0:
        raise PwpError(1, "pwp_layers_host_bytes")
    dev = torch.empty(nbytes, dtype=torch.uint8, device=device)
    stats = torch.zeros(nl * ctypes.sizeof(Stats), dtype=torch.uint8, device=device)
    arr = lambda ts: (_vp * nl)(*[_vp(t.data_ptr()) for t in ts])
    Wp, Xp, Op, Mp = arr(Ws_host), arr(Xs_host), arr(out_Ws), arr(out_masks)
    st = L.pwp_prune_layers_host(ctypes.byref(cfg), nl, Wp, wt, int(c), int(b), Xp, xt, int(n), Op, Mp,
                                 _vp(dev.data_ptr()), nbytes, _vp(stats.data_ptr()), _stream_ptr(stream))
    _check(st, "pwp_prune_layers_host")
    return out_Ws, out_masks, stats


def read_stats_list(stats_t):
    """The per-layer records of a stats tensor holding several (prune_layers_host)."""
    raw = stats_t.cpu().numpy().tobytes()
    sz = ctypes.sizeof(Stats)
    return [Stats.from_buffer_copy(raw[i:i + sz]) for i in range(0, len(raw), sz)]


def from_bf16_bits(u16: np.ndarray, device="cuda"):
    """Upload bf16 bit patterns (uint16 numpy array) as a torch.bfloat16 tensor."""
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16))
    return t.view(torch.bfloat16).to(device)
