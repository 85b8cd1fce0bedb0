"""Python binding of libs2o: S2O permuted, importance-ordered, early-stopped block-sparse causal
attention prefill on one B200.

The binding only marshals arguments: it checks tensor shapes, dtypes and devices, allocates
outputs and the workspace with PyTorch (device memory and streams are PyTorch's job), and passes
raw device pointers and the current CUDA stream to the C ABI declared in ``include/s2o.h``. Every
step of the method runs in the library's CUDA kernels; there is no CPU or PyTorch fallback — if
``libs2o.so`` cannot be loaded, importing this package raises.

Sources: "S2O: Early Stopping for Sparse Attention via Online Permutation" (Summary ¶2) for the
method, "AB-Sparse" Eq. (1) for the dense baseline.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

from . import build as _build

__all__ = [
    "Config", "Indices", "Stats", "S2OError", "workspace_size", "index_sizes", "alloc_indices",
    "alloc_workspace", "build_indices", "attention_prefill", "attention_prefill_with_indices",
    "dense_causal_prefill", "validate_indices", "index_stats", "workspace_views",
    "set_wait_limit_ns", "set_attention_max_ctas", "check_device_status", "exp64_eval", "library_path",
    "kernel_launch_count", "build_indices_static", "STATIC_WORKSPACE_BYTES",
    "prefill_workspace_size", "alloc_prefill_workspace", "attention_prefill_with_indices_ws",
    "set_permuted_copy", "layer_workspace_size", "layer_prefill", "WorkCounts", "attention_work",
    "attention_prefill_online_stop", "gemm_bf16",
]

STATUS = {0: "S2O_OK", 1: "S2O_ERR_INVALID_ARGUMENT", 2: "S2O_ERR_UNSUPPORTED",
          3: "S2O_ERR_WORKSPACE_TOO_SMALL", 4: "S2O_ERR_INVALID_INDICES", 5: "S2O_ERR_CUDA",
          6: "S2O_ERR_DEVICE_TIMEOUT"}


class S2OError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class _Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("seq_len", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("segment_len", ctypes.c_int),
                ("block_size", ctypes.c_int), ("tau", ctypes.c_float),
                ("query_perm", ctypes.c_int), ("shared_key_order", ctypes.c_int),
                ("int4_centroids", ctypes.c_int)]


class _Indices(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("perm_q", "perm_k", "sel_cnt", "sel_blk", "local_tiles")]


class _Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in
                ("local_tiles", "selected_tiles", "pairs", "causal_pairs")]


class _Work(ctypes.Structure):
    _fields_ = [("local_pass_tiles", ctypes.c_uint64), ("permuted_unit_tiles", ctypes.c_uint64),
                ("permuted_loaded_tiles", ctypes.c_uint64), ("packed", ctypes.c_int),
                ("merged", ctypes.c_int)]


class _View(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("qbar", "kbar_all", "kbar_top", "u", "kappa", "rho", "Qbar", "Kbar", "r", "n")]


@dataclasses.dataclass(frozen=True)
class Config:
    """One attention layer (the fields of ``s2o_config``)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    seq_len: int
    head_dim: int
    segment_len: int
    block_size: int
    tau: float
    query_perm: int = 1
    shared_key_order: int = 0
    int4_centroids: int = 0

    @classmethod
    def of(cls, obj, **overrides) -> "Config":
        f = {k.name: getattr(obj, k.name) for k in dataclasses.fields(cls)}
        f.update(overrides)
        return cls(**f)

    def _c(self) -> _Config:
        return _Config(self.batch, self.n_q_heads, self.n_kv_heads, self.seq_len, self.head_dim,
                       self.segment_len, self.block_size, float(self.tau), self.query_perm,
                       self.shared_key_order, self.int4_centroids)

    @property
    def n_blocks(self) -> int:
        return self.seq_len // self.block_size


@dataclasses.dataclass
class Indices:
    """Index arrays on the device (int32), shapes as in ``s2o_indices``."""
    perm_q: torch.Tensor
    perm_k: torch.Tensor
    sel_cnt: torch.Tensor
    sel_blk: torch.Tensor
    local_tiles: torch.Tensor

    def tensors(self):
        # Not dataclasses.astuple: that deep-copies its fields, and the library must see these
        # exact tensors.
        return (self.perm_q, self.perm_k, self.sel_cnt, self.sel_blk, self.local_tiles)

    def _c(self) -> _Indices:
        for t in self.tensors():
            if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError("index arrays must be contiguous int32 CUDA tensors")
        return _Indices(*(t.data_ptr() for t in self.tensors()))


@dataclasses.dataclass(frozen=True)
class Stats:
    local_tiles: int
    selected_tiles: int
    pairs: int
    causal_pairs: int

    @property
    def pair_sparsity(self) -> float:
        return 1.0 - self.pairs / self.causal_pairs

    @property
    def executed_tiles(self) -> int:
        return self.local_tiles + self.selected_tiles


_lib = None


class _LayerConfig(ctypes.Structure):
    _fields_ = [("intermediate", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_double), ("rope_factor", ctypes.c_double),
                ("rope_low_freq_factor", ctypes.c_double),
                ("rope_high_freq_factor", ctypes.c_double),
                ("rope_original_context", ctypes.c_int), ("dense_attention", ctypes.c_int)]


_LAYER_WEIGHTS = ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gu", "w_down")


class _LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _LAYER_WEIGHTS]


def _layer_config(shape, dense: bool) -> _LayerConfig:
    """From any object with the decoder-layer fields (e.g. ``gen.LayerShape``)."""
    return _LayerConfig(shape.intermediate, shape.rms_eps, shape.rope_theta, shape.rope_factor,
                        shape.rope_low_freq_factor, shape.rope_high_freq_factor,
                        shape.rope_original_context, 1 if dense else 0)


def library_path() -> str:
    return _build.LIB


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        vp, st, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        C, I = ctypes.POINTER(_Config), ctypes.POINTER(_Indices)
        sig = {
            "s2o_workspace_size": [C, ctypes.POINTER(sz)],
            "s2o_prefill_workspace_size": [C, ctypes.POINTER(sz)],
            "s2o_index_sizes": [C, ctypes.POINTER(sz * 5)],
            "s2o_build_indices": [C, vp, vp, I, vp, sz, vp],
            "s2o_build_indices_static": [C, vp, vp, I, vp],
            "s2o_workspace_views": [C, vp, sz, ctypes.POINTER(_View)],
            "s2o_attention_prefill": [C, vp, vp, vp, vp, I, vp, sz, vp],
            "s2o_attention_prefill_with_indices": [C, vp, vp, vp, I, vp, vp],
            "s2o_attention_prefill_with_indices_ws": [C, vp, vp, vp, I, vp, vp, sz, vp],
            "s2o_attention_prefill_online_stop": [C, vp, vp, vp, I, vp, vp, vp],
            "s2o_dense_causal_prefill": [C, vp, vp, vp, vp, vp],
            "s2o_validate_indices": [C, I, vp, sz, vp],
            "s2o_index_stats": [C, I, vp, sz, ctypes.POINTER(_Stats), vp],
            "s2o_attention_work": [C, I, vp, sz, ctypes.POINTER(_Work), vp],
            "s2o_check_device_status": [vp],
            "s2o_exp64_eval": [vp, vp, ctypes.c_int, vp],
            "s2o_gemm_bf16": [vp, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_int, vp],
            "s2o_layer_workspace_size": [C, ctypes.POINTER(_LayerConfig), ctypes.POINTER(sz)],
            "s2o_layer_prefill": [C, ctypes.POINTER(_LayerConfig), ctypes.POINTER(_LayerWeights),
                                  vp, vp, sz, vp],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = st
        lib.s2o_kernel_launch_count.argtypes = []
        lib.s2o_kernel_launch_count.restype = ctypes.c_uint64
        lib.s2o_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.s2o_set_wait_limit_ns.restype = None
        lib.s2o_set_attention_max_ctas.argtypes = [ctypes.c_int]
        lib.s2o_set_attention_max_ctas.restype = None
        lib.s2o_set_permuted_copy.argtypes = [ctypes.c_int]
        lib.s2o_set_permuted_copy.restype = None
        lib.s2o_status_string.argtypes = [st]
        lib.s2o_status_string.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise S2OError(status, where)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _bf16(t: torch.Tensor, shape, name: str):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _qkv(cfg: Config, q, k, v=None):
    _bf16(q, (cfg.batch, cfg.n_q_heads, cfg.seq_len, cfg.head_dim), "q")
    _bf16(k, (cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim), "k")
    if v is not None:
        _bf16(v, (cfg.batch, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim), "v")


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(_load().s2o_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(n)),
           "s2o_workspace_size")
    return n.value


def index_sizes(cfg: Config):
    arr = (ctypes.c_size_t * 5)()
    _check(_load().s2o_index_sizes(ctypes.byref(cfg._c()), ctypes.byref(arr)), "s2o_index_sizes")
    return list(arr)


def alloc_workspace(cfg: Config, device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(cfg), dtype=torch.uint8, device=device)


def prefill_workspace_size(cfg: Config) -> int:
    """Workspace bytes with which the prefill may also use the permuted copy of K and V."""
    n = ctypes.c_size_t(0)
    _check(_load().s2o_prefill_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(n)),
           "s2o_prefill_workspace_size")
    return n.value


def alloc_prefill_workspace(cfg: Config, device="cuda") -> torch.Tensor:
    return torch.empty(prefill_workspace_size(cfg), dtype=torch.uint8, device=device)


def alloc_indices(cfg: Config, device="cuda") -> Indices:
    B, H, N, nB = cfg.batch, cfg.n_q_heads, cfg.seq_len, cfg.n_blocks
    e = lambda *s: torch.empty(s, dtype=torch.int32, device=device)  # noqa: E731
    return Indices(e(B, H, N), e(B, H, N), e(B, H, nB), e(B, H, nB, nB), e(B, H, nB))


def build_indices(cfg: Config, q, k, out: Indices | None = None,
                  ws: torch.Tensor | None = None) -> Indices:
    _qkv(cfg, q, k)
    out = out or alloc_indices(cfg, q.device)
    ws = ws if ws is not None else alloc_workspace(cfg, q.device)
    idx = out._c()
    _check(_load().s2o_build_indices(ctypes.byref(cfg._c()), q.data_ptr(), k.data_ptr(),
                                     ctypes.byref(idx), ws.data_ptr(), ws.numel(),
                                     _stream(q.device)), "s2o_build_indices")
    return out


STATIC_WORKSPACE_BYTES = 48 << 20  # S2O_STATIC_WORKSPACE_BYTES in include/s2o.h


def build_indices_static(cfg: Config, q, k, out: Indices) -> Indices:
    """The index build for callers that cannot allocate device memory: the library's fixed
    scratch array (``STATIC_WORKSPACE_BYTES`` per GPU) replaces the caller workspace. ``out`` must
    be preallocated. Calls whose GPU work overlaps share that array and race; the first call on a
    device (and on each host thread) does a one-time set-up and should come before any stream
    capture. The call runs with q's device current, so it uses that device's array."""
    _qkv(cfg, q, k)
    idx = out._c()
    with torch.cuda.device(q.device):
        _check(_load().s2o_build_indices_static(ctypes.byref(cfg._c()), q.data_ptr(),
                                                k.data_ptr(), ctypes.byref(idx),
                                                _stream(q.device)),
               "s2o_build_indices_static")
    return out


def workspace_views(cfg: Config, ws: torch.Tensor) -> dict:
    """Intermediate values of the last index build held in ``ws`` (views, no copy)."""
    view = _View()
    _check(_load().s2o_workspace_views(ctypes.byref(cfg._c()), ws.data_ptr(), ws.numel(),
                                       ctypes.byref(view)), "s2o_workspace_views")
    B, Hq, Hkv, N, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim
    nB, nSeg = cfg.n_blocks, cfg.seq_len // cfg.segment_len
    shapes = dict(qbar=(B, Hq, d), kbar_all=(B, Hkv, d), kbar_top=(B, Hq, d), u=(B, Hq, d),
                  kappa=(B, Hq, N), rho=(B, Hq, N), Qbar=(B, Hq, nB, d), Kbar=(B, Hq, nB, d),
                  r=(B, Hq, nB, nB), n=(B, Hq, nSeg, nB))
    base = ws.data_ptr()
    out = {}
    for name, shape in shapes.items():
        off = getattr(view, name) - base
        count = 1
        for s in shape:
            count *= s
        dt = torch.int32 if name == "n" else torch.float32
        out[name] = ws[off:off + 4 * count].view(dt).view(shape)
    return out


def attention_prefill(cfg: Config, q, k, v, out: torch.Tensor | None = None,
                      idx: Indices | None = None, ws: torch.Tensor | None = None):
    """The whole S2O hot path: index build then gather-attention. Returns (O, indices)."""
    _qkv(cfg, q, k, v)
    o = out if out is not None else torch.empty_like(q)
    _bf16(o, q.shape, "out")
    idx = idx or alloc_indices(cfg, q.device)
    ws = ws if ws is not None else alloc_prefill_workspace(cfg, q.device)
    ci = idx._c()
    _check(_load().s2o_attention_prefill(ctypes.byref(cfg._c()), q.data_ptr(), k.data_ptr(),
                                         v.data_ptr(), o.data_ptr(), ctypes.byref(ci),
                                         ws.data_ptr(), ws.numel(), _stream(q.device)),
           "s2o_attention_prefill")
    return o, idx


def attention_prefill_with_indices(cfg: Config, q, k, v, idx: Indices,
                                   out: torch.Tensor | None = None) -> torch.Tensor:
    _qkv(cfg, q, k, v)
    o = out if out is not None else torch.empty_like(q)
    _bf16(o, q.shape, "out")
    ci = idx._c()
    _check(_load().s2o_attention_prefill_with_indices(ctypes.byref(cfg._c()), q.data_ptr(),
                                                      k.data_ptr(), v.data_ptr(),
                                                      ctypes.byref(ci), o.data_ptr(),
                                                      _stream(q.device)),
           "s2o_attention_prefill_with_indices")
    return o


def attention_prefill_with_indices_ws(cfg: Config, q, k, v, idx: Indices, ws: torch.Tensor,
                                      out: torch.Tensor | None = None) -> torch.Tensor:
    """Steps 3-4 on given indices with a workspace (the permuted copy needs
    ``prefill_workspace_size`` bytes)."""
    _qkv(cfg, q, k, v)
    o = out if out is not None else torch.empty_like(q)
    _bf16(o, q.shape, "out")
    if ws.dtype != torch.uint8 or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous uint8 CUDA tensor")
    ci = idx._c()
    _check(_load().s2o_attention_prefill_with_indices_ws(ctypes.byref(cfg._c()), q.data_ptr(),
                                                         k.data_ptr(), v.data_ptr(),
                                                         ctypes.byref(ci), o.data_ptr(),
                                                         ws.data_ptr(), ws.numel(),
                                                         _stream(q.device)),
           "s2o_attention_prefill_with_indices_ws")
    return o


def attention_prefill_online_stop(cfg: Config, q, k, v, idx: Indices,
                                  out: torch.Tensor | None = None):
    """Steps 3-4 with the measured-share early stop (labelled variant; stop threshold cfg.tau).
    Returns (O, stop_cnt): the listed blocks each query block kept, int32 [batch, Hq, nB]."""
    _qkv(cfg, q, k, v)
    o = out if out is not None else torch.empty_like(q)
    _bf16(o, q.shape, "out")
    stop = torch.empty((cfg.batch, cfg.n_q_heads, cfg.n_blocks), dtype=torch.int32,
                       device=q.device)
    ci = idx._c()
    _check(_load().s2o_attention_prefill_online_stop(ctypes.byref(cfg._c()), q.data_ptr(),
                                                     k.data_ptr(), v.data_ptr(), ctypes.byref(ci),
                                                     o.data_ptr(), stop.data_ptr(),
                                                     _stream(q.device)),
           "s2o_attention_prefill_online_stop")
    return o, stop


def dense_causal_prefill(cfg: Config, q, k, v, out: torch.Tensor | None = None) -> torch.Tensor:
    _qkv(cfg, q, k, v)
    o = out if out is not None else torch.empty_like(q)
    _bf16(o, q.shape, "out")
    _check(_load().s2o_dense_causal_prefill(ctypes.byref(cfg._c()), q.data_ptr(), k.data_ptr(),
                                            v.data_ptr(), o.data_ptr(), _stream(q.device)),
           "s2o_dense_causal_prefill")
    return o


def validate_indices(cfg: Config, idx: Indices, ws: torch.Tensor | None = None) -> bool:
    """True when the index arrays are valid (synchronises the current stream)."""
    dev = idx.perm_q.device
    ws = ws if ws is not None else alloc_workspace(cfg, dev)
    ci = idx._c()
    st = _load().s2o_validate_indices(ctypes.byref(cfg._c()), ctypes.byref(ci), ws.data_ptr(),
                                      ws.numel(), _stream(dev))
    if st == 4:
        return False
    _check(st, "s2o_validate_indices")
    return True


def index_stats(cfg: Config, idx: Indices, ws: torch.Tensor | None = None) -> Stats:
    dev = idx.perm_q.device
    ws = ws if ws is not None else alloc_workspace(cfg, dev)
    ci = idx._c()
    s = _Stats()
    _check(_load().s2o_index_stats(ctypes.byref(cfg._c()), ctypes.byref(ci), ws.data_ptr(),
                                   ws.numel(), ctypes.byref(s), _stream(dev)), "s2o_index_stats")
    return Stats(s.local_tiles, s.selected_tiles, s.pairs, s.causal_pairs)


@dataclasses.dataclass(frozen=True)
class WorkCounts:
    """Tile work of the last attention call on a prefill workspace (``s2o_work_counts``)."""
    local_pass_tiles: int
    permuted_unit_tiles: int
    permuted_loaded_tiles: int
    packed: bool
    merged: bool

    @property
    def unit_tiles(self) -> int:
        return self.local_pass_tiles + self.permuted_unit_tiles


def attention_work(cfg: Config, idx: Indices, ws: torch.Tensor) -> WorkCounts:
    """Tile products and loads of the last attention call that used ``ws`` (synchronises)."""
    dev = idx.perm_q.device
    ci = idx._c()
    w = _Work()
    _check(_load().s2o_attention_work(ctypes.byref(cfg._c()), ctypes.byref(ci), ws.data_ptr(),
                                      ws.numel(), ctypes.byref(w), _stream(dev)),
           "s2o_attention_work")
    return WorkCounts(w.local_pass_tiles, w.permuted_unit_tiles, w.permuted_loaded_tiles,
                      bool(w.packed), bool(w.merged))


def kernel_launch_count() -> int:
    """Kernel launches made by libs2o in this process so far."""
    return int(_load().s2o_kernel_launch_count())


def set_wait_limit_ns(ns: int) -> None:
    _load().s2o_set_wait_limit_ns(int(ns))


def layer_workspace_size(cfg: Config, shape, dense: bool = False) -> int:
    """Workspace bytes of ``layer_prefill`` (``shape``: the decoder-layer sizes, e.g.
    ``gen.LayerShape``)."""
    n = ctypes.c_size_t(0)
    lc = _layer_config(shape, dense)
    _check(_load().s2o_layer_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(lc),
                                            ctypes.byref(n)), "s2o_layer_workspace_size")
    return n.value


def layer_prefill(cfg: Config, shape, weights: dict, x: torch.Tensor,
                  ws: torch.Tensor | None = None, dense: bool = False) -> torch.Tensor:
    """One decoder layer in place on x [batch, N, H] (bf16, CUDA): S2O attention, or the dense
    causal baseline with ``dense``. ``weights``: bf16 CUDA tensors named as in s2o_layer_weights."""
    H = cfg.n_q_heads * cfg.head_dim
    _bf16(x, (cfg.batch, cfg.seq_len, H), "x")
    I = shape.intermediate
    shapes = {"attn_norm": (H,), "w_qkv": (H, (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim),
              "w_o": (H, H), "mlp_norm": (H,), "w_gu": (H, 2 * I), "w_down": (I, H)}
    for name, shp in shapes.items():
        _bf16(weights[name], shp, name)
    lc = _layer_config(shape, dense)
    ws = ws if ws is not None else torch.empty(layer_workspace_size(cfg, shape, dense),
                                               dtype=torch.uint8, device=x.device)
    wts = _LayerWeights(*(weights[n].data_ptr() for n in _LAYER_WEIGHTS))
    _check(_load().s2o_layer_prefill(ctypes.byref(cfg._c()), ctypes.byref(lc), ctypes.byref(wts),
                                     x.data_ptr(), ws.data_ptr(), ws.numel(), _stream(x.device)),
           "s2o_layer_prefill")
    return x


def set_permuted_copy(mode: int) -> None:
    """Packed streams from the permuted copy of K/V: 0 never (gathered rows), 1 when they pay
    (default), 2 always; 3 runs the path without a workspace even when one is given."""
    _load().s2o_set_permuted_copy(int(mode))


def set_attention_max_ctas(max_ctas: int) -> None:
    """Caps the persistent attention grid (0 = one CTA per SM); results do not depend on it."""
    _load().s2o_set_attention_max_ctas(int(max_ctas))


def check_device_status(device="cuda") -> int:
    """Synchronises and returns the library status (0 = S2O_OK, 6 = a bounded wait ran out)."""
    return _load().s2o_check_device_status(_stream(torch.device(device)))


def gemm_bf16(a: torch.Tensor, b: torch.Tensor, c: torch.Tensor | None = None,
              accumulate: bool = False) -> torch.Tensor:
    """C = A·B (+ C when ``accumulate``): row-major bf16 CUDA tensors, fp32 accumulation."""
    if a.dim() != 2 or b.dim() != 2 or a.shape[1] != b.shape[0]:
        raise ValueError("a [m, k] and b [k, n] expected")
    m, k = a.shape
    n = b.shape[1]
    _bf16(a, (m, k), "a")
    _bf16(b, (k, n), "b")
    if c is None:
        if accumulate:
            raise ValueError("accumulate needs c")
        c = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    _bf16(c, (m, n), "c")
    _check(_load().s2o_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), m, n, k,
                                 1 if accumulate else 0, _stream(a.device)), "s2o_gemm_bf16")
    return c


def exp64_eval(x: torch.Tensor) -> torch.Tensor:
    if x.dtype != torch.float64 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float64 CUDA tensor")
    y = torch.empty_like(x)
    _check(_load().s2o_exp64_eval(x.data_ptr(), y.data_ptr(), x.numel(), _stream(x.device)),
           "s2o_exp64_eval")
    return y
