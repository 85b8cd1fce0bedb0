"""CPU oracle for the S2O prefill path — TEST INFRASTRUCTURE, not part of the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module. It wraps ``s2o_oracle.c`` (plain C, written from the method's definition; see that file's
header for the passages it follows) through ctypes and builds it with gcc on first use.

Parity status per function (what pins it to something other than itself lives in
``tests/test_oracle_pins.py``):

* ``build_indices`` — pinned by the hand-worked case in ``tests/golden/``, by the hand-derived
  summation-order case, by a closed-form stop at p = τ (identical keys give p = 1/2 exactly), by
  invariants (permutations, sortedness, nesting in τ, Σp = 1) and by float64 re-derivations;
  ``tests/test_oracle_mutations.py`` checks that these pins reject planted mistakes.
* ``attention`` — pinned by torch's causal scaled-dot-product attention at τ = 0, by per-segment
  causal attention at τ > 1, and by permutation invariance.
* ``dense_causal`` — pinned by torch's causal scaled-dot-product attention.
* ``exp64`` — pinned by libm exp (≤ 2 ulp) and the constants by a 60-digit derivation.
* ``online_stop`` (the measured-share early stop, a labelled variant) — pinned by a hand-worked
  case (``tests/golden/online_stop_case.md``), by τ = 0 (nothing stops), by a brute-force
  restatement from whole-row softmax probabilities on small random inputs, and by the rule's
  consequences (stopping never adds a block; lists stay prefixes).
* ``layer.layer`` (the decoder layer around the attention, ``oracle/layer.py``) — pinned in
  ``tests/test_layer_oracle_pins.py`` (bf16 rounding against torch, closed-form norms, rotary
  invariants, the frequency scaling's regimes, the silu identity, zero projections = identity,
  and transformers' Llama decoder layer and rotary table on the same weights).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s2o_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
          "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle library with gcc (no-op when it is newer than its source)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("seq_len", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("segment_len", ctypes.c_int),
                ("block_size", ctypes.c_int), ("tau", ctypes.c_float),
                ("query_perm", ctypes.c_int), ("shared_key_order", ctypes.c_int),
                ("int4_centroids", ctypes.c_int)]


class _Debug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("qbar", "kbar_all", "kbar_top", "u", "kappa", "rho", "Qbar", "Kbar", "r", "n",
                 "p")]


def _load(path: str | None = None):
    global _lib
    with _lock:
        if _lib is None or path is not None:
            lib = ctypes.CDLL(path or build())
            vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
            lib.oracle_build_indices.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp, vp, vp,
                                                 vp, ctypes.POINTER(_Debug), i32]
            lib.oracle_build_indices.restype = i32
            lib.oracle_attention.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp, vp, vp, vp,
                                             vp, i64, vp, ctypes.POINTER(i64), i32]
            lib.oracle_attention.restype = i32
            lib.oracle_dense_causal.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp, i64, vp,
                                                i32]
            lib.oracle_dense_causal.restype = i32
            lib.oracle_online_stop.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp, vp, vp,
                                               vp, vp, i32]
            lib.oracle_online_stop.restype = i32
            lib.oracle_pair_count.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp]
            lib.oracle_pair_count.restype = i64
            lib.oracle_score_scale.argtypes = [ctypes.c_int]
            lib.oracle_score_scale.restype = ctypes.c_float
            lib.oracle_exp64.argtypes = [ctypes.c_double]
            lib.oracle_exp64.restype = ctypes.c_double
            if path is not None:
                return lib
            _lib = lib
    return _lib


class use_library:
    """Context manager that points this module at another build of the oracle source (used by
    the mutation tests, which compile deliberately broken copies and check the pins catch them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _load(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def config(w, **overrides) -> Config:
    """A ``Config`` from any object with the workload fields (e.g. ``gen.Workload``)."""
    f = {k: getattr(w, k) for k, _ in Config._fields_}
    f.update(overrides)
    return Config(**f)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _bits(x) -> np.ndarray:
    """bf16 input as contiguous uint16 bits (accepts a torch bf16 tensor or a uint16 array)."""
    if hasattr(x, "view") and not isinstance(x, np.ndarray):
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


def threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def build_indices(cfg: Config, q, k, debug: bool = False, n_threads: int | None = None):
    """Index arrays (and, with ``debug``, every intermediate value) as a dict of numpy arrays."""
    lib = _load()
    q, k = _bits(q), _bits(k)
    B, Hq, Hkv, N, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim
    nB, nSeg = N // cfg.block_size, N // cfg.segment_len
    out = dict(perm_q=np.empty((B, Hq, N), np.int32), perm_k=np.empty((B, Hq, N), np.int32),
               sel_cnt=np.empty((B, Hq, nB), np.int32),
               sel_blk=np.empty((B, Hq, nB, nB), np.int32),
               local_tiles=np.empty((B, Hq, nB), np.int32))
    dbg = None
    if debug:
        f32 = np.float32
        out.update(qbar=np.zeros((B, Hq, d), f32), kbar_all=np.zeros((B, Hkv, d), f32),
                   kbar_top=np.zeros((B, Hq, d), f32), u=np.zeros((B, Hq, d), f32),
                   kappa=np.zeros((B, Hq, N), f32), rho=np.zeros((B, Hq, N), f32),
                   Qbar=np.zeros((B, Hq, nB, d), f32), Kbar=np.zeros((B, Hq, nB, d), f32),
                   r=np.zeros((B, Hq, nB, nB), f32), n=np.zeros((B, Hq, nSeg, nB), np.int32),
                   p=np.zeros((B, Hq, nB, nB), np.float64))
        dbg = _Debug(**{name: _ptr(out[name]) for name, _ in _Debug._fields_})
    st = lib.oracle_build_indices(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(out["perm_q"]),
                                  _ptr(out["perm_k"]), _ptr(out["sel_cnt"]),
                                  _ptr(out["sel_blk"]), _ptr(out["local_tiles"]),
                                  ctypes.byref(dbg) if dbg is not None else None,
                                  n_threads or threads())
    if st != 0:
        raise ValueError(f"oracle_build_indices: status {st}")
    return out


def attention(cfg: Config, q, k, v, idx: dict, rows: np.ndarray | None = None,
              n_threads: int | None = None):
    """(out [n_rows, d] float64, Σ|K_i| over those rows) on the given index arrays."""
    lib = _load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    total = cfg.batch * cfg.n_q_heads * cfg.seq_len
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = total if rows_arr is None else len(rows_arr)
    out = np.empty((n_rows, cfg.head_dim), np.float64)
    pairs = ctypes.c_int64(0)
    arrs = [np.ascontiguousarray(idx[n], dtype=np.int32)
            for n in ("perm_q", "perm_k", "sel_cnt", "sel_blk")]
    st = lib.oracle_attention(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), *map(_ptr, arrs),
                              _ptr(rows_arr), n_rows, _ptr(out), ctypes.byref(pairs),
                              n_threads or threads())
    if st != 0:
        raise ValueError(f"oracle_attention: status {st}")
    return out, int(pairs.value)


def dense_causal(cfg: Config, q, k, v, rows: np.ndarray | None = None,
                 n_threads: int | None = None) -> np.ndarray:
    lib = _load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    total = cfg.batch * cfg.n_q_heads * cfg.seq_len
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = total if rows_arr is None else len(rows_arr)
    out = np.empty((n_rows, cfg.head_dim), np.float64)
    st = lib.oracle_dense_causal(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(rows_arr),
                                 n_rows, _ptr(out), n_threads or threads())
    if st != 0:
        raise ValueError(f"oracle_dense_causal: status {st}")
    return out


def online_stop(cfg: Config, q, k, idx: dict, n_threads: int | None = None):
    """The measured-share early stop (labelled variant): ``(stop_cnt [b, Hq, nB] int32,
    max_share [b, Hq, nB, nB] float64)`` — the listed blocks each query block keeps, and for every
    listed block the largest share over the block's rows (zero past the list)."""
    lib = _load()
    q, k = _bits(q), _bits(k)
    B, Hq, N = cfg.batch, cfg.n_q_heads, cfg.seq_len
    nB = N // cfg.block_size
    stop = np.empty((B, Hq, nB), np.int32)
    share = np.zeros((B, Hq, nB, nB), np.float64)
    arrs = [np.ascontiguousarray(idx[n], dtype=np.int32)
            for n in ("perm_q", "perm_k", "sel_cnt", "sel_blk")]
    st = lib.oracle_online_stop(ctypes.byref(cfg), _ptr(q), _ptr(k), *map(_ptr, arrs),
                                _ptr(stop), _ptr(share), n_threads or threads())
    if st != 0:
        raise ValueError(f"oracle_online_stop: status {st}")
    return stop, share


def with_counts(idx: dict, counts) -> dict:
    """The index arrays with sel_cnt replaced (the lists cut to the given lengths)."""
    out = dict(idx)
    out["sel_cnt"] = np.ascontiguousarray(counts, dtype=np.int32)
    return out


def pair_count(cfg: Config, idx: dict) -> int:
    lib = _load()
    arrs = [np.ascontiguousarray(idx[n], dtype=np.int32)
            for n in ("perm_q", "perm_k", "sel_cnt", "sel_blk")]
    return int(lib.oracle_pair_count(ctypes.byref(cfg), *map(_ptr, arrs)))


def score_scale(d: int) -> float:
    return _load().oracle_score_scale(int(d))


def exp64(x: float) -> float:
    return _load().oracle_exp64(float(x))
