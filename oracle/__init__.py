"""fp64 CPU oracle for the Avey-B ranker and neural-processor layer.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports or calls this package, and this package never imports the CUDA library.

The arithmetic lives in ``avey_oracle.c`` (plain C, naive fp64 loops); this
module only compiles it, marshals numpy arrays and strings the per-function
calls together in the order the method states:

  rank:      N(X) -> MaxSim scores -> top-k + divide by the best score
  compress:  X_hat = P [X_t ; w_1 X_c1 ; ... ; w_k X_ck] + X_t
  layers:    enricher -> head/tail -> static or dynamic mix -> fuser + residual

Every function works on float64 arrays; float32 inputs (bf16-representable for
the bf16 workloads) are widened exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "avey_oracle.c")
_LIB = os.path.join(_HERE, "libavey_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile avey_oracle.c into libavey_oracle.so (if missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            L.avey_orc_threads.restype = ctypes.c_int
            L.avey_orc_set_threads.argtypes = [ctypes.c_int]
            L.avey_orc_normalize.argtypes = [_D, ctypes.c_longlong, ctypes.c_int, _D]
            L.avey_orc_maxsim_rows.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, _I, _I, ctypes.c_int, _D]
            L.avey_orc_topk_row.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I, _D]
            L.avey_orc_topk_row.restype = ctypes.c_int
            L.avey_orc_topk_row_dir.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, _I, _D]
            L.avey_orc_topk_row_dir.restype = ctypes.c_int
            L.avey_orc_coupled_causal_mix.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_longlong, _D, ctypes.c_longlong]
            L.avey_orc_compress_rows.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, _I, _I, ctypes.c_int, _I, _D, _D,
                                                 _D]
            L.avey_orc_context_rows.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, _I, _I, ctypes.c_int, _I, _D, _D]
            L.avey_orc_static_mix.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_longlong, _D, ctypes.c_longlong]
            L.avey_orc_dynamic_weights.argtypes = [_D, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_longlong, ctypes.c_double, _D]
            L.avey_orc_dynamic_mix.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                               ctypes.c_double, _D, ctypes.c_longlong]
            L.avey_orc_layer.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, _D, _D, _D, _D]
            _lib = L
    return _lib


def threads() -> int:
    return lib().avey_orc_threads()


def set_threads(n: int) -> None:
    lib().avey_orc_set_threads(int(n))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _pd(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _pi(a: np.ndarray):
    return a.ctypes.data_as(_I)


# ---------------------------------------------------------------- ranker ----

def normalize(X) -> np.ndarray:
    """N(X) row-wise: x / max(||x||_2, 1e-12); X [..., d]."""
    X = _f64(X)
    out = np.empty_like(X)
    d = X.shape[-1]
    lib().avey_orc_normalize(_pd(X), X.size // d, d, _pd(out))
    return out


def maxsim_rows(X, S: int, sel) -> np.ndarray:
    """MaxSim scores of every split against the selected targets.

    X [B, N, d]; sel int [n_sel, 2] of (b, t).  Returns [n_sel, n] float64.
    """
    X = _f64(X)
    B, N, d = X.shape
    n = -(-N // S)
    sel = _i32(sel).reshape(-1, 2)
    sb, st = _i32(sel[:, 0]), _i32(sel[:, 1])
    Xn = normalize(X)
    out = np.empty((sel.shape[0], n), dtype=np.float64)
    lib().avey_orc_maxsim_rows(_pd(Xn), B, N, d, S, _pi(sb), _pi(st), sel.shape[0], _pd(out))
    return out


def all_targets(B: int, n: int) -> np.ndarray:
    bb, tt = np.meshgrid(np.arange(B), np.arange(n), indexing="ij")
    return np.stack([bb.ravel(), tt.ravel()], axis=1).astype(np.int32)


def topk(scores_rows, targets, k: int, causal: bool = False):
    """Top-k (self excluded, ties -> lower index) and w = s / s_best.

    scores_rows [n_sel, n]; targets [n_sel] target split index of each row;
    causal: candidates only c < t (unidirectional ranker).
    Returns idx int32 [n_sel, k] (-1 where fewer than k candidates) and
    w float64 [n_sel, k].
    """
    sc = _f64(scores_rows)
    n_sel, n = sc.shape
    idx = np.empty((n_sel, k), dtype=np.int32)
    w = np.empty((n_sel, k), dtype=np.float64)
    L = lib()
    for s in range(n_sel):
        row = np.ascontiguousarray(sc[s])
        L.avey_orc_topk_row_dir(_pd(row), n, int(targets[s]), k, int(bool(causal)), _pi(idx[s]),
                                _pd(w[s]))
    return idx, w


def rank(X, S: int, k: int, sel=None, causal: bool = False):
    """Ranker for the selected (b, t) targets (all targets when sel is None).

    Returns (sel, scores [n_sel, n], idx [n_sel, k], w [n_sel, k]).
    """
    X = _f64(X)
    B, N, _ = X.shape
    n = -(-N // S)
    sel = all_targets(B, n) if sel is None else _i32(sel).reshape(-1, 2)
    scores = maxsim_rows(X, S, sel)
    idx, w = topk(scores, sel[:, 1], k, causal)
    return sel, scores, idx, w


def compress(X, S: int, k: int, sel, idx, w, P) -> np.ndarray:
    """Neural compression + residual for the selected targets: [n_sel, S, d]."""
    X = _f64(X)
    B, N, d = X.shape
    sel = _i32(sel).reshape(-1, 2)
    sb, st = _i32(sel[:, 0]), _i32(sel[:, 1])
    idx, w, P = _i32(idx), _f64(w), _f64(P)
    out = np.empty((sel.shape[0], S, d), dtype=np.float64)
    lib().avey_orc_compress_rows(_pd(X), N, d, S, k, _pi(sb), _pi(st), sel.shape[0], _pi(idx),
                                 _pd(w), _pd(P), _pd(out))
    return out


def context(X, S: int, k: int, sel, idx, w) -> np.ndarray:
    """Uncompressed context of each selected target: [n_sel, (k+1)S, d] with
    rows [X_t ; w_1 X_c1 ; ... ; w_k X_ck] (the compressor's input, eq. 8)."""
    X = _f64(X)
    B, N, d = X.shape
    sel = _i32(sel).reshape(-1, 2)
    sb, st = _i32(sel[:, 0]), _i32(sel[:, 1])
    idx, w = _i32(idx), _f64(w)
    out = np.empty((sel.shape[0], (k + 1) * S, d), dtype=np.float64)
    lib().avey_orc_context_rows(_pd(X), N, d, S, k, _pi(sb), _pi(st), sel.shape[0], _pi(idx),
                                _pd(w), _pd(out))
    return out


# ----------------------------------------------------------------- layer ----

def static_mix(V, zt) -> np.ndarray:
    """c = V Z_t for one split; V [S, S], zt [S, mt]."""
    V, zt = _f64(V), _f64(zt)
    S, mt = zt.shape
    c = np.empty((S, mt), dtype=np.float64)
    lib().avey_orc_static_mix(_pd(V), _pd(zt), S, mt, mt, _pd(c), mt)
    return c


def coupled_causal_mix(V, zt) -> np.ndarray:
    """c = (V * N(Z)N(Z)^T, masked to j <= i) Z_t for one split (original Avey)."""
    V, zt = _f64(V), _f64(zt)
    S, mt = zt.shape
    c = np.empty((S, mt), dtype=np.float64)
    lib().avey_orc_coupled_causal_mix(_pd(V), _pd(zt), S, mt, mt, _pd(c), mt)
    return c


def dynamic_weights(zt, eps: float) -> np.ndarray:
    """Gt (eq. 6) for one split; zt [S, mt] -> [S, S]."""
    zt = _f64(zt)
    S, mt = zt.shape
    Gt = np.empty((S, S), dtype=np.float64)
    lib().avey_orc_dynamic_weights(_pd(zt), S, mt, mt, eps, _pd(Gt))
    return Gt


def dynamic_mix(zt, eps: float) -> np.ndarray:
    """c = Gt Z_t for one split; zt [S, mt]."""
    zt = _f64(zt)
    S, mt = zt.shape
    c = np.empty((S, mt), dtype=np.float64)
    lib().avey_orc_dynamic_mix(_pd(zt), S, mt, mt, eps, _pd(c), mt)
    return c


def dynamic_mix_blocks(zt_blocks, eps: float) -> np.ndarray:
    """Dynamic mix of many independent split blocks: zt [blocks, S, mt]."""
    zt = _f64(zt_blocks)
    return np.stack([dynamic_mix(zt[i], eps) for i in range(zt.shape[0])])


def layer(x_splits, lw, S: int, m_h: int, eps: float, prenorm: bool) -> np.ndarray:
    """One layer on independent splits x [n_splits, S, d]; returns a new array.

    lw: synthetic.LayerWeights (U [d, m], bU [m], V [S, S] or None, O [m, d]).
    """
    x = np.array(x_splits, dtype=np.float64, copy=True, order="C")
    n_sp, S_, d = x.shape
    assert S_ == S
    U, bU, O = _f64(lw.U), _f64(lw.bU), _f64(lw.O)
    m = U.shape[1]
    V = _f64(lw.V) if lw.V is not None else np.zeros((S, S))
    lib().avey_orc_layer(_pd(x), n_sp, S, d, m, m_h, int(lw.kind), int(bool(prenorm)), eps,
                         _pd(U), _pd(bU), _pd(V), _pd(O))
    return x


def forward(X, weights, wl, sel=None, causal: bool = False):
    """Ranker once, compression, then every layer, for selected targets.

    X [B, N, d]; weights: synthetic.Weights; wl: synthetic.Workload.
    The oracle always uses its own selection.
    Returns dict(sel, scores, idx, w, compressed, layers=[per-layer outputs]).
    """
    X = _f64(X)
    sel, scores, oidx, ow = rank(X, wl.S, wl.k, sel, causal)
    xc = compress(X, wl.S, wl.k, sel, oidx, ow, weights.P)
    outs = []
    x = xc
    for lw in weights.layers:
        x = layer(x, lw, wl.S, wl.m_h, wl.eps, wl.prenorm)
        outs.append(x)
    return dict(sel=sel, scores=scores, idx=oidx, w=ow, compressed=xc, layers=outs)


def forward_uncompressed(X, weights, wl, sel=None, causal: bool = False):
    """The processor without neural compression ([AB-sum] §4.3: the ablation
    that the 4.37x throughput figure compares against).

    Ranker once; each selected target's (k+1)S-token context
    [X_t ; w_1 X_c1 ; ... ; w_k X_ck] goes through every layer as one block, so
    the contextualizer mixes all (k+1)S tokens (V is (k+1)S x (k+1)S, from
    synthetic.gen_weights(wl, block=(k+1)S)); the first S rows of the last
    layer's block are the target split's output.
    Returns dict(sel, scores, idx, w, context, layers=[per-layer [n_sel, (k+1)S, d]],
    out [n_sel, S, d]).
    """
    X = _f64(X)
    sel, scores, oidx, ow = rank(X, wl.S, wl.k, sel, causal)
    ctx = context(X, wl.S, wl.k, sel, oidx, ow)
    L = (wl.k + 1) * wl.S
    outs = []
    x = ctx
    for lw in weights.layers:
        x = layer(x, lw, L, wl.m_h, wl.eps, wl.prenorm)
        outs.append(x)
    return dict(sel=sel, scores=scores, idx=oidx, w=ow, context=ctx, layers=outs,
                out=x[:, :wl.S, :].copy())
