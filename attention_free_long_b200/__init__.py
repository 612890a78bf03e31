"""Python binding of libavey.so, the B200 (sm_100a) Avey-B ranker and
neural-processor library.

This module only marshals arguments: it takes torch CUDA tensors, allocates
outputs and workspaces with torch (device memory and streams are all torch is
used for), and calls the C ABI declared in ``include/avey.h`` on the current
CUDA stream.  Every step of the computation runs in the library's kernels.
There is no fallback: if ``libavey.so`` is missing, importing the functions
raises.

Entry points (same names as the C ABI):
  avey_rank          MaxSim split scores -> top-k indices + divide-by-max weights
  avey_compress      eq. 8 neural compression with residual
  avey_dynamic_mix   eq. 6 row-normalised cosine mix of split blocks
  avey_layer_forward enricher -> static/dynamic mix -> fuser + residual
and ``encoder_forward`` which strings them together (ranker once, then every
layer), the call a user of the encoder makes; ``processor_forward`` is the
same forward after the ranker, for a selection the caller supplies.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libavey.so")

AVEY_F32, AVEY_BF16, AVEY_BF16X2 = 0, 1, 2
AVEY_STATIC, AVEY_DYNAMIC, AVEY_COUPLED_CAUSAL = 0, 1, 2
AVEY_RANK_UNIDIRECTIONAL = 1
STATUS = {0: "AVEY_OK", 1: "AVEY_ERR_INVALID_ARG", 2: "AVEY_ERR_UNSUPPORTED", 3: "AVEY_ERR_CUDA",
          4: "AVEY_ERR_DEVICE_TIMEOUT", 5: "AVEY_ERR_DEVICE_BOUNDS"}

_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


class AveyError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str):
        super().__init__(f"{fn}: {STATUS.get(code, code)}: {detail}")
        self.code = code


class LayerParams(ctypes.Structure):
    _fields_ = [("kind", _i), ("d", _i), ("m", _i), ("m_h", _i), ("S", _i), ("eps", ctypes.c_float),
                ("prenorm", _i), ("Ut", _vp), ("bU", _vp), ("V", _vp), ("Ot", _vp)]


def lib() -> ctypes.CDLL:
    """Loads libavey.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              f"`python -m attention_free_long_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        L.avey_rank.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]
        L.avey_rank.restype = _i
        L.avey_rank_ex.argtypes = [_vp, _i, _i, _i, _i, _i, _i, ctypes.c_uint32, _vp, _vp, _vp,
                                   _vp, _sz, _vp]
        L.avey_rank_ex.restype = _i
        L.avey_trace_begin.argtypes = [_i, _vp]
        L.avey_trace_begin.restype = _i
        L.avey_trace_end.argtypes = []
        L.avey_trace_end.restype = _i
        L.avey_trace_kernel_name.argtypes = [_i]
        L.avey_trace_kernel_name.restype = ctypes.c_char_p
        L.avey_trace_kernel_ms.argtypes = [_i, ctypes.POINTER(ctypes.c_float)]
        L.avey_trace_kernel_ms.restype = _i
        L.avey_rank_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.avey_rank_workspace_bytes.restype = _sz
        L.avey_compress.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]
        L.avey_compress.restype = _i
        L.avey_dynamic_mix.argtypes = [_vp, _i64, _i, _i, _i, _i, ctypes.c_float, _vp, _i64, _vp]
        L.avey_dynamic_mix.restype = _i
        L.avey_layer_forward.argtypes = [ctypes.POINTER(LayerParams), _i, _i, _vp, _vp, _vp, _vp,
                                         _vp, _sz, _vp]
        L.avey_layer_forward.restype = _i
        L.avey_layer_forward_ex.argtypes = [ctypes.POINTER(LayerParams), _i, _i, _vp, _vp, _vp, _vp,
                                            _vp, _vp, _vp, _sz, _vp]
        L.avey_layer_forward_ex.restype = _i
        L.avey_layer_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.avey_layer_workspace_bytes.restype = _sz
        L.avey_layer_workspace_bytes_ex.argtypes = [_i, _i, _i, _i, _i, _i, _i]
        L.avey_layer_workspace_bytes_ex.restype = _sz
        L.avey_context.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]
        L.avey_context.restype = _i
        L.avey_topk.argtypes = [_vp, _i, _i, _i, ctypes.c_uint32, _vp, _vp, _vp]
        L.avey_topk.restype = _i
        L.avey_static_mix.argtypes = [_vp, _vp, _i64, _i, _i, _i, _i, _vp, _i64, _vp]
        L.avey_static_mix.restype = _i
        L.avey_topk_rows.argtypes = [_vp, _i, _i, _i, _i, _i, ctypes.c_uint32, _vp, _vp, _vp]
        L.avey_topk_rows.restype = _i
        L.avey_maxsim_part.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]
        L.avey_maxsim_part.restype = _i
        L.avey_compress_rows.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp,
                                         _vp, _vp]
        L.avey_compress_rows.restype = _i
        L.avey_device_status.argtypes = [_vp]
        L.avey_device_status.restype = _i
        L.avey_status_string.argtypes = [_i]
        L.avey_status_string.restype = ctypes.c_char_p
        L.avey_last_error_detail.argtypes = []
        L.avey_last_error_detail.restype = ctypes.c_char_p
        L.avey_kernel_launches.argtypes = []
        L.avey_kernel_launches.restype = ctypes.c_uint64
        _lib = L
    return _lib


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise AveyError(fn, code, lib().avey_last_error_detail().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return AVEY_F32
    if t.dtype == torch.bfloat16:
        return AVEY_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _ws(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def kernel_launches() -> int:
    return int(lib().avey_kernel_launches())


class KernelTrace:
    """Per-kernel device times of the library's launches on the current stream.

    ``with KernelTrace(capacity) as tr: ...`` has the library record one of its
    own CUDA events before the block and one after every kernel it enqueues
    inside it (avey_trace_begin / avey_trace_end); after a synchronize,
    ``tr.kernels()`` gives [(name, ms)] in launch order.  For launches on one
    stream only.
    """

    def __init__(self, capacity: int = 256):
        self.capacity = int(capacity)
        self.count = 0
        self.names: List[str] = []

    def __enter__(self):
        _check("avey_trace_begin", lib().avey_trace_begin(self.capacity, _stream()))
        return self

    def __exit__(self, *exc):
        n = int(lib().avey_trace_end())
        if n < 0:
            raise AveyError("avey_trace_end", 3, lib().avey_last_error_detail().decode())
        if n > self.capacity:
            raise RuntimeError(f"kernel trace overflow: {n} launches, capacity {self.capacity}")
        self.count = n
        self.names = [lib().avey_trace_kernel_name(i).decode() for i in range(n)]
        return False

    def kernels(self):
        """[(name, ms)] of every traced launch (call after a synchronize)."""
        out = []
        ms = ctypes.c_float()
        for i in range(self.count):
            _check("avey_trace_kernel_ms", lib().avey_trace_kernel_ms(i, ctypes.byref(ms)))
            out.append((self.names[i], float(ms.value)))
        return out


def device_status(stream=None) -> int:
    s = _stream() if stream is None else ctypes.c_void_p(stream)
    return int(lib().avey_device_status(s))


# ------------------------------------------------------------------ ranker --

def rank_workspace_bytes(dtype: int, B: int, N: int, d: int, S: int) -> int:
    return int(lib().avey_rank_workspace_bytes(dtype, B, N, d, S))


def avey_rank(x: torch.Tensor, S: int, k: int, return_scores: bool = False,
              ws: Optional[torch.Tensor] = None, causal: bool = False):
    """x [B, N, d] fp32 or bf16 -> (idx int32 [B, n, k], w fp32 [B, n, k][, scores]).

    causal: candidates only the preceding splits (AVEY_RANK_UNIDIRECTIONAL).
    """
    _need(x, "x")
    B, N, d = x.shape
    n = -(-N // S)
    dt = _dt(x)
    idx = torch.empty((B, n, k), dtype=torch.int32, device=x.device)
    w = torch.empty((B, n, k), dtype=torch.float32, device=x.device)
    scores = torch.empty((B, n, n), dtype=torch.float32, device=x.device) if return_scores else None
    need = rank_workspace_bytes(dt, B, N, d, S)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    flags = AVEY_RANK_UNIDIRECTIONAL if causal else 0
    _check("avey_rank", lib().avey_rank_ex(_ptr(x), dt, B, N, d, S, k, flags, _ptr(idx), _ptr(w),
                                           _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return (idx, w, scores) if return_scores else (idx, w)


def avey_topk(scores: torch.Tensor, k: int, causal: bool = False):
    """Top-k selection and weights from precomputed scores [B, n, n] fp32."""
    _need(scores, "scores")
    if scores.dtype != torch.float32 or scores.dim() != 3 or scores.shape[1] != scores.shape[2]:
        raise TypeError("scores must be fp32 [B, n, n]")
    B, n, _ = scores.shape
    idx = torch.empty((B, n, k), dtype=torch.int32, device=scores.device)
    w = torch.empty((B, n, k), dtype=torch.float32, device=scores.device)
    flags = AVEY_RANK_UNIDIRECTIONAL if causal else 0
    _check("avey_topk", lib().avey_topk(_ptr(scores), B, n, k, flags, _ptr(idx), _ptr(w), _stream()))
    return idx, w


# ------------------------------------------------------------- compression --

def avey_compress(x: torch.Tensor, S: int, k: int, idx: torch.Tensor, w: torch.Tensor,
                  P: torch.Tensor, out: Optional[torch.Tensor] = None, lowp: bool = True):
    """eq. 8 compression + residual.  Returns (out fp32 [B, n*S, d], pair or None).

    For bf16 inputs the pair is the split activation [2, B*n*S, d] bf16.
    """
    for t, nm in ((x, "x"), (idx, "idx"), (w, "w"), (P, "P")):
        _need(t, nm)
    B, N, d = x.shape
    n = -(-N // S)
    dt = _dt(x)
    if P.dtype != x.dtype:
        raise TypeError("P must have the dtype of x")
    if out is None:
        out = torch.empty((B, n * S, d), dtype=torch.float32, device=x.device)
    pair = None
    if dt == AVEY_BF16 and lowp:
        pair = torch.empty((2, B * n * S, d), dtype=torch.bfloat16, device=x.device)
    _check("avey_compress", lib().avey_compress(_ptr(x), dt, B, N, d, S, k, _ptr(idx), _ptr(w),
                                                _ptr(P), _ptr(out), _ptr(pair), _stream()))
    return out, pair


def avey_context(x: torch.Tensor, S: int, k: int, idx: torch.Tensor, w: torch.Tensor,
                 out: Optional[torch.Tensor] = None, lowp: bool = True):
    """Uncompressed context [X_t ; w_1 X_c1 ; ... ; w_k X_ck] of every split.

    Returns (out fp32 [B, n, (k+1)S, d], pair [2, B*n*(k+1)S, d] bf16 or None).
    """
    for t, nm in ((x, "x"), (idx, "idx"), (w, "w")):
        _need(t, nm)
    B, N, d = x.shape
    n = -(-N // S)
    dt = _dt(x)
    L = (k + 1) * S
    if out is None:
        out = torch.empty((B, n, L, d), dtype=torch.float32, device=x.device)
    pair = None
    if dt == AVEY_BF16 and lowp:
        pair = torch.empty((2, B * n * L, d), dtype=torch.bfloat16, device=x.device)
    _check("avey_context", lib().avey_context(_ptr(x), dt, B, N, d, S, k, _ptr(idx), _ptr(w),
                                              _ptr(out), _ptr(pair), _stream()))
    return out, pair


# ------------------------------------------------------------- dynamic mix --

def avey_dynamic_mix(zt: torch.Tensor, S: int, eps: float, mt: Optional[int] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dynamic contextualizer on split blocks.

    zt: fp32 [rows, ld] or a bf16 split pair [2, rows, ld]; rows = blocks * S;
    the first ``mt`` (default ld) columns are mixed.  Returns out (same layout).
    """
    _need(zt, "zt")
    if zt.dtype == torch.float32:
        dt, rows, ld = AVEY_F32, zt.shape[0], zt.shape[1]
    elif zt.dtype == torch.bfloat16 and zt.dim() == 3 and zt.shape[0] == 2:
        dt, rows, ld = AVEY_BF16X2, zt.shape[1], zt.shape[2]
    else:
        raise TypeError("zt must be fp32 [rows, ld] or a bf16 pair [2, rows, ld]")
    mt = ld if mt is None else mt
    if out is None:
        out = torch.empty_like(zt)
    _need(out, "out")
    _check("avey_dynamic_mix", lib().avey_dynamic_mix(_ptr(zt), ld, dt, rows // S, S, mt, eps,
                                                      _ptr(out), out.shape[-1], _stream()))
    return out


def avey_static_mix(V: torch.Tensor, zt: torch.Tensor, S: int, mt: Optional[int] = None,
                    out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Static contextualizer c = V Z_t on split blocks (layouts as avey_dynamic_mix)."""
    _need(zt, "zt")
    _need(V, "V")
    if zt.dtype == torch.float32:
        dt, rows, ld = AVEY_F32, zt.shape[0], zt.shape[1]
    elif zt.dtype == torch.bfloat16 and zt.dim() == 3 and zt.shape[0] == 2:
        dt, rows, ld = AVEY_BF16X2, zt.shape[1], zt.shape[2]
    else:
        raise TypeError("zt must be fp32 [rows, ld] or a bf16 pair [2, rows, ld]")
    mt = ld if mt is None else mt
    if out is None:
        out = torch.empty_like(zt)
    _need(out, "out")
    _check("avey_static_mix", lib().avey_static_mix(_ptr(V), _ptr(zt), ld, dt, rows // S, S, mt,
                                                    _ptr(out), out.shape[-1], _stream()))
    return out


# ------------------------------------------------------------------ layer --

@dataclass
class DeviceLayer:
    """Device copies of one layer's weights in the layout the library takes."""
    kind: int
    Ut: torch.Tensor  # [m, d] (U transposed), bf16 or fp32
    bU: torch.Tensor  # [m] fp32
    V: Optional[torch.Tensor]  # [S, S] or None
    Ot: torch.Tensor  # [d, m] (O transposed)


def layer_workspace_bytes(dtype: int, T: int, d: int, m: int, prenorm: bool, S: int = 0,
                          kind: int = 1) -> int:
    """Workspace of one layer; S > 128 (blocks of (k+1)S tokens) adds what a
    dynamic layer over such blocks needs."""
    if S > 128:
        return int(lib().avey_layer_workspace_bytes_ex(dtype, T, d, m, int(bool(prenorm)), S, kind))
    return int(lib().avey_layer_workspace_bytes(dtype, T, d, m, int(bool(prenorm))))


def avey_layer_forward(layer: DeviceLayer, S: int, m_h: int, eps: float, prenorm: bool,
                       x_in: Optional[torch.Tensor], x_in_lowp: Optional[torch.Tensor] = None,
                       x_out: Optional[torch.Tensor] = None, lowp_out: bool = True,
                       x_out_lowp: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, fp32_out: bool = True,
                       x_in_rms: Optional[torch.Tensor] = None,
                       x_out_rms: Optional[torch.Tensor] = None):
    """One layer on x_in fp32 [T, d] (any leading shape that flattens to T rows).

    For a bf16 layer, x_in may be None when x_in_lowp (the split pair
    [2, T, d]) is given: the residual is then hi + lo.  fp32_out=False writes
    only the pair.  x_in_rms / x_out_rms (fp32 [T], optional): the prenorm
    row scales of x_in (used instead of computing them) and of x_out (written),
    as avey_layer_forward_ex takes them.  Returns (x_out fp32 or None,
    x_out_lowp pair or None).
    """
    m = layer.Ut.shape[0]
    dt = _dt(layer.Ut)
    if x_in is None:
        _need(x_in_lowp, "x_in_lowp")
        d = x_in_lowp.shape[-1]
        T = x_in_lowp.numel() // (2 * d)
        dev = x_in_lowp.device
    else:
        _need(x_in, "x_in")
        d = x_in.shape[-1]
        T = x_in.numel() // d
        dev = x_in.device
    if x_out is None and fp32_out:
        x_out = torch.empty_like(x_in) if x_in is not None else torch.empty((T, d), device=dev)
    if dt == AVEY_BF16 and lowp_out and x_out_lowp is None:
        x_out_lowp = torch.empty((2, T, d), dtype=torch.bfloat16, device=dev)
    need = layer_workspace_bytes(dt, T, d, m, prenorm, S, layer.kind)
    if ws is None or ws.numel() < need:
        ws = _ws(need, dev)
    p = LayerParams(layer.kind, d, m, m_h, S, eps, int(bool(prenorm)), layer.Ut.data_ptr(),
                    layer.bU.data_ptr(), None if layer.V is None else layer.V.data_ptr(),
                    layer.Ot.data_ptr())
    for t, nm in ((x_in_rms, "x_in_rms"), (x_out_rms, "x_out_rms")):
        if t is not None:
            _need(t, nm)
            if t.dtype != torch.float32 or t.numel() != T:
                raise TypeError(f"{nm} must be fp32 with T = {T} entries")
    _check("avey_layer_forward",
           lib().avey_layer_forward_ex(ctypes.byref(p), dt, T, _ptr(x_in), _ptr(x_in_lowp),
                                       _ptr(x_in_rms), _ptr(x_out),
                                       _ptr(x_out_lowp if dt == AVEY_BF16 else None), _ptr(x_out_rms),
                                       _ptr(ws), ws.numel(), _stream()))
    return x_out, (x_out_lowp if dt == AVEY_BF16 else None)


def device_layers(weights, dtype: torch.dtype, device) -> List[DeviceLayer]:
    """Device copies of host weights (U [d, m], bU, V, O [m, d] numpy arrays)."""
    out = []
    for lw in weights.layers:
        Ut = torch.from_numpy(lw.U.T.copy()).to(device=device, dtype=dtype).contiguous()
        Ot = torch.from_numpy(lw.O.T.copy()).to(device=device, dtype=dtype).contiguous()
        bU = torch.from_numpy(lw.bU).to(device=device, dtype=torch.float32).contiguous()
        V = None if lw.V is None else torch.from_numpy(lw.V).to(device=device, dtype=dtype).contiguous()
        out.append(DeviceLayer(int(lw.kind), Ut, bU, V, Ot))
    return out


@dataclass
class EncoderWorkspace:
    """Preallocated buffers for encoder_forward at one shape (reused per call)."""
    rank_ws: torch.Tensor
    layer_ws: torch.Tensor
    idx: torch.Tensor
    w: torch.Tensor
    x0: torch.Tensor
    x1: torch.Tensor
    pair0: Optional[torch.Tensor]
    pair1: Optional[torch.Tensor]
    rms0: Optional[torch.Tensor] = None  # per-row prenorm scales handed between layers
    rms1: Optional[torch.Tensor] = None


def make_workspace(B: int, N: int, d: int, S: int, k: int, m: int, dtype: torch.dtype, prenorm: bool,
                   device, uncompressed: bool = False) -> EncoderWorkspace:
    """Buffers for encoder_forward, or (uncompressed=True) for
    encoder_forward_uncompressed, whose layers run on B*n*(k+1)S tokens."""
    n = -(-N // S)
    blk = (k + 1) * S if uncompressed else S
    T = B * n * blk
    dt = AVEY_BF16 if dtype == torch.bfloat16 else AVEY_F32
    rank_ws = _ws(rank_workspace_bytes(dt, B, N, d, S), device)
    layer_ws = _ws(layer_workspace_bytes(dt, T, d, m, prenorm, blk, AVEY_DYNAMIC), device)
    idx = torch.empty((B, n, k), dtype=torch.int32, device=device)
    w = torch.empty((B, n, k), dtype=torch.float32, device=device)
    x0 = torch.empty((T, d), dtype=torch.float32, device=device)
    x1 = torch.empty((T, d), dtype=torch.float32, device=device)
    pair0 = pair1 = None
    if dt == AVEY_BF16:
        pair0 = torch.empty((2, T, d), dtype=torch.bfloat16, device=device)
        pair1 = torch.empty((2, T, d), dtype=torch.bfloat16, device=device)
    rms0 = rms1 = None
    if prenorm:
        rms0 = torch.empty((T,), dtype=torch.float32, device=device)
        rms1 = torch.empty((T,), dtype=torch.float32, device=device)
    return EncoderWorkspace(rank_ws, layer_ws, idx, w, x0, x1, pair0, pair1, rms0, rms1)


def _pair_stream(dt: int, layers) -> bool:
    """bf16 stacks pass the residual stream between the calls as its split pair
    alone; fp32 is written once, by the last layer."""
    return dt == AVEY_BF16 and len(layers) > 0


def _run_layers(L, layers, dt, T, d, m, m_h, S, eps, prenorm, ws, st, marks):
    """Every layer over the stream in (ws.x0, ws.pair0); returns the fp32 output
    buffer.  ``marks[3 + li]`` is recorded after layer li.  With prenorm, each
    layer but the last also writes its output's row scales for the next one."""
    pair_only = _pair_stream(dt, layers)
    hand_rms = bool(prenorm) and ws.rms0 is not None
    cur, nxt = (ws.x0, ws.pair0, ws.rms0), (ws.x1, ws.pair1, ws.rms1)
    for li, lay in enumerate(layers):
        last = li == len(layers) - 1
        p = LayerParams(lay.kind, d, m, m_h, S, eps, int(bool(prenorm)), lay.Ut.data_ptr(),
                        lay.bU.data_ptr(), None if lay.V is None else lay.V.data_ptr(),
                        lay.Ot.data_ptr())
        x_in = None if pair_only else _ptr(cur[0])
        x_out = _ptr(nxt[0]) if (last or not pair_only) else None
        x_out_lowp = None if (last and pair_only) else _ptr(nxt[1])
        rms_in = _ptr(cur[2]) if (hand_rms and li > 0) else None
        rms_out = _ptr(nxt[2]) if (hand_rms and not last) else None
        _check("avey_layer_forward",
               L.avey_layer_forward_ex(ctypes.byref(p), dt, T, x_in, _ptr(cur[1]), rms_in, x_out,
                                       x_out_lowp, rms_out, _ptr(ws.layer_ws), ws.layer_ws.numel(),
                                       st))
        if marks is not None:
            marks[3 + li].record()
        cur, nxt = nxt, cur
    return cur[0]


def encoder_forward(x: torch.Tensor, P: torch.Tensor, layers: Sequence[DeviceLayer], S: int, k: int,
                    m_h: int, eps: float, prenorm: bool,
                    ws: Optional[EncoderWorkspace] = None, marks=None,
                    causal: bool = False) -> torch.Tensor:
    """Ranker once, compression, then every layer (Avey-B paperlayer summary
    App. H: the ranker runs once per forward).  Returns fp32 [B, n*S, d].

    ``marks``: optional list of 3 + len(layers) torch.cuda.Event, recorded on
    the current stream before the ranker and after every C-ABI call.
    """
    B, N, d = x.shape
    m = layers[0].Ut.shape[0] if layers else d
    if ws is None:
        ws = make_workspace(B, N, d, S, k, m, x.dtype, prenorm, x.device)
    dt = _dt(x)
    L = lib()
    st = _stream()
    if marks is not None:
        marks[0].record()
    flags = AVEY_RANK_UNIDIRECTIONAL if causal else 0
    _check("avey_rank", L.avey_rank_ex(_ptr(x), dt, B, N, d, S, k, flags, _ptr(ws.idx),
                                       _ptr(ws.w), None, _ptr(ws.rank_ws), ws.rank_ws.numel(), st))
    if marks is not None:
        marks[1].record()
    return processor_forward(x, P, layers, S, k, m_h, eps, prenorm, ws.idx, ws.w, ws, marks)


def processor_forward(x: torch.Tensor, P: torch.Tensor, layers: Sequence[DeviceLayer], S: int,
                      k: int, m_h: int, eps: float, prenorm: bool, idx: torch.Tensor,
                      w: torch.Tensor, ws: Optional[EncoderWorkspace] = None,
                      marks=None) -> torch.Tensor:
    """Compression and every layer for a given selection (idx int32 [B, n, k],
    w fp32 [B, n, k], as avey_rank returns them): the part of the forward after
    the ranker, for a caller that ranks by other means.  Returns fp32
    [B, n*S, d].  ``marks[2 + i]`` is recorded after compression (i = 0) and
    after every layer.
    """
    B, N, d = x.shape
    n = -(-N // S)
    T = B * n * S
    dt = _dt(x)
    m = layers[0].Ut.shape[0] if layers else d
    if ws is None:
        ws = make_workspace(B, N, d, S, k, m, x.dtype, prenorm, x.device)
    for t, nm in ((idx, "idx"), (w, "w")):
        _need(t, nm)
        if t.numel() != B * n * k:
            raise ValueError(f"{nm} must have B*n*k = {B * n * k} entries")
    if idx.dtype != torch.int32 or w.dtype != torch.float32:
        raise TypeError("idx must be int32 and w fp32")
    L = lib()
    st = _stream()
    _check("avey_compress", L.avey_compress(_ptr(x), dt, B, N, d, S, k, _ptr(idx), _ptr(w),
                                            _ptr(P), None if _pair_stream(dt, layers) else _ptr(ws.x0),
                                            _ptr(ws.pair0), st))
    if marks is not None:
        marks[2].record()
    out = _run_layers(L, layers, dt, T, d, m, m_h, S, eps, prenorm, ws, st, marks)
    return out.view(B, n * S, d)


def encoder_forward_uncompressed(x: torch.Tensor, layers: Sequence[DeviceLayer], S: int, k: int,
                                 m_h: int, eps: float, prenorm: bool,
                                 ws: Optional[EncoderWorkspace] = None, marks=None,
                                 causal: bool = False) -> torch.Tensor:
    """The processor without neural compression (Avey-B paperlayer summary
    §4.3): ranker once, then each split's (k+1)S-token context
    [X_t ; w_1 X_c1 ; ... ; w_k X_ck] goes through every layer as one block
    (the layers' V are (k+1)S x (k+1)S).  Returns fp32 [B, n, S, d], the first
    S rows of every block (a view).

    ``marks``: optional list of 3 + len(layers) torch.cuda.Event, recorded on
    the current stream before the ranker and after every C-ABI call.
    """
    B, N, d = x.shape
    m = layers[0].Ut.shape[0] if layers else d
    if ws is None:
        ws = make_workspace(B, N, d, S, k, m, x.dtype, prenorm, x.device, uncompressed=True)
    dt = _dt(x)
    L = lib()
    st = _stream()
    if marks is not None:
        marks[0].record()
    _check("avey_rank", L.avey_rank_ex(_ptr(x), dt, B, N, d, S, k,
                                       AVEY_RANK_UNIDIRECTIONAL if causal else 0, _ptr(ws.idx),
                                       _ptr(ws.w), None, _ptr(ws.rank_ws), ws.rank_ws.numel(), st))
    if marks is not None:
        marks[1].record()
    return processor_forward_uncompressed(x, layers, S, k, m_h, eps, prenorm, ws.idx, ws.w, ws,
                                          marks)


def processor_forward_uncompressed(x: torch.Tensor, layers: Sequence[DeviceLayer], S: int, k: int,
                                   m_h: int, eps: float, prenorm: bool, idx: torch.Tensor,
                                   w: torch.Tensor, ws: Optional[EncoderWorkspace] = None,
                                   marks=None) -> torch.Tensor:
    """The uncompressed processor for a given selection (idx int32 [B, n, k],
    w fp32 [B, n, k]): every split's context through every layer.  Returns
    fp32 [B, n, S, d] (a view); ``marks`` as in processor_forward."""
    B, N, d = x.shape
    n = -(-N // S)
    L_ = (k + 1) * S
    T = B * n * L_
    dt = _dt(x)
    m = layers[0].Ut.shape[0] if layers else d
    if ws is None:
        ws = make_workspace(B, N, d, S, k, m, x.dtype, prenorm, x.device, uncompressed=True)
    for t, nm in ((idx, "idx"), (w, "w")):
        _need(t, nm)
        if t.numel() != B * n * k:
            raise ValueError(f"{nm} must have B*n*k = {B * n * k} entries")
    if idx.dtype != torch.int32 or w.dtype != torch.float32:
        raise TypeError("idx must be int32 and w fp32")
    L = lib()
    st = _stream()
    _check("avey_context", L.avey_context(_ptr(x), dt, B, N, d, S, k, _ptr(idx), _ptr(w),
                                          _ptr(ws.x0), _ptr(ws.pair0), st))
    if marks is not None:
        marks[2].record()
    cur, nxt = (ws.x0, ws.pair0), (ws.x1, ws.pair1)
    for li, lay in enumerate(layers):
        p = LayerParams(lay.kind, d, m, m_h, L_, eps, int(bool(prenorm)), lay.Ut.data_ptr(),
                        lay.bU.data_ptr(), None if lay.V is None else lay.V.data_ptr(),
                        lay.Ot.data_ptr())
        _check("avey_layer_forward",
               L.avey_layer_forward(ctypes.byref(p), dt, T, _ptr(cur[0]), _ptr(cur[1]),
                                    _ptr(nxt[0]), _ptr(nxt[1]), _ptr(ws.layer_ws),
                                    ws.layer_ws.numel(), st))
        if marks is not None:
            marks[3 + li].record()
        cur, nxt = nxt, cur
    return cur[0].view(B, n, L_, d)[:, :, :S, :]


# ------------------------------------------- one sequence across several GPUs --

def shard_targets(n: int, world: int, rank: int):
    """Contiguous, balanced target-split range [t0, t1) of ``rank``."""
    base, extra = divmod(n, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def avey_maxsim_part(x: torch.Tensor, S: int, part: int, nparts: int, scores: torch.Tensor,
                     ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Adds part ``part`` of ``nparts`` of the split scores into the zeroed
    ``scores`` [B, n, n] (its entries only; see include/avey.h)."""
    _need(x, "x")
    _need(scores, "scores")
    B, N, d = x.shape
    dt = _dt(x)
    need = rank_workspace_bytes(dt, B, N, d, S)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    _check("avey_maxsim_part", lib().avey_maxsim_part(_ptr(x), dt, B, N, d, S, part, nparts,
                                                      _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return scores


@dataclass
class ShardWorkspace:
    """Buffers of encoder_forward_sharded for one rank at one shape."""
    t0: int
    t1: int
    rank_ws: torch.Tensor
    scores: torch.Tensor
    layer_ws: torch.Tensor
    idx: torch.Tensor
    w: torch.Tensor
    x0: torch.Tensor
    x1: torch.Tensor
    pair0: Optional[torch.Tensor]
    pair1: Optional[torch.Tensor]
    rms0: Optional[torch.Tensor] = None  # per-row prenorm scales handed between layers
    rms1: Optional[torch.Tensor] = None


def make_shard_workspace(B: int, N: int, d: int, S: int, k: int, m: int, dtype: torch.dtype,
                         prenorm: bool, rank: int, world: int, device) -> ShardWorkspace:
    n = -(-N // S)
    t0, t1 = shard_targets(n, world, rank)
    T = B * (t1 - t0) * S
    dt = AVEY_BF16 if dtype == torch.bfloat16 else AVEY_F32
    pair = lambda: (torch.empty((2, T, d), dtype=torch.bfloat16, device=device)
                    if dt == AVEY_BF16 else None)
    rms = (lambda: torch.empty((max(T, 1),), dtype=torch.float32, device=device)
           if prenorm else None)
    return ShardWorkspace(
        t0, t1, _ws(rank_workspace_bytes(dt, B, N, d, S), device),
        torch.empty((B, n, n), dtype=torch.float32, device=device),
        _ws(layer_workspace_bytes(dt, max(T, S), d, m, prenorm), device),
        torch.empty((B, t1 - t0, k), dtype=torch.int32, device=device),
        torch.empty((B, t1 - t0, k), dtype=torch.float32, device=device),
        torch.empty((max(T, 1), d), dtype=torch.float32, device=device),
        torch.empty((max(T, 1), d), dtype=torch.float32, device=device), pair(), pair(), rms(),
        rms())


def encoder_forward_sharded(x: torch.Tensor, P: torch.Tensor, layers: Sequence[DeviceLayer], S: int,
                            k: int, m_h: int, eps: float, prenorm: bool, rank: int, world: int,
                            allreduce, ws: Optional[ShardWorkspace] = None, marks=None,
                            causal: bool = False) -> torch.Tensor:
    """One long sequence (or batch) split across ``world`` GPUs; this is rank
    ``rank``'s share.  Every rank holds the whole input x.

    1. MaxSim: the triangular tiles are dealt round-robin; this rank writes its
       tiles' entries into zeroed scores, and ``allreduce(scores)`` (an
       in-place sum over the ranks, e.g. torch.distributed.all_reduce) makes
       every rank's scores the full matrix: the one exchange step.
    2. Top-k, compression and every layer for this rank's target splits
       [t0, t1) only (each split's processing is independent).
    Returns fp32 [B, (t1-t0)*S, d], the rows of targets t0 .. t1-1.

    ``marks``: optional list of 3 + len(layers) torch.cuda.Event, recorded
    before MaxSim, after the all-reduce, after compression and after every layer.
    """
    B, N, d = x.shape
    dt = _dt(x)
    if dt != AVEY_BF16:
        raise TypeError("the sharded forward takes bf16 embeddings")
    n = -(-N // S)
    m = layers[0].Ut.shape[0] if layers else d
    if ws is None:
        ws = make_shard_workspace(B, N, d, S, k, m, x.dtype, prenorm, rank, world, x.device)
    L = lib()
    st = _stream()
    if marks is not None:
        marks[0].record()
    ws.scores.zero_()
    _check("avey_maxsim_part", L.avey_maxsim_part(_ptr(x), dt, B, N, d, S, rank, world,
                                                  _ptr(ws.scores), _ptr(ws.rank_ws),
                                                  ws.rank_ws.numel(), st))
    allreduce(ws.scores)
    if marks is not None:
        marks[1].record()
    t0, t1 = ws.t0, ws.t1
    T = B * (t1 - t0) * S
    if T == 0:
        return ws.x0[:0].view(B, 0, d)
    flags = AVEY_RANK_UNIDIRECTIONAL if causal else 0
    _check("avey_topk_rows", L.avey_topk_rows(_ptr(ws.scores), B, n, t0, t1, k, flags, _ptr(ws.idx),
                                              _ptr(ws.w), st))
    _check("avey_compress_rows", L.avey_compress_rows(
        _ptr(x), dt, B, N, d, S, k, t0, t1, _ptr(ws.idx), _ptr(ws.w), _ptr(P),
        None if _pair_stream(dt, layers) else _ptr(ws.x0), _ptr(ws.pair0), st))
    if marks is not None:
        marks[2].record()
    out = _run_layers(L, layers, dt, T, d, m, m_h, S, eps, prenorm, ws, st, marks)
    return out[:T].view(B, (t1 - t0) * S, d)
