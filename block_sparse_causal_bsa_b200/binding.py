"""ctypes binding of libbsa.so (the C ABI in include/bsa.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream. There is no CPU
fallback; if the library is missing or fails to load, calls raise.

The raw entry points keep the C names (``bsa_score``, ``bsa_select``,
``bsa_attend``, ``bsa_decode`` and the sizing helpers) and take torch tensors
or raw pointers; ``score``/``select``/``attend``/``decode``/``prefill`` allocate
outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

BSA_OK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA = 0, 1, 2, 3
BSA_DEV_OK, BSA_DEV_BAD_INDEX, BSA_DEV_TIMEOUT, BSA_DEV_BAD_SCORE = 0, 1, 2, 4
BSA_BF16, BSA_F32 = 0, 1
BSA_SCORE_MEAN, BSA_SCORE_MEAN_VNORM, BSA_SCORE_MEAN_VLOG, BSA_SCORE_KMINMAX = 0, 1, 2, 3
BSA_PATH_CUDA_CORES, BSA_PATH_TENSOR_CORES = 0, 1
SCORE_KINDS = {"mean": BSA_SCORE_MEAN, "vnorm": BSA_SCORE_MEAN_VNORM, "vlog": BSA_SCORE_MEAN_VLOG,
               "kminmax": BSA_SCORE_KMINMAX}

EXPORTS = ("bsa_score_workspace_bytes", "bsa_score", "bsa_kv_idx_width",
           "bsa_select_workspace_bytes", "bsa_select", "bsa_attend", "bsa_decode",
           "bsa_status_string", "bsa_last_error", "bsa_select_noalloc_max_bytes",
           "bsa_select_noalloc", "bsa_selftest_wait", "bsa_decode_list", "bsa_score_ex",
           "bsa_attend_vs_workspace_bytes", "bsa_attend_vs", "bsa_score_select_workspace_bytes",
           "bsa_score_select", "bsa_score_path", "bsa_attend_path", "bsa_decode_path")


class BsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libbsa status {status}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("block_k", ctypes.c_int),
                ("tile_q", ctypes.c_int), ("dtype", ctypes.c_int)]


class ScoreParams(ctypes.Structure):
    _fields_ = [("beta", ctypes.c_float)]


class SelectParams(ctypes.Structure):
    _fields_ = [("k_first", ctypes.c_int), ("k_last", ctypes.c_int), ("rho", ctypes.c_int),
                ("gate_quantile", ctypes.c_float), ("gate_threshold", ctypes.c_float)]


class DecodeShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("L", ctypes.c_int), ("d", ctypes.c_int), ("block_kv", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("tau", ctypes.c_float), ("phi", ctypes.c_float), ("patience", ctypes.c_int),
                ("enable", ctypes.c_int), ("n_probe", ctypes.c_int),
                ("probe_dims", ctypes.POINTER(ctypes.c_int))]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbsa.so (built by ``block_sparse_causal_bsa_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run python -m block_sparse_causal_bsa_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32p, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
        sp, pp = ctypes.POINTER(Shape), ctypes.POINTER(SelectParams)
        dsp, dpp = ctypes.POINTER(DecodeShape), ctypes.POINTER(DecodeParams)
        L.bsa_score_workspace_bytes.argtypes = [sp, ctypes.c_int]
        L.bsa_score_workspace_bytes.restype = sz
        L.bsa_score.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, i32p, vp, sz, vp]
        L.bsa_score.restype = ctypes.c_int
        L.bsa_score_ex.argtypes = [sp, ctypes.c_int, ctypes.POINTER(ScoreParams), vp, vp, vp, vp, i32p,
                                   vp, sz, vp]
        L.bsa_score_ex.restype = ctypes.c_int
        L.bsa_kv_idx_width.argtypes = [sp, pp]
        L.bsa_kv_idx_width.restype = ctypes.c_int
        L.bsa_select_workspace_bytes.argtypes = [sp, pp]
        L.bsa_select_workspace_bytes.restype = sz
        L.bsa_select.argtypes = [sp, pp, vp, i32p, i32p, vp, vp, vp, vp, i32p, vp, sz, vp]
        L.bsa_select.restype = ctypes.c_int
        L.bsa_attend.argtypes = [sp, vp, vp, vp, i32p, i32p, ctypes.c_int, ctypes.c_float, vp, vp,
                                 i32p, vp]
        L.bsa_attend.restype = ctypes.c_int
        L.bsa_decode.argtypes = [dsp, dpp, vp, vp, vp, ctypes.c_float, vp, i32p, vp, i32p, vp]
        L.bsa_decode.restype = ctypes.c_int
        L.bsa_decode_list.argtypes = [dsp, dpp, vp, vp, vp, i32p, i32p, ctypes.c_int, ctypes.c_float,
                                      vp, i32p, vp, i32p, vp]
        L.bsa_decode_list.restype = ctypes.c_int
        L.bsa_score_select_workspace_bytes.argtypes = [sp, ctypes.c_int, pp]
        L.bsa_score_select_workspace_bytes.restype = sz
        L.bsa_score_select.argtypes = [sp, ctypes.c_int, ctypes.POINTER(ScoreParams), pp, vp, vp, vp, vp,
                                       i32p, i32p, vp, vp, vp, vp, i32p, vp, sz, vp]
        L.bsa_score_select.restype = ctypes.c_int
        L.bsa_select_noalloc_max_bytes.argtypes = []
        L.bsa_select_noalloc_max_bytes.restype = sz
        L.bsa_select_noalloc.argtypes = [sp, pp, vp, i32p, i32p, vp, vp, vp, vp, i32p, vp]
        L.bsa_select_noalloc.restype = ctypes.c_int
        L.bsa_attend_vs_workspace_bytes.argtypes = [sp, ctypes.c_int, ctypes.c_int]
        L.bsa_attend_vs_workspace_bytes.restype = sz
        L.bsa_attend_vs.argtypes = [sp, vp, vp, vp, i32p, i32p, ctypes.c_int, i32p, i32p, ctypes.c_int,
                                    ctypes.c_float, vp, vp, i32p, vp, sz, vp]
        L.bsa_attend_vs.restype = ctypes.c_int
        L.bsa_selftest_wait.argtypes = [ctypes.c_int, i32p, i32p, vp]
        L.bsa_selftest_wait.restype = ctypes.c_int
        L.bsa_score_path.argtypes = [sp, ctypes.c_int]
        L.bsa_score_path.restype = ctypes.c_int
        L.bsa_attend_path.argtypes = [sp, ctypes.c_int]
        L.bsa_attend_path.restype = ctypes.c_int
        L.bsa_decode_path.argtypes = [dsp]
        L.bsa_decode_path.restype = ctypes.c_int
        L.bsa_status_string.argtypes = [ctypes.c_int]
        L.bsa_status_string.restype = ctypes.c_char_p
        L.bsa_last_error.argtypes = []
        L.bsa_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != BSA_OK:
        raise BsaError(status, lib().bsa_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BSA_BF16
    if t.dtype == torch.float32:
        return BSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


@dataclasses.dataclass
class SelectConfig:
    """Selection parameters (mirrors bsa_select_params)."""
    k_first: int
    k_last: Optional[int] = None
    rho: int = 1
    gate_quantile: float = 0.25
    gate_threshold: float = float("nan")

    def c(self) -> SelectParams:
        kl = self.k_first if self.k_last is None else self.k_last
        return SelectParams(self.k_first, kl, self.rho, self.gate_quantile, self.gate_threshold)


def make_shape(q: torch.Tensor, k: torch.Tensor, block_k: int, tile_q: int) -> Shape:
    B, Hq, N, d = q.shape
    return Shape(B, Hq, k.shape[1], N, d, block_k, tile_q, _dtype_code(q))


# ---------------------------------------------------------------------------
# raw entry points (C names)

def bsa_score_workspace_bytes(shape: Shape, kind: int) -> int:
    return lib().bsa_score_workspace_bytes(ctypes.byref(shape), kind)


def bsa_score(shape, kind, q, k, v, scores, dev_status, ws, ws_bytes, stream=None) -> None:
    _check(lib().bsa_score(ctypes.byref(shape), kind, _ptr(q), _ptr(k), _ptr(v), _ptr(scores),
                           _ptr(dev_status), _ptr(ws), ws_bytes, _stream(stream)))


def bsa_score_ex(shape, kind, params, q, k, v, scores, dev_status, ws, ws_bytes, stream=None) -> None:
    _check(lib().bsa_score_ex(ctypes.byref(shape), kind, ctypes.byref(params) if params is not None else None,
                              _ptr(q), _ptr(k), _ptr(v), _ptr(scores), _ptr(dev_status), _ptr(ws),
                              ws_bytes, _stream(stream)))


def bsa_kv_idx_width(shape: Shape, params: SelectParams) -> int:
    return lib().bsa_kv_idx_width(ctypes.byref(shape), ctypes.byref(params))


def bsa_select_workspace_bytes(shape: Shape, params: SelectParams) -> int:
    return lib().bsa_select_workspace_bytes(ctypes.byref(shape), ctypes.byref(params))


def bsa_select(shape, params, scores, kv_idx, kv_cnt, sigma, sigma_bar, trigger, theta,
               dev_status, ws, ws_bytes, stream=None) -> None:
    _check(lib().bsa_select(ctypes.byref(shape), ctypes.byref(params), _ptr(scores), _ptr(kv_idx),
                            _ptr(kv_cnt), _ptr(sigma), _ptr(sigma_bar), _ptr(trigger), _ptr(theta),
                            _ptr(dev_status), _ptr(ws), ws_bytes, _stream(stream)))


def bsa_score_select_workspace_bytes(shape: Shape, kind: int, params: SelectParams) -> int:
    return lib().bsa_score_select_workspace_bytes(ctypes.byref(shape), kind, ctypes.byref(params))


def bsa_score_select(shape, kind, score_params, params, q, k, v, scores, kv_idx, kv_cnt, sigma,
                     sigma_bar, trigger, theta, dev_status, ws, ws_bytes, stream=None) -> None:
    _check(lib().bsa_score_select(ctypes.byref(shape), kind,
                                  ctypes.byref(score_params) if score_params is not None else None,
                                  ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(scores),
                                  _ptr(kv_idx), _ptr(kv_cnt), _ptr(sigma), _ptr(sigma_bar),
                                  _ptr(trigger), _ptr(theta), _ptr(dev_status), _ptr(ws), ws_bytes,
                                  _stream(stream)))


def bsa_select_noalloc(shape, params, scores, kv_idx, kv_cnt, sigma, sigma_bar, trigger, theta,
                       dev_status, stream=None) -> None:
    """bsa_select with the library's static scratch instead of a workspace (no allocation)."""
    _check(lib().bsa_select_noalloc(ctypes.byref(shape), ctypes.byref(params), _ptr(scores),
                                    _ptr(kv_idx), _ptr(kv_cnt), _ptr(sigma), _ptr(sigma_bar),
                                    _ptr(trigger), _ptr(theta), _ptr(dev_status),
                                    _stream(stream)))


def bsa_score_path(shape: Shape, kind: int) -> int:
    return lib().bsa_score_path(ctypes.byref(shape), kind)


def bsa_attend_path(shape: Shape, W: int) -> int:
    return lib().bsa_attend_path(ctypes.byref(shape), int(W))


def bsa_decode_path(shape: DecodeShape) -> int:
    return lib().bsa_decode_path(ctypes.byref(shape))


def bsa_attend_vs_workspace_bytes(shape: Shape, Wv: int, Ws: int) -> int:
    return lib().bsa_attend_vs_workspace_bytes(ctypes.byref(shape), int(Wv), int(Ws))


def bsa_attend_vs(shape, q, k, v, v_idx, v_cnt, Wv, s_off, s_cnt, Ws, scale, out, lse, dev_status, ws,
                  ws_bytes, stream=None) -> None:
    _check(lib().bsa_attend_vs(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(v_idx), _ptr(v_cnt),
                               int(Wv), _ptr(s_off), _ptr(s_cnt), int(Ws), scale, _ptr(out), _ptr(lse),
                               _ptr(dev_status), _ptr(ws), ws_bytes, _stream(stream)))


def bsa_selftest_wait(mode, dev_status, completed, stream=None) -> None:
    """Bounded-wait self-test: mode 0 lets a wait run out (BSA_DEV_TIMEOUT), mode 1 completes it."""
    _check(lib().bsa_selftest_wait(int(mode), _ptr(dev_status), _ptr(completed), _stream(stream)))


def bsa_attend(shape, q, k, v, kv_idx, kv_cnt, W, scale, out, lse, dev_status, stream=None) -> None:
    _check(lib().bsa_attend(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_idx),
                            _ptr(kv_cnt), W, scale, _ptr(out), _ptr(lse), _ptr(dev_status),
                            _stream(stream)))


def bsa_decode(shape, params, q, k_cache, v_cache, scale, out, blocks_used, probe_trace,
               dev_status, stream=None) -> None:
    _check(lib().bsa_decode(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k_cache),
                            _ptr(v_cache), scale, _ptr(out), _ptr(blocks_used), _ptr(probe_trace),
                            _ptr(dev_status), _stream(stream)))


def bsa_decode_list(shape, params, q, k_cache, v_cache, block_list, list_cnt, list_width, scale,
                    out, blocks_used, probe_trace, dev_status, stream=None) -> None:
    _check(lib().bsa_decode_list(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(block_list), _ptr(list_cnt), int(list_width),
                                 scale, _ptr(out), _ptr(blocks_used), _ptr(probe_trace),
                                 _ptr(dev_status), _stream(stream)))


# ---------------------------------------------------------------------------
# convenience wrappers (torch allocation + the raw calls)

def _empty_bytes(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)


def score(q, k, v=None, *, block_k: int, tile_q: int, output_aware: bool = False, stream=None,
          status: Optional[torch.Tensor] = None, kind: Optional[str] = None, beta: float = 0.0):
    """Block scores. kind: "mean", "vnorm" (output_aware=True), "vlog" (additive value
    term with weight beta) or "kminmax"."""
    shape = make_shape(q, k, block_k, tile_q)
    if kind is None:
        kind = "vnorm" if output_aware else "mean"
    code = SCORE_KINDS[kind]
    B, Hq, N, _ = q.shape
    scores = torch.empty(B, Hq, N // tile_q, N // block_k, dtype=torch.float32, device=q.device)
    nb = bsa_score_workspace_bytes(shape, code)
    ws = _empty_bytes(nb, q.device)
    uses_v = kind in ("vnorm", "vlog")
    bsa_score_ex(shape, code, ScoreParams(beta), q, k, v if uses_v else None, scores, status, ws, nb,
                 stream)
    return scores


def select(scores, *, shape: Shape, cfg: SelectConfig, stream=None):
    dev = scores.device
    p = cfg.c()
    W = bsa_kv_idx_width(shape, p)
    if W < 0:
        raise BsaError(BSA_ERR_INVALID_ARG, lib().bsa_last_error().decode())
    B, Hq, n_qt, _ = scores.shape
    r = dict(
        kv_idx=torch.empty(B, Hq, n_qt, W, dtype=torch.int32, device=dev),
        kv_cnt=torch.empty(B, Hq, n_qt, dtype=torch.int32, device=dev),
        sigma=torch.empty(B, Hq, n_qt, dtype=torch.float32, device=dev),
        sigma_bar=torch.empty(B, n_qt, dtype=torch.float32, device=dev),
        trigger=torch.empty(B, n_qt, dtype=torch.uint8, device=dev),
        theta=torch.empty(1, dtype=torch.float32, device=dev),
        dev_status=torch.zeros(1, dtype=torch.int32, device=dev),
        W=W)
    nb = bsa_select_workspace_bytes(shape, p)
    ws = _empty_bytes(nb, dev)
    bsa_select(shape, p, scores, r["kv_idx"], r["kv_cnt"], r["sigma"], r["sigma_bar"],
               r["trigger"], r["theta"], r["dev_status"], ws, nb, stream)
    return r


def attend(q, k, v, kv_idx, kv_cnt, *, block_k: int, tile_q: int, scale: Optional[float] = None,
           want_lse: bool = False, stream=None):
    shape = make_shape(q, k, block_k, tile_q)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    st = torch.zeros(1, dtype=torch.int32, device=q.device)
    bsa_attend(shape, q, k, v, kv_idx, kv_cnt, kv_idx.shape[-1], scale, out, lse, st, stream)
    return out, lse, st


def attend_vs(q, k, v, v_idx, v_cnt, s_off, s_cnt, *, scale: Optional[float] = None,
              want_lse: bool = False, stream=None):
    """Vertical-slash attention (bsa_attend_vs): v_idx [B,Hq,Wv], s_off [B,Hq,Ws] and
    their counts [B,Hq] as device int32 tensors. Returns (out, lse or None, status)."""
    shape = make_shape(q, k, 64, 128)
    Wv, Ws = v_idx.shape[-1], s_off.shape[-1]
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    nb = bsa_attend_vs_workspace_bytes(shape, Wv, Ws)
    if nb == 0:
        raise BsaError(BSA_ERR_UNSUPPORTED, lib().bsa_last_error().decode())
    ws = _empty_bytes(nb, q.device)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    st = torch.zeros(1, dtype=torch.int32, device=q.device)
    bsa_attend_vs(shape, q, k, v, v_idx, v_cnt, Wv, s_off, s_cnt, Ws, scale, out, lse, st, ws, nb, stream)
    return out, lse, st


def decode(q, k_cache, v_cache, *, block_kv: int, tau: float, phi: float, patience: int = 1,
           enable: bool = True, probe_dims: Sequence[int], scale: Optional[float] = None,
           want_trace: bool = False, block_list=None, list_cnt=None, stream=None):
    """Decode with run-time termination; with block_list [B,Hkv,W] / list_cnt [B,Hkv]
    (device int32) the listed blocks are visited in list order (bsa_decode_list)."""
    B, Hq, d = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    shape = DecodeShape(B, Hq, Hkv, L, d, block_kv, BSA_BF16)
    dims = (ctypes.c_int * len(probe_dims))(*[int(x) for x in probe_dims])
    params = DecodeParams(tau, phi, patience, int(enable), len(probe_dims), dims)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty_like(q)
    used = torch.empty(B, Hkv, dtype=torch.int32, device=q.device)
    steps = L // block_kv if block_list is None else block_list.shape[-1]
    trace = (torch.full((B, Hkv, steps, len(probe_dims)), float("nan"),
                        dtype=torch.float32, device=q.device) if want_trace else None)
    st = torch.zeros(1, dtype=torch.int32, device=q.device)
    if block_list is None:
        bsa_decode(shape, params, q, k_cache, v_cache, scale, out, used, trace, st, stream)
    else:
        bsa_decode_list(shape, params, q, k_cache, v_cache, block_list, list_cnt,
                        block_list.shape[-1], scale, out, used, trace, st, stream)
    return out, used, trace, st


def score_select(q, k, v=None, *, block_k: int, tile_q: int, cfg: SelectConfig, kind: str = "mean",
                 beta: float = 0.0, want_scores: bool = True, stream=None):
    """Scores and selection in one call (bsa_score_select). Returns the selection dict of
    ``select`` plus "scores" (None unless want_scores)."""
    shape = make_shape(q, k, block_k, tile_q)
    code = SCORE_KINDS[kind]
    p = cfg.c()
    dev = q.device
    W = bsa_kv_idx_width(shape, p)
    if W < 0:
        raise BsaError(BSA_ERR_INVALID_ARG, lib().bsa_last_error().decode())
    B, Hq, N, _ = q.shape
    n_qt, n_kb = N // tile_q, N // block_k
    r = dict(
        kv_idx=torch.empty(B, Hq, n_qt, W, dtype=torch.int32, device=dev),
        kv_cnt=torch.empty(B, Hq, n_qt, dtype=torch.int32, device=dev),
        sigma=torch.empty(B, Hq, n_qt, dtype=torch.float32, device=dev),
        sigma_bar=torch.empty(B, n_qt, dtype=torch.float32, device=dev),
        trigger=torch.empty(B, n_qt, dtype=torch.uint8, device=dev),
        theta=torch.empty(1, dtype=torch.float32, device=dev),
        dev_status=torch.zeros(1, dtype=torch.int32, device=dev),
        scores=(torch.empty(B, Hq, n_qt, n_kb, dtype=torch.float32, device=dev) if want_scores else None),
        W=W)
    nb = bsa_score_select_workspace_bytes(shape, code, p)
    if nb == 0:
        raise BsaError(BSA_ERR_INVALID_ARG, lib().bsa_last_error().decode())
    ws = _empty_bytes(nb, dev)
    uses_v = kind in ("vnorm", "vlog")
    bsa_score_select(shape, code, ScoreParams(beta), p, q, k, v if uses_v else None, r["scores"],
                     r["kv_idx"], r["kv_cnt"], r["sigma"], r["sigma_bar"], r["trigger"], r["theta"],
                     r["dev_status"], ws, nb, stream)
    return r


def prefill(q, k, v, *, block_k: int, tile_q: int, cfg: SelectConfig, output_aware: bool = False,
            scale: Optional[float] = None, stream=None, kind: Optional[str] = None, beta: float = 0.0,
            fused: bool = True):
    """score -> select -> attend on the current stream; returns (out, selection dict, status).
    fused: scores and selection in one bsa_score_select call (scores written out too);
    otherwise bsa_score then bsa_select."""
    shape = make_shape(q, k, block_k, tile_q)
    if kind is None:
        kind = "vnorm" if output_aware else "mean"
    if fused:
        sel = score_select(q, k, v, block_k=block_k, tile_q=tile_q, cfg=cfg, kind=kind, beta=beta,
                           want_scores=True, stream=stream)
        sel["score_status"] = torch.zeros(1, dtype=torch.int32, device=q.device)
    else:
        st_score = torch.zeros(1, dtype=torch.int32, device=q.device)
        s = score(q, k, v, block_k=block_k, tile_q=tile_q, stream=stream, status=st_score, kind=kind,
                  beta=beta)
        sel = select(s, shape=shape, cfg=cfg, stream=stream)
        sel["score_status"] = st_score
        sel["scores"] = s
    out, _, st = attend(q, k, v, sel["kv_idx"], sel["kv_cnt"], block_k=block_k, tile_q=tile_q,
                        scale=scale, stream=stream)
    return out, sel, st
