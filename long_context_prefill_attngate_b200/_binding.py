"""ctypes binding for libseer.so (the C ABI in include/seer.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and streams.  The
functions keep the C names; they take torch tensors, allocate any missing
output or workspace with torch (the library itself never allocates), call
the C entry point and raise ``SeerError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libseer.so")

SEER_OK = 0
SEER_ERR_INVALID_ARG = 1
SEER_ERR_UNSUPPORTED = 2
SEER_ERR_WORKSPACE = 3
SEER_ERR_CUDA = 4
SEER_ERR_TIMEOUT = 5
SEER_ERR_DEVICE = 6

SEER_MASK_THRESHOLD = 0
SEER_MASK_TOPK = 1

SEER_CALL_GATE_SCORES = 0
SEER_CALL_BLOCK_SPARSE_PREFILL = 1
SEER_CALL_ATTN_POOLED_MAP = 2
SEER_CALL_DECODE_GATE_SCORES = 3
SEER_CALL_BLOCK_SPARSE_DECODE = 4
SEER_CALL_GATE_KEY_CACHE = 5
SEER_CALL_DECODE_GATE_CACHED = 6

BLOCK = 64

# Every symbol include/seer.h declares.
EXPORTS = (
    "seer_gate_scores", "seer_block_mask", "seer_compact_mask", "seer_block_sparse_prefill",
    "seer_attn_pooled_map", "seer_workspace_bytes", "seer_check_status", "seer_set_wait_timeout_ns",
    "seer_last_error", "seer_version", "seer_gate_scores_noalloc", "seer_distill_loss",
    "seer_decode_gate_scores", "seer_decode_block_mask", "seer_block_sparse_decode",
    "seer_gate_key_cache", "seer_decode_gate_scores_cached", "seer_topk_from_density",
)


class SeerError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"status {status}: {msg}")
        self.status = status


class seer_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("S", ctypes.c_int),
                ("d", ctypes.c_int)]


SEER_KPOOL_AVG = 0
SEER_KPOOL_MAXMIN = 1


class seer_gate_params(ctypes.Structure):
    _fields_ = [("d_gate", ctypes.c_int), ("rope_theta", ctypes.c_float), ("wq_head_stride", ctypes.c_longlong),
                ("wk_head_stride", ctypes.c_longlong), ("k_pooling", ctypes.c_int)]


class seer_mask_params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("threshold", ctypes.c_float), ("density", ctypes.c_double),
                ("k_fixed", ctypes.c_int), ("k_per_row", ctypes.c_void_p), ("force_first", ctypes.c_int),
                ("force_diag", ctypes.c_int)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libseer.so (built in-tree).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libseer.so not found at {LIB_PATH}: build it with "
                    "`python -m long_context_prefill_attngate_b200.build` (there is no fallback path)")
            L = ctypes.CDLL(LIB_PATH)
            P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
            SP = ctypes.POINTER(seer_shape)
            L.seer_gate_scores.argtypes = [SP, P, P, P, P, ctypes.POINTER(seer_gate_params), P, P, Z, P]
            L.seer_gate_scores_noalloc.argtypes = [SP, P, P, P, P, ctypes.POINTER(seer_gate_params), P, P]
            L.seer_block_mask.argtypes = [SP, P, ctypes.POINTER(seer_mask_params), P, P]
            L.seer_compact_mask.argtypes = [SP, P, P, P, P]
            L.seer_distill_loss.argtypes = [SP, P, P, P, P, P, P]
            L.seer_block_sparse_prefill.argtypes = [SP, P, P, P, P, F, P, P, P, Z, P]
            L.seer_attn_pooled_map.argtypes = [SP, P, P, P, F, P, P, P, Z, P]
            L.seer_decode_gate_scores.argtypes = [SP, P, P, P, P, ctypes.POINTER(seer_gate_params), P, P, Z, P]
            L.seer_decode_block_mask.argtypes = [SP, P, ctypes.POINTER(seer_mask_params), P, P]
            L.seer_block_sparse_decode.argtypes = [SP, P, P, P, P, F, P, P, P, Z, P]
            L.seer_gate_key_cache.argtypes = [SP, P, P, ctypes.POINTER(seer_gate_params), I, P, P, Z, P]
            L.seer_decode_gate_scores_cached.argtypes = [SP, P, P, P, ctypes.POINTER(seer_gate_params), P, P, Z, P]
            L.seer_topk_from_density.argtypes = [ctypes.c_double, I, I, I, ctypes.POINTER(ctypes.c_int32)]
            for fn in ("seer_gate_scores", "seer_gate_scores_noalloc", "seer_block_mask", "seer_compact_mask",
                       "seer_block_sparse_prefill", "seer_attn_pooled_map", "seer_check_status",
                       "seer_distill_loss", "seer_decode_gate_scores", "seer_decode_block_mask",
                       "seer_block_sparse_decode", "seer_gate_key_cache", "seer_decode_gate_scores_cached",
                       "seer_topk_from_density"):
                getattr(L, fn).restype = I
            L.seer_workspace_bytes.argtypes = [I, SP]
            L.seer_workspace_bytes.restype = Z
            L.seer_check_status.argtypes = [P]
            L.seer_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
            L.seer_set_wait_timeout_ns.restype = None
            L.seer_last_error.restype = ctypes.c_char_p
            L.seer_version.restype = ctypes.c_char_p
            _lib = L
    return _lib


def _check(status: int) -> None:
    if status != SEER_OK:
        raise SeerError(status, lib().seer_last_error().decode())


def _torch():
    import torch
    return torch


def _stream_ptr(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(getattr(stream, "cuda_stream", stream))


def shape_of(q, k) -> seer_shape:
    B, Hq, S, d = q.shape
    return seer_shape(B, Hq, k.shape[1], S, d)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def seer_version() -> str:
    return lib().seer_version().decode()


def seer_last_error() -> str:
    return lib().seer_last_error().decode()


def seer_set_wait_timeout_ns(ns: int) -> None:
    lib().seer_set_wait_timeout_ns(int(ns))


def seer_workspace_bytes(which: int, shape: seer_shape) -> int:
    return int(lib().seer_workspace_bytes(int(which), ctypes.byref(shape)))


def seer_check_status(stream=None) -> None:
    _check(lib().seer_check_status(ctypes.c_void_p(_stream_ptr(stream))))


def _workspace(which: int, sh: seer_shape, device, workspace):
    n = seer_workspace_bytes(which, sh)
    if workspace is None and n > 0:
        workspace = _torch().empty(n, dtype=_torch().uint8, device=device)
    return workspace, (0 if workspace is None else workspace.numel() * workspace.element_size())


def seer_gate_scores(q, k, wq, wk, rope_theta: float = 5e5, scores=None, workspace=None, stream=None,
                     wq_head_stride: int | None = None, wk_head_stride: int | None = None,
                     k_maxmin: bool = False):
    """AttnGate soft scores fp32 [B,Hq,nb,nb] (see include/seer.h)."""
    torch = _torch()
    _need(q.is_contiguous() and k.is_contiguous() and wq.is_contiguous() and wk.is_contiguous(),
          "tensors must be contiguous")
    _need(q.dtype == k.dtype == wq.dtype == wk.dtype == torch.bfloat16, "q, k, wq, wk must be bf16")
    sh = shape_of(q, k)
    d, dg = sh.d, wq.shape[-1]
    nb = -(-sh.S // BLOCK)
    if wq_head_stride is None:
        wq_head_stride = 0 if wq.dim() == 2 else d * dg
    if wk_head_stride is None:
        wk_head_stride = 0 if wk.dim() == 2 else (2 * d if k_maxmin else d) * dg
    _need(wk.shape[-2] == (2 * d if k_maxmin else d) and wk.shape[-1] == dg,
          "wk must be [.., %d, %d] for %s K pooling" % (2 * d if k_maxmin else d, dg, "max+min" if k_maxmin else "average"))
    if scores is None:
        scores = torch.empty((sh.B, sh.Hq, nb, nb), dtype=torch.float32, device=q.device)
    workspace, wsb = _workspace(SEER_CALL_GATE_SCORES, sh, q.device, workspace)
    gp = seer_gate_params(int(dg), float(rope_theta), int(wq_head_stride), int(wk_head_stride), int(bool(k_maxmin)))
    _check(lib().seer_gate_scores(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk), ctypes.byref(gp),
                                  _ptr(scores), _ptr(workspace), wsb, _stream_ptr(stream)))
    return scores


def seer_gate_scores_noalloc(q, k, wq, wk, rope_theta: float = 5e5, scores=None, stream=None,
                             wq_head_stride: int | None = None, wk_head_stride: int | None = None,
                             k_maxmin: bool = False):
    """seer_gate_scores without a workspace: the library's fixed scratch is used
    (for callers that cannot allocate device memory; shapes needing more than
    24 MiB of gate scratch raise SeerError)."""
    torch = _torch()
    _need(q.is_contiguous() and k.is_contiguous() and wq.is_contiguous() and wk.is_contiguous(),
          "tensors must be contiguous")
    sh = shape_of(q, k)
    d, dg = sh.d, wq.shape[-1]
    nb = -(-sh.S // BLOCK)
    if wq_head_stride is None:
        wq_head_stride = 0 if wq.dim() == 2 else d * dg
    if wk_head_stride is None:
        wk_head_stride = 0 if wk.dim() == 2 else (2 * d if k_maxmin else d) * dg
    _need(wk.shape[-2] == (2 * d if k_maxmin else d) and wk.shape[-1] == dg,
          "wk must be [.., %d, %d] for %s K pooling" % (2 * d if k_maxmin else d, dg, "max+min" if k_maxmin else "average"))
    if scores is None:
        scores = torch.empty((sh.B, sh.Hq, nb, nb), dtype=torch.float32, device=q.device)
    gp = seer_gate_params(int(dg), float(rope_theta), int(wq_head_stride), int(wk_head_stride), int(bool(k_maxmin)))
    _check(lib().seer_gate_scores_noalloc(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk), ctypes.byref(gp),
                                          _ptr(scores), _stream_ptr(stream)))
    return scores


def seer_block_mask(scores, mode: str = "topk", threshold: float = 0.0, density: float = 1.0, k_fixed: int = 0,
                    k_per_row=None, force_first: bool = True, force_diag: bool = True, mask=None, stream=None,
                    Hkv: int = 1, d: int = 64):
    """Binary block mask u8 [B,Hq,nb,nb] from scores (threshold or per-row TopK)."""
    torch = _torch()
    _need(scores.dtype == torch.float32 and scores.is_contiguous(), "scores must be contiguous fp32")
    B, Hq, nb, _ = scores.shape
    sh = seer_shape(B, Hq, Hkv if Hq % Hkv == 0 else 1, nb * BLOCK, d)
    if mask is None:
        mask = torch.empty((B, Hq, nb, nb), dtype=torch.uint8, device=scores.device)
    m = {"threshold": SEER_MASK_THRESHOLD, "topk": SEER_MASK_TOPK}[mode]
    if k_per_row is not None:
        _need(k_per_row.dtype == torch.int32 and k_per_row.is_cuda, "k_per_row must be a device int32 tensor")
    mp = seer_mask_params(m, float(threshold), float(density), int(k_fixed), _ptr(k_per_row),
                          int(bool(force_first)), int(bool(force_diag)))
    _check(lib().seer_block_mask(ctypes.byref(sh), _ptr(scores), ctypes.byref(mp), _ptr(mask),
                                 _stream_ptr(stream)))
    return mask


def seer_compact_mask(mask, lists=None, counts=None, stream=None):
    """Causal-packed ascending active-block lists int32 [B,Hq,nb(nb+1)/2] and counts [B,Hq,nb]."""
    torch = _torch()
    _need(mask.dtype == torch.uint8 and mask.is_contiguous(), "mask must be contiguous uint8")
    B, Hq, nb, _ = mask.shape
    sh = seer_shape(B, Hq, 1, nb * BLOCK, 64)
    if lists is None:
        lists = torch.full((B, Hq, nb * (nb + 1) // 2), -1, dtype=torch.int32, device=mask.device)
    if counts is None:
        counts = torch.empty((B, Hq, nb), dtype=torch.int32, device=mask.device)
    _check(lib().seer_compact_mask(ctypes.byref(sh), _ptr(mask), _ptr(lists), _ptr(counts), _stream_ptr(stream)))
    return lists, counts


def seer_block_sparse_prefill(q, k, v, mask, softmax_scale: float = 0.0, o=None, lse=None, return_lse: bool = False,
                              workspace=None, stream=None):
    """Block-sparse causal attention (GQA); returns O (and LSE if requested)."""
    torch = _torch()
    _need(all(t.is_contiguous() for t in (q, k, v, mask)), "tensors must be contiguous")
    _need(q.dtype == k.dtype == v.dtype == torch.bfloat16 and mask.dtype == torch.uint8, "bf16 q/k/v, u8 mask")
    sh = shape_of(q, k)
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((sh.B, sh.Hq, sh.S), dtype=torch.float32, device=q.device)
    workspace, wsb = _workspace(SEER_CALL_BLOCK_SPARSE_PREFILL, sh, q.device, workspace)
    _check(lib().seer_block_sparse_prefill(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(mask),
                                           float(softmax_scale), _ptr(o), _ptr(lse), _ptr(workspace), wsb,
                                           _stream_ptr(stream)))
    return (o, lse) if (return_lse or lse is not None) else o


def seer_attn_pooled_map(q, k, v, softmax_scale: float = 0.0, o=None, A=None, workspace=None, stream=None):
    """Dense causal attention returning (O, A) with A the 64x64 max-pooled map."""
    torch = _torch()
    _need(all(t.is_contiguous() for t in (q, k, v)), "tensors must be contiguous")
    _need(q.dtype == k.dtype == v.dtype == torch.bfloat16, "bf16 q/k/v")
    sh = shape_of(q, k)
    nb = -(-sh.S // BLOCK)
    if o is None:
        o = torch.empty_like(q)
    if A is None:
        A = torch.empty((sh.B, sh.Hq, nb, nb), dtype=torch.float32, device=q.device)
    workspace, wsb = _workspace(SEER_CALL_ATTN_POOLED_MAP, sh, q.device, workspace)
    _check(lib().seer_attn_pooled_map(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), float(softmax_scale), _ptr(o),
                                      _ptr(A), _ptr(workspace), wsb, _stream_ptr(stream)))
    return o, A


def seer_distill_loss(scores, A, want_norm: bool = False, stream=None, Hkv: int = 1, d: int = 64):
    """Row-normalised target, per-row squared error and per-head MSE (see include/seer.h).

    Returns (loss [B,Hq], loss_rows [B,Hq,nb], A_norm or None)."""
    torch = _torch()
    _need(scores.dtype == A.dtype == torch.float32 and scores.is_contiguous() and A.is_contiguous(),
          "scores and A must be contiguous fp32")
    _need(scores.shape == A.shape, "scores and A must have the same shape")
    B, Hq, nb, _ = scores.shape
    sh = seer_shape(B, Hq, Hkv if Hq % Hkv == 0 else 1, nb * BLOCK, d)
    rows = torch.empty((B, Hq, nb), dtype=torch.float32, device=scores.device)
    loss = torch.empty((B, Hq), dtype=torch.float32, device=scores.device)
    an = torch.empty_like(A) if want_norm else None
    _check(lib().seer_distill_loss(ctypes.byref(sh), _ptr(scores), _ptr(A), _ptr(an), _ptr(rows), _ptr(loss),
                                   _stream_ptr(stream)))
    return loss, rows, an


# ------------------------------------------------------------------ decode step
def _decode_shape(q_tok, k):
    _need(q_tok.dim() == 3 and k.dim() == 4, "q_tok must be [B,Hq,d] and k [B,Hkv,L,d]")
    B, Hq, d = q_tok.shape
    _need(k.shape[0] == B and k.shape[3] == d, "q_tok / k shapes disagree")
    return seer_shape(B, Hq, k.shape[1], k.shape[2], d)


def seer_decode_gate_scores(q_tok, k, wq, wk, rope_theta: float = 5e5, scores=None, workspace=None, stream=None,
                            wq_head_stride: int | None = None, wk_head_stride: int | None = None,
                            k_maxmin: bool = False):
    """Decode gate row fp32 [B,Hq,nb] of the token at position L-1 (see include/seer.h)."""
    torch = _torch()
    _need(q_tok.is_contiguous() and k.is_contiguous() and wq.is_contiguous() and wk.is_contiguous(),
          "tensors must be contiguous")
    _need(q_tok.dtype == k.dtype == wq.dtype == wk.dtype == torch.bfloat16, "q_tok, k, wq, wk must be bf16")
    sh = _decode_shape(q_tok, k)
    d, dg = sh.d, wq.shape[-1]
    nb = -(-sh.S // BLOCK)
    if wq_head_stride is None:
        wq_head_stride = 0 if wq.dim() == 2 else d * dg
    if wk_head_stride is None:
        wk_head_stride = 0 if wk.dim() == 2 else (2 * d if k_maxmin else d) * dg
    _need(wk.shape[-2] == (2 * d if k_maxmin else d) and wk.shape[-1] == dg, "wk shape does not match k pooling")
    if scores is None:
        scores = torch.empty((sh.B, sh.Hq, nb), dtype=torch.float32, device=q_tok.device)
    workspace, wsb = _workspace(SEER_CALL_DECODE_GATE_SCORES, sh, q_tok.device, workspace)
    gp = seer_gate_params(int(dg), float(rope_theta), int(wq_head_stride), int(wk_head_stride), int(bool(k_maxmin)))
    _check(lib().seer_decode_gate_scores(ctypes.byref(sh), _ptr(q_tok), _ptr(k), _ptr(wq), _ptr(wk),
                                         ctypes.byref(gp), _ptr(scores), _ptr(workspace), wsb, _stream_ptr(stream)))
    return scores


def seer_gate_key_cache(k, wk, kt=None, first_block: int = 0, rope_theta: float = 5e5, d_gate: int | None = None,
                        workspace=None, stream=None, wk_head_stride: int | None = None, k_maxmin: bool = False):
    """The gate's key rows fp32 [B,Hkv,nb,d_gate] for blocks first_block.. of the cache k [B,Hkv,L,d]
    (rows below first_block of a given kt are left as they are)."""
    torch = _torch()
    _need(k.is_contiguous() and wk.is_contiguous() and k.dtype == wk.dtype == torch.bfloat16, "bf16 contiguous k, wk")
    Bsz, Hkv, L, d = k.shape
    dg = wk.shape[-1] if d_gate is None else d_gate
    nb = -(-L // BLOCK)
    sh = seer_shape(Bsz, Hkv, Hkv, L, d)
    if wk_head_stride is None:
        wk_head_stride = 0 if wk.dim() == 2 else (2 * d if k_maxmin else d) * dg
    if kt is None:
        kt = torch.empty((Bsz, Hkv, nb, dg), dtype=torch.float32, device=k.device)
    _need(kt.dtype == torch.float32 and kt.is_contiguous() and tuple(kt.shape) == (Bsz, Hkv, nb, dg), "kt shape")
    workspace, wsb = _workspace(SEER_CALL_GATE_KEY_CACHE, sh, k.device, workspace)
    gp = seer_gate_params(int(dg), float(rope_theta), 0, int(wk_head_stride), int(bool(k_maxmin)))
    _check(lib().seer_gate_key_cache(ctypes.byref(sh), _ptr(k), _ptr(wk), ctypes.byref(gp), int(first_block), _ptr(kt),
                                     _ptr(workspace), wsb, _stream_ptr(stream)))
    return kt


def seer_decode_gate_scores_cached(q_tok, kt, wq, L: int, Hkv: int, rope_theta: float = 5e5, scores=None,
                                   workspace=None, stream=None, wq_head_stride: int | None = None):
    """Decode gate row fp32 [B,Hq,nb] from cached key rows kt [B,Hkv,nb,d_gate] (cache of L tokens)."""
    torch = _torch()
    _need(q_tok.is_contiguous() and wq.is_contiguous() and kt.is_contiguous(), "tensors must be contiguous")
    Bsz, Hq, d = q_tok.shape
    dg = wq.shape[-1]
    nb = -(-L // BLOCK)
    _need(tuple(kt.shape) == (Bsz, Hkv, nb, dg) and kt.dtype == torch.float32, "kt must be fp32 [B,Hkv,nb,d_gate]")
    sh = seer_shape(Bsz, Hq, Hkv, L, d)
    if wq_head_stride is None:
        wq_head_stride = 0 if wq.dim() == 2 else d * dg
    if scores is None:
        scores = torch.empty((Bsz, Hq, nb), dtype=torch.float32, device=q_tok.device)
    workspace, wsb = _workspace(SEER_CALL_DECODE_GATE_CACHED, sh, q_tok.device, workspace)
    gp = seer_gate_params(int(dg), float(rope_theta), int(wq_head_stride), 0, 0)
    _check(lib().seer_decode_gate_scores_cached(ctypes.byref(sh), _ptr(q_tok), _ptr(kt), _ptr(wq), ctypes.byref(gp),
                                                _ptr(scores), _ptr(workspace), wsb, _stream_ptr(stream)))
    return scores


def seer_decode_block_mask(scores, mode: str = "topk", threshold: float = 0.0, density: float = 1.0,
                           k_fixed: int = 0, force_first: bool = True, force_diag: bool = True, mask=None,
                           stream=None):
    """Decode mask row u8 [B,Hq,nb] from the gate row (threshold or TopK)."""
    torch = _torch()
    _need(scores.dtype == torch.float32 and scores.is_contiguous() and scores.dim() == 3,
          "scores must be contiguous fp32 [B,Hq,nb]")
    B, Hq, nb = scores.shape
    sh = seer_shape(B, Hq, 1, nb * BLOCK, 64)
    if mask is None:
        mask = torch.empty((B, Hq, nb), dtype=torch.uint8, device=scores.device)
    m = {"threshold": SEER_MASK_THRESHOLD, "topk": SEER_MASK_TOPK}[mode]
    mp = seer_mask_params(m, float(threshold), float(density), int(k_fixed), None,
                          int(bool(force_first)), int(bool(force_diag)))
    _check(lib().seer_decode_block_mask(ctypes.byref(sh), _ptr(scores), ctypes.byref(mp), _ptr(mask),
                                        _stream_ptr(stream)))
    return mask


def seer_block_sparse_decode(q_tok, k, v, mask, softmax_scale: float = 0.0, o=None, lse=None,
                             return_lse: bool = False, workspace=None, stream=None):
    """Attention of the token at position L-1 over its active KV blocks; returns o [B,Hq,d] bf16."""
    torch = _torch()
    _need(all(t.is_contiguous() for t in (q_tok, k, v, mask)), "tensors must be contiguous")
    _need(q_tok.dtype == k.dtype == v.dtype == torch.bfloat16 and mask.dtype == torch.uint8, "bf16 q/k/v, u8 mask")
    sh = _decode_shape(q_tok, k)
    if o is None:
        o = torch.empty_like(q_tok)
    if return_lse and lse is None:
        lse = torch.empty((sh.B, sh.Hq), dtype=torch.float32, device=q_tok.device)
    workspace, wsb = _workspace(SEER_CALL_BLOCK_SPARSE_DECODE, sh, q_tok.device, workspace)
    _check(lib().seer_block_sparse_decode(ctypes.byref(sh), _ptr(q_tok), _ptr(k), _ptr(v), _ptr(mask),
                                          float(softmax_scale), _ptr(o), _ptr(lse), _ptr(workspace), wsb,
                                          _stream_ptr(stream)))
    return (o, lse) if (return_lse or lse is not None) else o


def seer_topk_from_density(density: float, nb: int, force_first: bool = True, force_diag: bool = True) -> list[int]:
    """Per-row TopK counts k_i for a density, computed by the C library."""
    out = (ctypes.c_int32 * nb)()
    _check(lib().seer_topk_from_density(ctypes.c_double(float(density)), int(nb), int(bool(force_first)),
                                        int(bool(force_diag)), out))
    return list(out)