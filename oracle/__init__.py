"""fp64 CPU oracle for the SeerAttention prefill hot path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product library
never does.  The arithmetic lives in ``seer_oracle.c`` (plain C, fp64, OpenMP
over independent units); this module builds it with gcc and marshals numpy
arrays through ctypes.  It shares nothing with the CUDA library.

Inputs are the raw bf16 bit patterns as ``np.uint16`` arrays, so the oracle
reads exactly the values the GPU reads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "seer_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 64


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            LL = ctypes.c_longlong
            D = ctypes.c_double
            F = ctypes.c_float
            lib.oracle_pool_avg.argtypes = [P, I, I, I, I, P]
            lib.oracle_block_rope.argtypes = [P, I, I, D]
            lib.oracle_project_rope.argtypes = [P, I, I, I, I, P, LL, I, D, P]
            lib.oracle_block_softmax.argtypes = [P, P, I, I, I, I, I, P]
            lib.oracle_gate_scores.argtypes = [P, P, I, I, I, I, I, P, LL, P, LL, I, D, P]
            lib.oracle_topk_count.argtypes = [D, I, I]
            lib.oracle_topk_count.restype = I
            lib.oracle_block_mask.argtypes = [P, I, I, I, I, F, P, I, I, P]
            lib.oracle_compact.argtypes = [P, I, I, I, P, P]
            lib.oracle_masked_attention.argtypes = [P, P, P, I, I, I, I, I, P, D, P, I, P, P]
            lib.oracle_pooled_map.argtypes = [P, P, P, I, I, I, I, I, D, P, I, P, P]
            lib.oracle_distill_loss.argtypes = [P, P, I, I, I, P, P, P]
            lib.oracle_pool_maxmin.argtypes = [P, I, I, I, I, P]
            lib.oracle_gate_scores_kpool.argtypes = [P, P, I, I, I, I, I, P, LL, P, LL, I, D, I, P]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns as uint16, got {a.dtype}")
    return a


def set_threads(n: int) -> None:
    """Set the OpenMP thread count used by the oracle (call before first use)."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))


def pool_avg(x: np.ndarray) -> np.ndarray:
    """a1: mean over each 64-row block; bf16 [B,H,S,d] -> f64 [B,H,ceil(S/64),d]; the last block of a ragged S averages its real tokens."""
    x = _u16(x)
    B, H, S, d = x.shape
    out = np.empty((B, H, -(-S // BLOCK), d), np.float64)
    _load().oracle_pool_avg(_ptr(x), B, H, S, d, _ptr(out))
    return out


def pool_maxmin(x: np.ndarray) -> np.ndarray:
    """a1': per-block max and min, concatenated; bf16 [B,H,S,d] -> f64 [B,H,ceil(S/64),2d]."""
    x = _u16(x)
    B, H, S, d = x.shape
    out = np.empty((B, H, -(-S // BLOCK), 2 * d), np.float64)
    _load().oracle_pool_maxmin(_ptr(x), B, H, S, d, _ptr(out))
    return out


def block_rope(x: np.ndarray, p: int, theta: float) -> np.ndarray:
    """Block RoPE of one f64 vector at block position ``p`` (returns a copy)."""
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    _load().oracle_block_rope(_ptr(y), y.shape[0], int(p), float(theta))
    return y


def project_rope(xp: np.ndarray, w: np.ndarray, theta: float, head_stride: int | None = None) -> np.ndarray:
    """a2: RoPE_i(xp[b,h,i] @ W[h]); w bf16 [H,d,dg] (or [d,dg] shared)."""
    xp = np.ascontiguousarray(xp, dtype=np.float64)
    w = _u16(w)
    B, H, nb, d = xp.shape
    dg = w.shape[-1]
    if head_stride is None:
        head_stride = 0 if w.ndim == 2 else d * dg
    out = np.empty((B, H, nb, dg), np.float64)
    _load().oracle_project_rope(_ptr(xp), B, H, nb, d, _ptr(w), int(head_stride), dg, float(theta), _ptr(out))
    return out


def block_softmax(qt: np.ndarray, kt: np.ndarray) -> np.ndarray:
    """a3 core: causal block softmax of qt.kt/sqrt(dg); f64 [B,Hq,nb,nb]."""
    qt = np.ascontiguousarray(qt, dtype=np.float64)
    kt = np.ascontiguousarray(kt, dtype=np.float64)
    B, Hq, nb, dg = qt.shape
    Hkv = kt.shape[1]
    out = np.empty((B, Hq, nb, nb), np.float64)
    _load().oracle_block_softmax(_ptr(qt), _ptr(kt), B, Hq, Hkv, nb, dg, _ptr(out))
    return out


def gate_scores(q, k, wq, wk, theta: float = 5e5, wq_head_stride=None, wk_head_stride=None,
                k_maxmin: bool = False) -> np.ndarray:
    """a1-a3: AttnGate soft scores, f64 [B,Hq,nb,nb].  With k_maxmin, K is
    pooled by [max | min] and wk is [Hkv, 2d, dg]."""
    q, k, wq, wk = _u16(q), _u16(k), _u16(wq), _u16(wk)
    B, Hq, S, d = q.shape
    Hkv = k.shape[1]
    dg = wq.shape[-1]
    dk = 2 * d if k_maxmin else d
    if wq_head_stride is None:
        wq_head_stride = 0 if wq.ndim == 2 else d * dg
    if wk_head_stride is None:
        wk_head_stride = 0 if wk.ndim == 2 else dk * dg
    nb = -(-S // BLOCK)
    out = np.empty((B, Hq, nb, nb), np.float64)
    _load().oracle_gate_scores_kpool(_ptr(q), _ptr(k), B, Hq, Hkv, S, d, _ptr(wq), int(wq_head_stride),
                                     _ptr(wk), int(wk_head_stride), dg, float(theta), int(bool(k_maxmin)), _ptr(out))
    return out


def topk_count(density: float, i: int, n_forced: int) -> int:
    """k_i = ceil(density*(i+1)) clamped to [n_forced, i+1]."""
    return int(_load().oracle_topk_count(float(density), int(i), int(n_forced)))


def topk_counts(density: float, nb: int, force_first: bool = True, force_diag: bool = True) -> np.ndarray:
    """Per-row k for a density, as int32 [nb]."""
    out = np.empty(nb, np.int32)
    for i in range(nb):
        nf = (1 if force_first else 0) + (1 if (force_diag and not (force_first and i == 0)) else 0)
        out[i] = topk_count(density, i, nf)
    return out


def block_mask(scores: np.ndarray, mode: str, threshold: float = 0.0, k_row=None,
               force_first: bool = True, force_diag: bool = True) -> np.ndarray:
    """a4: threshold / per-row TopK mask from f32 scores; u8 [B,Hq,nb,nb]."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    B, Hq, nb, _ = s.shape
    m = {"threshold": 0, "topk": 1}[mode]
    if m == 1:
        kr = np.ascontiguousarray(k_row, dtype=np.int32)
        assert kr.shape == (nb,)
    else:
        kr = np.zeros(nb, np.int32)
    out = np.empty((B, Hq, nb, nb), np.uint8)
    _load().oracle_block_mask(_ptr(s), B, Hq, nb, m, float(np.float32(threshold)), _ptr(kr),
                              int(bool(force_first)), int(bool(force_diag)), _ptr(out))
    return out


def compact(mask: np.ndarray):
    """a5: causal-packed ascending active lists + counts per (b,h,i)."""
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    B, Hq, nb, _ = m.shape
    tri = nb * (nb + 1) // 2
    lists = np.full((B, Hq, tri), -1, np.int32)
    counts = np.empty((B, Hq, nb), np.int32)
    _load().oracle_compact(_ptr(m), B, Hq, nb, _ptr(lists), _ptr(counts))
    return lists, counts


def all_units(B: int, H: int, nb: int) -> np.ndarray:
    """Every (b, h, i) query-block unit, as int32 [n, 3]."""
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(nb), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], 1).astype(np.int32)


def masked_attention(q, k, v, mask, scale: float | None = None, units=None):
    """a6: explicit masked causal attention for the given (b,h,i) units.

    Returns (o f64 [n,64,d], lse f64 [n,64]); rows at or past S (a ragged
    last block) are 0 with LSE -inf.
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, S, d = q.shape
    Hkv = k.shape[1]
    nb = -(-S // BLOCK)
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    assert m.shape == (B, Hq, nb, nb)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if units is None:
        units = all_units(B, Hq, nb)
    units = np.ascontiguousarray(units, dtype=np.int32)
    n = units.shape[0]
    o = np.empty((n, BLOCK, d), np.float64)
    lse = np.empty((n, BLOCK), np.float64)
    _load().oracle_masked_attention(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, S, d, _ptr(m), float(scale),
                                    _ptr(units), n, _ptr(o), _ptr(lse))
    return o, lse


def pooled_map(q, k, v, scale: float | None = None, units=None):
    """a7: dense causal O plus the max-pooled map rows A[b,h,i,:].

    Returns (o f64 [n,64,d], A f64 [n,nb]); rows at or past S are 0 and do
    not enter A.
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, S, d = q.shape
    Hkv = k.shape[1]
    nb = -(-S // BLOCK)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if units is None:
        units = all_units(B, Hq, nb)
    units = np.ascontiguousarray(units, dtype=np.int32)
    n = units.shape[0]
    o = np.empty((n, BLOCK, d), np.float64)
    A = np.empty((n, nb), np.float64)
    _load().oracle_pooled_map(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, S, d, float(scale),
                              _ptr(units), n, _ptr(o), _ptr(A))
    return o, A


# --------------------------------------------------------------------------- decode
# "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning" (abstract):
# the decode form keeps the self-distilled gate but drops query pooling, and
# runs a block-sparse decoding kernel; "SeerAttention" rebuttal Weakness 4 on
# decode: a per-Q-token AttnGate without pooling, on the same linear weights.
# Reading: one new token per sequence at position L - 1 of a KV cache of L
# tokens (its own k, v included), nb = ceil(L / 64).  Its query block is the
# last one, i = nb - 1: the gate row is the prefill gate's row i with the
# pooled query replaced by the token's own q, the mask row is the prefill
# mask's row i, and the attention is the prefill attention of query row L - 1.
# Each function below is exactly that: the pinned prefill functions applied
# to arrays whose row i (or token L - 1) holds the decode data.
def decode_gate_scores(q_tok, k, wq, wk, theta: float = 5e5, wq_head_stride=None, wk_head_stride=None,
                       k_maxmin: bool = False) -> np.ndarray:
    """Decode gate: q_tok bf16 [B,Hq,d] (no pooling), k bf16 [B,Hkv,L,d] -> f64 [B,Hq,nb]."""
    q_tok, k = _u16(q_tok), _u16(k)
    B, Hq, d = q_tok.shape
    nb = -(-k.shape[2] // BLOCK)
    dk = 2 * d if k_maxmin else d
    dg = _u16(wq).shape[-1]
    if wq_head_stride is None:
        wq_head_stride = 0 if _u16(wq).ndim == 2 else d * dg
    if wk_head_stride is None:
        wk_head_stride = 0 if _u16(wk).ndim == 2 else dk * dg
    kt = project_rope(pool_maxmin(k) if k_maxmin else pool_avg(k), wk, theta, head_stride=wk_head_stride)
    xq = np.zeros((B, Hq, nb, d), np.float64)
    xq[:, :, nb - 1] = (q_tok.astype(np.uint32) << 16).view(np.float32)     # bf16 bits -> value
    qt = project_rope(xq, wq, theta, head_stride=wq_head_stride)
    return block_softmax(qt, kt)[:, :, nb - 1, :].copy()


def decode_mask(scores, mode: str, threshold: float = 0.0, k: int | None = None, force_first: bool = True,
                force_diag: bool = True) -> np.ndarray:
    """Decode mask row from f32 scores [B,Hq,nb] -> u8 [B,Hq,nb]; TopK keeps k
    blocks (clamped to the forced set and to nb); the last block is the
    token's own ("diagonal")."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    B, Hq, nb = s.shape
    full = np.zeros((B, Hq, nb, nb), np.float32)
    full[:, :, nb - 1] = s
    kr = np.ones(nb, np.int32)
    if mode == "topk":
        kr[nb - 1] = int(k)
    return block_mask(full, mode, threshold=threshold, k_row=kr, force_first=force_first,
                      force_diag=force_diag)[:, :, nb - 1].copy()


def decode_attention(q_tok, k, v, mask_row, scale: float | None = None):
    """Decode attention of token L-1 over the active blocks of its mask row:
    q_tok bf16 [B,Hq,d], k/v bf16 [B,Hkv,L,d], mask_row u8 [B,Hq,nb]
    -> (o f64 [B,Hq,d], lse f64 [B,Hq])."""
    q_tok, k, v = _u16(q_tok), _u16(k), _u16(v)
    B, Hq, d = q_tok.shape
    L = k.shape[2]
    nb = -(-L // BLOCK)
    Q = np.zeros((B, Hq, L, d), np.uint16)
    Q[:, :, L - 1] = q_tok
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    mask[:, :, nb - 1] = np.asarray(mask_row, np.uint8)
    units = np.array([(b, h, nb - 1) for b in range(B) for h in range(Hq)], np.int32)
    o, lse = masked_attention(Q, k, v, mask, scale=scale, units=units)
    r = L - 1 - BLOCK * (nb - 1)
    return o[:, r].reshape(B, Hq, d), lse[:, r].reshape(B, Hq)


def distill_loss(G, A):
    """Row-normalised target Ahat, per-row squared error and per-head mean
    (over causal block entries) of MSE(G, Ahat); G, A f32 [B,Hq,nb,nb]."""
    G = np.ascontiguousarray(G, dtype=np.float32)
    A = np.ascontiguousarray(A, dtype=np.float32)
    B, Hq, nb, _ = G.shape
    assert A.shape == G.shape
    ahat = np.empty((B, Hq, nb, nb), np.float64)
    rows = np.empty((B, Hq, nb), np.float64)
    heads = np.empty((B, Hq), np.float64)
    _load().oracle_distill_loss(_ptr(G), _ptr(A), B, Hq, nb, _ptr(ahat), _ptr(rows), _ptr(heads))
    return ahat, rows, heads
