"""CPU oracle for the hybrid sparse attention forward (HCA + MLA-DSA), and for the
gradients of its attention and compression steps (backward pass).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path (the CUDA library and
its binding) never imports this package, and this package never imports the
product.  The arithmetic lives in ``oracle.c`` (plain C, OpenMP over query
rows); this module only compiles it with gcc and marshals numpy arrays.

Every function evaluates the definitions stated in ``oracle.c``; the pins that
tie those definitions to the pages and to independent mathematics are in
``tests/test_oracle_pins.py``.  Parity status of each function: pinned (see the
pin tests), except the large-configuration attention values, which are pinned
only through the special cases and invariants the tests check.  The backward
functions are pinned to torch fp64 autograd and to closed forms.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_long
            D = ctypes.c_double
            lib.oracle_version.restype = I
            lib.oracle_f32_to_bf16.argtypes = [P, P, L]
            lib.oracle_bf16_to_f32.argtypes = [P, P, L]
            lib.oracle_hca_compress.argtypes = [P, P, P, I, I, I, I, I]
            lib.oracle_hca_compress.restype = I
            lib.oracle_hca_window_start.argtypes = [I, I]
            lib.oracle_hca_window_start.restype = I
            lib.oracle_hca_n_compressed.argtypes = [I, I, I]
            lib.oracle_hca_n_compressed.restype = I
            lib.oracle_hca_attn.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, I, I, I,
                                            D, P, I, P, P]
            lib.oracle_hca_attn.restype = I
            lib.oracle_hca_attn_latent.argtypes = [P, P, I, P, I, I, I, I, I, I, I, I, I, I, I, D, P, I, P, P]
            lib.oracle_hca_attn_latent.restype = I
            lib.oracle_dsa_scores.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P]
            lib.oracle_dsa_scores.restype = I
            lib.oracle_dsa_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, P]
            lib.oracle_dsa_topk.restype = I
            lib.oracle_csa_n_candidates.argtypes = [I, I, I]
            lib.oracle_csa_n_candidates.restype = I
            lib.oracle_csa_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, I, P]
            lib.oracle_csa_topk.restype = I
            lib.oracle_dsa_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, D, P, I, P, P]
            lib.oracle_gate_vha.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
            lib.oracle_gate_vha.restype = I
            lib.oracle_dsa_attn.restype = I
            lib.oracle_hca_attn_bwd.argtypes = [P, P, P, I, P, P, I, I, P, I, I, I, I, I, I, I, I, D,
                                                P, P, P, P, P]
            lib.oracle_hca_attn_bwd.restype = I
            lib.oracle_dsa_attn_bwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, D, P, P, P]
            lib.oracle_dsa_attn_bwd.restype = I
            lib.oracle_hca_compress_bwd.argtypes = [P, P, P, I, I, I, I, I, P, P]
            lib.oracle_hca_compress_bwd.restype = I
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _rows(rows, total):
    if rows is None:
        rows = np.arange(total, dtype=np.int64)
    return _c(rows, np.int64)


def _check(status, what):
    if status != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {status})")


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_f32_to_bf16(_ptr(x), _ptr(out), x.size)
    return out


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.uint16)
    out = np.empty(x.shape, np.float32)
    _load().oracle_bf16_to_f32(_ptr(x), _ptr(out), x.size)
    return out


def hca_window_start(t: int, W: int) -> int:
    return _load().oracle_hca_window_start(t, W)


def hca_n_compressed(t: int, W: int, blk: int) -> int:
    return _load().oracle_hca_n_compressed(t, W, blk)


def hca_compress(X: np.ndarray, w: np.ndarray, blk: int) -> np.ndarray:
    """X: [B, L, H, d] bf16 bits (uint16); w: [blk] fp32 -> [B, L//blk, H, d] bf16 bits."""
    X = _c(X, np.uint16)
    w = _c(w, np.float32)
    B, L, H, d = X.shape
    assert w.shape == (blk,)
    out = np.empty((B, L // blk, H, d), np.uint16)
    _check(_load().oracle_hca_compress(_ptr(X), _ptr(w), _ptr(out), B, L, H, d, blk), "hca_compress")
    return out


def hca_attn(Q, Kc, Vc, Kw, Vw, *, win_start=0, q_offset=0, blk=128, W=128, scale=None,
             rows=None, with_lse=False):
    """Q [B,Lq,Hq,d], Kc/Vc [B,n_c,Hkv,d], Kw/Vw [B,n_w,Hkv,d] (bf16 bits).

    Returns O [n_rows, Hq, d] fp64 (and lse [n_rows, Hq]) for the flat rows b*Lq+r listed
    in ``rows`` (all rows when None)."""
    Q = _c(Q, np.uint16)
    Kw = _c(Kw, np.uint16)
    Vw = _c(Vw, np.uint16)
    B, Lq, Hq, d = Q.shape
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    if Kc is None or Kc.shape[1] == 0:
        n_c, Kc_, Vc_ = 0, None, None
    else:
        Kc_, Vc_ = _c(Kc, np.uint16), _c(Vc, np.uint16)
        n_c = Kc_.shape[1]
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    rows = _rows(rows, B * Lq)
    O = np.empty((rows.size, Hq, d), np.float64)
    lse = np.empty((rows.size, Hq), np.float64) if with_lse else None
    st = _load().oracle_hca_attn(_ptr(Q), _ptr(Kc_), _ptr(Vc_), n_c, _ptr(Kw), _ptr(Vw), win_start,
                                 n_w, B, Lq, q_offset, Hq, Hkv, d, blk, W, float(scale), _ptr(rows),
                                 rows.size, _ptr(O), _ptr(lse))
    _check(st, "hca_attn")
    return (O, lse) if with_lse else O


def hca_attn_latent(Q, Kc, Kw, dv, *, win_start=0, q_offset=0, blk=128, W=128, scale=None, rows=None,
                    with_lse=False):
    """HCA attention with a shared latent: Q [B,Lq,Hq,dqk], Kc [B,n_c,Hkv,dqk] (or None), Kw
    [B,n_w,Hkv,dqk] bf16 bits; the value of a key is the first dv columns of its row.  Returns O
    [n_rows, Hq, dv] fp64 (and lse [n_rows, Hq])."""
    Q = _c(Q, np.uint16)
    Kw = _c(Kw, np.uint16)
    B, Lq, Hq, dqk = Q.shape
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    if Kc is None or Kc.shape[1] == 0:
        n_c, Kc_ = 0, None
    else:
        Kc_ = _c(Kc, np.uint16)
        n_c = Kc_.shape[1]
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(dqk)))
    rows = _rows(rows, B * Lq)
    O = np.empty((rows.size, Hq, dv), np.float64)
    lse = np.empty((rows.size, Hq), np.float64) if with_lse else None
    st = _load().oracle_hca_attn_latent(_ptr(Q), _ptr(Kc_), n_c, _ptr(Kw), win_start, n_w, B, Lq, q_offset, Hq, Hkv,
                                        dqk, dv, blk, W, float(scale), _ptr(rows), rows.size, _ptr(O), _ptr(lse))
    _check(st, "hca_attn_latent")
    return (O, lse) if with_lse else O


def dsa_scores(q_idx, k_idx, w_idx, b, r, n):
    q_idx = _c(q_idx, np.int8)
    k_idx = _c(k_idx, np.int8)
    w_idx = _c(w_idx, np.int32)
    B, Lq, H_idx, d_idx = q_idx.shape
    Lk = k_idx.shape[1]
    out = np.empty(n, np.int64)
    st = _load().oracle_dsa_scores(_ptr(q_idx), _ptr(k_idx), _ptr(w_idx), B, Lq, Lk, H_idx, d_idx,
                                   b, r, n, _ptr(out))
    _check(st, "dsa_scores")
    return out


def dsa_topk(q_idx, k_idx, w_idx, k, *, q_offset=0, rows=None):
    """q_idx [B,Lq,H_idx,d_idx] int8, k_idx [B,Lk,d_idx] int8, w_idx [H_idx] int32.

    Returns idx [n_rows, k] int32: ascending positions, -1 padded."""
    q_idx = _c(q_idx, np.int8)
    k_idx = _c(k_idx, np.int8)
    w_idx = _c(w_idx, np.int32)
    B, Lq, H_idx, d_idx = q_idx.shape
    Lk = k_idx.shape[1]
    rows = _rows(rows, B * Lq)
    out = np.empty((rows.size, k), np.int32)
    st = _load().oracle_dsa_topk(_ptr(q_idx), _ptr(k_idx), _ptr(w_idx), B, Lq, q_offset, Lk, H_idx,
                                 d_idx, k, _ptr(rows), rows.size, _ptr(out))
    _check(st, "dsa_topk")
    return out


def csa_n_candidates(t: int, blk: int, n_c: int) -> int:
    return _load().oracle_csa_n_candidates(t, blk, n_c)


def csa_topk(q_idx, kc_idx, w_idx, k, blk, *, q_offset=0, rows=None):
    """CSA selection over compressed entries: q_idx [B,Lq,H_idx,d_idx] int8, kc_idx [B,n_c,d_idx]
    int8 (one indexer key per entry), w_idx [H_idx] int32; the query at t sees the entries
    j < floor((t+1)/blk).  Returns idx [n_rows, k] int32: ascending entry numbers, -1 padded."""
    q_idx = _c(q_idx, np.int8)
    kc_idx = _c(kc_idx, np.int8)
    w_idx = _c(w_idx, np.int32)
    B, Lq, H_idx, d_idx = q_idx.shape
    n_c = kc_idx.shape[1]
    rows = _rows(rows, B * Lq)
    out = np.empty((rows.size, k), np.int32)
    st = _load().oracle_csa_topk(_ptr(q_idx), _ptr(kc_idx), _ptr(w_idx), B, Lq, q_offset, n_c, H_idx, d_idx,
                                 k, blk, _ptr(rows), rows.size, _ptr(out))
    _check(st, "csa_topk")
    return out


def dsa_attn(Q, K, V, idx_rows, *, scale=None, rows=None, with_lse=False):
    """Q [B,Lq,Hq,d], K/V [B,Lk,d] (one shared head; a [B,Lk,1,d] view is accepted),
    idx_rows [n_rows, k] int32 aligned with ``rows``."""
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, Lq, Hq, d = Q.shape
    Lk = K.shape[1]
    rows = _rows(rows, B * Lq)
    idx_rows = _c(idx_rows, np.int32)
    assert idx_rows.shape[0] == rows.size
    k = idx_rows.shape[1]
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    O = np.empty((rows.size, Hq, d), np.float64)
    lse = np.empty((rows.size, Hq), np.float64) if with_lse else None
    st = _load().oracle_dsa_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx_rows), B, Lq, Lk, Hq, d, k,
                                 float(scale), _ptr(rows), rows.size, _ptr(O), _ptr(lse))
    _check(st, "dsa_attn")
    return (O, lse) if with_lse else O


def gate_vha(O, cq, Wg, U, V):
    """Attention epilogue: Y = sigmoid(cq . Wg^T) * (O + U (V^T O)) per token, channel by channel.

    O [B,L,H,dv], cq [B,L,rq], Wg [H*dv, rq] (bf16 bits); U, V [H, r] fp32 (r may be 0).
    Returns Y [B,L,H,dv] fp64."""
    O = _c(O, np.uint16)
    cq = _c(cq, np.uint16)
    Wg = _c(Wg, np.uint16)
    B, L, H, dv = O.shape
    rq = cq.shape[-1]
    assert cq.shape == (B, L, rq) and Wg.shape == (H * dv, rq)
    U = _c(U, np.float32).reshape(H, -1)
    V = _c(V, np.float32).reshape(H, -1)
    r = U.shape[1]
    assert V.shape == (H, r)
    Y = np.empty((B, L, H, dv), np.float64)
    st = _load().oracle_gate_vha(_ptr(O), _ptr(cq), _ptr(Wg), _ptr(U) if r else None, _ptr(V) if r else None,
                                 B, L, H, dv, rq, r, _ptr(Y))
    _check(st, "gate_vha")
    return Y


# ---------------------------------------------------------------- backward pass


def hca_attn_bwd(Q, Kc, Vc, Kw, Vw, dO, *, win_start=0, q_offset=0, blk=128, W=128, scale=None):
    """Gradients of sum(O * dO) for hca_attn over every query row.

    Q [B,Lq,Hq,d], Kc/Vc [B,n_c,Hkv,d], Kw/Vw [B,n_w,Hkv,d] bf16 bits; dO [B,Lq,Hq,d] fp64.
    Returns fp64 (dQ, dKc, dVc, dKw, dVw) shaped like their inputs (dKc/dVc None when n_c = 0)."""
    Q = _c(Q, np.uint16)
    Kw = _c(Kw, np.uint16)
    Vw = _c(Vw, np.uint16)
    dO = _c(dO, np.float64)
    B, Lq, Hq, d = Q.shape
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    assert dO.shape == Q.shape
    if Kc is None or Kc.shape[1] == 0:
        n_c, Kc_, Vc_, dKc, dVc = 0, None, None, None, None
    else:
        Kc_, Vc_ = _c(Kc, np.uint16), _c(Vc, np.uint16)
        n_c = Kc_.shape[1]
        dKc = np.empty(Kc_.shape, np.float64)
        dVc = np.empty(Kc_.shape, np.float64)
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    dQ = np.empty(Q.shape, np.float64)
    dKw = np.empty(Kw.shape, np.float64)
    dVw = np.empty(Kw.shape, np.float64)
    st = _load().oracle_hca_attn_bwd(_ptr(Q), _ptr(Kc_), _ptr(Vc_), n_c, _ptr(Kw), _ptr(Vw), win_start,
                                     n_w, _ptr(dO), B, Lq, q_offset, Hq, Hkv, d, blk, W, float(scale),
                                     _ptr(dQ), _ptr(dKc), _ptr(dVc), _ptr(dKw), _ptr(dVw))
    _check(st, "hca_attn_bwd")
    return dQ, dKc, dVc, dKw, dVw


def dsa_attn_bwd(Q, K, V, idx, dO, *, scale=None):
    """Gradients of sum(O * dO) for dsa_attn over every query row.

    Q [B,Lq,Hq,d], K/V [B,Lk,d] bf16 bits; idx [B,Lq,k] int32 (-1 padding); dO [B,Lq,Hq,d]
    fp64.  Returns fp64 (dQ, dK, dV)."""
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    dO = _c(dO, np.float64)
    idx = _c(idx, np.int32)
    B, Lq, Hq, d = Q.shape
    Lk = K.shape[1]
    k = idx.shape[-1]
    assert idx.size == B * Lq * k and dO.shape == Q.shape
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    dQ = np.empty(Q.shape, np.float64)
    dK = np.empty((B, Lk, d), np.float64)
    dV = np.empty((B, Lk, d), np.float64)
    st = _load().oracle_dsa_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO), B, Lq, Lk, Hq, d, k,
                                     float(scale), _ptr(dQ), _ptr(dK), _ptr(dV))
    _check(st, "dsa_attn_bwd")
    return dQ, dK, dV


def hca_compress_bwd(X, w, dXc, blk):
    """Adjoint of the compressor as the exact linear map Xc[j] = sum_i w[i] X[blk*j + i].

    X [B,L,H,d] bf16 bits, w [blk] fp32, dXc [B,L//blk,H,d] fp64 -> (dX [B,L,H,d], dw [blk]) fp64."""
    X = _c(X, np.uint16)
    w = _c(w, np.float32)
    dXc = _c(dXc, np.float64)
    B, L, H, d = X.shape
    assert w.shape == (blk,) and dXc.shape == (B, L // blk, H, d)
    dX = np.empty(X.shape, np.float64)
    dw = np.empty(blk, np.float64)
    st = _load().oracle_hca_compress_bwd(_ptr(X), _ptr(w), _ptr(dXc), B, L, H, d, blk, _ptr(dX), _ptr(dw))
    _check(st, "hca_compress_bwd")
    return dX, dw
