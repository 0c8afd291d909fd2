"""Python binding of libhcadsa.so: hybrid sparse attention forward (HCA + MLA-DSA) on B200.

Thin argument marshalling over the C ABI declared in include/hcadsa.h: every step of
the computation runs in the library's CUDA kernels.  PyTorch supplies device memory
and the current CUDA stream.  There is no fallback: if the library is missing or the
tensors are not on a CUDA device, the calls raise.

Functions (same names as the C ABI):
    hca_compress_kv(K, V, w, blk=128)                 -> (Kc, Vc)
    hca_attn_fwd(Q, Kc, Vc, Kw, Vw, ...)              -> O  (or (O, lse))
    hca_attn_fwd_latent(Q, Kc, Kw, ...)               -> O  (qk 576 / v 512, values = latent part of K)
    dsa_index_topk(q_idx, k_idx, w_idx, k, ...)       -> idx
    csa_index_topk(q_idx, kc_idx, w_idx, k, blk, ...) -> idx (over compressed entries)
    dsa_sparse_attn_fwd(Q, K, V, idx, ...)            -> O  (or (O, lse))
    attn_gate_vha_fwd(O, cq, Wg, U, V)                -> Y (output gate + virtual-head mix)
    hcadsa_check_device_error()                       -> raises on a recorded device error
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhcadsa.so")

_lock = threading.Lock()
_lib = None

STATUS = {
    0: "HCADSA_OK", -1: "HCADSA_ERR_NULL", -2: "HCADSA_ERR_SHAPE", -3: "HCADSA_ERR_ALIGN",
    -4: "HCADSA_ERR_UNSUPPORTED", -5: "HCADSA_ERR_WORKSPACE", -6: "HCADSA_ERR_CUDA",
    -7: "HCADSA_ERR_TIMEOUT", -8: "HCADSA_ERR_DEVICE_BOUNDS",
}


class HcaDsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing; build it with "
                                  "`python -m sparse_attention_hca_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            L.hcadsa_version.restype = I
            L.hcadsa_status_string.argtypes = [I]
            L.hcadsa_status_string.restype = ctypes.c_char_p
            L.hcadsa_last_error_string.argtypes = []
            L.hcadsa_last_error_string.restype = ctypes.c_char_p
            L.hcadsa_selftest_bounded_wait.argtypes = [ctypes.c_uint, P]
            L.hcadsa_selftest_bounded_wait.restype = I
            L.hcadsa_check_device_error.argtypes = [P]
            L.hcadsa_check_device_error.restype = I
            L.hca_compress_kv.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
            L.hca_compress_kv.restype = I
            L.hca_attn_fwd_workspace_size.argtypes = [I] * 9
            L.hca_attn_fwd_workspace_size.restype = S
            L.hca_attn_fwd.argtypes = [P, P, P, I, P, P, I, I, P, P, I, I, I, I, I, I, I, I, F, P, S, P]
            L.hca_attn_fwd.restype = I
            L.hca_attn_fwd_latent_workspace_size.argtypes = [I] * 10
            L.hca_attn_fwd_latent_workspace_size.restype = S
            L.hca_attn_fwd_latent.argtypes = [P, P, I, P, I, I, P, P, I, I, I, I, I, I, I, I, I, F, P, S, P]
            L.hca_attn_fwd_latent.restype = I
            L.dsa_index_topk_workspace_size.argtypes = [I, I, I, I, I]
            L.dsa_index_topk_workspace_size.restype = S
            L.dsa_index_topk.argtypes = [P, P, P, P, P, S, I, I, I, I, I, I, I, P]
            L.dsa_index_topk.restype = I
            L.csa_index_topk_workspace_size.argtypes = [I, I, I, I, I, I]
            L.csa_index_topk_workspace_size.restype = S
            L.csa_index_topk.argtypes = [P, P, P, P, P, S, I, I, I, I, I, I, I, I, P]
            L.csa_index_topk.restype = I
            L.dsa_index_topk_noalloc_max_scratch_bytes.argtypes = []
            L.dsa_index_topk_noalloc_max_scratch_bytes.restype = S
            L.dsa_index_topk_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P]
            L.dsa_index_topk_noalloc.restype = I
            L.dsa_sparse_attn_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P]
            L.dsa_sparse_attn_fwd.restype = I
            L.dsa_sparse_attn_fwd_workspace_size.argtypes = [I, I, I]
            L.dsa_sparse_attn_fwd_workspace_size.restype = S
            L.dsa_sparse_attn_fwd_ws.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P, S, P]
            L.dsa_sparse_attn_fwd_ws.restype = I
            L.attn_gate_vha_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
            L.attn_gate_vha_fwd.restype = I
            L.hca_compress_bwd.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
            L.hca_compress_bwd.restype = I
            L.dsa_sparse_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
            L.dsa_sparse_attn_bwd.restype = I
            L.hca_attn_bwd_workspace_size.argtypes = [I] * 9
            L.hca_attn_bwd_workspace_size.restype = S
            L.hca_attn_bwd.argtypes = [P, P, P, I, P, P, I, I, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P,
                                       S, P]
            L.hca_attn_bwd.restype = I
            _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        if status == -6:
            what = f"{what} ({lib().hcadsa_last_error_string().decode(errors='replace')})"
        raise HcaDsaError(status, what)


def _need(t, dtype, name, shape=None):
    """dtype, contiguity and (optionally) exact shape; the device is checked by _on_device."""
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _need_numel(t, n, name, what):
    if t.numel() != n:
        raise ValueError(f"{name} has {t.numel()} elements, expected {n} ({what})")


def _on_device(*tensors):
    """Every tensor must be a CUDA tensor on the current device: the library launches on the
    current device's stream and reads the pointers there."""
    cur = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("every tensor must be a CUDA tensor")
        if cur is None:
            cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"tensor on {t.device}, but the current device is cuda:{cur}; "
                             f"call under torch.cuda.device({t.device})")


def _bf16(t):
    return t.view(torch.int16) if t is not None else None


def hcadsa_check_device_error(stream=None):
    """Synchronises the stream and raises if a kernel recorded a device-side error."""
    _check(lib().hcadsa_check_device_error(_stream(stream)), "device")


def hca_compress_kv(K, V, w, blk: int = 128, *, Kc=None, Vc=None, stream=None):
    """K, V: [B, L, Hkv, d] bf16; w: [blk] fp32 -> Kc, Vc: [B, L // blk, Hkv, d] bf16."""
    _need(K, torch.bfloat16, "K")
    B, L, Hkv, d = K.shape
    _need(V, torch.bfloat16, "V", K.shape)
    _need(w, torch.float32, "w", (blk,))
    shape = (B, L // blk, Hkv, d)
    if Kc is not None:
        _need(Kc, torch.bfloat16, "Kc", shape)
    if Vc is not None:
        _need(Vc, torch.bfloat16, "Vc", shape)
    _on_device(K, V, w, Kc, Vc)
    Kc = torch.empty(shape, dtype=torch.bfloat16, device=K.device) if Kc is None else Kc
    Vc = torch.empty(shape, dtype=torch.bfloat16, device=K.device) if Vc is None else Vc
    st = lib().hca_compress_kv(_ptr(K), _ptr(V), _ptr(w), _ptr(Kc), _ptr(Vc), B, L, Hkv, d, blk,
                               _stream(stream))
    _check(st, "hca_compress_kv")
    return Kc, Vc


def hca_attn_fwd(Q, Kc, Vc, Kw, Vw, *, win_start: int = 0, q_offset: int = 0, blk: int = 128,
                 W: int = 128, scale: float | None = None, O=None, lse=None, return_lse=False,
                 workspace=None, stream=None):
    """Q: [B, Lq, Hq, d]; Kc/Vc: [B, n_c, Hkv, d] (or None); Kw/Vw: [B, n_w, Hkv, d]."""
    _need(Q, torch.bfloat16, "Q")
    B, Lq, Hq, d = Q.shape
    _need(Kw, torch.bfloat16, "Kw")
    if Kw.dim() != 4 or Kw.shape[0] != B or Kw.shape[3] != d:
        raise ValueError(f"Kw has shape {tuple(Kw.shape)}, expected [{B}, n_w, Hkv, {d}]")
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    _need(Vw, torch.bfloat16, "Vw", Kw.shape)
    n_c = 0 if Kc is None else Kc.shape[1]
    if n_c:
        _need(Kc, torch.bfloat16, "Kc", (B, n_c, Hkv, d))
        _need(Vc, torch.bfloat16, "Vc", (B, n_c, Hkv, d))
    if O is not None:
        _need(O, torch.bfloat16, "O", Q.shape)
    if lse is not None:
        _need(lse, torch.float32, "lse", (B, Lq, Hq))
    if workspace is not None and not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device(Q, Kw, Vw, Kc if n_c else None, Vc if n_c else None, O, lse, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = torch.empty_like(Q) if O is None else O
    if return_lse and lse is None:
        lse = torch.empty((B, Lq, Hq), dtype=torch.float32, device=Q.device)
    L = lib()
    ws_bytes = L.hca_attn_fwd_workspace_size(B, Lq, q_offset, Hq, Hkv, d, n_c, blk, W)
    if workspace is None:
        if ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    else:
        ws_bytes = workspace.numel() * workspace.element_size()
    st = L.hca_attn_fwd(_ptr(Q), _ptr(Kc) if n_c else None, _ptr(Vc) if n_c else None, n_c, _ptr(Kw),
                        _ptr(Vw), win_start, n_w, _ptr(O), _ptr(lse), B, Lq, q_offset, Hq, Hkv, d, blk, W,
                        float(scale), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "hca_attn_fwd")
    return (O, lse) if return_lse else O


def hca_attn_fwd_latent(Q, Kc, Kw, *, dv: int = 512, win_start: int = 0, q_offset: int = 0, blk: int = 128,
                        W: int = 128, scale: float | None = None, O=None, lse=None, return_lse=False,
                        workspace=None, stream=None):
    """FlashMask-4's head shape: Q [B, Lq, Hq, 576]; Kc [B, n_c, Hkv, 576] (or None); Kw [B, n_w,
    Hkv, 576]; the value of a key is the first dv = 512 columns of its row -> O [B, Lq, Hq, 512]."""
    _need(Q, torch.bfloat16, "Q")
    B, Lq, Hq, dqk = Q.shape
    _need(Kw, torch.bfloat16, "Kw")
    if Kw.dim() != 4 or Kw.shape[0] != B or Kw.shape[3] != dqk:
        raise ValueError(f"Kw has shape {tuple(Kw.shape)}, expected [{B}, n_w, Hkv, {dqk}]")
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    n_c = 0 if Kc is None else Kc.shape[1]
    if n_c:
        _need(Kc, torch.bfloat16, "Kc", (B, n_c, Hkv, dqk))
    if O is not None:
        _need(O, torch.bfloat16, "O", (B, Lq, Hq, dv))
    if lse is not None:
        _need(lse, torch.float32, "lse", (B, Lq, Hq))
    if workspace is not None and not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device(Q, Kw, Kc if n_c else None, O, lse, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    O = torch.empty((B, Lq, Hq, dv), dtype=torch.bfloat16, device=Q.device) if O is None else O
    if return_lse and lse is None:
        lse = torch.empty((B, Lq, Hq), dtype=torch.float32, device=Q.device)
    L = lib()
    ws_bytes = L.hca_attn_fwd_latent_workspace_size(B, Lq, q_offset, Hq, Hkv, dqk, dv, n_c, blk, W)
    if workspace is None:
        if ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    else:
        ws_bytes = workspace.numel() * workspace.element_size()
    st = L.hca_attn_fwd_latent(_ptr(Q), _ptr(Kc) if n_c else None, n_c, _ptr(Kw), win_start, n_w, _ptr(O), _ptr(lse),
                               B, Lq, q_offset, Hq, Hkv, dqk, dv, blk, W, float(scale), _ptr(workspace), ws_bytes,
                               _stream(stream))
    _check(st, "hca_attn_fwd_latent")
    return (O, lse) if return_lse else O


def dsa_index_topk_workspace_size(B, Lq, q_offset, Lk, k) -> int:
    return lib().dsa_index_topk_workspace_size(B, Lq, q_offset, Lk, k)


def _check_index_args(q_idx, k_idx, w_idx, k, idx):
    _need(q_idx, torch.int8, "q_idx")
    B, Lq, H_idx, d_idx = q_idx.shape
    _need(k_idx, torch.int8, "k_idx")
    if k_idx.shape[0] != B or k_idx.shape[-1] != d_idx:
        raise ValueError(f"k_idx has shape {tuple(k_idx.shape)}, expected [{B}, Lk, {d_idx}]")
    Lk = k_idx.shape[1]
    _need_numel(k_idx, B * Lk * d_idx, "k_idx", f"[{B}, {Lk}, {d_idx}]")
    _need(w_idx, torch.int32, "w_idx", (H_idx,))
    if idx is not None:
        _need(idx, torch.int32, "idx", (B, Lq, k))
    return B, Lq, H_idx, d_idx, Lk


def dsa_index_topk(q_idx, k_idx, w_idx, k: int, *, q_offset: int = 0, idx=None, workspace=None,
                   stream=None):
    """q_idx: [B, Lq, 4, 64] int8; k_idx: [B, Lk, 64] int8; w_idx: [4] int32 -> idx [B, Lq, k] int32."""
    B, Lq, H_idx, d_idx, Lk = _check_index_args(q_idx, k_idx, w_idx, k, idx)
    if workspace is not None and not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device(q_idx, k_idx, w_idx, idx, workspace)
    idx = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device) if idx is None else idx
    ws_bytes = dsa_index_topk_workspace_size(B, Lq, q_offset, Lk, k)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q_idx.device)
    st = lib().dsa_index_topk(_ptr(q_idx), _ptr(k_idx), _ptr(w_idx), _ptr(idx), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), B, Lq, q_offset, Lk, H_idx,
                              d_idx, k, _stream(stream))
    _check(st, "dsa_index_topk")
    return idx


def csa_index_topk(q_idx, kc_idx, w_idx, k: int, blk: int = 4, *, q_offset: int = 0, idx=None, workspace=None,
                   stream=None):
    """q_idx: [B, Lq, 4, 64] int8; kc_idx: [B, n_c, 64] int8 (one key per compressed entry);
    w_idx: [4] int32 -> idx [B, Lq, k] int32 (entry numbers; the query at t sees the entries of
    complete blocks, j < (t + 1) // blk)."""
    B, Lq, H_idx, d_idx, n_c = _check_index_args(q_idx, kc_idx, w_idx, k, idx)
    if workspace is not None and not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device(q_idx, kc_idx, w_idx, idx, workspace)
    idx = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device) if idx is None else idx
    ws_bytes = lib().csa_index_topk_workspace_size(B, Lq, q_offset, n_c, k, blk)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q_idx.device)
    st = lib().csa_index_topk(_ptr(q_idx), _ptr(kc_idx), _ptr(w_idx), _ptr(idx), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), B, Lq, q_offset, n_c, H_idx, d_idx,
                              k, blk, _stream(stream))
    _check(st, "csa_index_topk")
    return idx


def dsa_index_topk_noalloc(q_idx, k_idx, w_idx, k: int, *, q_offset: int = 0, idx=None, stream=None):
    """dsa_index_topk for callers that cannot allocate device memory: the score rows go to a
    fixed 64 MiB array inside the library (see include/hcadsa.h for its limits and sharing).
    The output tensor is still the caller's; pass ``idx`` to avoid allocating it here."""
    B, Lq, H_idx, d_idx, Lk = _check_index_args(q_idx, k_idx, w_idx, k, idx)
    _on_device(q_idx, k_idx, w_idx, idx)
    idx = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device) if idx is None else idx
    st = lib().dsa_index_topk_noalloc(_ptr(q_idx), _ptr(k_idx), _ptr(w_idx), _ptr(idx), B, Lq, q_offset, Lk,
                                      H_idx, d_idx, k, _stream(stream))
    _check(st, "dsa_index_topk_noalloc")
    return idx


def dsa_sparse_attn_fwd(Q, K, V, idx, *, scale: float | None = None, O=None, lse=None,
                        return_lse=False, split: bool = True, workspace=None, stream=None):
    """Q: [B, Lq, 64, 256]; K, V: [B, Lk, 256]; idx: [B, Lq, k] int32 -> O [B, Lq, 64, 256].

    With split (the default), calls with few query rows divide each row's key tiles among
    several CTAs through a workspace (allocated here unless given); split=False always runs
    one CTA per query row."""
    _need(Q, torch.bfloat16, "Q")
    B, Lq, Hq, d = Q.shape
    _need(K, torch.bfloat16, "K")  # [B, Lk, d] (a [B, Lk, 1, d] view of one shared head is accepted)
    if K.shape[0] != B or K.shape[-1] != d:
        raise ValueError(f"K has shape {tuple(K.shape)}, expected [{B}, Lk, {d}]")
    Lk = K.shape[1]
    _need_numel(K, B * Lk * d, "K", f"[{B}, {Lk}, {d}]: one shared K/V head")
    _need(V, torch.bfloat16, "V", K.shape)
    _need(idx, torch.int32, "idx")
    if idx.dim() != 3 or idx.shape[0] != B or idx.shape[1] != Lq:
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected [{B}, {Lq}, k]")
    k = idx.shape[-1]
    if O is not None:
        _need(O, torch.bfloat16, "O", Q.shape)
    if lse is not None:
        _need(lse, torch.float32, "lse", (B, Lq, Hq))
    _on_device(Q, K, V, idx, O, lse)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = torch.empty_like(Q) if O is None else O
    if return_lse and lse is None:
        lse = torch.empty((B, Lq, Hq), dtype=torch.float32, device=Q.device)
    L = lib()
    if not split:
        st = L.dsa_sparse_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(O), _ptr(lse), B, Lq, Lk,
                                   Hq, d, k, float(scale), _stream(stream))
        _check(st, "dsa_sparse_attn_fwd")
        return (O, lse) if return_lse else O
    ws_bytes = L.dsa_sparse_attn_fwd_workspace_size(B, Lq, k)
    if workspace is None:
        if ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    else:
        if not workspace.is_contiguous():
            raise ValueError("workspace must be contiguous")
        _on_device(workspace)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = L.dsa_sparse_attn_fwd_ws(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(O), _ptr(lse), B, Lq, Lk, Hq, d, k,
                                  float(scale), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "dsa_sparse_attn_fwd_ws")
    return (O, lse) if return_lse else O


def attn_gate_vha_fwd(O, cq, Wg, U=None, V=None, *, Y=None, stream=None):
    """O: [B, L, H, dv] bf16; cq: [B, L, rq] bf16; Wg: [H*dv, rq] bf16; U, V: [H, r] fp32 (or None)
    -> Y = sigmoid(cq Wg^T) * (O + U (V^T O)) per token, [B, L, H, dv] bf16."""
    _need(O, torch.bfloat16, "O")
    B, L, H, dv = O.shape
    _need(cq, torch.bfloat16, "cq")
    if cq.dim() != 3 or cq.shape[0] != B or cq.shape[1] != L:
        raise ValueError(f"cq has shape {tuple(cq.shape)}, expected [{B}, {L}, rq]")
    rq = cq.shape[2]
    _need(Wg, torch.bfloat16, "Wg", (H * dv, rq))
    r = 0
    if U is not None or V is not None:
        if U is None or V is None:
            raise ValueError("U and V go together")
        _need(U, torch.float32, "U")
        if U.dim() != 2 or U.shape[0] != H:
            raise ValueError(f"U has shape {tuple(U.shape)}, expected [{H}, r]")
        r = U.shape[1]
        _need(V, torch.float32, "V", (H, r))
    if Y is not None:
        _need(Y, torch.bfloat16, "Y", O.shape)
    _on_device(O, cq, Wg, U, V, Y)
    Y = torch.empty_like(O) if Y is None else Y
    st = lib().attn_gate_vha_fwd(_ptr(O), _ptr(cq), _ptr(Wg), _ptr(U) if r else None, _ptr(V) if r else None,
                                 _ptr(Y), B, L, H, dv, rq, r, _stream(stream))
    _check(st, "attn_gate_vha_fwd")
    return Y


def hca_compress_bwd(X, w, dXc, blk: int = 128, *, dX=None, dw=None, stream=None):
    """Adjoint of hca_compress_kv: X [B, L, H, d] bf16, w [blk] fp32, dXc [B, L//blk, H, d] fp32 ->
    (dX [B, L, H, d] fp32, dw [blk] fp32), both added to when given (zeros otherwise)."""
    _need(X, torch.bfloat16, "X")
    B, L, H, d = X.shape
    _need(w, torch.float32, "w", (blk,))
    _need(dXc, torch.float32, "dXc", (B, L // blk, H, d))
    if dX is not None:
        _need(dX, torch.float32, "dX", X.shape)
    if dw is not None:
        _need(dw, torch.float32, "dw", (blk,))
    _on_device(X, w, dXc, dX, dw)
    dX = torch.zeros(X.shape, dtype=torch.float32, device=X.device) if dX is None else dX
    dw = torch.zeros(blk, dtype=torch.float32, device=X.device) if dw is None else dw
    st = lib().hca_compress_bwd(_ptr(X), _ptr(w), _ptr(dXc), _ptr(dX), _ptr(dw), B, L, H, d, blk, _stream(stream))
    _check(st, "hca_compress_bwd")
    return dX, dw


def dsa_sparse_attn_bwd(Q, K, V, idx, O, dO, lse, *, scale: float | None = None, dK=None, dV=None, stream=None):
    """Gradients of the DSA sparse attention: Q, O, dO [B, Lq, 64, 256] bf16, K, V [B, Lk, 256] bf16,
    idx [B, Lq, k] int32, lse [B, Lq, 64] fp32 (from the forward) -> (dQ [B, Lq, 64, 256] fp32,
    dK, dV [B, Lk, 256] fp32; dK and dV are added to when given, zeros otherwise)."""
    _need(Q, torch.bfloat16, "Q")
    B, Lq, Hq, d = Q.shape
    _need(K, torch.bfloat16, "K")
    if K.shape[0] != B or K.shape[-1] != d:
        raise ValueError(f"K has shape {tuple(K.shape)}, expected [{B}, Lk, {d}]")
    Lk = K.shape[1]
    _need_numel(K, B * Lk * d, "K", f"[{B}, {Lk}, {d}]")
    _need(V, torch.bfloat16, "V", K.shape)
    _need(idx, torch.int32, "idx")
    if idx.dim() != 3 or idx.shape[0] != B or idx.shape[1] != Lq:
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected [{B}, {Lq}, k]")
    k = idx.shape[-1]
    _need(O, torch.bfloat16, "O", Q.shape)
    _need(dO, torch.bfloat16, "dO", Q.shape)
    _need(lse, torch.float32, "lse", (B, Lq, Hq))
    if dK is not None:
        _need_numel(dK, B * Lk * d, "dK", "fp32 like K")
    if dV is not None:
        _need_numel(dV, B * Lk * d, "dV", "fp32 like V")
    _on_device(Q, K, V, idx, O, dO, lse, dK, dV)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    dK = torch.zeros((B, Lk, d), dtype=torch.float32, device=Q.device) if dK is None else dK
    dV = torch.zeros((B, Lk, d), dtype=torch.float32, device=Q.device) if dV is None else dV
    st = lib().dsa_sparse_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(O), _ptr(dO), _ptr(lse), _ptr(dQ),
                                   _ptr(dK), _ptr(dV), B, Lq, Lk, Hq, d, k, float(scale), _stream(stream))
    _check(st, "dsa_sparse_attn_bwd")
    return dQ, dK, dV


def hca_attn_bwd(Q, Kc, Vc, Kw, Vw, O, dO, lse, *, win_start: int = 0, q_offset: int = 0, blk: int = 128,
                 W: int = 128, scale: float | None = None, dKc=None, dVc=None, dKw=None, dVw=None, workspace=None,
                 stream=None):
    """Gradients of the HCA attention: Q, O, dO [B, Lq, Hq, 512] bf16, Kc/Vc [B, n_c, Hkv, 512] (or
    None), Kw/Vw [B, n_w, Hkv, 512] bf16, lse [B, Lq, Hq] fp32 from the forward ->
    (dQ fp32 like Q, dKc, dVc fp32 like Kc (None if n_c = 0), dKw, dVw fp32 like Kw); the key and
    value gradients are added to when given, zeros otherwise."""
    _need(Q, torch.bfloat16, "Q")
    B, Lq, Hq, d = Q.shape
    _need(Kw, torch.bfloat16, "Kw")
    if Kw.dim() != 4 or Kw.shape[0] != B or Kw.shape[3] != d:
        raise ValueError(f"Kw has shape {tuple(Kw.shape)}, expected [{B}, n_w, Hkv, {d}]")
    n_w, Hkv = Kw.shape[1], Kw.shape[2]
    _need(Vw, torch.bfloat16, "Vw", Kw.shape)
    n_c = 0 if Kc is None else Kc.shape[1]
    if n_c:
        _need(Kc, torch.bfloat16, "Kc", (B, n_c, Hkv, d))
        _need(Vc, torch.bfloat16, "Vc", (B, n_c, Hkv, d))
    _need(O, torch.bfloat16, "O", Q.shape)
    _need(dO, torch.bfloat16, "dO", Q.shape)
    _need(lse, torch.float32, "lse", (B, Lq, Hq))
    for t, n, shp in ((dKc, "dKc", (B, n_c, Hkv, d)), (dVc, "dVc", (B, n_c, Hkv, d)), (dKw, "dKw", Kw.shape),
                      (dVw, "dVw", Kw.shape)):
        if t is not None:
            _need(t, torch.float32, n, shp)
    if workspace is not None and not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device(Q, Kw, Vw, Kc if n_c else None, Vc if n_c else None, O, dO, lse, dKc, dVc, dKw, dVw, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = Q.device
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    if n_c:
        dKc = torch.zeros((B, n_c, Hkv, d), dtype=torch.float32, device=dev) if dKc is None else dKc
        dVc = torch.zeros((B, n_c, Hkv, d), dtype=torch.float32, device=dev) if dVc is None else dVc
    dKw = torch.zeros(tuple(Kw.shape), dtype=torch.float32, device=dev) if dKw is None else dKw
    dVw = torch.zeros(tuple(Kw.shape), dtype=torch.float32, device=dev) if dVw is None else dVw
    L = lib()
    ws_bytes = L.hca_attn_bwd_workspace_size(B, Lq, q_offset, Hq, Hkv, d, n_c, blk, W)
    if workspace is None:
        if ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    else:
        ws_bytes = workspace.numel() * workspace.element_size()
    st = L.hca_attn_bwd(_ptr(Q), _ptr(Kc) if n_c else None, _ptr(Vc) if n_c else None, n_c, _ptr(Kw), _ptr(Vw),
                        win_start, n_w, _ptr(O), _ptr(dO), _ptr(lse), _ptr(dQ), _ptr(dKc) if n_c else None,
                        _ptr(dVc) if n_c else None, _ptr(dKw), _ptr(dVw), B, Lq, q_offset, Hq, Hkv, d, blk, W,
                        float(scale), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "hca_attn_bwd")
    return dQ, (dKc if n_c else None), (dVc if n_c else None), dKw, dVw
