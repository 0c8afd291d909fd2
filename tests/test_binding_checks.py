"""The Python binding rejects inconsistent tensors before anything reaches the library (CPU):
a caller-provided output or secondary input of the wrong shape or dtype would otherwise be
read or written past its end by a kernel, and a tensor that is not on the current CUDA device
would hand the library a pointer it cannot use."""
import pytest
import torch

import sparse_attention_hca_b200 as hd

bf, i8, i32, f32 = torch.bfloat16, torch.int8, torch.int32, torch.float32
L = 256


def _hca():
    Q = torch.zeros(1, L, 16, 512, dtype=bf)
    K = torch.zeros(1, L, 1, 512, dtype=bf)
    Kc = torch.zeros(1, L // 128, 1, 512, dtype=bf)
    return Q, K, Kc


def _dsa():
    Q = torch.zeros(1, L, 64, 256, dtype=bf)
    K = torch.zeros(1, L, 256, dtype=bf)
    idx = torch.zeros(1, L, 64, dtype=i32)
    return Q, K, idx


@pytest.mark.parametrize("case", ["O", "lse", "Vc", "Vw", "Kw_d"])
def test_hca_attn_rejects_mismatched_tensors(case):
    Q, K, Kc = _hca()
    kw = {}
    Vc, Vw, Kw = Kc, K, K
    if case == "O":
        kw["O"] = torch.zeros(1, L, 16, 256, dtype=bf)
    elif case == "lse":
        kw["lse"] = torch.zeros(1, L, 8, dtype=f32)
    elif case == "Vc":
        Vc = Kc[:, :1].contiguous()
    elif case == "Vw":
        Vw = K[:, : L // 2].contiguous()
    else:
        Kw = torch.zeros(1, L, 1, 256, dtype=bf)
    with pytest.raises(ValueError, match="shape"):
        hd.hca_attn_fwd(Q, Kc, Vc, Kw, Vw if case != "Kw_d" else Kw, **kw)


def test_compress_rejects_small_outputs_and_weights():
    _, K, Kc = _hca()
    with pytest.raises(ValueError, match="shape"):
        hd.hca_compress_kv(K, K, torch.zeros(128, dtype=f32), 128, Kc=Kc[:, :1].contiguous())
    with pytest.raises(ValueError, match="shape"):
        hd.hca_compress_kv(K, K, torch.zeros(64, dtype=f32), 128)


@pytest.mark.parametrize("case", ["V", "idx_rows", "O"])
def test_dsa_attn_rejects_mismatched_tensors(case):
    Q, K, idx = _dsa()
    V, kw = K, {}
    if case == "V":
        V = K[:, :100].contiguous()
    elif case == "idx_rows":
        idx = idx[:, :10].contiguous()
    else:
        kw["O"] = torch.zeros(1, L, 64, 128, dtype=bf)
    with pytest.raises(ValueError, match="shape"):
        hd.dsa_sparse_attn_fwd(Q, K, V, idx, **kw)


def test_index_topk_rejects_mismatched_tensors():
    q = torch.zeros(1, L, 4, 64, dtype=i8)
    k = torch.zeros(1, L, 64, dtype=i8)
    w = torch.zeros(4, dtype=i32)
    with pytest.raises(ValueError, match="shape"):
        hd.dsa_index_topk(q, k, w, 64, idx=torch.zeros(1, L, 32, dtype=i32))
    with pytest.raises(ValueError, match="shape"):
        hd.dsa_index_topk(q, torch.zeros(2, L, 64, dtype=i8), w, 64)
    with pytest.raises(ValueError, match="shape"):
        hd.dsa_index_topk(q, k, torch.zeros(3, dtype=i32), 64)
    with pytest.raises(ValueError, match="int32"):
        hd.dsa_index_topk(q, k, torch.zeros(4, dtype=torch.int64), 64)


def test_consistent_cpu_tensors_are_refused_as_not_cuda():
    Q, K, Kc = _hca()
    with pytest.raises(ValueError, match="CUDA"):
        hd.hca_attn_fwd(Q, Kc, Kc, K, K)
    Qd, Kd, idx = _dsa()
    with pytest.raises(ValueError, match="CUDA"):
        hd.dsa_sparse_attn_fwd(Qd, Kd, Kd, idx)
