"""GPU parity of HCA attention with FlashMask-4's head shape (qk 576 / v 512, the value of a key
being the first 512 columns of its 576-wide row) against the CPU oracle.  Bars as for the
512-wide HCA attention: max-abs 2e-2, mean-abs 2e-3, relative RMS 1e-2, lse within 2e-3 (2e-2
for sigma = 1 inputs)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
DQK, DV = 576, 512


@pytest.fixture(scope="module")
def hd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_hca_b200 import build

    build.build()
    import sparse_attention_hca_b200 as m

    oracle.build()
    return m


def bits(x):
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check(O, ref, what, s=1.0):
    g = O.float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(g - ref)
    rel = math.sqrt(float((err ** 2).sum()) / float((ref ** 2).sum()))
    assert err.max() <= 2e-2 * s and err.mean() <= 2e-3 * s and rel <= 1e-2, (what, err.max(), err.mean(), rel)


def _prefill(hd, B, L, Hq, Hkv, sigma, seed, blk=128, W=128, rows=None):
    Q = synth.normal_bf16((B, L, Hq, DQK), sigma, seed, "Q")
    K = synth.normal_bf16((B, L, Hkv, DQK), sigma, seed, "K")
    w = synth.uniform_f32((blk,), 0.0, 2.0 / blk, seed, "w")
    Kd = K.cuda()
    # entries: the compressor over all 576 columns (latent and positional slice alike)
    Kc, _ = hd.hca_compress_kv(Kd, Kd, w.cuda(), blk)
    O, lse = hd.hca_attn_fwd_latent(Q.cuda(), Kc, Kd, blk=blk, W=W, return_lse=True)
    hd.hcadsa_check_device_error()
    Kc_o = oracle.hca_compress(bits(K), w.numpy(), blk)
    assert np.array_equal(bits(Kc), Kc_o)
    ref, ref_lse = oracle.hca_attn_latent(bits(Q), Kc_o, bits(K), DV, blk=blk, W=W, rows=rows, with_lse=True)
    O = O.reshape(B * L, Hq, DV)
    lse = lse.reshape(B * L, Hq)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        O, lse = O[r], lse[r]
    return O, lse.cpu().numpy(), ref, ref_lse


@pytest.mark.parametrize("B,L,Hq,Hkv,sigma", [
    (1, 2048, 4, 4, None),     # the tiny configuration's heads, all rows
    (2, 700, 8, 2, 1.0),       # sharper softmax, 4 heads per K/V head, two sequences
    (1, 1003, 16, 1, 1.0),     # 16 heads on one K/V head (8-token row tiles), ragged length
])
def test_latent_hca_all_rows(hd, B, L, Hq, Hkv, sigma):
    s = sigma if sigma is not None else 1.0 / math.sqrt(DQK)
    O, lse, ref, ref_lse = _prefill(hd, B, L, Hq, Hkv, s, 700 + L)
    check(O, ref, f"latent L={L}", max(1.0, s))
    np.testing.assert_allclose(lse, ref_lse, atol=2e-3 if sigma is None else 2e-2, rtol=0)


def test_latent_hca_32k_sampled(hd):
    L = 32768
    rows = np.array([0, 1, 127, 128, 255, 256, 1000, 4095, 4096, 16384, 32000, 32766, 32767])
    O, lse, ref, ref_lse = _prefill(hd, 1, L, 16, 1, 1.0 / math.sqrt(DQK), 733, rows=rows)
    check(O, ref, "latent 32k")
    np.testing.assert_allclose(lse, ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("B,t", [(2, 5000), (32, 200000)])
def test_latent_hca_decode(hd, B, t):
    """One query per sequence at t over [entries | window] (the split / stream-K path)."""
    n_c = (t + 1) // 128
    ws = t - 127
    Kc = synth.normal_bf16((B, n_c, 1, DQK), 1.0, 741, "K")
    Kw = synth.normal_bf16((B, 128, 1, DQK), 1.0, 742, "K")
    Q = synth.normal_bf16((B, 1, 16, DQK), 1.0, 743, "Q")
    O, lse = hd.hca_attn_fwd_latent(Q.cuda(), Kc.cuda(), Kw.cuda(), win_start=ws, q_offset=t, return_lse=True)
    hd.hcadsa_check_device_error()
    ref, ref_lse = oracle.hca_attn_latent(bits(Q), bits(Kc), bits(Kw), DV, win_start=ws, q_offset=t, with_lse=True)
    check(O, ref, f"latent decode B={B}")
    np.testing.assert_allclose(lse.reshape(B, 16).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)
