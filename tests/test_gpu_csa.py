"""GPU parity of the CSA path (compressed sparse attention: 4:1 compression, indexer + top-k over
the compressed entries, sparse attention over the selected entries) against the CPU oracle.

The CSA layer runs three library calls: hca_compress_kv with a 4-token block, csa_index_topk,
and dsa_sparse_attn_fwd over the compressed K/V.  Bars as everywhere: compression and top-k
bit-exact, attention within max-abs 2e-2 / mean-abs 2e-3 / relative RMS 1e-2 of the fp64
oracle, lse within 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

BLK = 4


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


def check_attn(gpu, ref, what):
    g = gpu.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(g - ref)
    rel = np.sqrt((err ** 2).sum() / max((ref ** 2).sum(), 1e-300))
    assert err.max() <= 2e-2 and err.mean() <= 2e-3 and rel <= 1e-2, (what, err.max(), err.mean(), rel)


def _inputs(B, L, seed, sigma=None):
    cfg = synth.DsaConfig("csa", B=B, L=L, Hq=64, sigma=sigma)
    x = synth.dsa_inputs(cfg, seed=seed)
    n_c = L // BLK
    x["kc_idx"] = synth.randint((B, n_c, 64), -8, 8, seed + 1, "k_idx", torch.int8)
    x["w4"] = synth.uniform_f32((BLK,), 0.0, 2.0 / BLK, seed, "w")
    return x, n_c


@pytest.mark.parametrize("B,L,k", [(2, 1200, 64), (1, 3000, 256), (1, 700, 2048)])
def test_csa_topk_bit_exact_all_rows(hd, B, L, k):
    """Many query rows (the fused tensor-core selection), candidates = complete 4-token blocks."""
    x, n_c = _inputs(B, L, 301 + k)
    idx = hd.csa_index_topk(x["q_idx"].cuda(), x["kc_idx"].cuda(), x["w_idx"].cuda(), k, BLK)
    hd.hcadsa_check_device_error()
    ref = oracle.csa_topk(x["q_idx"].numpy(), x["kc_idx"].numpy(), x["w_idx"].numpy(), k, BLK)
    assert np.array_equal(idx.cpu().numpy().reshape(B * L, k), ref)


@pytest.mark.parametrize("B,t,n_c", [(3, 40003, 10000), (2, 150001, 37500)])
def test_csa_topk_decode_form(hd, B, t, n_c):
    """One query per sequence at position t: the streaming scorer over the entries, with the
    single-block selection (10000 entries) and the multi-CTA selection (37500 entries)."""
    g = torch.Generator().manual_seed(t)
    q = torch.randint(-8, 9, (B, 1, 4, 64), generator=g).to(torch.int8)
    kc = torch.randint(-8, 9, (B, n_c, 64), generator=g).to(torch.int8)
    w = torch.tensor([3, 1, 4, 2], dtype=torch.int32)
    idx = hd.csa_index_topk(q.cuda(), kc.cuda(), w.cuda(), 2048, BLK, q_offset=t)
    hd.hcadsa_check_device_error()
    ref = oracle.csa_topk(q.numpy(), kc.numpy(), w.numpy(), 2048, BLK, q_offset=t)
    assert np.array_equal(idx.cpu().numpy().reshape(B, 2048), ref)


def test_csa_layer_pipeline_all_rows(hd):
    """Compress 4:1 (bit-exact), select over complete blocks (bit-exact), attend over the selected
    entries: every row against the oracle, O and lse; the first three queries have no complete
    block, so O = 0 and lse = -inf."""
    B, L, k = 1, 1500, 128
    x, n_c = _inputs(B, L, 311, sigma=1.0)
    K4 = x["K"].view(B, L, 1, 256).cuda()
    V4 = x["V"].view(B, L, 1, 256).cuda()
    Kc, Vc = hd.hca_compress_kv(K4, V4, x["w4"].cuda(), BLK)
    idx = hd.csa_index_topk(x["q_idx"].cuda(), x["kc_idx"].cuda(), x["w_idx"].cuda(), k, BLK)
    O, lse = hd.dsa_sparse_attn_fwd(x["Q"].cuda(), Kc.view(B, n_c, 256), Vc.view(B, n_c, 256), idx, return_lse=True)
    hd.hcadsa_check_device_error()
    w4 = x["w4"].numpy()
    Kc_o = oracle.hca_compress(bits(x["K"]).reshape(B, L, 1, 256), w4, BLK)
    Vc_o = oracle.hca_compress(bits(x["V"]).reshape(B, L, 1, 256), w4, BLK)
    assert np.array_equal(bits(Kc), Kc_o) and np.array_equal(bits(Vc), Vc_o)
    idx_o = oracle.csa_topk(x["q_idx"].numpy(), x["kc_idx"].numpy(), x["w_idx"].numpy(), k, BLK)
    assert np.array_equal(idx.cpu().numpy().reshape(L, k), idx_o)
    ref, ref_lse = oracle.dsa_attn(bits(x["Q"]), Kc_o.reshape(B, n_c, 256), Vc_o.reshape(B, n_c, 256), idx_o,
                                   with_lse=True)
    O = O.reshape(L, 64, 256)
    lse = lse.reshape(L, 64).cpu().numpy()
    assert torch.count_nonzero(O[:BLK - 1]).item() == 0 and np.all(np.isneginf(lse[:BLK - 1]))
    check_attn(O[BLK - 1:], ref[BLK - 1:], "csa pipeline")
    np.testing.assert_allclose(lse[BLK - 1:], ref_lse[BLK - 1:], atol=2e-3, rtol=0)


def test_csa_layer_32k_sampled(hd):
    """The CSA layer at the MLA-DSA layer's size (L = 32768, 64 heads of 256, top-2048 of up to
    8192 entries): sampled rows against the oracle."""
    B, L, k = 1, 32768, 2048
    x, n_c = _inputs(B, L, 321)
    dev = {n: v.cuda() for n, v in x.items()}
    Kc, Vc = hd.hca_compress_kv(dev["K"].view(B, L, 1, 256), dev["V"].view(B, L, 1, 256), dev["w4"], BLK)
    idx = hd.csa_index_topk(dev["q_idx"], dev["kc_idx"], dev["w_idx"], k, BLK)
    O, lse = hd.dsa_sparse_attn_fwd(dev["Q"], Kc.view(B, n_c, 256), Vc.view(B, n_c, 256), idx, return_lse=True)
    hd.hcadsa_check_device_error()
    rows = np.array([3, 4, 100, 8191, 8192, 8195, 8196, 20000, 32766, 32767], np.int64)
    w4 = x["w4"].numpy()
    Kc_o = oracle.hca_compress(bits(x["K"]).reshape(B, L, 1, 256), w4, BLK).reshape(B, n_c, 256)
    Vc_o = oracle.hca_compress(bits(x["V"]).reshape(B, L, 1, 256), w4, BLK).reshape(B, n_c, 256)
    assert np.array_equal(bits(Kc).reshape(B, n_c, 256), Kc_o)
    idx_o = oracle.csa_topk(x["q_idx"].numpy(), x["kc_idx"].numpy(), x["w_idx"].numpy(), k, BLK, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    assert np.array_equal(idx.reshape(L, k)[r].cpu().numpy(), idx_o)
    ref, ref_lse = oracle.dsa_attn(bits(x["Q"]), Kc_o, Vc_o, idx_o, rows=rows, with_lse=True)
    check_attn(O.reshape(L, 64, 256)[r], ref, "csa 32k sampled")
    np.testing.assert_allclose(lse.reshape(L, 64)[r].cpu().numpy(), ref_lse, atol=2e-3, rtol=0)
