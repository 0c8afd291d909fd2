"""GPU parity of the backward kernels against the CPU oracle's fp64 gradients (which are pinned
to torch autograd in test_oracle_pins.py).

Tolerances: gradients are fp32 on the GPU (atomic sums in a free order) against fp64; relative
max error 1e-4 of the gradient's scale for the compressor's exact linear map."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("B,L,H,d,blk", [(1, 32768, 1, 512, 128), (2, 1000, 2, 512, 128), (1, 300, 1, 256, 4)])
def test_compress_bwd_matches_oracle(hd, B, L, H, d, blk):
    cfg = synth.HcaConfig("cb", B=B, L=L, Hq=H, Hkv=H, d=d, blk=blk)
    x = synth.hca_inputs(cfg, seed=811)
    g = torch.Generator().manual_seed(812)
    dXc = torch.randn(B, L // blk, H, d, generator=g)
    dX, dw = hd.hca_compress_bwd(x["K"].cuda(), x["w"].cuda(), dXc.cuda(), blk)
    hd.hcadsa_check_device_error()
    rdX, rdw = oracle.hca_compress_bwd(bits(x["K"]), x["w"].numpy(), dXc.double().numpy(), blk)
    np.testing.assert_allclose(dX.cpu().numpy(), rdX, rtol=0, atol=1e-6 * np.abs(rdX).max())
    np.testing.assert_allclose(dw.cpu().numpy(), rdw, rtol=0, atol=1e-4 * np.abs(rdw).max())
    # accumulation: a second call adds the same amounts again
    hd.hca_compress_bwd(x["K"].cuda(), x["w"].cuda(), dXc.cuda(), blk, dX=dX, dw=dw)
    hd.hcadsa_check_device_error()
    np.testing.assert_allclose(dX.cpu().numpy(), 2 * rdX, rtol=0, atol=2e-6 * np.abs(rdX).max())


def _check_grad(g, ref, what, rel_rms=2e-2, rel_max=1e-1):
    g = g.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(g - ref)
    scale = np.abs(ref).max()
    rr = float(np.sqrt((err ** 2).sum() / max((ref ** 2).sum(), 1e-300)))
    assert rr <= rel_rms and err.max() <= rel_max * scale, (what, rr, err.max(), scale)


def _random_rows(Lq, Lk, k, seed, pad_every=0):
    """Distinct positions per row (padding -1 at random slots when k > Lk or every pad_every-th
    row left empty); rows overlap heavily when k is close to Lk, so dK / dV sum many tokens."""
    rng = np.random.default_rng(seed)
    idx = np.full((Lq, k), -1, np.int32)
    for t in range(Lq):
        if pad_every and t % pad_every == 3:
            continue
        n = min(k, Lk) if t % 2 == 0 else int(rng.integers(1, min(k, Lk) + 1))
        idx[t, rng.choice(k, size=n, replace=False)] = rng.choice(Lk, size=n, replace=False)
    return idx


def _bwd_case(hd, Lq, Lk, k, seed, sigma=None, pad_every=0):
    cfg = synth.DsaConfig("bwd", B=1, L=Lk, Hq=64, k=k, sigma=sigma)
    x = synth.dsa_inputs(cfg, seed=seed)
    Q = x["Q"][:, :Lq].contiguous()
    idx = _random_rows(Lq, Lk, k, seed + 1, pad_every).reshape(1, Lq, k)
    g = torch.Generator().manual_seed(seed + 2)
    dO = (torch.randn(1, Lq, 64, 256, generator=g) * 0.1).to(torch.bfloat16)
    Qd, Kd, Vd = Q.cuda(), x["K"].cuda(), x["V"].cuda()
    idd = torch.as_tensor(idx).cuda()
    O, lse = hd.dsa_sparse_attn_fwd(Qd, Kd, Vd, idd, return_lse=True)
    dQ, dK, dV = hd.dsa_sparse_attn_bwd(Qd, Kd, Vd, idd, O, dO.cuda(), lse)
    hd.hcadsa_check_device_error()
    ref = oracle.dsa_attn_bwd(bits(Q), bits(x["K"]), bits(x["V"]), idx, dO.double().numpy())
    return (dQ, dK, dV), ref, idx


@pytest.mark.parametrize("Lq,Lk,k,sigma", [(64, 300, 64, 1.0), (96, 300, 256, None), (40, 5000, 2048, None),
                                           (24, 9000, 4096, None), (100, 700, 100, 1.0)])
def test_dsa_attn_bwd_matches_oracle(hd, Lq, Lk, k, sigma):
    """Forward on the GPU (O, lse), then the backward, against the oracle's fp64 gradients (which
    redo the forward themselves): dQ, dK, dV over every row, one to 32 key tiles per token, a
    ragged last tile (k = 100), heavy key overlap between tokens (Lk = 300)."""
    got, ref, _ = _bwd_case(hd, Lq, Lk, k, 820 + k, sigma)
    for g, r, what in zip(got, ref, ("dQ", "dK", "dV")):
        _check_grad(g, r, what)


def test_dsa_attn_bwd_padding_rows(hd):
    """-1 padding at random slots and every 37th row empty: empty rows get dQ = 0 and add
    nothing to dK / dV."""
    got, ref, idx = _bwd_case(hd, 120, 400, 128, 831, 1.0, pad_every=37)
    empty = [t for t in range(120) if t % 37 == 3]
    assert torch.count_nonzero(got[0][0, empty]).item() == 0
    for g, r, what in zip(got, ref, ("dQ", "dK", "dV")):
        _check_grad(g, r, what)
