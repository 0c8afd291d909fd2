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
