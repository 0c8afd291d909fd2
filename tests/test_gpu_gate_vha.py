"""GPU parity of the fused output gate + virtual-head mix (attn_gate_vha_fwd) against the CPU
oracle: Y = sigmoid(cq Wg^T) * (O + U (V^T O)) per token and channel.  Bars: max-abs 2e-2,
mean-abs 2e-3 and relative RMS 1e-2 of the fp64 oracle, as for the attention outputs."""
import math

import numpy as np
import pytest
import torch

import oracle

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


def _case(B, L, H, dv, rq, r, seed, o_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    O = (torch.randn(B, L, H, dv, generator=g) * o_scale).to(torch.bfloat16)
    cq = torch.randn(B, L, rq, generator=g).to(torch.bfloat16)
    Wg = (torch.randn(H * dv, rq, generator=g) / math.sqrt(rq)).to(torch.bfloat16)
    U = (torch.randn(H, r, generator=g) * 0.25).float()
    V = (torch.randn(H, r, generator=g) * 0.25).float()
    return O, cq, Wg, U, V


def _check(Y, ref, what):
    g = Y.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    rel = math.sqrt(float((err ** 2).sum()) / float((ref ** 2).sum()))
    assert err.max() <= 2e-2 and err.mean() <= 2e-3 and rel <= 1e-2, (what, err.max(), err.mean(), rel)


@pytest.mark.parametrize("B,L,H,dv,rq,r", [
    (1, 300, 16, 512, 1024, 4),   # HCA heads: 16 x 512, latent 1024 (ragged token tile)
    (2, 130, 64, 256, 1024, 2),   # DSA heads: 64 x 256
    (1, 257, 32, 128, 192, 3),    # 32 heads, short latent, odd rank
    (1, 128, 16, 256, 64, 0),     # gate only (no mix)
])
def test_gate_vha_matches_oracle(hd, B, L, H, dv, rq, r):
    O, cq, Wg, U, V = _case(B, L, H, dv, rq, r, 500 + H + r)
    Y = hd.attn_gate_vha_fwd(O.cuda(), cq.cuda(), Wg.cuda(), U.cuda() if r else None, V.cuda() if r else None)
    hd.hcadsa_check_device_error()
    ref = oracle.gate_vha(bits(O), bits(cq), bits(Wg), U.numpy(), V.numpy())
    _check(Y, ref, f"gate+vha H={H} dv={dv} rq={rq} r={r}")


def test_gate_vha_on_hca_output_32k_sampled(hd):
    """The HCA layer's output size (L = 32768, 16 heads of 512, latent 1024, rank 4): sampled
    tokens against the oracle."""
    B, L, H, dv, rq, r = 1, 32768, 16, 512, 1024, 4
    O, cq, Wg, U, V = _case(B, L, H, dv, rq, r, 555, o_scale=0.05)
    Y = hd.attn_gate_vha_fwd(O.cuda(), cq.cuda(), Wg.cuda(), U.cuda(), V.cuda())
    hd.hcadsa_check_device_error()
    rows = np.array([0, 1, 127, 128, 5000, 16383, 16384, 32766, 32767])
    ref = oracle.gate_vha(bits(O[:, rows]), bits(cq[:, rows]), bits(Wg), U.numpy(), V.numpy())
    _check(Y[:, torch.as_tensor(rows)], ref, "gate+vha 32k")
