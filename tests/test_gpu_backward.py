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


def _hca_bwd_gpu(hd, Q, Kc, Vc, Kw, Vw, dO, **kw):
    """Forward (O, lse) then backward on the GPU, over the given cache tensors."""
    dev = [t.cuda() if t is not None else None for t in (Q, Kc, Vc, Kw, Vw, dO)]
    Qd, Kcd, Vcd, Kwd, Vwd, dOd = dev
    O, lse = hd.hca_attn_fwd(Qd, Kcd, Vcd, Kwd, Vwd, return_lse=True, **kw)
    out = hd.hca_attn_bwd(Qd, Kcd, Vcd, Kwd, Vwd, O, dOd, lse, **kw)
    hd.hcadsa_check_device_error()
    return out


@pytest.mark.parametrize("B,L,Hq,Hkv,blk,W,sigma", [
    (1, 600, 16, 1, 128, 128, None),   # the HCA layer's head grouping, 3 entries
    (2, 700, 8, 2, 64, 96, 1.0),       # 4 heads per K/V head, two sequences, ragged last row tile
    (1, 300, 2, 2, 16, 64, 1.0),       # one head per K/V head: 128-token row tiles, 3 window tiles
    (1, 200, 128, 1, 32, 64, 1.0),     # 128 heads per K/V head: one-token row tiles
    (1, 1200, 4, 1, 4, 128, 1.0),      # 268 entries: 3 entry tiles, dK/dV units over several chunks
])
def test_hca_attn_bwd_matches_oracle(hd, B, L, Hq, Hkv, blk, W, sigma):
    """Every row and every key: dQ, dKc, dVc (compressed entries) and dKw, dVw (raw window keys)
    against the oracle's fp64 gradients."""
    cfg = synth.HcaConfig("hbwd", B=B, L=L, Hq=Hq, Hkv=Hkv, blk=blk, W=W, sigma=sigma)
    x = synth.hca_inputs(cfg, seed=841 + L)
    w = x["w"].numpy()
    Kc = torch.as_tensor(oracle.hca_compress(bits(x["K"]), w, blk).view(np.int16)).view(torch.bfloat16)
    Vc = torch.as_tensor(oracle.hca_compress(bits(x["V"]), w, blk).view(np.int16)).view(torch.bfloat16)
    g = torch.Generator().manual_seed(842)
    dO = (torch.randn(B, L, Hq, 512, generator=g) * 0.1).to(torch.bfloat16)
    dQ, dKc, dVc, dKw, dVw = _hca_bwd_gpu(hd, x["Q"], Kc, Vc, x["K"], x["V"], dO, blk=blk, W=W)
    ref = oracle.hca_attn_bwd(bits(x["Q"]), bits(Kc), bits(Vc), bits(x["K"]), bits(x["V"]), dO.double().numpy(),
                              blk=blk, W=W)
    for got, r, what in zip((dQ, dKc, dVc, dKw, dVw), ref, ("dQ", "dKc", "dVc", "dKw", "dVw")):
        _check_grad(got, r, what)


def test_hca_attn_bwd_chunk_at_offset(hd):
    """A chunk of 300 query tokens at positions 4000..4299 of two sequences over the entries stored
    so far and a window buffer that starts at the first query's window."""
    d, Hq, blk, W, B, Lq, t0 = 512, 16, 128, 128, 2, 300, 4000
    t_last = t0 + Lq - 1
    n_c = (t_last - W + 1) // blk
    ws = t0 - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 851, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 851, "V")
    Kw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 852, "K")
    Vw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 852, "V")
    Q = synth.normal_bf16((B, Lq, Hq, d), 1.0, 853, "Q")
    g = torch.Generator().manual_seed(854)
    dO = (torch.randn(B, Lq, Hq, d, generator=g) * 0.1).to(torch.bfloat16)
    got = _hca_bwd_gpu(hd, Q, Kc, Vc, Kw, Vw, dO, win_start=ws, q_offset=t0)
    ref = oracle.hca_attn_bwd(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), dO.double().numpy(), win_start=ws,
                              q_offset=t0)
    for gg, r, what in zip(got, ref, ("dQ", "dKc", "dVc", "dKw", "dVw")):
        _check_grad(gg, r, what)


def test_hca_attn_bwd_32k(hd):
    """The HCA layer's size (L = 32768, 16 heads on one K/V head, 256 entries): dQ of sampled row
    chunks against the oracle; the raw-key gradients of two window keys exactly (the oracle over
    the W + 1 query rows that see them); and two sums that hold at any size: the value gradients
    of all keys add up to the sum of dO over all rows (each row's probabilities sum to 1), and the
    key gradients to ~0 (each row's dS sums to 0)."""
    cfg = synth.HCA_32K
    B, L, Hq, blk, W = cfg.B, cfg.L, cfg.Hq, cfg.blk, cfg.W
    x = synth.hca_inputs(cfg, seed=861)
    dev = {n: v.cuda() for n, v in x.items()}
    Kc, Vc = hd.hca_compress_kv(dev["K"], dev["V"], dev["w"], blk)
    g = torch.Generator(device="cuda").manual_seed(862)
    dO = (torch.randn(B, L, Hq, 512, generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    O, lse = hd.hca_attn_fwd(dev["Q"], Kc, Vc, dev["K"], dev["V"], return_lse=True)
    dQ, dKc, dVc, dKw, dVw = hd.hca_attn_bwd(dev["Q"], Kc, Vc, dev["K"], dev["V"], O, dO, lse)
    hd.hcadsa_check_device_error()
    Kc_h, Vc_h = bits(Kc), bits(Vc)
    dO_h = dO.cpu()
    Kb, Vb = bits(x["K"]), bits(x["V"])
    for r0, n in ((0, 24), (16380, 24), (32744, 24)):
        ref = oracle.hca_attn_bwd(bits(x["Q"][:, r0:r0 + n]), Kc_h, Vc_h, Kb, Vb,
                                  dO_h[:, r0:r0 + n].double().numpy(), q_offset=r0)
        _check_grad(dQ[:, r0:r0 + n], ref[0], f"dQ rows {r0}..")
    s = 20000  # keys s and s + 1 are seen by the rows s .. s + W exactly
    ref = oracle.hca_attn_bwd(bits(x["Q"][:, s:s + W + 1]), Kc_h, Vc_h, Kb, Vb,
                              dO_h[:, s:s + W + 1].double().numpy(), q_offset=s)
    _check_grad(dKw[:, s:s + 2], ref[3][:, s:s + 2], "dKw keys 20000, 20001")
    _check_grad(dVw[:, s:s + 2], ref[4][:, s:s + 2], "dVw keys 20000, 20001")
    sum_dv = (dVc.double().sum(dim=(0, 1, 2)) + dVw.double().sum(dim=(0, 1, 2))).cpu().numpy()
    sum_do = dO.double().sum(dim=(0, 1, 2)).cpu().numpy()
    assert np.abs(sum_dv - sum_do).max() <= 1e-2 * np.abs(sum_do).max() + 1e-3, np.abs(sum_dv - sum_do).max()
    sum_dk = (dKc.double().sum(dim=(0, 1, 2)) + dKw.double().sum(dim=(0, 1, 2))).cpu().numpy()
    abs_dk = (dKc.double().abs().sum(dim=(0, 1, 2)) + dKw.double().abs().sum(dim=(0, 1, 2))).cpu().numpy()
    assert np.all(np.abs(sum_dk) <= 1e-2 * abs_dk), (np.abs(sum_dk) / abs_dk).max()


def test_dsa_attn_bwd_two_sequences(hd):
    """Two sequences with their own K/V: gradients land in each sequence's own dK / dV rows."""
    B, Lq, Lk, k = 2, 48, 1500, 512
    cfg = synth.DsaConfig("bwdb2", B=B, L=Lk, Hq=64, k=k, sigma=1.0)
    x = synth.dsa_inputs(cfg, seed=871)
    Q = x["Q"][:, :Lq].contiguous()
    idx = np.stack([_random_rows(Lq, Lk, k, 872 + b) for b in range(B)])
    g = torch.Generator().manual_seed(873)
    dO = (torch.randn(B, Lq, 64, 256, generator=g) * 0.1).to(torch.bfloat16)
    Qd, Kd, Vd, idd = Q.cuda(), x["K"].cuda(), x["V"].cuda(), torch.as_tensor(idx).cuda()
    O, lse = hd.dsa_sparse_attn_fwd(Qd, Kd, Vd, idd, return_lse=True)
    got = hd.dsa_sparse_attn_bwd(Qd, Kd, Vd, idd, O, dO.cuda(), lse)
    hd.hcadsa_check_device_error()
    ref = oracle.dsa_attn_bwd(bits(Q), bits(x["K"]), bits(x["V"]), idx, dO.double().numpy())
    for gg, r, what in zip(got, ref, ("dQ", "dK", "dV")):
        _check_grad(gg, r, what)


def test_dsa_attn_bwd_index_out_of_range_is_reported(hd):
    """An index entry >= Lk: the backward skips it (no read or reduction outside K/V and dK/dV),
    records HCADSA_ERR_DEVICE_BOUNDS, and the gradients are those of the other entries (the
    forward skips the same entries)."""
    Lq, Lk, k = 40, 600, 256
    cfg = synth.DsaConfig("bwdoob", B=1, L=Lk, Hq=64, k=k, sigma=1.0)
    x = synth.dsa_inputs(cfg, seed=881)
    Q = x["Q"][:, :Lq].contiguous()
    idx = _random_rows(Lq, Lk, k, 882)
    bad = idx.copy()
    bad[0, 5] = Lk
    bad[7, 200] = Lk + 999
    bad[39, 255] = 2 ** 30
    g = torch.Generator().manual_seed(883)
    dO = (torch.randn(1, Lq, 64, 256, generator=g) * 0.1).to(torch.bfloat16)
    Qd, Kd, Vd = Q.cuda(), x["K"].cuda(), x["V"].cuda()
    idd = torch.as_tensor(bad).reshape(1, Lq, k).cuda()
    hd.hcadsa_check_device_error()  # start from a clear error word
    O, lse = hd.dsa_sparse_attn_fwd(Qd, Kd, Vd, idd, return_lse=True)
    got = hd.dsa_sparse_attn_bwd(Qd, Kd, Vd, idd, O, dO.cuda(), lse)
    with pytest.raises(hd.HcaDsaError) as e:
        hd.hcadsa_check_device_error()
    assert e.value.status == -8
    hd.hcadsa_check_device_error()  # reading the word cleared it
    skipped = np.where(bad >= Lk, -1, bad).reshape(1, Lq, k)
    ref = oracle.dsa_attn_bwd(bits(Q), bits(x["K"]), bits(x["V"]), skipped, dO.double().numpy())
    for gg, r, what in zip(got, ref, ("dQ", "dK", "dV")):
        _check_grad(gg, r, what)


def test_dsa_attn_bwd_32k(hd):
    """The MLA-DSA layer's size (L = 32768, 64 heads of 256, top-2048 from the fused indexer):
    dQ of sampled query rows against the oracle (a row's dQ depends only on that row), and two
    sums that hold at any size: the value gradients of all keys add up to the sum of dO over all
    rows with a selection (each row's probabilities sum to 1), and the key gradients to ~0."""
    cfg = synth.DSA_32K
    B, L, k = cfg.B, cfg.L, cfg.k
    x = synth.dsa_inputs(cfg, seed=891)
    dev = {n: v.cuda() for n, v in x.items()}
    idx = hd.dsa_index_topk(dev["q_idx"], dev["k_idx"], dev["w_idx"], k)
    g = torch.Generator(device="cuda").manual_seed(892)
    dO = (torch.randn(B, L, 64, 256, generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    O, lse = hd.dsa_sparse_attn_fwd(dev["Q"], dev["K"], dev["V"], idx, return_lse=True)
    dQ, dK, dV = hd.dsa_sparse_attn_bwd(dev["Q"], dev["K"], dev["V"], idx, O, dO, lse)
    hd.hcadsa_check_device_error()
    rows = np.array([0, 1, 2047, 2048, 16385, 32767], np.int64)
    r = torch.as_tensor(rows, device="cuda")
    idx_rows = idx.reshape(L, k)[r].cpu().numpy().reshape(1, len(rows), k)
    Qb = bits(x["Q"]).reshape(L, 64, 256)[rows].reshape(1, len(rows), 64, 256)
    dO_rows = dO.reshape(L, 64, 256)[r].cpu().double().numpy().reshape(1, len(rows), 64, 256)
    ref = oracle.dsa_attn_bwd(Qb, bits(x["K"]), bits(x["V"]), idx_rows, dO_rows)
    _check_grad(dQ.reshape(L, 64, 256)[r], ref[0].reshape(len(rows), 64, 256), "dQ sampled rows")
    sum_dv = dV.double().sum(dim=(0, 1)).cpu().numpy()
    sum_do = dO.double().sum(dim=(0, 1, 2)).cpu().numpy()  # every row selects >= 1 key
    assert np.abs(sum_dv - sum_do).max() <= 1e-2 * np.abs(sum_do).max() + 1e-3, np.abs(sum_dv - sum_do).max()
    sum_dk = dK.double().sum(dim=(0, 1)).cpu().numpy()
    abs_dk = dK.double().abs().sum(dim=(0, 1)).cpu().numpy()
    assert np.all(np.abs(sum_dk) <= 1e-2 * abs_dk), (np.abs(sum_dk) / abs_dk).max()
