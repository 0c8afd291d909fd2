"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bars: compression and top-k bit-exact; attention outputs (bf16) within max-abs 2e-2
and mean-abs 2e-3 of the fp64 oracle, plus a relative RMS error <= 1e-2 (the absolute
bars alone would accept an all-zero output at sigma = 1/sqrt(d)).  Inputs come from
the seeded generators in synth; every expected value comes from the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, REL_RMS = 2e-2, 2e-3, 1e-2


@pytest.fixture(scope="module")
def hd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_hca_b200 import build

    build.build()
    import sparse_attention_hca_b200 as m

    oracle.build()
    return m


def bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_attn(gpu: torch.Tensor, ref: np.ndarray, what: str, value_scale: float = 1.0):
    """value_scale: standard deviation of V when it is not O(1) (stress inputs with sigma > 1);
    the absolute bars are stated for O(1) values and scale with it, the relative bar does not."""
    g = gpu.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(g - ref)
    rel = math.sqrt(float((err ** 2).sum()) / max(float((ref ** 2).sum()), 1e-300))
    msg = f"{what}: max_abs={err.max():.3e} mean_abs={err.mean():.3e} rel_rms={rel:.3e}"
    s = max(1.0, value_scale)
    assert err.max() <= MAX_ABS * s and err.mean() <= MEAN_ABS * s and rel <= REL_RMS, msg
    return msg


def no_device_error(hd):
    hd.hcadsa_check_device_error()


# ------------------------------------------------------------------ compression

@pytest.mark.parametrize("cfg", [
    synth.HCA_TINY,
    synth.HCA_32K,
    synth.HcaConfig("ragged_L1000_hkv2", B=2, L=1000, Hq=4, Hkv=2),
])
def test_compress_bit_exact(hd, cfg):
    inp = synth.hca_inputs(cfg)
    Kc, Vc = hd.hca_compress_kv(inp["K"].cuda(), inp["V"].cuda(), inp["w"].cuda(), cfg.blk)
    no_device_error(hd)
    w = inp["w"].numpy()
    assert np.array_equal(bits(Kc), oracle.hca_compress(bits(inp["K"]), w, cfg.blk))
    assert np.array_equal(bits(Vc), oracle.hca_compress(bits(inp["V"]), w, cfg.blk))


def test_compress_block_one_is_identity(hd):
    cfg = synth.HcaConfig("blk1", B=1, L=77, Hq=1, Hkv=1, d=64, blk=1)
    inp = synth.hca_inputs(cfg)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    Kc, _ = hd.hca_compress_kv(inp["K"].cuda(), inp["V"].cuda(), one, 1)
    assert torch.equal(Kc.cpu(), inp["K"])


# ------------------------------------------------------------------ HCA attention

def _hca_gpu_and_oracle(hd, cfg, rows=None, W=None):
    W = cfg.W if W is None else W
    inp = synth.hca_inputs(cfg)
    Kd, Vd, Qd = inp["K"].cuda(), inp["V"].cuda(), inp["Q"].cuda()
    Kc, Vc = hd.hca_compress_kv(Kd, Vd, inp["w"].cuda(), cfg.blk)
    O, lse = hd.hca_attn_fwd(Qd, Kc, Vc, Kd, Vd, blk=cfg.blk, W=W, return_lse=True)
    no_device_error(hd)
    w = inp["w"].numpy()
    Kc_o = oracle.hca_compress(bits(inp["K"]), w, cfg.blk)
    Vc_o = oracle.hca_compress(bits(inp["V"]), w, cfg.blk)
    ref, ref_lse = oracle.hca_attn(bits(inp["Q"]), Kc_o, Vc_o, bits(inp["K"]), bits(inp["V"]), blk=cfg.blk,
                                   W=W, rows=rows, with_lse=True)
    Of = O.reshape(cfg.B * cfg.L, cfg.Hq, cfg.d)
    lf = lse.reshape(cfg.B * cfg.L, cfg.Hq)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        Of, lf = Of[r], lf[r]
    return Of, lf, ref, ref_lse


def test_hca_tiny_all_rows(hd):
    O, lse, ref, ref_lse = _hca_gpu_and_oracle(hd, synth.HCA_TINY)
    print(check_attn(O, ref, "hca tiny"))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("cfg,W", [
    (synth.HcaConfig("stress_sigma1_L1003_hq16", B=1, L=1003, Hq=16, Hkv=1, sigma=1.0), 128),
    (synth.HcaConfig("stress_sigma1_L700_hq8_hkv2_B2", B=2, L=700, Hq=8, Hkv=2, sigma=1.0), 128),
    (synth.HcaConfig("wide_window_L300", B=1, L=300, Hq=16, Hkv=1, sigma=1.0), 512),
    (synth.HcaConfig("sharp_L600_blk64_W96", B=1, L=600, Hq=16, Hkv=1, blk=64, W=96, sigma=2.0), 96),
    # one head per K/V head (128-token row tiles) with W = 64 and blk = 32: a band tile can start
    # after a row's last key, and a compressed tile after a row's last entry (empty intervals)
    (synth.HcaConfig("g1_W64_blk32_L4400_hq2", B=1, L=4400, Hq=2, Hkv=2, blk=32, W=64, sigma=1.0), 64),
    # blk = 16 walks the last compressed tile through every fill (1..128 entries), so the band's
    # overhang shares that tile (merged tiles) or not, for 8- and 16-token row tiles
    (synth.HcaConfig("merge_blk16_L2400_hq16", B=1, L=2400, Hq=16, Hkv=1, blk=16, sigma=1.0), 128),
    (synth.HcaConfig("merge_g8_blk16_L2400_hq16_hkv2", B=1, L=2400, Hq=16, Hkv=2, blk=16, sigma=1.0), 128),
    # 32 and 128 query heads per K/V head: row tiles of 4 tokens (band overhang 3, merged
    # tiles) and of a single token
    (synth.HcaConfig("g32_L700_hq32", B=1, L=700, Hq=32, Hkv=1, sigma=1.0), 128),
    (synth.HcaConfig("g128_L300_hq128", B=1, L=300, Hq=128, Hkv=1, sigma=1.0), 128),
    # 618 entries of 4 tokens: row tiles of 7 key tiles, the long-row ring (three groups,
    # rows stored straight from registers)
    (synth.HcaConfig("deep_ring_blk4_L2600_hq4", B=1, L=2600, Hq=4, Hkv=1, blk=4, sigma=1.0), 128),
])
def test_hca_stress(hd, cfg, W):
    O, lse, ref, ref_lse = _hca_gpu_and_oracle(hd, cfg, W=W)
    print(check_attn(O, ref, cfg.name, value_scale=cfg.sigma or 1.0))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_hca_forced_rescales(hd):
    """Keys whose scale grows along the sequence: later key tiles raise the running max by far
    more than the lazy-rescale threshold, so O is rescaled in both halves of d_v."""
    cfg = synth.HcaConfig("ramp_L1500_hq16", B=1, L=1500, Hq=16, Hkv=1, sigma=1.0)
    inp = synth.hca_inputs(cfg)
    ramp = 1.0 + 6.0 * torch.arange(cfg.L, dtype=torch.float32) / cfg.L
    K = (inp["K"].float() * ramp.view(1, -1, 1, 1)).to(torch.bfloat16)
    Kd, Vd, Qd = K.cuda(), inp["V"].cuda(), inp["Q"].cuda()
    Kc, Vc = hd.hca_compress_kv(Kd, Vd, inp["w"].cuda(), cfg.blk)
    O, lse = hd.hca_attn_fwd(Qd, Kc, Vc, Kd, Vd, return_lse=True)
    O2 = hd.hca_attn_fwd(Qd, Kc, Vc, Kd, Vd)
    no_device_error(hd)
    assert torch.equal(O, O2)  # deterministic: no atomics, fixed accumulation order
    w = inp["w"].numpy()
    Kc_o = oracle.hca_compress(bits(K), w, cfg.blk)
    Vc_o = oracle.hca_compress(bits(inp["V"]), w, cfg.blk)
    ref, ref_lse = oracle.hca_attn(bits(inp["Q"]), Kc_o, Vc_o, bits(K), bits(inp["V"]), with_lse=True)
    print(check_attn(O.reshape(cfg.L, cfg.Hq, cfg.d), ref, "hca forced rescales"))
    np.testing.assert_allclose(lse.reshape(cfg.L, cfg.Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_hca_workspace_size_and_check(hd):
    """The workspace holds one probability-tile slot per key tile for each resident CTA; a
    short workspace is rejected before launch."""
    lib = hd.lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    L, Hq = 32768, 16
    TT = 128 // Hq
    nc_last = (L - 1 - 128 + 1) // 128
    J_max = -(-nc_last // 128) + (TT + 128 - 2 + 128) // 128
    want = min(L // TT, sms) * J_max * (128 * 128 * 2 + 128 * 4)
    assert lib.hca_attn_fwd_workspace_size(1, L, 0, Hq, 1, 512, L // 128, 128, 128) == want
    L = 1024
    Q = torch.zeros(1, L, Hq, 512, dtype=torch.bfloat16, device="cuda")
    K = torch.zeros(1, L, 1, 512, dtype=torch.bfloat16, device="cuda")
    Kc = torch.zeros(1, L // 128, 1, 512, dtype=torch.bfloat16, device="cuda")
    need = lib.hca_attn_fwd_workspace_size(1, L, 0, Hq, 1, 512, L // 128, 128, 128)
    assert need > 0
    with pytest.raises(hd.HcaDsaError) as e:
        hd.hca_attn_fwd(Q, Kc, Kc, K, K, workspace=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == -5


def _sample_rows(L, B=1, extra=()):
    toks = {0, 1, 2, 126, 127, 128, 129, 254, 255, 256, 257, 383, 384, 1000, 4095, 4096, L // 2, L - 2, L - 1}
    toks |= set(extra)
    toks = sorted(t for t in toks if 0 <= t < L)
    return np.array([b * L + t for b in range(B) for t in toks], np.int64)


def test_hca_32k_sampled(hd):
    cfg = synth.HCA_32K
    rows = _sample_rows(cfg.L, extra=(8191, 16384, 32000))
    O, lse, ref, ref_lse = _hca_gpu_and_oracle(hd, cfg, rows=rows)
    print(check_attn(O, ref, "hca 32k sampled"))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


def test_hca_131k_sampled(hd):
    cfg = synth.HCA_131K
    rows = _sample_rows(cfg.L, extra=(65536, 100000, 131000))
    O, lse, ref, ref_lse = _hca_gpu_and_oracle(hd, cfg, rows=rows)
    print(check_attn(O, ref, "hca 131k sampled"))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("B,t", [(2, 5000), (3, 130)])
def test_hca_decode_form(hd, B, t):
    """One query token per sequence at position t over [entries | window buffer]."""
    d, Hq, blk, W = 512, 16, 128, 128
    n_c = (t + 1) // blk
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 7, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 7, "V")
    ws = max(0, t - W + 1)
    Kw = synth.normal_bf16((B, t + 1 - ws, 1, d), 1.0, 8, "K")
    Vw = synth.normal_bf16((B, t + 1 - ws, 1, d), 1.0, 8, "V")
    Q = synth.normal_bf16((B, 1, Hq, d), 1.0, 9, "Q")
    O = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t, blk=blk, W=W)
    no_device_error(hd)
    ref = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t, blk=blk, W=W)
    print(check_attn(O.reshape(B, Hq, d), ref, f"hca decode t={t}"))


def test_hca_split_key_ranges(hd):
    """Few row tiles: every row tile's key tiles are split over several CTAs and the partial
    softmax results are combined (3 query tokens per sequence, 4 sequences, lse checked)."""
    d, Hq, blk, W, B, Lq, t0 = 512, 16, 128, 128, 4, 3, 20000
    t_last = t0 + Lq - 1
    n_c = (t_last + 1) // blk
    ws = t0 - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 21, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 21, "V")
    Kw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 22, "K")
    Vw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 22, "V")
    Q = synth.normal_bf16((B, Lq, Hq, d), 1.0, 23, "Q")
    O, lse = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t0,
                             return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t0,
                                   with_lse=True)
    print(check_attn(O.reshape(B * Lq, Hq, d), ref, "hca split key ranges"))
    np.testing.assert_allclose(lse.reshape(B * Lq, Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_hca_decode_uneven_splits(hd):
    """32 sequences at t = 200000: 32 equal row tiles of 14 key tiles, so every CTA takes an
    equal share of all 448 key tiles laid end to end (stream-K), and row tiles are recombined
    from the pieces of 4-6 CTAs."""
    d, Hq, blk, W, B, t = 512, 16, 128, 128, 32, 200000
    n_c = (t + 1) // blk
    ws = t - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 51, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 51, "V")
    Kw = synth.normal_bf16((B, W, 1, d), 1.0, 52, "K")
    Vw = synth.normal_bf16((B, W, 1, d), 1.0, 52, "V")
    Q = synth.normal_bf16((B, 1, Hq, d), 1.0, 53, "Q")
    O, lse = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t,
                             return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t,
                                   with_lse=True)
    print(check_attn(O.reshape(B, Hq, d), ref, "hca decode uneven splits"))
    np.testing.assert_allclose(lse.reshape(B, Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_hca_chunked_prefill(hd):
    """A prefill chunk: 1500 query tokens at positions 4000..5499 of two sequences, over the
    entries stored so far and a window buffer that starts at the first query's window (many
    row tiles: the unsplit path, with merged key tiles at an offset)."""
    d, Hq, blk, W, B, Lq, t0 = 512, 16, 128, 128, 2, 1500, 4000
    t_last = t0 + Lq - 1
    n_c = (t_last - W + 1) // blk
    ws = t0 - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 71, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 71, "V")
    Kw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 72, "K")
    Vw = synth.normal_bf16((B, t_last + 1 - ws, 1, d), 1.0, 72, "V")
    Q = synth.normal_bf16((B, Lq, Hq, d), 1.0, 73, "Q")
    O, lse = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t0,
                             return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t0,
                                   with_lse=True)
    print(check_attn(O.reshape(B * Lq, Hq, d), ref, "hca chunked prefill"))
    np.testing.assert_allclose(lse.reshape(B * Lq, Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_hca_decode_stream_k_short_rows(hd):
    """70 sequences at t = 20000 (3 key tiles each, 210 in all): with stream-K most CTAs take
    one or two key tiles, often the end of one row tile and the start of the next."""
    d, Hq, blk, W, B, t = 512, 16, 128, 128, 70, 20000
    n_c = (t - W + 1) // blk
    ws = t - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 81, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 81, "V")
    Kw = synth.normal_bf16((B, W, 1, d), 1.0, 82, "K")
    Vw = synth.normal_bf16((B, W, 1, d), 1.0, 82, "V")
    Q = synth.normal_bf16((B, 1, Hq, d), 1.0, 83, "Q")
    O, lse = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t,
                             return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t,
                                   with_lse=True)
    print(check_attn(O.reshape(B, Hq, d), ref, "hca decode stream-K short rows"))
    np.testing.assert_allclose(lse.reshape(B, Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


@pytest.mark.parametrize("B", [1, 2])
def test_hca_decode_many_units(hd, B):
    """One or two sequences at t = 1,048,575: 65 key tiles per row tile, split over the SMs
    into the maximum of 64 units per row tile, so the combine pass gathers units 32-63 too."""
    d, Hq, blk, W, t = 512, 16, 128, 128, 1048575
    n_c = (t + 1) // blk - 1  # entries the query needs (8191), as a decode cache holds them
    ws = t - W + 1
    Kc = synth.normal_bf16((B, n_c, 1, d), 1.0, 61, "K")
    Vc = synth.normal_bf16((B, n_c, 1, d), 1.0, 61, "V")
    Kw = synth.normal_bf16((B, W, 1, d), 1.0, 62, "K")
    Vw = synth.normal_bf16((B, W, 1, d), 1.0, 62, "V")
    Q = synth.normal_bf16((B, 1, Hq, d), 1.0, 63, "Q")
    O, lse = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t,
                             return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t,
                                   with_lse=True)
    print(check_attn(O.reshape(B, Hq, d), ref, f"hca decode B={B} t=1M"))
    np.testing.assert_allclose(lse.reshape(B, Hq).cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


# ------------------------------------------------------------------ DSA indexer + top-k

def _dsa_cfg(name, L, B=1, k=2048, sigma=None):
    return synth.DsaConfig(name, B=B, L=L, Hq=64, k=k, sigma=sigma)


@pytest.mark.parametrize("L,k,B", [(3000, 2048, 1), (700, 64, 2), (200, 16, 1), (130, 200, 1)])
def test_topk_bit_exact_all_rows(hd, L, k, B):
    cfg = _dsa_cfg("topk", L, B=B, k=k)
    inp = synth.dsa_inputs(cfg)
    idx = hd.dsa_index_topk(inp["q_idx"].cuda(), inp["k_idx"].cuda(), inp["w_idx"].cuda(), k)
    no_device_error(hd)
    ref = oracle.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), k)
    assert np.array_equal(idx.cpu().numpy().reshape(B * L, k), ref)


def test_topk_heavy_ties(hd):
    L, k = 2500, 300
    g = torch.Generator().manual_seed(5)
    q = torch.randint(-1, 2, (1, L, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-1, 2, (1, L, 64), generator=g).to(torch.int8)
    w = torch.tensor([1, 1, 2, 1], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), k)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), k)
    assert np.array_equal(idx.cpu().numpy().reshape(L, k), ref)


def test_topk_all_equal_scores(hd):
    L, k = 600, 100
    q = torch.zeros(1, L, 4, 64, dtype=torch.int8)
    kk = synth.dsa_inputs(_dsa_cfg("x", L))["k_idx"]
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), torch.tensor([1, 2, 3, 4], dtype=torch.int32).cuda(), k)
    exp = np.array([list(range(min(k, t + 1))) + [-1] * (k - min(k, t + 1)) for t in range(L)], np.int32)
    assert np.array_equal(idx.cpu().numpy().reshape(L, k), exp)


def test_topk_wide_weights_and_extreme_int8(hd):
    L, k = 900, 50
    g = torch.Generator().manual_seed(6)
    q = torch.randint(-128, 128, (1, L, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-128, 128, (1, L, 64), generator=g).to(torch.int8)
    w = torch.tensor([7, -3, 100, 1], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), k)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), k)
    assert np.array_equal(idx.cpu().numpy().reshape(L, k), ref)


@pytest.mark.parametrize("B,t", [(2, 70000), (1, 3000)])
def test_topk_decode_form(hd, B, t):
    """Lq = 1 at position t (streaming scorer; t + 1 > shared-memory row capacity for 70000)."""
    Lk = t + 1
    g = torch.Generator().manual_seed(t)
    q = torch.randint(-8, 9, (B, 1, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-8, 9, (B, Lk, 64), generator=g).to(torch.int8)
    w = torch.tensor([1, 4, 2, 3], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), 2048, q_offset=t)
    no_device_error(hd)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), 2048, q_offset=t)
    assert np.array_equal(idx.cpu().numpy().reshape(B, 2048), ref)


def test_topk_decode_ties_overflow_candidates(hd):
    """Decode shape where every score ties (q_idx = 0): the threshold bin holds all 50000 keys,
    more than the candidate list takes, so the row falls back to the exact single-CTA select;
    ties go to the lowest positions."""
    B, t, k = 2, 49999, 2048
    q = torch.zeros(B, 1, 4, 64, dtype=torch.int8)
    kk = synth.randint((B, t + 1, 64), -8, 8, 31, "k_idx", torch.int8)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), torch.tensor([1, 2, 3, 4], dtype=torch.int32).cuda(), k,
                            q_offset=t)
    no_device_error(hd)
    exp = np.tile(np.arange(k, dtype=np.int32), (B, 1))
    assert np.array_equal(idx.cpu().numpy().reshape(B, k), exp)


def test_topk_decode_many_rows_split_select(hd):
    """Lq = 3 rows per sequence over 40000+ keys: the multi-CTA selection path, bit-exact."""
    B, Lq, t0, k = 3, 3, 40000, 2048
    g = torch.Generator().manual_seed(41)
    q = torch.randint(-8, 9, (B, Lq, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-8, 9, (B, t0 + Lq, 64), generator=g).to(torch.int8)
    w = torch.tensor([2, 1, 4, 3], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), k, q_offset=t0)
    no_device_error(hd)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), k, q_offset=t0)
    assert np.array_equal(idx.cpu().numpy().reshape(B * Lq, k), ref)


def test_topk_chunked_prefill(hd):
    """A prefill chunk: 600 query rows at positions 3000..3599 over 3600 keys (the tiled scorer
    and single-block selection with a query offset), bit-exact on every row."""
    B, Lq, t0, k = 2, 600, 3000, 2048
    g = torch.Generator().manual_seed(43)
    q = torch.randint(-8, 9, (B, Lq, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-8, 9, (B, t0 + Lq, 64), generator=g).to(torch.int8)
    w = torch.tensor([3, 1, 2, 4], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), k, q_offset=t0)
    no_device_error(hd)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), k, q_offset=t0)
    assert np.array_equal(idx.cpu().numpy().reshape(B * Lq, k), ref)


def test_topk_32k_sampled_rows(hd):
    cfg = synth.DSA_32K
    inp = synth.dsa_inputs(cfg)
    idx = hd.dsa_index_topk(inp["q_idx"].cuda(), inp["k_idx"].cuda(), inp["w_idx"].cuda(), cfg.k)
    no_device_error(hd)
    rows = _sample_rows(cfg.L, extra=(2046, 2047, 2048, 2049, 12345, 30000))
    ref = oracle.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), cfg.k, rows=rows)
    got = idx.reshape(cfg.L, cfg.k)[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal(got, ref)


def test_topk_131k_sampled_rows(hd):
    """The long-context prefill length through the fused indexer + selection (no score matrix:
    the workspace is 512 bytes), bit-exact on sampled rows."""
    cfg = synth.DsaConfig("topk131k", B=1, L=131072, Hq=64)
    g = torch.Generator().manual_seed(131)
    q = torch.randint(-8, 9, (1, cfg.L, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-8, 9, (1, cfg.L, 64), generator=g).to(torch.int8)
    w = torch.tensor([2, 4, 1, 3], dtype=torch.int32)
    assert hd.dsa_index_topk_workspace_size(1, cfg.L, 0, cfg.L, cfg.k) == 512
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), cfg.k)
    no_device_error(hd)
    rows = _sample_rows(cfg.L, extra=(2047, 2048, 65535, 65536, 100000, 131071))
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), cfg.k, rows=rows)
    got = idx.reshape(cfg.L, cfg.k)[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal(got, ref)


def test_topk_ragged_batches_offset_odd_k(hd):
    """Three sequences, 300 query rows each at positions 1000..1299 (a ragged last tile of 44
    rows), k = 77 (rows not 16-byte aligned: scalar stores), bit-exact on every row."""
    B, Lq, t0, k = 3, 300, 1000, 77
    g = torch.Generator().manual_seed(77)
    q = torch.randint(-8, 9, (B, Lq, 4, 64), generator=g).to(torch.int8)
    kk = torch.randint(-8, 9, (B, t0 + Lq, 64), generator=g).to(torch.int8)
    w = torch.tensor([1, 3, 2, 4], dtype=torch.int32)
    idx = hd.dsa_index_topk(q.cuda(), kk.cuda(), w.cuda(), k, q_offset=t0)
    no_device_error(hd)
    ref = oracle.dsa_topk(q.numpy(), kk.numpy(), w.numpy(), k, q_offset=t0)
    assert np.array_equal(idx.cpu().numpy().reshape(B * Lq, k), ref)


# ------------------------------------------------------------------ DSA sparse attention

def _dsa_attn_case(hd, cfg, rows, split=True):
    """GPU attention fed the ORACLE's index rows for the sampled queries; returns the GPU and
    oracle outputs and log-sum-exps of those rows."""
    inp = synth.dsa_inputs(cfg)
    idx_o = oracle.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), cfg.k, rows=rows)
    Qs = inp["Q"].reshape(cfg.B * cfg.L, 1, cfg.Hq, cfg.d)[torch.as_tensor(rows)]   # one query per sequence row
    # every sampled row becomes its own "token" of a batch-1 call over the key sequence of its batch
    outs, lses = [], []
    for b in range(cfg.B):
        sel = (rows // cfg.L) == b
        if not sel.any():
            continue
        q_b = Qs[torch.as_tensor(np.nonzero(sel)[0])].reshape(1, -1, cfg.Hq, cfg.d)
        O, lse = hd.dsa_sparse_attn_fwd(q_b.cuda(), inp["K"][b:b + 1].cuda(), inp["V"][b:b + 1].cuda(),
                                        torch.as_tensor(idx_o[sel]).reshape(1, -1, cfg.k).cuda(), return_lse=True,
                                        split=split)
        outs.append(O.reshape(-1, cfg.Hq, cfg.d))
        lses.append(lse.reshape(-1, cfg.Hq))
    no_device_error(hd)
    ref, ref_lse = oracle.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx_o, rows=rows, with_lse=True)
    return torch.cat(outs), torch.cat(lses), ref, ref_lse


@pytest.mark.parametrize("L,k,sigma", [(3000, 2048, None), (2000, 256, 1.0), (300, 2048, 1.0), (500, 100, 2.0),
                                         (5000, 4096, 1.0)])
def test_dsa_attn_against_oracle(hd, L, k, sigma):
    cfg = _dsa_cfg("dsa", L, k=k, sigma=sigma)
    rows = _sample_rows(L, extra=(k - 1, k, k + 1, L - 3))
    O, lse, ref, ref_lse = _dsa_attn_case(hd, cfg, rows)
    print(check_attn(O, ref, f"dsa L={L} k={k} sigma={sigma}", value_scale=sigma or 1.0))
    # natural-log log-sum-exp of the selected scores, per head (the backward consumes it)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-3 * max(1.0, (sigma or 1.0) ** 2), rtol=0)


def test_dsa_attn_max_k_one_cta_per_row(hd):
    """k = 4096, the largest index row (32 key tiles, every bit of the tile mask), with one CTA
    per query row (the split path of the same rows is in test_dsa_attn_against_oracle)."""
    cfg = _dsa_cfg("dsa", 5000, k=4096, sigma=1.0)
    rows = _sample_rows(cfg.L, extra=(4095, 4096, 4097, 4998))
    O, lse, ref, ref_lse = _dsa_attn_case(hd, cfg, rows, split=False)
    print(check_attn(O, ref, "dsa k=4096 one CTA per row"))
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


def test_dsa_pipeline_32k_sampled(hd):
    """Indexer -> top-k -> sparse attention, all on the GPU at the 32K configuration."""
    cfg = synth.DSA_32K
    inp = synth.dsa_inputs(cfg)
    dev = {k: v.cuda() for k, v in inp.items()}
    idx = hd.dsa_index_topk(dev["q_idx"], dev["k_idx"], dev["w_idx"], cfg.k)
    O, lse = hd.dsa_sparse_attn_fwd(dev["Q"], dev["K"], dev["V"], idx, return_lse=True)
    no_device_error(hd)
    rows = _sample_rows(cfg.L, extra=(2047, 2048, 20000))
    idx_o = oracle.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), cfg.k, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    assert np.array_equal(idx.reshape(cfg.L, cfg.k)[r].cpu().numpy(), idx_o)
    ref, ref_lse = oracle.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx_o, rows=rows, with_lse=True)
    print(check_attn(O.reshape(cfg.L, cfg.Hq, cfg.d)[r], ref, "dsa 32k pipeline"))
    np.testing.assert_allclose(lse.reshape(cfg.L, cfg.Hq)[r].cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


def test_dsa_padding_and_order(hd):
    """Index rows with -1 padding in arbitrary places and shuffled order."""
    cfg = _dsa_cfg("pad", 400, k=64, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    rng = np.random.default_rng(3)
    idx = np.full((cfg.L, cfg.k), -1, np.int32)
    for t in range(cfg.L):
        n = min(cfg.k, t + 1, int(rng.integers(1, cfg.k + 1)))
        sel = rng.choice(t + 1, size=n, replace=False)
        pos = rng.choice(cfg.k, size=n, replace=False)
        idx[t, pos] = sel
    O = hd.dsa_sparse_attn_fwd(inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(),
                               torch.as_tensor(idx).reshape(1, cfg.L, cfg.k).cuda())
    no_device_error(hd)
    ref = oracle.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx)
    print(check_attn(O, ref, "dsa padded/shuffled"))


def test_dsa_forced_rescales(hd):
    """Keys whose scale grows with their position and index rows in ascending order: later
    128-entry tiles raise a head's running max by far more than the lazy-rescale threshold, so
    that head's O row is rescaled in TMEM (while other heads of the same warp keep theirs); a
    few padded entries in the middle of some rows mix partial tiles with fully valid ones."""
    cfg = _dsa_cfg("ramp", 1500, k=1024, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    ramp = 1.0 + 6.0 * torch.arange(cfg.L, dtype=torch.float32) / cfg.L
    K = (inp["K"].float() * ramp.view(1, -1, 1)).to(torch.bfloat16)
    rng = np.random.default_rng(11)
    idx = np.full((cfg.L, cfg.k), -1, np.int32)
    for t in range(cfg.L):
        n = min(cfg.k, t + 1)
        idx[t, :n] = np.sort(rng.choice(t + 1, size=n, replace=False))
        if t % 3 == 0 and n > 300:
            idx[t, 200:210] = -1
    O, lse = hd.dsa_sparse_attn_fwd(inp["Q"].cuda(), K.cuda(), inp["V"].cuda(),
                                    torch.as_tensor(idx).reshape(1, cfg.L, cfg.k).cuda(), return_lse=True)
    no_device_error(hd)
    rows = _sample_rows(cfg.L, extra=(300, 1023, 1024, 1200, 1497))
    ref, ref_lse = oracle.dsa_attn(bits(inp["Q"]), bits(K), bits(inp["V"]), idx[rows], rows=rows, with_lse=True)
    r = torch.as_tensor(rows, device="cuda")
    print(check_attn(O.reshape(cfg.L, cfg.Hq, cfg.d)[r], ref, "dsa forced rescales"))
    np.testing.assert_allclose(lse.reshape(cfg.L, cfg.Hq)[r].cpu().numpy(), ref_lse, atol=2e-2, rtol=0)


def test_dsa_all_padding_rows_and_lse(hd):
    """Rows whose index list holds no valid entry (all -1) give O = 0 and lse = -inf, the
    oracle's empty-set case; their neighbours (partly padded, shuffled) still match the oracle
    in O and lse."""
    cfg = _dsa_cfg("allpad", 300, k=256, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    rng = np.random.default_rng(17)
    idx = np.full((cfg.L, cfg.k), -1, np.int32)
    empty = {0, 1, 5, 128, 129, 200, 299}
    for t in range(cfg.L):
        if t in empty:
            continue
        n = min(cfg.k, t + 1, int(rng.integers(1, cfg.k + 1)))
        idx[t, rng.choice(cfg.k, size=n, replace=False)] = rng.choice(t + 1, size=n, replace=False)
    O, lse = hd.dsa_sparse_attn_fwd(inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(),
                                    torch.as_tensor(idx).reshape(1, cfg.L, cfg.k).cuda(), return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx, with_lse=True)
    O = O.reshape(cfg.L, cfg.Hq, cfg.d)
    lse = lse.reshape(cfg.L, cfg.Hq).cpu().numpy()
    e = sorted(empty)
    assert torch.count_nonzero(O[e]).item() == 0
    assert np.all(np.isneginf(lse[e])) and np.all(np.isneginf(ref_lse[e]))
    assert np.all(ref[e] == 0.0)
    keep = np.array([t for t in range(cfg.L) if t not in empty])
    print(check_attn(O[torch.as_tensor(keep, device="cuda")], ref[keep], "dsa all-padding neighbours"))
    np.testing.assert_allclose(lse[keep], ref_lse[keep], atol=2e-3, rtol=0)


def test_dsa_split_matches_oracle_and_unsplit(hd):
    """Few query rows (a decode-sized call): each row's key tiles are divided among several CTAs
    whose partial outputs the combine pass merges.  Rows with every entry valid, with entries in
    only two tiles (most parts empty), with none (every part empty) and with scattered padding;
    compared with the oracle and with the one-CTA-per-row path."""
    Lk, n_q, k = 5000, 12, 2048
    cfg = _dsa_cfg("split", Lk, k=k, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    assert hd.lib().dsa_sparse_attn_fwd_workspace_size(1, n_q, k) > 0  # this call splits
    rng = np.random.default_rng(23)
    idx = np.full((n_q, k), -1, np.int32)
    for r in range(n_q):
        if r == 3:
            continue  # no valid entry
        if r == 5:
            idx[r, 700:790] = rng.choice(Lk, 90, replace=False)  # tiles 5 and 6 only
            continue
        idx[r] = rng.choice(Lk, k, replace=False)
        if r == 8:
            idx[r, rng.random(k) < 0.3] = -1
    qpos = torch.as_tensor(rng.choice(Lk, n_q, replace=False))
    q = inp["Q"].reshape(Lk, cfg.Hq, cfg.d)[qpos].reshape(1, n_q, cfg.Hq, cfg.d)
    args = (q.cuda(), inp["K"].cuda(), inp["V"].cuda(), torch.as_tensor(idx).reshape(1, n_q, k).cuda())
    O_s, lse_s = hd.dsa_sparse_attn_fwd(*args, return_lse=True)
    O_u, lse_u = hd.dsa_sparse_attn_fwd(*args, return_lse=True, split=False)
    no_device_error(hd)
    ref, ref_lse = oracle.dsa_attn(bits(q), bits(inp["K"]), bits(inp["V"]), idx, with_lse=True)
    for O, lse, name in ((O_s, lse_s, "split"), (O_u, lse_u, "one CTA per row")):
        O = O.reshape(n_q, cfg.Hq, cfg.d)
        lse = lse.reshape(n_q, cfg.Hq).cpu().numpy()
        assert torch.count_nonzero(O[3]).item() == 0 and np.all(np.isneginf(lse[3]))
        keep = [r for r in range(n_q) if r != 3]
        print(check_attn(O[keep], ref[keep], f"dsa {name}, {n_q} rows"))
        np.testing.assert_allclose(lse[keep], ref_lse[keep], atol=2e-3, rtol=0)


def test_dsa_split_two_sequences(hd):
    """The split path with a batch: 2 sequences of 3000 keys, 5 query rows each; every unit reads
    the K/V rows of its own sequence."""
    cfg = synth.DsaConfig("split2", B=2, L=3000, Hq=64, k=1024, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    n_q = 5
    assert hd.lib().dsa_sparse_attn_fwd_workspace_size(cfg.B, n_q, cfg.k) > 0
    rng = np.random.default_rng(29)
    idx = np.stack([np.stack([rng.choice(cfg.L, cfg.k, replace=False) for _ in range(n_q)]) for _ in range(cfg.B)])
    idx = idx.astype(np.int32)
    idx[1, 2, 500:] = -1  # a short row in the second sequence
    q = inp["Q"][:, :n_q].contiguous()
    O, lse = hd.dsa_sparse_attn_fwd(q.cuda(), inp["K"].cuda(), inp["V"].cuda(), torch.as_tensor(idx).cuda(),
                                    return_lse=True)
    no_device_error(hd)
    ref, ref_lse = oracle.dsa_attn(bits(q), bits(inp["K"]), bits(inp["V"]), idx.reshape(cfg.B * n_q, cfg.k),
                                   with_lse=True)
    print(check_attn(O.reshape(cfg.B * n_q, cfg.Hq, cfg.d), ref, "dsa split, two sequences"))
    np.testing.assert_allclose(lse.reshape(cfg.B * n_q, cfg.Hq).cpu().numpy(), ref_lse, atol=2e-3, rtol=0)


def test_dsa_index_out_of_range_is_reported(hd):
    """An index entry >= Lk is a caller error the host cannot see: the kernel skips it (no read
    outside K/V), records HCADSA_ERR_DEVICE_BOUNDS, and the row is the attention over its other
    entries."""
    cfg = _dsa_cfg("oob", 260, k=128, sigma=1.0)
    inp = synth.dsa_inputs(cfg)
    rows = np.array([10, 129, 259], np.int64)
    idx_o = oracle.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), cfg.k, rows=rows)
    bad = idx_o.copy()
    bad[0, 3] = cfg.L          # one past the end
    bad[1, 0] = cfg.L + 12345  # far past the end
    bad[2, 127] = 2 ** 30
    q = inp["Q"].reshape(cfg.L, cfg.Hq, cfg.d)[torch.as_tensor(rows)].reshape(1, len(rows), cfg.Hq, cfg.d)
    hd.hcadsa_check_device_error()  # start from a clear error word
    O = hd.dsa_sparse_attn_fwd(q.cuda(), inp["K"].cuda(), inp["V"].cuda(),
                               torch.as_tensor(bad).reshape(1, len(rows), cfg.k).cuda())
    with pytest.raises(hd.HcaDsaError) as e:
        hd.hcadsa_check_device_error()
    assert e.value.status == -8
    hd.hcadsa_check_device_error()  # reading the word cleared it
    skipped = np.where(bad >= cfg.L, -1, bad)
    qb = bits(inp["Q"]).reshape(cfg.L, cfg.Hq, cfg.d)[rows].reshape(1, len(rows), cfg.Hq, cfg.d)
    ref = oracle.dsa_attn(qb, bits(inp["K"]), bits(inp["V"]), skipped)
    print(check_attn(O.reshape(len(rows), cfg.Hq, cfg.d), ref, "dsa out-of-range entries skipped"))


def test_dsa_decode_1m_batch32_sampled(hd):
    """The benchmarked decode call exactly: 32 sequences, one query each at t = 1,048,575, top-2048
    and sparse attention in one launch each; top-k (bit-exact), O and lse checked against the
    oracle on 4 of the 32 sequences.  Inputs are drawn on the device with torch's seeded generator
    (the same laws as the synthetic generators; 34 GB of caches) and copied to the host for the
    oracle."""
    cfg = synth.DECODE_1M
    B, t, Lk = cfg.B, cfg.t, cfg.t + 1
    dev = torch.device("cuda")
    seed = 91
    q_idx = synth.randint((B, 1, 4, 64), -8, 8, seed, "q_idx", torch.int8, dev)
    k_idx = synth.randint((B, Lk, 64), -8, 8, seed, "k_idx", torch.int8, dev)
    w_idx = synth.randint((4,), 1, 4, seed, "w_idx", torch.int32, dev)
    Q = synth.normal_bf16((B, 1, 64, 256), 1.0, seed, "Q", dev)
    K = synth.normal_bf16((B, Lk, 256), 1.0, seed, "K", dev)
    V = synth.normal_bf16((B, Lk, 256), 1.0, seed, "V", dev)
    idx = hd.dsa_index_topk(q_idx, k_idx, w_idx, cfg.k, q_offset=t)
    O, lse = hd.dsa_sparse_attn_fwd(Q, K, V, idx, return_lse=True)
    no_device_error(hd)
    for b in (0, 7, 19, 31):
        sl = slice(b, b + 1)
        idx_o = oracle.dsa_topk(q_idx[sl].cpu().numpy(), k_idx[sl].cpu().numpy(), w_idx.cpu().numpy(), cfg.k,
                                q_offset=t)
        assert np.array_equal(idx[b].cpu().numpy(), idx_o), f"sequence {b}"
        ref, ref_lse = oracle.dsa_attn(bits(Q[sl]), bits(K[sl]), bits(V[sl]), idx_o, with_lse=True)
        print(check_attn(O[b].reshape(1, 64, 256), ref, f"dsa decode B=32 sequence {b}"))
        np.testing.assert_allclose(lse[b].reshape(1, 64).cpu().numpy(), ref_lse, atol=2e-3, rtol=0)
    del K, V, k_idx
    torch.cuda.empty_cache()


def test_dsa_decode_1m_sampled_batch(hd):
    """The 1M-context decode shape for 2 of the 32 sequences (each sequence is independent)."""
    cfg = synth.DECODE_1M
    B, t, Lk = 2, cfg.t, cfg.t + 1
    g = 11
    q_idx = synth.randint((B, 1, 4, 64), -8, 8, g, "q_idx", torch.int8)
    k_idx = synth.randint((B, Lk, 64), -8, 8, g, "k_idx", torch.int8)
    w_idx = synth.randint((4,), 1, 4, g, "w_idx", torch.int32)
    Q = synth.normal_bf16((B, 1, 64, 256), 1.0, g, "Q")
    K = synth.normal_bf16((B, Lk, 256), 1.0, g, "K")
    V = synth.normal_bf16((B, Lk, 256), 1.0, g, "V")
    idx = hd.dsa_index_topk(q_idx.cuda(), k_idx.cuda(), w_idx.cuda(), cfg.k, q_offset=t)
    O = hd.dsa_sparse_attn_fwd(Q.cuda(), K.cuda(), V.cuda(), idx)
    no_device_error(hd)
    idx_o = oracle.dsa_topk(q_idx.numpy(), k_idx.numpy(), w_idx.numpy(), cfg.k, q_offset=t)
    assert np.array_equal(idx.cpu().numpy().reshape(B, cfg.k), idx_o)
    ref = oracle.dsa_attn(bits(Q), bits(K), bits(V), idx_o)
    print(check_attn(O.reshape(B, 64, 256), ref, "dsa decode 1M"))


def test_hca_decode_1m_sampled_batch(hd):
    cfg = synth.DECODE_1M
    B, t = 2, cfg.t
    n_c = cfg.n_c
    g = 12
    Kc = synth.normal_bf16((B, n_c, 1, 512), 1.0, g, "K")
    Vc = synth.normal_bf16((B, n_c, 1, 512), 1.0, g, "V")
    ws = t - cfg.W + 1
    Kw = synth.normal_bf16((B, cfg.W, 1, 512), 1.0, g + 1, "K")
    Vw = synth.normal_bf16((B, cfg.W, 1, 512), 1.0, g + 1, "V")
    Q = synth.normal_bf16((B, 1, 16, 512), 1.0, g, "Q")
    O = hd.hca_attn_fwd(Q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), win_start=ws, q_offset=t)
    no_device_error(hd)
    ref = oracle.hca_attn(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), win_start=ws, q_offset=t)
    print(check_attn(O.reshape(B, 16, 512), ref, "hca decode 1M"))
