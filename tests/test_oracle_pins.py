"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test ties one oracle function to something the pages or mathematics fix:
a hand-derived worked example (tests/golden), a closed form, a special case
that reduces to a library routine (torch's fp64 scaled-dot-product attention,
numpy integer einsum, Python's sort), or brute force on tiny inputs.  A
plausible slip in the oracle (dropped term, off-by-one in the visible set,
wrong head mapping, wrong tie order, transposed operand) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2 = float(np.float32(math.log(2.0)))


def bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def bf16(x) -> np.ndarray:
    return bits(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def sdpa_ref(Q, K, V, mask, scale):
    """torch fp64 SDPA on [B,L,H,d] bf16 inputs, K/V expanded to Hq heads; mask [Lq, Lk] bool."""
    q = Q.double().permute(0, 2, 1, 3)
    k = K.double().permute(0, 2, 1, 3)
    v = V.double().permute(0, 2, 1, 3)
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_torch(oracle_mod):
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000).astype(np.float32) * 3
    # exact ties: low 16 bits = 0x8000 with both parities of the kept lsb
    ties = (rng.integers(0, 0x7f00, 2000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, ties, np.float32([0.0, -0.0, 1e-40, 3.4e38, -1.0, 65504.0])])
    ours = oracle_mod.f32_to_bf16_bits(x)
    ref = bits(torch.from_numpy(x).to(torch.bfloat16))
    assert np.array_equal(ours, ref)
    assert np.array_equal(oracle_mod.bf16_bits_to_f32(ref), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


# ---------------------------------------------------------------- compressor

def _rand_bf16(shape, seed, scale=1.0):
    return bits(synth.normal_bf16(shape, scale, seed, "K"))


def test_compress_one_hot_weight_selects_a_row(oracle_mod):
    B, L, H, d, blk = 2, 37, 3, 8, 8           # ragged tail of 5 rows is dropped
    X = _rand_bf16((B, L, H, d), 3)
    for i in (0, 3, blk - 1):
        w = np.zeros(blk, np.float32)
        w[i] = 1.0
        Xc = oracle_mod.hca_compress(X, w, blk)
        assert Xc.shape == (B, L // blk, H, d)
        assert np.array_equal(Xc, X[:, i:(L // blk) * blk:blk])


def test_compress_uniform_weight_is_exact_block_mean_on_dyadic_inputs(oracle_mod):
    B, L, H, d, blk = 1, 256, 2, 16, 128
    rng = np.random.default_rng(5)
    vals = rng.integers(-64, 65, (B, L, H, d)).astype(np.float64) / 8.0   # exact in bf16
    X = bf16(vals)
    w = np.full(blk, 1.0 / blk, np.float32)
    Xc = oracle_mod.hca_compress(X, w, blk)
    mean = vals.reshape(B, L // blk, blk, H, d).mean(axis=2)          # exact in fp32 here
    assert np.array_equal(Xc, bf16(mean))


def test_compress_block_one_weight_one_is_identity(oracle_mod):
    X = _rand_bf16((2, 19, 2, 32), 7)
    assert np.array_equal(oracle_mod.hca_compress(X, np.ones(1, np.float32), 1), X)


def test_compress_within_one_bf16_ulp_of_exact_weighted_sum(oracle_mod):
    cfg = synth.HcaConfig("t", B=1, L=512, Hq=1, Hkv=2, d=64)
    inp = synth.hca_inputs(cfg, seed=11)
    X, w = bits(inp["K"]), inp["w"].numpy()
    Xc = oracle_mod.hca_compress(X, w, cfg.blk)
    xf = inp["K"].double().numpy().reshape(1, cfg.n_c, cfg.blk, 2, 64)
    exact = np.einsum("i,bjihc->bjhc", w.astype(np.float64), xf)          # fp64, products exact
    ref = bf16(exact)
    diff = np.abs(Xc.astype(np.int32) - ref.astype(np.int32))              # same-sign -> ulp distance
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.99


def test_compress_is_linear_in_power_of_two_weight_scaling(oracle_mod):
    X = _rand_bf16((1, 256, 1, 32), 13)
    w = synth.uniform_f32((128,), 0.0, 2.0 / 128, 13, "w").numpy()
    a = oracle_mod.bf16_bits_to_f32(oracle_mod.hca_compress(X, w, 128))
    b = oracle_mod.bf16_bits_to_f32(oracle_mod.hca_compress(X, (w * 4).astype(np.float32), 128))
    assert np.array_equal(a * 4, b)
    assert np.abs(a).max() > 0


# ---------------------------------------------------------------- HCA visible set

@pytest.mark.parametrize("W,blk", [(128, 128), (5, 4), (1, 1), (3, 8), (200, 16), (2, 2)])
def test_hca_visible_set_matches_enumeration(oracle_mod, W, blk):
    for t in range(1024):
        ws = max(0, t - W + 1)
        assert oracle_mod.hca_window_start(t, W) == ws
        # definition: block j is visible iff every position of it precedes the window start
        vis = [j for j in range(t // blk + 1) if all(p < ws for p in range(blk * j, blk * j + blk))]
        assert vis == list(range(len(vis)))
        assert oracle_mod.hca_n_compressed(t, W, blk) == len(vis)


# ---------------------------------------------------------------- HCA attention

def _hca_case(B, L, Hq, Hkv, d, seed, sigma=None):
    cfg = synth.HcaConfig("t", B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, sigma=sigma)
    return synth.hca_inputs(cfg, seed=seed)


def test_hca_wide_window_is_dense_causal(oracle_mod):
    B, L, Hq, Hkv, d, blk = 2, 37, 4, 2, 16, 4
    inp = _hca_case(B, L, Hq, Hkv, d, 21, sigma=1.0)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    w = np.full(blk, 1.0 / blk, np.float32)
    Kc, Vc = oracle_mod.hca_compress(bits(K), w, blk), oracle_mod.hca_compress(bits(V), w, blk)
    scale = 0.3
    O = oracle_mod.hca_attn(bits(Q), Kc, Vc, bits(K), bits(V), blk=blk, W=L, scale=scale)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    ref = sdpa_ref(Q, K, V, mask, scale).reshape(B * L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [1, 3, 10])
def test_hca_block_one_identity_compressor_is_dense_causal(oracle_mod, W):
    B, L, Hq, Hkv, d = 1, 29, 4, 1, 8
    inp = _hca_case(B, L, Hq, Hkv, d, 23, sigma=1.0)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    one = np.ones(1, np.float32)
    Kc, Vc = oracle_mod.hca_compress(bits(K), one, 1), oracle_mod.hca_compress(bits(V), one, 1)
    O = oracle_mod.hca_attn(bits(Q), Kc, Vc, bits(K), bits(V), blk=1, W=W, scale=0.5)
    ref = sdpa_ref(Q, K, V, torch.ones(L, L, dtype=torch.bool).tril(), 0.5).reshape(L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


def test_hca_general_matches_masked_sdpa_over_entries_and_window(oracle_mod):
    B, L, Hq, Hkv, d, blk, W = 2, 45, 4, 2, 8, 4, 6
    inp = _hca_case(B, L, Hq, Hkv, d, 25, sigma=1.0)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    w = synth.uniform_f32((blk,), 0.0, 2.0 / blk, 25, "w").numpy()
    Kc, Vc = oracle_mod.hca_compress(bits(K), w, blk), oracle_mod.hca_compress(bits(V), w, blk)
    n_c = L // blk
    O, lse = oracle_mod.hca_attn(bits(Q), Kc, Vc, bits(K), bits(V), blk=blk, W=W, scale=0.4,
                                 with_lse=True)
    # keys = [all entries | all raw tokens]; mask built from the set definition by enumeration
    Kall = torch.cat([from_bits(Kc), K], dim=1)
    Vall = torch.cat([from_bits(Vc), V], dim=1)
    mask = torch.zeros(L, n_c + L, dtype=torch.bool)
    for t in range(L):
        ws = max(0, t - W + 1)
        for j in range(n_c):
            mask[t, j] = (blk * j + blk - 1) < ws
        for s in range(ws, t + 1):
            mask[t, n_c + s] = True
    ref = sdpa_ref(Q, Kall, Vall, mask, 0.4).reshape(B * L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    # log-sum-exp against the explicit scores
    g = Hq // Hkv
    for flat in (0, 17, B * L - 1):
        b, t = divmod(flat, L)
        for h in range(Hq):
            kk = Kall[b, mask[t], h // g].double()
            s = 0.4 * kk @ Q[b, t, h].double()
            assert abs(lse[flat, h] - torch.logsumexp(s, 0).item()) < 1e-12


def test_hca_golden_three_tokens(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "hca_three_token.json")))
    Q = bf16(np.array(g["Q"], np.float32).reshape(1, 3, 1, 2))
    K = bf16(np.array(g["K"], np.float32).reshape(1, 3, 1, 2))
    V = bf16(np.array(g["V"], np.float32).reshape(1, 3, 1, 2))
    O, lse = oracle_mod.hca_attn(Q, None, None, K, V, blk=g["blk"], W=g["W"], scale=LN2, with_lse=True)
    np.testing.assert_allclose(O[:, 0], np.array(g["O"]), atol=g["tolerance"], rtol=0)
    np.testing.assert_allclose(lse[:, 0], np.array(g["lse"]), atol=g["tolerance"], rtol=0)


def test_hca_golden_blocks_and_gap(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "hca_blocks_gap.json")))
    L, blk, W = g["L"], g["blk"], g["W"]
    s = np.arange(L, dtype=np.float32)
    K = bf16(np.stack([s, 0 * s], 1).reshape(1, L, 1, 2))
    V = bf16(np.stack([1 + 0 * s, s], 1).reshape(1, L, 1, 2))
    Q = bf16(np.tile(np.float32([1, 0]), (L, 1)).reshape(1, L, 1, 2))
    w = np.array(g["w"], np.float32)
    Kc, Vc = oracle_mod.hca_compress(K, w, blk), oracle_mod.hca_compress(V, w, blk)
    for t, (ents, win) in enumerate(g["visible"]):
        assert oracle_mod.hca_n_compressed(t, W, blk) == len(ents)
        assert oracle_mod.hca_window_start(t, W) == win[0]
    O = oracle_mod.hca_attn(Q, Kc, Vc, K, V, blk=blk, W=W, scale=LN2)
    np.testing.assert_allclose(O[:, 0, 0], 1.0, atol=1e-12)
    np.testing.assert_allclose(O[:, 0, 1], np.array(g["O1"]), atol=g["tolerance"], rtol=0)


def test_hca_constant_values_give_constant_output(oracle_mod):
    B, L, Hq, Hkv, d, blk, W = 1, 300, 2, 1, 16, 128, 16
    inp = _hca_case(B, L, Hq, Hkv, d, 27, sigma=1.0)
    V = torch.ones(B, L, Hkv, d, dtype=torch.bfloat16)
    w = np.full(blk, 1.0 / blk, np.float32)
    Kc, Vc = oracle_mod.hca_compress(bits(inp["K"]), w, blk), oracle_mod.hca_compress(bits(V), w, blk)
    O = oracle_mod.hca_attn(bits(inp["Q"]), Kc, Vc, bits(inp["K"]), bits(V), blk=blk, W=W)
    np.testing.assert_allclose(O, 1.0, atol=1e-12)


def test_hca_softmax_rows_sum_to_one(oracle_mod):
    # one-hot values make the output row equal to the probability row
    B, L, Hq, d = 1, 40, 2, 64
    inp = _hca_case(B, L, Hq, 1, d, 29, sigma=1.0)
    V = torch.zeros(B, L, 1, d, dtype=torch.bfloat16)
    V[0, torch.arange(L), 0, torch.arange(L)] = 1.0
    O = oracle_mod.hca_attn(bits(inp["Q"]), None, None, bits(inp["K"]), bits(V), blk=128, W=L)
    np.testing.assert_allclose(O.sum(-1), 1.0, atol=1e-12)
    for t in range(L):
        assert np.all(O[t, :, t + 1:] == 0.0) and np.all(O[t, :, : t + 1] > 0.0)


def test_hca_decode_form_equals_prefill_row(oracle_mod):
    B, L, Hq, Hkv, d, blk, W = 2, 700, 4, 1, 16, 128, 128
    inp = _hca_case(B, L, Hq, Hkv, d, 31)
    K, V, Q = bits(inp["K"]), bits(inp["V"]), bits(inp["Q"])
    w = inp["w"].numpy()
    Kc, Vc = oracle_mod.hca_compress(K, w, blk), oracle_mod.hca_compress(V, w, blk)
    t = L - 1
    rows = np.array([t, L + t], np.int64)
    O_pre = oracle_mod.hca_attn(Q, Kc, Vc, K, V, blk=blk, W=W, rows=rows)
    ws = t - W + 1
    O_dec = oracle_mod.hca_attn(Q[:, t:t + 1], Kc, Vc, K[:, ws:t + 1], V[:, ws:t + 1], win_start=ws,
                                q_offset=t, blk=blk, W=W)
    np.testing.assert_array_equal(O_dec, O_pre)


# ---------------------------------------------------------------- DSA indexer / top-k

def _dsa_small(B, L, Hq, d, seed, H_idx=4, d_idx=64):
    cfg = synth.DsaConfig("t", B=B, L=L, Hq=Hq, d=d, H_idx=H_idx, d_idx=d_idx, sigma=1.0)
    return synth.dsa_inputs(cfg, seed=seed)


def test_dsa_scores_match_integer_einsum(oracle_mod):
    inp = _dsa_small(2, 50, 2, 8, 41)
    q, k, w = inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy()
    ref = np.einsum("j,btjc,bsc->bts", w.astype(np.int64), q.astype(np.int64), k.astype(np.int64))
    for b in range(2):
        for r in (0, 7, 49):
            assert np.array_equal(oracle_mod.dsa_scores(q, k, w, b, r, r + 1), ref[b, r, : r + 1])


def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda s: (-int(scores[s]), s))[:k]
    return sorted(order) + [-1] * (k - len(order))


@pytest.mark.parametrize("k", [1, 7, 64])
def test_dsa_topk_matches_brute_force_sort_with_ties(oracle_mod, k):
    B, L, H_idx, d_idx = 2, 60, 2, 3
    g = torch.Generator().manual_seed(43 + k)
    q = torch.randint(-1, 2, (B, L, H_idx, d_idx), generator=g).to(torch.int8).numpy()
    kk = torch.randint(-1, 2, (B, L, d_idx), generator=g).to(torch.int8).numpy()
    w = np.array([1, 2], np.int32)
    idx = oracle_mod.dsa_topk(q, kk, w, k)
    sc = np.einsum("j,btjc,bsc->bts", w.astype(np.int64), q.astype(np.int64), kk.astype(np.int64))
    for b in range(B):
        for t in range(L):
            assert idx[b * L + t].tolist() == _brute_topk(sc[b, t, : t + 1], k)


def test_dsa_topk_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "dsa_topk_hand.json")))
    L = len(g["k_idx"])
    q = np.ones((1, L, 1, 1), np.int8)
    kk = np.array(g["k_idx"], np.int8).reshape(1, L, 1)
    idx = oracle_mod.dsa_topk(q, kk, np.array([1], np.int32), g["k"])
    assert idx.tolist() == g["idx"]


def test_dsa_topk_all_equal_scores_take_lowest_positions(oracle_mod):
    L, k = 40, 16
    q = np.zeros((1, L, 4, 64), np.int8)
    kk = _dsa_small(1, L, 1, 8, 45)["k_idx"].numpy()
    idx = oracle_mod.dsa_topk(q, kk, np.array([1, 2, 3, 4], np.int32), k)
    for t in range(L):
        n = min(k, t + 1)
        assert idx[t].tolist() == list(range(n)) + [-1] * (k - n)


def test_dsa_topk_large_k_keeps_every_candidate(oracle_mod):
    inp = _dsa_small(1, 33, 1, 8, 47)
    idx = oracle_mod.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), 40)
    for t in range(33):
        assert idx[t].tolist() == list(range(t + 1)) + [-1] * (40 - t - 1)


def test_dsa_topk_constructed_order(oracle_mod):
    # score(t, s) = 3 * key value of s; key values are a known permutation
    L, k = 50, 5
    perm = np.random.default_rng(49).permutation(L)                       # distinct values
    kk = np.zeros((1, L, 64), np.int8)
    kk[0, :, 0] = (perm % 17 - 8).astype(np.int8)
    kk[0, :, 1] = (perm // 17).astype(np.int8)
    q = np.zeros((1, L, 4, 64), np.int8)
    q[0, :, 0, 0] = 1
    q[0, :, 0, 1] = 17                                                    # 17*hi + lo - 8: injective
    idx = oracle_mod.dsa_topk(q, kk, np.array([3, 1, 1, 1], np.int32), k)
    for t in range(L):
        order = np.argsort(-perm[: t + 1], kind="stable")[:k]
        exp = sorted(order.tolist()) + [-1] * (k - min(k, t + 1))
        assert idx[t].tolist() == exp


def test_dsa_topk_decode_offset_equals_prefill_row(oracle_mod):
    inp = _dsa_small(2, 300, 1, 8, 51)
    q, kk, w = inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy()
    t = 299
    pre = oracle_mod.dsa_topk(q, kk, w, 32, rows=np.array([t, 300 + t]))
    dec = oracle_mod.dsa_topk(q[:, t:t + 1], kk, w, 32, q_offset=t)
    assert np.array_equal(pre, dec)


# ---------------------------------------------------------------- qk 576 / v 512 (shared latent)

def _sdpa_latent(Q, K, dv, mask, scale):
    """torch fp64 SDPA with keys of width dqk and values = the first dv columns of the keys."""
    q = Q.double().permute(0, 2, 1, 3)
    k = K.double().permute(0, 2, 1, 3)
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, k[..., :dv].contiguous(), attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def test_hca_latent_wide_window_is_dense_causal_with_positional_slice(oracle_mod):
    """W >= L: dense causal attention with 24-wide scores (16-wide latent + an 8-wide positional
    slice that changes the scores) and values = the latent part of the keys (torch fp64 SDPA)."""
    B, L, Hq, Hkv, dqk, dv = 2, 40, 4, 2, 24, 16
    g = torch.Generator().manual_seed(601)
    Q = torch.randn(B, L, Hq, dqk, generator=g).to(torch.bfloat16)
    K = torch.randn(B, L, Hkv, dqk, generator=g).to(torch.bfloat16)
    O, lse = oracle_mod.hca_attn_latent(bits(Q), None, bits(K), dv, W=L, scale=0.3, with_lse=True)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    np.testing.assert_allclose(O, _sdpa_latent(Q, K, dv, mask, 0.3).reshape(B * L, Hq, dv), rtol=0, atol=1e-12)
    # the positional slice is part of the score: zeroing it changes the result
    Q0 = Q.clone()
    Q0[..., dv:] = 0
    O0 = oracle_mod.hca_attn_latent(bits(Q0), None, bits(K), dv, W=L, scale=0.3)
    assert np.abs(O0 - O).max() > 1e-3
    s = 0.3 * K[1, :8, 1].double() @ Q[1, 7, 3].double()
    assert abs(lse[L + 7, 3] - torch.logsumexp(s, 0).item()) < 1e-12


def test_hca_latent_general_matches_masked_sdpa_over_entries_and_window(oracle_mod):
    """Entries + window (W = 5, blk = 4) with shared-latent values against SDPA over [entries ||
    window] with the visible set enumerated from its definition."""
    B, L, Hq, dqk, dv, blk, W = 1, 37, 2, 24, 16, 4, 5
    g = torch.Generator().manual_seed(603)
    Q = torch.randn(B, L, Hq, dqk, generator=g).to(torch.bfloat16)
    K = torch.randn(B, L, 1, dqk, generator=g).to(torch.bfloat16)
    w = np.full(blk, 0.25, np.float32)
    Kc = oracle_mod.hca_compress(bits(K), w, blk)
    O = oracle_mod.hca_attn_latent(bits(Q), Kc, bits(K), dv, blk=blk, W=W, scale=0.2)
    n_c = L // blk
    Kall = torch.cat([from_bits(Kc).view(B, n_c, 1, dqk), K], dim=1)
    mask = torch.zeros(L, n_c + L, dtype=torch.bool)
    for t in range(L):
        for j in range(n_c):
            if blk * (j + 1) <= t - W + 1:
                mask[t, j] = True
        for s in range(max(0, t - W + 1), t + 1):
            mask[t, n_c + s] = True
    np.testing.assert_allclose(O, _sdpa_latent(Q, Kall, dv, mask, 0.2).reshape(L, Hq, dv), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- CSA (top-k over compressed entries)

@pytest.mark.parametrize("blk", [1, 4, 7])
def test_csa_candidates_match_block_completion_enumeration(oracle_mod, blk):
    """Entry j (tokens blk*j .. blk*j + blk - 1) is a candidate of the query at t exactly when its
    last token is at or before t; the stored entries cap the count."""
    for n_c in (3, 1000):
        for t in range(200):
            want = sum(1 for j in range(n_c) if blk * j + blk - 1 <= t)
            assert oracle_mod.csa_n_candidates(t, blk, n_c) == want


@pytest.mark.parametrize("blk,k", [(4, 1), (4, 9), (3, 30)])
def test_csa_topk_matches_brute_force_sort_over_complete_blocks(oracle_mod, blk, k):
    B, L, H_idx, d_idx = 2, 90, 2, 3
    n_c = L // blk
    g = torch.Generator().manual_seed(211 + blk + k)
    q = torch.randint(-1, 2, (B, L, H_idx, d_idx), generator=g).to(torch.int8).numpy()
    kc = torch.randint(-1, 2, (B, n_c, d_idx), generator=g).to(torch.int8).numpy()
    w = np.array([2, 1], np.int32)
    idx = oracle_mod.csa_topk(q, kc, w, k, blk)
    sc = np.einsum("j,btjc,bsc->bts", w.astype(np.int64), q.astype(np.int64), kc.astype(np.int64))
    for b in range(B):
        for t in range(L):
            n = min((t + 1) // blk, n_c)
            assert idx[b * L + t].tolist() == _brute_topk(sc[b, t, :n], k)


def test_csa_with_block_one_is_dsa(oracle_mod):
    """blk = 1 makes every position its own entry: the CSA candidates are DSA's (0 .. t)."""
    inp = _dsa_small(2, 120, 1, 8, 213)
    q, kk, w = inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy()
    assert np.array_equal(oracle_mod.csa_topk(q, kk, w, 17, 1), oracle_mod.dsa_topk(q, kk, w, 17))
    assert np.array_equal(oracle_mod.csa_topk(q[:, 100:], kk, w, 17, 1, q_offset=100),
                          oracle_mod.dsa_topk(q[:, 100:], kk, w, 17, q_offset=100))


def test_csa_layer_with_identity_compressor_and_large_k_is_dense_causal(oracle_mod):
    """The whole CSA chain -- compress (blk = 1, w = [1]), select over complete blocks with
    k >= L, attend over the selected entries -- is dense causal attention (torch fp64 SDPA)."""
    B, L, Hq, d = 1, 40, 4, 16
    inp = _dsa_small(B, L, Hq, d, 215)
    K4 = bits(inp["K"]).reshape(B, L, 1, d)
    V4 = bits(inp["V"]).reshape(B, L, 1, d)
    one = np.ones(1, np.float32)
    Kc = oracle_mod.hca_compress(K4, one, 1).reshape(B, L, d)
    Vc = oracle_mod.hca_compress(V4, one, 1).reshape(B, L, d)
    idx = oracle_mod.csa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), 64, 1)
    O = oracle_mod.dsa_attn(bits(inp["Q"]), Kc, Vc, idx, scale=0.25)
    ref = sdpa_ref(inp["Q"], inp["K"].unsqueeze(2), inp["V"].unsqueeze(2),
                   torch.ones(L, L, dtype=torch.bool).tril(), 0.25).reshape(B * L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


def test_csa_attention_over_4to1_entries_matches_masked_sdpa(oracle_mod):
    """4:1 entries, top-5 of the complete blocks: attention over the selected entries equals SDPA
    over the compressed keys with the selection as the mask (a query with no complete block sees
    nothing: O = 0)."""
    B, L, Hq, d, blk, k = 1, 64, 2, 16, 4, 5
    n_c = L // blk
    inp = _dsa_small(B, L, Hq, d, 217)
    w4 = np.array([0.125, 0.25, 0.375, 0.25], np.float32)
    Kc = oracle_mod.hca_compress(bits(inp["K"]).reshape(B, L, 1, d), w4, blk).reshape(B, n_c, d)
    Vc = oracle_mod.hca_compress(bits(inp["V"]).reshape(B, L, 1, d), w4, blk).reshape(B, n_c, d)
    kc_idx = torch.randint(-8, 9, (B, n_c, 64), generator=torch.Generator().manual_seed(219)).to(torch.int8)
    idx = oracle_mod.csa_topk(inp["q_idx"].numpy(), kc_idx.numpy(), inp["w_idx"].numpy(), k, blk)
    O = oracle_mod.dsa_attn(bits(inp["Q"]), Kc, Vc, idx, scale=0.25)
    mask = torch.zeros(L, n_c, dtype=torch.bool)
    for t in range(L):
        for j in idx[t]:
            if j >= 0:
                assert blk * j + blk - 1 <= t
                mask[t, j] = True
    Kt, Vt = from_bits(Kc).view(B, n_c, 1, d), from_bits(Vc).view(B, n_c, 1, d)
    seen = mask.any(1)
    ref = sdpa_ref(inp["Q"][:, seen], Kt, Vt, mask[seen], 0.25).reshape(-1, Hq, d)
    np.testing.assert_allclose(O[seen.numpy()], ref, rtol=0, atol=1e-12)
    assert np.all(O[~seen.numpy()] == 0.0) and (~seen).sum() == blk - 1


# ---------------------------------------------------------------- output gate + virtual-head mix

def _gate_inputs(B, L, H, dv, rq, r, seed):
    g = torch.Generator().manual_seed(seed)
    O = (torch.randn(B, L, H, dv, generator=g) * 0.1).to(torch.bfloat16)
    cq = torch.randn(B, L, rq, generator=g).to(torch.bfloat16)
    Wg = (torch.randn(H * dv, rq, generator=g) / math.sqrt(rq)).to(torch.bfloat16)
    U = (torch.randn(H, r, generator=g) * 0.3).numpy().astype(np.float32)
    V = (torch.randn(H, r, generator=g) * 0.3).numpy().astype(np.float32)
    return O, cq, Wg, U, V


def test_gate_vha_zero_gate_weights_and_no_mix_halve_the_output(oracle_mod):
    """W_g = 0 gives sigmoid(0) = 1/2 everywhere; U = 0 switches the mix off: Y = O / 2 exactly."""
    O, cq, _, _, _ = _gate_inputs(2, 5, 4, 8, 16, 2, 401)
    Wg = torch.zeros(4 * 8, 16, dtype=torch.bfloat16)
    Y = oracle_mod.gate_vha(bits(O), bits(cq), bits(Wg), np.zeros((4, 2), np.float32), np.ones((4, 2), np.float32))
    np.testing.assert_array_equal(Y, O.double().numpy() / 2)


def test_gate_vha_without_mix_is_sigmoid_of_latent_projection(oracle_mod):
    """No mix (rank 0): Y = sigmoid(cq W_g^T) * O, the gate through torch's fp64 matmul and sigmoid."""
    B, L, H, dv, rq = 2, 6, 4, 8, 32
    O, cq, Wg, _, _ = _gate_inputs(B, L, H, dv, rq, 1, 403)
    Y = oracle_mod.gate_vha(bits(O), bits(cq), bits(Wg), np.zeros((H, 0), np.float32), np.zeros((H, 0), np.float32))
    z = (cq.double().reshape(B * L, rq) @ Wg.double().t()).reshape(B, L, H, dv)
    np.testing.assert_allclose(Y, (torch.sigmoid(z) * O.double()).numpy(), rtol=0, atol=1e-13)


def test_gate_vha_mix_orientation_copies_one_head(oracle_mod):
    """I + U V^T with U = [[1], [0]], V = [[-1], [1]] has rows [0, 1] and [0, 1]: both heads
    become head 1 (U and V swapped would give [[0, 0], [1, 2]] instead)."""
    B, L, H, dv, rq = 1, 3, 2, 8, 16
    O, cq, _, _, _ = _gate_inputs(B, L, H, dv, rq, 1, 405)
    Wg = torch.zeros(H * dv, rq, dtype=torch.bfloat16)
    U = np.array([[1.0], [0.0]], np.float32)
    V = np.array([[-1.0], [1.0]], np.float32)
    Y = oracle_mod.gate_vha(bits(O), bits(cq), bits(Wg), U, V)
    o = O.double().numpy()
    np.testing.assert_array_equal(Y[:, :, 0], o[:, :, 1] / 2)
    np.testing.assert_array_equal(Y[:, :, 1], o[:, :, 1] / 2)


def test_gate_vha_full_rank_negative_identity_mix_cancels_the_output(oracle_mod):
    """U V^T = -I (rank H) removes the identity path: Y = 0."""
    O, cq, Wg, _, _ = _gate_inputs(1, 4, 3, 8, 16, 3, 407)
    Y = oracle_mod.gate_vha(bits(O), bits(cq), bits(Wg), -np.eye(3, dtype=np.float32), np.eye(3, dtype=np.float32))
    np.testing.assert_allclose(Y, 0.0, rtol=0, atol=1e-15)


def test_gate_vha_mix_matches_matrix_form_per_channel(oracle_mod):
    """With the gate fixed at 1/2, each token's output is (I + U V^T) applied to its H x dv block,
    checked against a torch fp64 matrix product (heads mix, channels do not)."""
    B, L, H, dv, rq, r = 2, 3, 16, 32, 16, 4
    O, cq, _, U, V = _gate_inputs(B, L, H, dv, rq, r, 409)
    Wg = torch.zeros(H * dv, rq, dtype=torch.bfloat16)
    Y = oracle_mod.gate_vha(bits(O), bits(cq), bits(Wg), U, V)
    M = torch.eye(H, dtype=torch.float64) + torch.from_numpy(U).double() @ torch.from_numpy(V).double().t()
    ref = torch.einsum("hg,btgc->bthc", M, O.double()) / 2
    np.testing.assert_allclose(Y, ref.numpy(), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- DSA attention

def test_dsa_attention_with_large_k_is_dense_causal(oracle_mod):
    B, L, Hq, d = 2, 31, 4, 16
    inp = _dsa_small(B, L, Hq, d, 61)
    idx = oracle_mod.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), 40)
    O = oracle_mod.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx, scale=0.25)
    ref = sdpa_ref(inp["Q"], inp["K"].unsqueeze(2), inp["V"].unsqueeze(2),
                   torch.ones(L, L, dtype=torch.bool).tril(), 0.25).reshape(B * L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


def test_dsa_attention_matches_sdpa_masked_by_selection(oracle_mod):
    B, L, Hq, d, k = 1, 64, 4, 16, 9
    inp = _dsa_small(B, L, Hq, d, 63)
    idx = oracle_mod.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), k)
    O, lse = oracle_mod.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx, scale=0.25,
                                 with_lse=True)
    mask = torch.zeros(L, L, dtype=torch.bool)
    for t in range(L):
        for s in idx[t]:
            if s >= 0:
                mask[t, s] = True
    ref = sdpa_ref(inp["Q"], inp["K"].unsqueeze(2), inp["V"].unsqueeze(2), mask, 0.25).reshape(L, Hq, d)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    t, h = 50, 3
    s = 0.25 * inp["K"][0, mask[t]].double() @ inp["Q"][0, t, h].double()
    assert abs(lse[t, h] - torch.logsumexp(s, 0).item()) < 1e-12


def test_dsa_attention_ignores_index_order_and_padding(oracle_mod):
    B, L, Hq, d, k = 1, 64, 2, 16, 12
    inp = _dsa_small(B, L, Hq, d, 65)
    idx = oracle_mod.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), k)
    rng = np.random.default_rng(67)
    shuffled = np.stack([rng.permutation(row) for row in idx])
    a = oracle_mod.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx)
    b = oracle_mod.dsa_attn(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), shuffled)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- backward pass
# The gradients are pinned to torch's fp64 autograd through an explicitly masked softmax
# attention (the visible set enumerated from its definition, as above), to closed forms,
# and, for the compressor, to autograd of the exact weighted block sum.

def _masked_attention_grads(Q, Kall, Vall, mask, scale, dO):
    """fp64 autograd of sum(O * dO) with O = softmax(scale q.k, masked) v; K/V [B,Lk,Hkv,d]
    shared by the Hq/Hkv query heads of a group.  Returns dQ, dK, dV (numpy fp64)."""
    q = Q.double().clone().requires_grad_(True)
    k = Kall.double().clone().requires_grad_(True)
    v = Vall.double().clone().requires_grad_(True)
    g = q.shape[2] // k.shape[2]
    kk = k.repeat_interleave(g, dim=2)
    vv = v.repeat_interleave(g, dim=2)
    s = scale * torch.einsum("bthc,bshc->bhts", q, kk)
    s = s.masked_fill(~mask.view(1, 1, *mask.shape), float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = torch.einsum("bhts,bshc->bthc", p, vv)
    (o * torch.as_tensor(dO)).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def test_hca_attn_bwd_matches_autograd_over_entries_and_window(oracle_mod):
    B, L, Hq, Hkv, d, blk, W, scale = 2, 45, 4, 2, 8, 4, 6, 0.4
    inp = _hca_case(B, L, Hq, Hkv, d, 91, sigma=1.0)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    w = synth.uniform_f32((blk,), 0.0, 2.0 / blk, 91, "w").numpy()
    Kc, Vc = oracle_mod.hca_compress(bits(K), w, blk), oracle_mod.hca_compress(bits(V), w, blk)
    n_c = L // blk
    dO = np.random.default_rng(92).standard_normal((B, L, Hq, d))
    dQ, dKc, dVc, dKw, dVw = oracle_mod.hca_attn_bwd(bits(Q), Kc, Vc, bits(K), bits(V), dO, blk=blk, W=W,
                                                     scale=scale)
    Kall = torch.cat([from_bits(Kc), K], dim=1)
    Vall = torch.cat([from_bits(Vc), V], dim=1)
    mask = torch.zeros(L, n_c + L, dtype=torch.bool)
    for t in range(L):
        ws = max(0, t - W + 1)
        for j in range(n_c):
            mask[t, j] = (blk * j + blk - 1) < ws
        for s in range(ws, t + 1):
            mask[t, n_c + s] = True
    rQ, rK, rV = _masked_attention_grads(Q, Kall, Vall, mask, scale, dO)
    np.testing.assert_allclose(dQ, rQ, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dKc, rK[:, :n_c], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dVc, rV[:, :n_c], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dKw, rK[:, n_c:], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dVw, rV[:, n_c:], rtol=0, atol=1e-11)


def test_hca_attn_bwd_decode_offset_matches_autograd(oracle_mod):
    """One query per sequence at t = 300 over an entry cache and a window buffer that starts at
    the window (q_offset and win_start both in play)."""
    B, Hq, Hkv, d, blk, W, t = 2, 4, 1, 8, 16, 20, 300
    n_c = (t - W + 1) // blk
    ws = t - W + 1
    g = torch.Generator().manual_seed(93)
    Q = torch.randn(B, 1, Hq, d, generator=g).to(torch.bfloat16)
    Kc = torch.randn(B, n_c, Hkv, d, generator=g).to(torch.bfloat16)
    Vc = torch.randn(B, n_c, Hkv, d, generator=g).to(torch.bfloat16)
    Kw = torch.randn(B, W, Hkv, d, generator=g).to(torch.bfloat16)
    Vw = torch.randn(B, W, Hkv, d, generator=g).to(torch.bfloat16)
    dO = np.random.default_rng(94).standard_normal((B, 1, Hq, d))
    dQ, dKc, dVc, dKw, dVw = oracle_mod.hca_attn_bwd(bits(Q), bits(Kc), bits(Vc), bits(Kw), bits(Vw), dO,
                                                     win_start=ws, q_offset=t, blk=blk, W=W, scale=0.3)
    mask = torch.ones(1, n_c + W, dtype=torch.bool)  # every stored entry and window row is visible
    rQ, rK, rV = _masked_attention_grads(Q, torch.cat([Kc, Kw], 1), torch.cat([Vc, Vw], 1), mask, 0.3, dO)
    np.testing.assert_allclose(dQ, rQ, rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.concatenate([dKc, dKw], 1), rK, rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.concatenate([dVc, dVw], 1), rV, rtol=0, atol=1e-11)


def test_hca_attn_bwd_closed_forms(oracle_mod):
    """Token 0 sees only itself (p = 1): its dQ is 0 and its own V row receives dO.  With every
    V row equal, O no longer depends on the scores, so dQ and all key gradients vanish."""
    B, L, Hq, Hkv, d, blk, W = 1, 12, 2, 1, 4, 4, 5
    inp = _hca_case(B, L, Hq, Hkv, d, 95, sigma=1.0)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    w = np.full(blk, 1.0 / blk, np.float32)
    Kc, Vc = oracle_mod.hca_compress(bits(K), w, blk), oracle_mod.hca_compress(bits(V), w, blk)
    dO = np.zeros((B, L, Hq, d))
    dO[0, 0] = np.random.default_rng(96).standard_normal((Hq, d))
    dQ, dKc, dVc, dKw, dVw = oracle_mod.hca_attn_bwd(bits(Q), Kc, Vc, bits(K), bits(V), dO, blk=blk, W=W)
    assert np.all(dQ == 0.0) and np.all(dKc == 0.0) and np.all(dVc == 0.0)
    np.testing.assert_allclose(dVw[0, 0, 0], dO[0, 0].sum(0), rtol=0, atol=1e-15)  # both heads share kv 0
    assert np.all(dVw[0, 1:] == 0.0) and np.all(dKw == 0.0)
    Vconst = torch.ones_like(V) * 0.75
    Vc1 = oracle_mod.hca_compress(bits(Vconst), w, blk)  # entries of a constant row stay 0.75
    dO = np.random.default_rng(97).standard_normal((B, L, Hq, d))
    dQ, dKc, dVc, dKw, dVw = oracle_mod.hca_attn_bwd(bits(Q), Kc, Vc1, bits(K), bits(Vconst), dO, blk=blk, W=W)
    assert np.abs(dQ).max() < 1e-14 and np.abs(dKc).max() < 1e-14 and np.abs(dKw).max() < 1e-14
    # the value gradients still sum to the total dO of each kv head (softmax rows sum to 1)
    np.testing.assert_allclose(dVc.sum((1,)) + dVw.sum((1,)), dO.sum(1).reshape(B, Hkv, Hq // Hkv, d).sum(2),
                               rtol=0, atol=1e-12)


def test_dsa_attn_bwd_matches_autograd_over_selection(oracle_mod):
    B, L, Hq, d, k, scale = 2, 40, 4, 16, 7, 0.25
    inp = _dsa_small(B, L, Hq, d, 98)
    idx = oracle_mod.dsa_topk(inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w_idx"].numpy(), k)
    rng = np.random.default_rng(99)
    idx = np.stack([rng.permutation(row) for row in idx]).reshape(B, L, k)  # order must not matter
    dO = rng.standard_normal((B, L, Hq, d))
    dQ, dK, dV = oracle_mod.dsa_attn_bwd(bits(inp["Q"]), bits(inp["K"]), bits(inp["V"]), idx, dO, scale=scale)
    for b in range(B):
        mask = torch.zeros(L, L, dtype=torch.bool)
        for t in range(L):
            for s in idx[b, t]:
                if s >= 0:
                    mask[t, s] = True
        rQ, rK, rV = _masked_attention_grads(inp["Q"][b:b + 1], inp["K"][b:b + 1].unsqueeze(2),
                                             inp["V"][b:b + 1].unsqueeze(2), mask, scale, dO[b:b + 1])
        np.testing.assert_allclose(dQ[b:b + 1], rQ, rtol=0, atol=1e-11)
        np.testing.assert_allclose(dK[b], rK[0, :, 0], rtol=0, atol=1e-11)
        np.testing.assert_allclose(dV[b], rV[0, :, 0], rtol=0, atol=1e-11)


def test_compress_bwd_matches_autograd_and_one_hot(oracle_mod):
    B, L, H, d, blk = 2, 23, 3, 5, 4  # 5 complete blocks and a partial tail of 3 tokens
    X = synth.normal_bf16((B, L, H, d), 1.0, 100, "K")
    w = synth.uniform_f32((blk,), 0.0, 2.0 / blk, 100, "w").numpy()
    n_c = L // blk
    dXc = np.random.default_rng(101).standard_normal((B, n_c, H, d))
    dX, dw = oracle_mod.hca_compress_bwd(bits(X), w, dXc, blk)
    x = X.double().clone().requires_grad_(True)
    wt = torch.as_tensor(w, dtype=torch.float64).clone().requires_grad_(True)
    xc = torch.einsum("i,bjihc->bjhc", wt, x[:, : n_c * blk].reshape(B, n_c, blk, H, d))
    (xc * torch.as_tensor(dXc)).sum().backward()
    np.testing.assert_allclose(dX, x.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-13, atol=1e-12)
    assert np.all(dX[:, n_c * blk:] == 0.0)  # the partial tail block feeds no entry
    onehot = np.zeros(blk, np.float32)
    onehot[2] = 1.0
    dX1, _ = oracle_mod.hca_compress_bwd(bits(X), onehot, dXc, blk)
    np.testing.assert_array_equal(dX1[:, 2: n_c * blk: blk], dXc)  # row 2 of each block takes dXc
    assert np.count_nonzero(dX1) == np.count_nonzero(dXc)
