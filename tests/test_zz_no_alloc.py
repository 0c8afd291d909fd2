"""The allocation-free top-k entry point, for callers that cannot allocate device memory
(hot paths that must not call cudaMalloc/cudaFree, plugins whose host framework owns all
device memory, callers with no workspace allocator).

dsa_index_topk_noalloc keeps its score rows in a fixed array inside the library.  Its GPU
test compares it, through the C ABI, against dsa_index_topk (which uses a caller workspace)
on two calls in a row with different inputs, so a second call that saw stale scratch from
the first would show, and checks sampled rows of both against the CPU oracle.  This file sorts last so a stop-at-first-failure run has already run
every other test; the test also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth


def _lib():
    from sparse_attention_hca_b200 import build

    build.build()
    import sparse_attention_hca_b200 as m

    return m, m.lib()


def test_noalloc_rejects_oversized_calls_before_any_cuda_call():
    _, lib = _lib()
    cap = lib.dsa_index_topk_noalloc_max_scratch_bytes()
    assert cap == 64 << 20
    fake = ctypes.c_void_p(1 << 20)     # never dereferenced: the size check comes first
    # 32768 x 32768 scores need 4 GiB > 64 MiB
    assert lib.dsa_index_topk_noalloc(fake, fake, fake, fake, 1, 32768, 0, 32768, 4, 64, 2048, None) == -5
    # 17 sequences of 1M keys (Lq = 1) exceed it, 16 would fit (their int32 score rows: 64 MiB)
    assert 16 * 1048576 * 4 <= cap
    assert lib.dsa_index_topk_noalloc(fake, fake, fake, fake, 17, 1, 1048575, 1048576, 4, 64, 2048, None) == -5


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    m, lib = _lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    cases = [
        # prefill: 3000 x 3000 scores (36 MB of scratch), rows above and below k
        dict(B=1, L=3000, Lq=3000, q_offset=0, k=2048, seed=101),
        # decode: 3 sequences, one query each at position 200000, different inputs
        dict(B=3, L=200001, Lq=1, q_offset=200000, k=2048, seed=202),
    ]
    for c in cases:
        g = torch.Generator().manual_seed(c["seed"])
        q = torch.randint(-8, 9, (c["B"], c["Lq"], 4, 64), generator=g).to(torch.int8).cuda()
        kk = torch.randint(-8, 9, (c["B"], c["L"], 64), generator=g).to(torch.int8).cuda()
        w = torch.randint(1, 5, (4,), generator=g).to(torch.int32).cuda()
        need = lib.dsa_index_topk_workspace_size(c["B"], c["Lq"], c["q_offset"], c["L"], c["k"])
        assert need <= lib.dsa_index_topk_noalloc_max_scratch_bytes()
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        ref = torch.empty((c["B"], c["Lq"], c["k"]), dtype=torch.int32, device="cuda")
        got = torch.full_like(ref, -7)
        st = lib.dsa_index_topk(ptr(q), ptr(kk), ptr(w), ptr(ref), ptr(ws), ws.numel(), c["B"], c["Lq"],
                                c["q_offset"], c["L"], 4, 64, c["k"], stream)
        assert st == 0
        st = lib.dsa_index_topk_noalloc(ptr(q), ptr(kk), ptr(w), ptr(got), c["B"], c["Lq"], c["q_offset"], c["L"],
                                        4, 64, c["k"], stream)
        assert st == 0
        assert lib.hcadsa_check_device_error(stream) == 0
        # top-k indices: the tolerance of every top-k test here is bit-exact
        assert torch.equal(got, ref)
        assert (got[..., 0] >= 0).all()
        # ... and both equal the oracle on sampled rows (the two entries share their scoring
        # kernels, so the comparison above alone would not see a scoring fault)
        rows = np.unique(np.linspace(0, c["B"] * c["Lq"] - 1, 12).astype(np.int64))
        want = oracle.dsa_topk(q.cpu().numpy(), kk.cpu().numpy(), w.cpu().numpy(), c["k"], q_offset=c["q_offset"],
                               rows=rows)
        flat = got.reshape(c["B"] * c["Lq"], c["k"])[torch.as_tensor(rows, device="cuda")].cpu().numpy()
        assert np.array_equal(flat, want)
