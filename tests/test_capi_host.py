"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects invalid arguments with the documented status codes
before touching any device memory."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hcadsa.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_hca_b200 import build

    build.build()
    import sparse_attention_hca_b200 as m

    return m.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z][a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("hca_compress_kv", "hca_attn_fwd", "dsa_index_topk", "dsa_sparse_attn_fwd",
              "hcadsa_check_device_error", "hcadsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    assert lib.hcadsa_version() >= 100
    for code in range(0, -9, -1):
        s = lib.hcadsa_status_string(code).decode()
        assert s.startswith("HCADSA_")
    assert b"unknown" in lib.hcadsa_status_string(-99)


FAKE = ctypes.c_void_p(1 << 20)      # never dereferenced: every call below fails its checks first
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def test_compress_argument_errors(lib):
    f = lib.hca_compress_kv
    assert f(None, FAKE, FAKE, FAKE, FAKE, 1, 256, 1, 512, 128, None) == -1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 256, 0, 512, 128, None) == -2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 256, 1, 500, 128, None) == -4
    assert f(FAKE, MISALIGNED, FAKE, FAKE, FAKE, 1, 256, 1, 512, 128, None) == -3
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 1, 512, 128, None) == 0   # no complete block: nothing to do


def test_hca_attn_argument_errors(lib):
    f = lib.hca_attn_fwd
    args = dict(Q=FAKE, Kc=FAKE, Vc=FAKE, n_c=8, Kw=FAKE, Vw=FAKE, ws=0, n_w=1024, O=FAKE, lse=None, B=1,
                Lq=1024, q0=0, Hq=16, Hkv=1, d=512, blk=128, W=128, scale=0.04, wsp=None, wsb=0, s=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(*a.values())

    assert call(Q=None) == -1
    assert call(Hkv=3) == -2             # 16 % 3
    assert call(d=256) == -4
    assert call(Hq=48, Hkv=1) == -4      # group 48 does not divide 128
    assert call(O=MISALIGNED) == -3
    assert call(n_w=1000) == -2          # window of the last query not stored
    assert call(n_c=6) == -2             # entries of the last query not stored
    assert call(ws=1, n_w=1023) == -2    # the window buffer starts after the first query's window
    assert call(q0=-1) == -2
    assert call(lse=ctypes.c_void_p(FAKE.value + 2)) == -3   # lse must be 4-byte aligned
    assert call(Lq=0) == 0


def test_dsa_argument_errors(lib):
    t = lib.dsa_index_topk
    assert t(None, FAKE, FAKE, FAKE, FAKE, 1 << 30, 1, 64, 0, 64, 4, 64, 16, None) == -1
    assert t(FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 1, 64, 0, 64, 8, 64, 16, None) == -4
    assert t(FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 1, 64, 0, 64, 4, 64, 0, None) == -2
    assert t(FAKE, FAKE, FAKE, FAKE, None, 0, 1, 4096, 0, 4096, 4, 64, 16, None) == -5
    assert t(FAKE, FAKE, FAKE, FAKE, FAKE, 16, 1, 4096, 0, 4096, 4, 64, 16, None) == -5
    a = lib.dsa_sparse_attn_fwd
    assert a(FAKE, FAKE, FAKE, FAKE, None, None, 1, 8, 8, 64, 256, 16, 0.06, None) == -1
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 32, 256, 16, 0.06, None) == -4
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 512, 16, 0.06, None) == -4
    assert a(FAKE, FAKE, MISALIGNED, FAKE, FAKE, None, 1, 8, 8, 64, 256, 16, 0.06, None) == -3
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 256, 4097, 0.06, None) == -4  # k > 4096
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 256, 16, 0.0, None) == -2    # scale <= 0
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 256, 16, float("nan"), None) == -2
    w = lib.dsa_sparse_attn_fwd_ws  # same argument checks before any device query or launch
    assert w(FAKE, FAKE, FAKE, None, FAKE, None, 1, 8, 8, 64, 256, 16, 0.06, None, 0, None) == -1
    assert w(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 128, 16, 0.06, None, 0, None) == -4
    assert w(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 256, 16, -1.0, None, 0, None) == -2
    assert w(FAKE, MISALIGNED, FAKE, FAKE, FAKE, None, 1, 8, 8, 64, 256, 16, 0.06, None, 0, None) == -3
    assert lib.dsa_sparse_attn_fwd_workspace_size(1, 8, 0) == 0        # invalid k
    assert lib.dsa_sparse_attn_fwd_workspace_size(1, 8, 4097) == 0     # unsupported k


def test_workspace_size_queries(lib):
    # 64 or more query rows per sequence: the fused indexer + selection keeps no score rows, only
    # the per-channel min / max of k_idx (2 x 64 int32 per sequence) -- at 32K as at 131K
    assert lib.dsa_index_topk_workspace_size(1, 32768, 0, 32768, 2048) == 2 * 64 * 4
    assert lib.dsa_index_topk_workspace_size(3, 131072, 0, 131072, 2048) == 3 * 2 * 64 * 4
    # fewer rows (decode shapes) keep their int32 score rows: 63 rows over 5000 keys
    assert lib.dsa_index_topk_workspace_size(1, 63, 4937, 5000, 2048) == 63 * 5120 * 4
    # few rows over many keys add the multi-CTA selection state: per row 16 bytes + a 2048-bin
    # histogram + 8192 (score, position) candidates
    assert lib.dsa_index_topk_workspace_size(2, 1, 1048575, 1048576, 2048) == 2 * 1048576 * 4 + 2 * (
        16 + 2048 * 4 + 8192 * 8)
    # HCA's workspace holds one probability-tile slot per resident CTA, so it is sized for the
    # current device; unsupported shapes (and a machine with no device to size for) give 0
    assert lib.hca_attn_fwd_workspace_size(1, 32768, 0, 16, 1, 256, 256, 128, 128) == 0
    assert lib.hca_attn_fwd_workspace_size(1, 32768, 0, 16, 3, 512, 256, 128, 128) == 0


def test_next_row_entry_argument_errors(lib):
    """Gate + head mix, qk 576 / v 512 HCA, CSA selection: documented host-side errors."""
    g = lib.attn_gate_vha_fwd
    assert g(None, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 16, 512, 1024, 4, None) == -1
    assert g(FAKE, FAKE, FAKE, None, FAKE, FAKE, 1, 128, 16, 512, 1024, 4, None) == -1   # r > 0 needs U, V
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 16, 512, 1024, -1, None) == -2
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 12, 512, 1024, 4, None) == -4   # H not 16/32/64
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 16, 512, 1000, 4, None) == -4   # rq % 64
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 16, 512, 1024, 5, None) == -4   # rank > 4
    assert g(FAKE, MISALIGNED, FAKE, FAKE, FAKE, FAKE, 1, 128, 16, 512, 1024, 4, None) == -3
    assert lib.hca_attn_fwd_latent_workspace_size(1, 4096, 0, 16, 1, 512, 512, 31, 128, 128) == 0  # dqk != 576
    la = lib.hca_attn_fwd_latent
    assert la(FAKE, FAKE, 1, FAKE, 0, 256, FAKE, None, 1, 256, 0, 16, 1, 512, 512, 128, 128, 0.04, FAKE, 1 << 30,
              None) == -4
    c = lib.csa_index_topk
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 1, 64, 0, 16, 4, 64, 16, 0, None) == -2  # blk < 1


def test_backward_argument_errors(lib):
    """The three backward calls: documented host-side errors before anything is enqueued."""
    d = lib.dsa_sparse_attn_bwd
    args = [FAKE] * 10 + [1, 8, 8, 64, 256, 16, 0.0625, None]
    assert d(*([None] + args[1:])) == -1
    assert d(*(args[:13] + [32] + args[14:])) == -4        # Hq != 64
    assert d(*(args[:14] + [512] + args[15:])) == -4       # d != 256
    assert d(*(args[:15] + [5000] + args[16:])) == -4      # k > 4096
    assert d(*(args[:15] + [0] + args[16:])) == -2         # k < 1
    assert d(*(args[:7] + [MISALIGNED] + args[8:])) == -3  # dQ misaligned
    h = lib.hca_attn_bwd
    # Q, Kc, Vc, n_c, Kw, Vw, win_start, n_w, O, dO, lse, dQ, dKc, dVc, dKw, dVw,
    # B, Lq, q_offset, Hq, Hkv, d, blk, W, scale, ws, ws_bytes, stream
    base = [FAKE, FAKE, FAKE, 1, FAKE, FAKE, 0, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            1, 256, 0, 16, 1, 512, 128, 128, 0.04, FAKE, 1 << 40, None]

    def call(**kw):
        a = list(base)
        pos = {"Q": 0, "n_w": 7, "Hq": 19, "Hkv": 20, "d": 21, "ws_bytes": 26, "dQ": 11, "win_start": 6}
        for k, v in kw.items():
            a[pos[k]] = v
        return h(*a)

    assert call(Q=None) == -1
    assert call(d=256) == -4
    assert call(Hq=16, Hkv=3) == -2
    assert call(n_w=200) == -2                # the last query's window is past the raw buffer
    assert call(win_start=5) == -2            # the first query's window starts before it
    assert call(ws_bytes=1024) == -5
    assert call(dQ=MISALIGNED) == -3
    # one fp32 D per query row (256-rounded) + P and dS blocks: 4096 row tiles x (2 entry + 3
    # window slots) x 2 x 32 KB at L = 32768, 16 heads on one K/V head
    assert lib.hca_attn_bwd_workspace_size(1, 32768, 0, 16, 1, 512, 256, 128, 128) == \
        32768 * 16 * 4 + 2 * 4096 * 5 * 128 * 128 * 2
    assert lib.hca_attn_bwd_workspace_size(1, 32768, 0, 16, 1, 256, 256, 128, 128) == 0
    cb = lib.hca_compress_bwd
    assert cb(None, FAKE, FAKE, FAKE, FAKE, 1, 256, 1, 512, 128, None) == -1
    assert cb(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 256, 1, 500, 128, None) == -4
    assert cb(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 256, 1, 512, 2048, None) == -4
    assert cb(FAKE, FAKE, FAKE, MISALIGNED, FAKE, 1, 256, 1, 512, 128, None) == -3
    assert cb(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 1, 512, 128, None) == 0  # no complete block: nothing to do
