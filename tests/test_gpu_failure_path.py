"""Device-side failure detection without faulting the GPU: a bounded wait that nothing
satisfies must give up and be reported through the error word, and the context must stay
usable afterwards."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_is_reported():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_hca_b200 import build

    build.build()
    import sparse_attention_hca_b200 as hd

    lib = hd.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.hcadsa_check_device_error(s) == 0
    assert lib.hcadsa_selftest_bounded_wait(20000, s) == 0          # 20 ms limit
    assert lib.hcadsa_check_device_error(s) == -7                   # HCADSA_ERR_TIMEOUT, then cleared
    assert lib.hcadsa_check_device_error(s) == 0
    # the context still works: a real call succeeds afterwards
    x = torch.randn(1, 256, 1, 64, device="cuda").to(torch.bfloat16)
    w = torch.full((128,), 1.0 / 128, device="cuda")
    Kc, _ = hd.hca_compress_kv(x, x, w, 128)
    torch.cuda.synchronize()
    ref = x.float().reshape(2, 128, 64).mean(1).to(torch.bfloat16)
    assert (Kc.reshape(2, 64).float() - ref.float()).abs().max() <= 2 ** -8
