"""The allocation-free forward entry point, for callers that cannot allocate
device memory (plug-ins inside a framework that owns all device memory,
deployments that forbid allocation after start-up).  It must give the same
result as the ordinary forward, which takes a caller-allocated workspace,
call after call even though every call reuses one fixed scratch array.

Collected last on purpose (file name), so a stop-at-first-failure run has
already run every other test when it gets here."""
from __future__ import annotations

import ctypes

import pytest
import torch

from _parity import assert_close

pytestmark = pytest.mark.gpu


def _noalloc(L, q, X, w, A, B, scale, Y, T):
    st = w.c_struct()
    return L.qlora_linear_forward_noalloc(X.data_ptr(), X.shape[0], ctypes.byref(st),
                                          A.data_ptr(), B.data_ptr(), A.shape[0], float(scale),
                                          Y.data_ptr(), T.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)


def test_noalloc_forward_matches_workspace_forward_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as q
    q.lib()
    L = ctypes.CDLL(q._lib.LIB_PATH)
    vp = ctypes.c_void_p
    L.qlora_linear_forward_noalloc.argtypes = [vp, ctypes.c_int64, ctypes.POINTER(q._lib._Tensor),
                                               vp, vp, ctypes.c_int, ctypes.c_float, vp, vp, vp]
    L.qlora_linear_forward_noalloc.restype = ctypes.c_int
    gen = torch.Generator(device="cuda").manual_seed(7)
    # two calls in a row: a tensor-core GEMM shape, then a decode GEMV shape
    for (M, N, K, r) in ((200, 264, 320, 16), (4, 512, 1024, 8)):
        W = torch.randn(N, K, device="cuda", generator=gen) * 0.02
        w = q.qlora_quantize(W)
        X = torch.randn(M, K, device="cuda", generator=gen).bfloat16()
        A = (torch.randn(r, K, device="cuda", generator=gen) / K ** 0.5).bfloat16()
        B = (torch.randn(N, r, device="cuda", generator=gen) * 0.01).bfloat16()
        T_ref = torch.empty(M, r, dtype=torch.float32, device="cuda")
        Y_ref = q.qlora_linear_forward(X, w, A, B, 2.0, T_save=T_ref)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(L, q, X, w, A, B, 2.0, Y, T) == 0
        # the kernels' error word of this call, read from the library's array
        word = ctypes.c_int(-1)
        L.qlora_linear_forward_noalloc_error_word.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
        assert L.qlora_linear_forward_noalloc_error_word(
            ctypes.byref(word), torch.cuda.current_stream().cuda_stream) == 0
        torch.cuda.synchronize()
        assert word.value == 0, f"device error word {word.value}"
        assert_close("Y", Y, Y_ref.double().cpu().numpy())
        assert_close("T", T, T_ref.double().cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as q
    L = ctypes.CDLL(q._lib.LIB_PATH)
    vp = ctypes.c_void_p
    L.qlora_linear_forward_noalloc.argtypes = [vp, ctypes.c_int64, ctypes.POINTER(q._lib._Tensor),
                                               vp, vp, ctypes.c_int, ctypes.c_float, vp, vp, vp]
    # 65536 tokens x 16384 x 16384, r = 128 needs far more than 16 MiB; the
    # call must refuse before touching any (fake) pointer.
    t = q._lib._Tensor(0x10000, 0x20000, 0x30000, 16384, 16384)
    fake = 0x40000
    assert L.qlora_linear_forward_noalloc(fake, 65536, ctypes.byref(t), fake, fake, 128, 1.0,
                                          fake, None, None) == q._lib.QLORA_ERR_WORKSPACE
