"""GPU parity of the storage kernels through the C-ABI: packed indices, FP8
scale codes and meta scales bit-exact with the oracle, and the dequantised
bf16 weight bit-exact."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _gpu_store(q, W):
    t = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    if t.dim() == 1:
        t = t.view(1, -1)
    w = q.qlora_quantize(t)
    torch.cuda.synchronize()
    return w


def _compare_store(q, W, numel=None):
    w = _gpu_store(q, W)
    packed, sc, meta = o.quantize(W)
    gp = w.packed.cpu().numpy()
    gs = w.scale_codes.cpu().numpy()
    gm = w.meta_scale.cpu().numpy()
    assert gp.shape == packed.shape and np.array_equal(gp, packed), \
        f"packed differs at {np.flatnonzero(gp != packed)[:10]}"
    assert np.array_equal(gs, sc), f"scale codes differ at {np.flatnonzero(gs != sc)[:10]}"
    assert np.array_equal(gm.view(np.uint32), meta.view(np.uint32)), "meta scales differ"
    # dequantised bf16, bit-exact
    deq = q.qlora_dequantize(w)
    torch.cuda.synchronize()
    bits = deq.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    ref = o.dequantize_bits(packed, sc, meta, W.size)
    assert np.array_equal(bits, ref), f"dequant differs at {np.flatnonzero(bits != ref)[:10]}"
    return w


def test_single_layer_weight(q):
    lin = syn.WORKLOADS["single_256x512_m64_r8"].layers[0]
    W = syn.make_weight(lin, np.random.default_rng(lin.seed))
    _compare_store(q, W)


@pytest.mark.parametrize("shape", [(3, 100), (1, 37), (1, 64), (2, 64 * 256 * 2 + 70),
                                   (17, 1000), (64, 64 * 5)])
def test_ragged_shapes(q, shape):
    rng = np.random.default_rng(sum(shape))
    W = rng.normal(0, 0.02, shape).astype(np.float32)
    _compare_store(q, W)


def test_edge_values(q):
    """Zero blocks, an all-zero group, exact midpoint ties, tiny scale ratios
    (subnormal FP8 codes) and sign patterns."""
    codes, mids = o.nf4_codebook()
    nblk = 256 * 3
    W = np.random.default_rng(11).normal(0, 0.02, (nblk, 64)).astype(np.float32)
    W[3] = 0.0                                       # zero block
    W[256:512] = 0.0                                 # all-zero group
    W[600, 0] = 1.0                                  # absmax 1: x = w exactly
    W[600, 1:16] = mids                              # ties at every midpoint
    W[600, 16:31] = np.nextafter(mids, np.float32(2))
    W[600, 31:46] = np.nextafter(mids, np.float32(-2))
    W[601] = np.float32(-0.5) * codes[np.arange(64) % 16]
    W[700, 5] = 300.0                                # one huge block in the group
    W[701:703] *= np.float32(0.1)                    # subnormal E4M3 scale codes
    W[703:705] *= np.float32(1e-3)                   # scale codes that round to zero
    W[705] = np.float32(1e-30)                       # near-underflow block
    _compare_store(q, W.reshape(-1))


def test_attn_projection_full(q):
    lin = syn.WORKLOADS["llama7b_attn_proj_4096x4096_m4096_r16"].layers[0]
    W = syn.make_weight(lin, np.random.default_rng(lin.seed))
    _compare_store(q, W)


@pytest.mark.parametrize("workload", ["decode_gemv_28672x8192_m1", "decode_gemv_8192x28672_m1"])
def test_decode_weights_in_full(q, workload):
    """Both decode weights (235 M parameters each) quantised and dequantised
    on the GPU and compared with the oracle in full: SHA-256 digests of every
    packed byte, scale code, meta scale and dequantised bf16, the oracle run
    in a spawned process."""
    import _oracle_pool as op
    lin = syn.WORKLOADS[workload].layers[0]
    with op.pool(1) as px:
        want = px.submit(op.oracle_storage_digests, lin)
        W = syn.make_weight(lin, np.random.default_rng(lin.seed))
        w = _gpu_store(q, W)
        deq = q.qlora_dequantize(w)
        got = op.gpu_storage_digests(w, deq)
        assert got == want.result()


def test_nonfinite_status_from_the_c_call(q):
    """The C entry point itself returns QLORA_ERR_NONFINITE when the caller
    passes a flag (it synchronises the stream); without a flag it returns
    QLORA_OK at once and checks nothing."""
    import ctypes
    L = q._lib.lib()
    W = torch.ones(4, 128, device="cuda")
    W[1, 70] = float("-inf")
    w = q._lib.empty_nf4(4, 128)
    st = w.c_struct()
    flag = torch.full((1,), 123, dtype=torch.int32, device="cuda")   # stale value: cleared
    s = torch.cuda.current_stream().cuda_stream
    assert L.qlora_quantize(W.data_ptr(), ctypes.byref(st), flag.data_ptr(), s) == \
        q._lib.QLORA_ERR_NONFINITE
    assert L.qlora_quantize(W.data_ptr(), ctypes.byref(st), None, s) == q._lib.QLORA_OK
    W[1, 70] = 2.0
    flag.fill_(123)
    assert L.qlora_quantize(W.data_ptr(), ctypes.byref(st), flag.data_ptr(), s) == q._lib.QLORA_OK
    assert flag.item() == 0
    Wb = W.bfloat16()
    Wb[3, 3] = float("nan")
    assert L.qlora_quantize_bf16(Wb.data_ptr(), ctypes.byref(st), flag.data_ptr(), s) == \
        q._lib.QLORA_ERR_NONFINITE


def test_nonfinite_is_reported(q):
    W = torch.ones(4, 128, device="cuda")
    W[2, 5] = float("nan")
    with pytest.raises(q.QloraError) as ei:
        q.qlora_quantize(W)
    assert ei.value.status == q._lib.QLORA_ERR_NONFINITE
    W[2, 5] = float("inf")
    with pytest.raises(q.QloraError):
        q.qlora_quantize(W)
    q.qlora_quantize(torch.ones(4, 128, device="cuda"))      # finite: no error


def _digests(w):
    return [t.cpu().numpy().tobytes() for t in (w.packed, w.scale_codes, w.meta_scale)]


@pytest.mark.parametrize("bf16", [False, True])
def test_quantize_many_equals_one_by_one(q, bf16):
    """qlora_quantize_many over 18 weights (two launches of at most 16; ragged
    last groups and blocks; one empty weight): every stored byte equals the
    single call's for that weight, fp32 and bf16 inputs alike."""
    rng = np.random.default_rng(31 + bf16)
    shapes = [(64, 256 * 64), (3, 100), (1024, 4096), (17, 1000), (2, 64 * 256 * 2 + 70),
              (256, 512), (1, 64), (4096, 96)] * 2 + [(512, 1024)]
    Ws = []
    for r, c in shapes:
        W = torch.from_numpy((rng.standard_normal((r, c)) * 0.02).astype(np.float32)).cuda()
        W.view(-1)[:64] = 0.0                          # a zero block
        Ws.append(W.bfloat16() if bf16 else W)
    Ws.append(Ws[0][:0])                               # empty: torch gives it a NULL pointer
    many = q.qlora_quantize_many([(W, None) for W in Ws])
    torch.cuda.synchronize()
    assert many[-1].packed.numel() == 0
    for i, (W, w) in enumerate(zip(Ws[:-1], many)):
        one = q.qlora_quantize_bf16(W) if bf16 else q.qlora_quantize(W)
        torch.cuda.synchronize()
        assert _digests(w) == _digests(one), f"job {i} {tuple(W.shape)}"


def test_quantize_many_nonfinite(q):
    """One non-finite weight among several: the call reports it with
    QLORA_ERR_NONFINITE; without it the same call succeeds."""
    Ws = [torch.ones(64, 512, device="cuda") * 0.01 for _ in range(5)]
    Ws[3][7, 300] = float("inf")
    with pytest.raises(q.QloraError) as ei:
        q.qlora_quantize_many([(W, None) for W in Ws])
    assert ei.value.status == q._lib.QLORA_ERR_NONFINITE
    Ws[3][7, 300] = 0.5
    q.qlora_quantize_many([(W, None) for W in Ws])
