"""GPU parity of the merge for export (qlora_merge) and of the re-quantisation
of a bf16 weight (qlora_quantize_bf16) against the oracle, through the C-ABI.

Merge tolerance.  The library forms W~ + gamma B A in fp32 (B A accumulated
on the tensor cores from exact bf16 products, then one fused multiply-add
with W~) and rounds once to bf16; the oracle forms it exactly (fp64) and
rounds once.  With S = |gamma| sum_j |B_nj A_jk|, the fp32 value is within
e = (2r + 4) 2^-24 (|w~| + S) of the exact one (r additions that lose at most
one fp32 unit each, the rounding of the fused multiply-add, and margin), so
each output must lie between the bf16 roundings of exact - e and exact + e.
Those two coincide for almost every element, which makes the check
bit-exact there; the test also reports how many elements match the oracle's
bits outright.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

from _parity import groups_of_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_merge_close(name, got: torch.Tensor, exact, Wt, A, B, gamma, r,
                       min_exact_frac=0.99) -> float:
    g_bits = got.view(torch.int16).cpu().numpy().view(np.uint16)
    g = _bits_to_f64(g_bits)
    S = abs(float(np.float32(gamma))) * (np.abs(B) @ np.abs(A))
    e = (2 * r + 4) * 2.0 ** -24 * (np.abs(Wt) + S)
    lo = _bits_to_f64(o.bf16_rne_f64(exact - e))
    hi = _bits_to_f64(o.bf16_rne_f64(exact + e))
    bad = ~((g >= lo) & (g <= hi))
    assert not bad.any(), (f"{name}: {int(bad.sum())} elements outside one rounding of the exact "
                           f"merge, first at {np.argwhere(bad)[0].tolist()}")
    same = float(np.mean(g == _bits_to_f64(o.bf16_rne_f64(exact))))
    assert same >= min_exact_frac, f"{name}: only {same:.5f} of elements match the oracle's bits"
    return same


def _layer(N, K, r, seed, alpha=32.0, b_scale=1.0):
    lin = syn.Linear(f"merge_{N}x{K}_r{r}", 1, N, K, r, alpha, 0.02, seed % 2 == 1, seed)
    d = syn.make_layer(lin, with_grad=False)
    if b_scale != 1.0:
        d["B"] = syn.to_bf16(syn.as_f64(d["B"]).astype(np.float32) * np.float32(b_scale))
    return lin, d


CASES = [
    # (N, K, r, seed, b_scale)
    (16, 64, 8, 1, 1.0),           # one warp tile
    (8, 128, 16, 2, 1.0),          # fewer rows than a tile
    (40, 768, 24, 3, 1.0),         # ragged rows (40 = 2.5 tiles), r % 16 == 8
    (1000, 2304, 16, 4, 1.0),      # N % 16 == 8, many strips per warp
    (256, 4352, 128, 5, 1.0),      # largest rank
    (24, 512, 64, 6, 30.0),        # adapter as large as the base: cancellation
    (513 * 8, 1024, 32, 7, 1.0),   # several warps share a strip
]


@pytest.mark.parametrize("N,K,r,seed,b_scale", CASES)
def test_merge_matches_oracle(q, N, K, r, seed, b_scale):
    lin, d = _layer(N, K, r, seed, b_scale=b_scale)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    A, B = d["A"].cuda(), d["B"].cuda()
    got = q.qlora_merge(w, A, B, lin.gamma)
    torch.cuda.synchronize()
    p, s, m = o.quantize(d["W"])
    A64, B64 = syn.as_f64(d["A"]), syn.as_f64(d["B"])
    exact, _ = o.merge(p, s, m, N, K, A64, B64, lin.gamma)
    Wt = o.dequantize(p, s, m, N, K)
    assert_merge_close(lin.name, got, exact, Wt, A64, B64, lin.gamma, r)


def test_merge_full_attention_projection(q):
    """The whole 4096 x 4096 weight of the attention-projection workload
    (r = 16, gamma = 2), every element against the oracle."""
    lin = syn.WORKLOADS["llama7b_attn_proj_4096x4096_m4096_r16"].layers[0]
    d = syn.make_layer(lin, with_grad=False)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    got = q.qlora_merge(w, d["A"].cuda(), d["B"].cuda(), lin.gamma)
    torch.cuda.synchronize()
    p, s, m = o.quantize(d["W"])
    A64, B64 = syn.as_f64(d["A"]), syn.as_f64(d["B"])
    exact, _ = o.merge(p, s, m, lin.N, lin.K, A64, B64, lin.gamma)
    Wt = o.dequantize(p, s, m, lin.N, lin.K)
    frac = assert_merge_close(lin.name, got, exact, Wt, A64, B64, lin.gamma, lin.r)
    print(f"merge 4096x4096: {frac:.6f} of elements bit-equal to the oracle")


def test_merge_decoder_mlp_sampled_rows(q):
    """An 11008 x 4096 MLP weight of the decoder workload; the oracle quantises
    only whole double-quantisation groups around sampled rows."""
    lin = [l for l in syn.WORKLOADS["llama7b_decoder_32layers_m4096_r16"].layers
           if l.name == "layer5.gate"][0]
    d = syn.make_layer(lin, with_grad=False)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    got = q.qlora_merge(w, d["A"].cuda(), d["B"].cuda(), lin.gamma).cpu()
    A64, B64 = syn.as_f64(d["A"]), syn.as_f64(d["B"])
    rows = sorted(set([0, 1, lin.N - 1] + np.random.default_rng(3).integers(0, lin.N, 24).tolist()))
    flat = d["W"].reshape(-1)
    for (e0, e1), row in zip(groups_of_rows(rows, lin.K), rows):
        p, s, m = o.quantize(flat[e0:e1])
        r0 = e0 // lin.K
        nr = (e1 - e0) // lin.K
        exact, _ = o.merge(p, s, m, nr, lin.K, A64, B64[r0:r0 + nr], lin.gamma)
        Wt = o.dequantize(p, s, m, nr, lin.K)
        i = row - r0
        assert_merge_close(f"{lin.name} row {row}", got[row:row + 1], exact[i:i + 1],
                           Wt[i:i + 1], A64, B64[row:row + 1], lin.gamma, lin.r, 0.98)


@pytest.mark.parametrize("zero", ["B", "gamma"])
def test_merge_without_adapter_is_dequantize(q, zero):
    lin, d = _layer(520, 1024, 16, 8)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    B = torch.zeros_like(d["B"]).cuda() if zero == "B" else d["B"].cuda()
    gamma = 0.0 if zero == "gamma" else lin.gamma
    got = q.qlora_merge(w, d["A"].cuda(), B, gamma).float().cpu().numpy()
    p, s, m = o.quantize(d["W"])
    ref = o.dequantize(p, s, m, lin.N, lin.K)
    assert np.array_equal(got, ref)            # values: -0 and +0 compare equal


def test_merge_stream_and_empty(q):
    lin, d = _layer(64, 256, 8, 9)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = q.qlora_merge(w, d["A"].cuda(), d["B"].cuda(), lin.gamma, stream=s)
    s.synchronize()
    ref = q.qlora_merge(w, d["A"].cuda(), d["B"].cuda(), lin.gamma)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    e = q.empty_nf4(0, 256)
    out = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    q.qlora_merge(e, d["A"].cuda(), d["B"].cuda()[:0], lin.gamma, out=out)


def test_merge_many_equals_one_by_one(q):
    """qlora_merge_many over 21 weights of different shapes and ranks (two
    launches of at most 16, one empty weight among them): every output equals
    qlora_merge's for that weight bit for bit, and qlora_merge is checked
    against the oracle above."""
    shapes = [CASES[i % len(CASES)][:3] for i in range(20)] + [(4096, 1024, 16)]
    jobs, singles = [], []
    for i, (N, K, r) in enumerate(shapes):
        lin, d = _layer(N, K, r, 100 + i)
        w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
        A, B = d["A"].cuda(), d["B"].cuda()
        jobs.append((w, A, B, lin.gamma, None))
        singles.append(q.qlora_merge(w, A, B, lin.gamma))
    e = q.empty_nf4(0, 256)
    jobs.insert(7, (e, jobs[0][1][:, :256].contiguous(), jobs[0][2][:0], 2.0,
                    torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")))
    outs = q.qlora_merge_many(jobs)
    torch.cuda.synchronize()
    outs.pop(7)
    assert len(outs) == len(singles)
    for i, (got, ref) in enumerate(zip(outs, singles)):
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"job {i} {shapes[i]}"


@pytest.mark.parametrize("N,K,seed", [(4096, 4096, 11), (40, 768, 12), (3, 100, 13), (1, 1, 14)])
def test_quantize_bf16_matches_oracle(q, N, K, seed):
    """Re-quantisation of a bf16 weight: bit-exact with the oracle's quantiser
    on the same values, including a partial final group and block."""
    rng = np.random.default_rng(seed)
    Wb = syn.to_bf16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    w = q.qlora_quantize_bf16(Wb.cuda())
    torch.cuda.synchronize()
    p, s, m = o.quantize(syn.as_f64(Wb).astype(np.float32))
    assert np.array_equal(w.packed.cpu().numpy(), p)
    assert np.array_equal(w.scale_codes.cpu().numpy(), s)
    assert np.array_equal(w.meta_scale.cpu().numpy().view(np.uint32), m.view(np.uint32))


def test_requantise_the_oracle_merge(q):
    """The export chain's second step on the oracle's merged weight: the
    library's bf16 quantiser reproduces the oracle's quantisation of it."""
    lin, d = _layer(512, 2048, 16, 15)
    p, s, m = o.quantize(d["W"])
    _, bits = o.merge(p, s, m, lin.N, lin.K, syn.as_f64(d["A"]), syn.as_f64(d["B"]), lin.gamma)
    Wm = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    w2 = q.qlora_quantize_bf16(Wm.cuda())
    torch.cuda.synchronize()
    p2, s2, m2 = o.quantize(_bits_to_f64(bits).astype(np.float32))
    assert np.array_equal(w2.packed.cpu().numpy(), p2)
    assert np.array_equal(w2.scale_codes.cpu().numpy(), s2)
    assert np.array_equal(w2.meta_scale.cpu().numpy().view(np.uint32), m2.view(np.uint32))
