"""Pins for the CPU oracle (CPU only, no GPU, no CUDA library).

Each test ties an oracle function to something other than the oracle itself:
values the pages print (fixtures under tests/golden/, each citing its source),
closed forms, independent library routines (stdlib/scipy quantiles, torch's
float8 and bf16 casts), brute force on tiny inputs and finite differences.
"""
from __future__ import annotations

import math
import os
import statistics

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _golden_table(name):
    out = {}
    for ln in _golden_lines(name):
        k, v, tol = ln.split()
        out[k] = (float(v), float(tol))
    return out


# --------------------------------------------------------------------------
# Codebook
# --------------------------------------------------------------------------
def test_codebook_matches_printed_digits():
    codes, _ = o.nf4_codebook()
    for ln in _golden_lines("nf4_printed_codes.txt"):
        i, v = ln.split()
        assert abs(float(codes[int(i)]) - float(v)) <= 5e-5, (i, codes[int(i)], v)


def test_codebook_structure():
    codes, mids = o.nf4_codebook()
    assert codes.dtype == np.float32 and codes.shape == (16,)
    assert np.all(np.diff(codes) > 0)
    assert codes[7] == 0.0 and codes[0] == -1.0 and codes[15] == 1.0
    # 8 levels on the negative side and 9 on the positive side, sharing zero
    assert (codes < 0).sum() == 7 and (codes > 0).sum() == 8
    assert mids.shape == (15,)
    assert np.all(mids > codes[:-1]) and np.all(mids < codes[1:])


@pytest.mark.parametrize("ppf", [statistics.NormalDist().inv_cdf,
                                 pytest.importorskip("scipy.special").ndtri])
def test_codebook_independent_quantile_routines(ppf):
    ours = o.nf4_codebook()[0]
    theirs = o.nf4_levels_fp64(ppf=lambda p: float(ppf(p))).astype(np.float32)
    assert np.array_equal(ours.view(np.uint32), theirs.view(np.uint32))


def test_norm_ppf_closed_forms():
    assert o.norm_ppf(0.5) == pytest.approx(0.0, abs=1e-15)
    # Phi(1.959963984540054) = 0.975 (textbook value)
    assert o.norm_ppf(0.975) == pytest.approx(1.959963984540054, abs=1e-13)
    assert o.norm_ppf(0.025) == pytest.approx(-1.959963984540054, abs=1e-13)


def test_codebook_alternative_offsets_fail_printed_digits():
    """The offset reading is pinned: the two single-sided offsets miss."""
    printed = {int(a): float(b) for a, b in (ln.split() for ln in _golden_lines("nf4_printed_codes.txt"))}
    for delta in (1 - 1 / 30, 1 - 1 / 32):
        pos = [o.norm_ppf(delta - i * (delta - 0.5) / 8) for i in range(8)]
        neg = [-o.norm_ppf(delta - j * (delta - 0.5) / 7) for j in range(7)]
        lv = np.array(sorted(neg + [0.0] + pos)) / o.norm_ppf(delta)
        assert max(abs(lv[i] - v) for i, v in printed.items()) > 5e-5


def test_midpoints_are_rounded_exact_averages():
    codes, mids = o.nf4_codebook()
    for i in range(15):
        exact = (float(codes[i]) + float(codes[i + 1])) / 2
        m = float(mids[i])
        below = float(np.nextafter(mids[i], np.float32(-2)))
        above = float(np.nextafter(mids[i], np.float32(2)))
        assert abs(m - exact) <= abs(below - exact) and abs(m - exact) <= abs(above - exact)


# --------------------------------------------------------------------------
# Blockwise quantisation
# --------------------------------------------------------------------------
def _worked():
    d = {}
    for ln in _golden_lines("worked_example_block8.txt"):
        k, v = ln.split(":")
        d[k] = [float(t) for t in v.split()]
    return d


def test_worked_example_block_of_eight():
    d = _worked()
    codes, mids = o.nf4_codebook()
    w = np.array(d["weights"], dtype=np.float32)
    c = o.block_absmax(w, block=8)
    assert c.shape == (1,) and abs(c[0] - d["absmax"][0]) < 1e-7
    x = o.normalise_blocks(w, c, block=8)
    assert np.allclose(x, d["normalised"], atol=5e-4)
    idx = o.nearest_code_index(x, mids)
    assert idx.tolist() == [int(v) for v in d["indices"]]
    rec = codes[idx] * c[0]
    assert np.allclose(rec, d["reconstructed"], atol=5e-5)
    assert np.allclose(np.abs(rec - w), d["abs_error"], atol=5e-5)
    assert rec[3] == w[3]        # the absmax element is reconstructed exactly


def test_nearest_index_agrees_with_brute_force():
    rng = np.random.default_rng(1)
    codes, mids = o.nf4_codebook()
    x = rng.uniform(-1, 1, 20000).astype(np.float32)
    x = np.concatenate([x, codes, -np.abs(codes)])
    fast = o.nearest_code_index(x, mids)
    brute = o.brute_nearest_index(x, codes)
    on_mid = np.isin(x, mids)
    assert np.array_equal(fast[~on_mid], brute[~on_mid])


def test_tie_rule_goes_to_lower_code():
    codes, mids = o.nf4_codebook()
    for i, m in enumerate(mids):
        assert o.nearest_code_index(np.array([m]), mids)[0] == i
        up = np.nextafter(m, np.float32(2))
        dn = np.nextafter(m, np.float32(-2))
        assert o.nearest_code_index(np.array([up]), mids)[0] == i + 1
        assert o.nearest_code_index(np.array([dn]), mids)[0] == i


def test_roundtrip_of_exact_codes():
    """Blocks made of codes times a power of two, each holding a +-1, quantise
    back to the very indices they were built from."""
    rng = np.random.default_rng(2)
    codes, mids = o.nf4_codebook()
    idx = rng.integers(0, 16, size=(40, 64)).astype(np.uint8)
    idx[:, 5] = np.where(rng.random(40) < 0.5, 0, 15)
    scale = (2.0 ** rng.integers(-20, 5, size=(40, 1))).astype(np.float32)
    w = (codes[idx] * scale).astype(np.float32)
    packed, _, _ = o.quantize(w)
    got = o.unpack_nibbles(packed, w.size).reshape(40, 64)
    assert np.array_equal(got, idx)


def test_error_bound_half_local_gap():
    rng = np.random.default_rng(3)
    codes, mids = o.nf4_codebook()
    w = rng.normal(0, 0.02, 64 * 500).astype(np.float32)
    c = o.block_absmax(w)
    x = o.normalise_blocks(w, c)
    idx = o.nearest_code_index(x, mids)
    q = codes[idx].astype(np.float64)
    lo = codes[np.maximum(idx.astype(int) - 1, 0)]
    hi = codes[np.minimum(idx.astype(int) + 1, 15)]
    gap = np.maximum(q - lo, hi - q)
    ulp = np.spacing(np.abs(x).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(x - q) <= 0.5 * gap + ulp)
    err = np.abs(w.astype(np.float64) - q * np.repeat(c, 64))
    assert np.all(err <= (0.5 * gap + 2 * ulp) * np.repeat(c, 64))


def test_pack_nibble_order_and_padding():
    idx = np.array([1, 2, 3, 4, 15, 0, 9], dtype=np.uint8)
    p = o.pack_nibbles(idx)
    assert p.tolist() == [0x21, 0x43, 0x0F, 0x79]
    assert o.unpack_nibbles(p, 7).tolist() == idx.tolist()


def test_zero_block_and_partial_tail():
    w = np.zeros(64 * 3 + 10, dtype=np.float32)
    w[64:128] = np.linspace(-1, 1, 64, dtype=np.float32)
    w[-3] = 0.5
    packed, sc, meta = o.quantize(w)
    nb, ng = 4, 1
    assert packed.size == nb * 32 and sc.size == nb and meta.size == ng
    idx = o.unpack_nibbles(packed, nb * 64)
    assert np.all(idx[:64] == 7)                       # zero block -> zero code
    assert np.all(idx[192 + 10:] == 7)                 # padding -> zero code
    deq = o.bf16_bits_to_float(o.dequantize_bits(packed, sc, meta, w.size))
    assert np.all(deq[:64] == 0)
    assert deq[-3] > 0


def test_all_zero_tensor():
    packed, sc, meta = o.quantize(np.zeros((4, 64), np.float32))
    assert np.all(packed == 0x77) and np.all(sc == 0) and np.all(meta == 0)


def test_nonfinite_rejected():
    w = np.ones(128, np.float32)
    for bad in (np.nan, np.inf, -np.inf):
        w2 = w.copy()
        w2[7] = bad
        with pytest.raises(o.NonFiniteWeight):
            o.quantize(w2)


def test_quantize_against_per_element_loop():
    """Brute force on a tiny tensor, one element at a time in plain Python."""
    rng = np.random.default_rng(4)
    codes, _ = o.nf4_codebook()
    w = rng.normal(0, 0.02, (3, 128)).astype(np.float32)
    w[1, 7] *= 10
    packed, _, _ = o.quantize(w)
    flat = w.reshape(-1)
    got = o.unpack_nibbles(packed, flat.size)
    for b in range(flat.size // 64):
        blk = flat[b * 64:(b + 1) * 64]
        c = max(abs(float(v)) for v in blk)
        for j, v in enumerate(blk):
            xv = float(np.float32(v) / np.float32(c))
            dist = [abs(xv - float(q)) for q in codes]
            best = min(range(16), key=lambda i: (dist[i], i))
            assert got[b * 64 + j] == best


# --------------------------------------------------------------------------
# FP8 scales and bf16
# --------------------------------------------------------------------------
def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        o.e4m3_value_table().astype(np.float32),
        ((o.e4m3_value_table()[:-1] + o.e4m3_value_table()[1:]) / 2).astype(np.float32),
        rng.uniform(0, 464, 3000).astype(np.float32),
        (2.0 ** rng.uniform(-12, -5, 1000)).astype(np.float32),
        np.array([0.0, 2 ** -10, 3 * 2 ** -10, 448.0, 460.0, 464.0], np.float32),
    ])
    ours = o.e4m3_encode(vals)
    theirs = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)
    assert o.e4m3_encode(np.array([465.0, 1e30], np.float32)).tolist() == [0x7E, 0x7E]


def _e4m3_probe_values(n_random):
    """Every E4M3 value, every midpoint between neighbours and its two fp32
    neighbours, values above the top code, and random values over the whole
    range (uniform and log-uniform)."""
    rng = np.random.default_rng(11)
    tab = o.e4m3_value_table()
    mids = ((tab[:-1] + tab[1:]) / 2).astype(np.float32)
    return np.concatenate([
        tab.astype(np.float32), mids,
        np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
        np.array([448.0, 455.9, 460.0, 464.0, 1e3, 1e30], np.float32),
        rng.uniform(0, 464, n_random // 2).astype(np.float32),
        (2.0 ** rng.uniform(-16, 8.8, n_random // 2)).astype(np.float32),
    ])


def test_e4m3_encode_sorted_equals_enumeration():
    vals = _e4m3_probe_values(200_000)
    assert np.array_equal(o.e4m3_encode_sorted(vals), o.e4m3_encode(vals))


def test_e4m3_encode_sorted_matches_torch_cast():
    vals = _e4m3_probe_values(2_000_000)
    vals = vals[vals <= 464.0]                      # torch's cast saturates only up to there
    ours = o.e4m3_encode_sorted(vals)
    theirs = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert vals.size > 1_000_000 and np.array_equal(ours, theirs)
    assert o.e4m3_encode_sorted(np.array([465.0, 1e30], np.float32)).tolist() == [0x7E, 0x7E]
    with pytest.raises(ValueError):
        o.e4m3_encode_sorted(np.array([-1.0], np.float32))


def test_double_quantize_matches_per_group_enumeration():
    """The whole-array double quantisation equals the group-by-group one with
    the enumerating encoder (all-zero groups, a partial last group)."""
    rng = np.random.default_rng(12)
    c = np.abs(rng.standard_normal(256 * 9 + 77)).astype(np.float32) * np.float32(0.05)
    c[256:512] = 0.0
    c[600] = 0.0
    sc, meta = o.double_quantize(c)
    ngroups = -(-c.size // 256)
    for g in range(ngroups):
        part = c[g * 256:(g + 1) * 256]
        m = np.float32(part.max() / np.float32(448.0))
        assert meta[g] == m
        want = (o.e4m3_encode((part / m).astype(np.float32)) if m > 0
                else np.zeros(part.size, np.uint8))
        assert np.array_equal(sc[g * 256:g * 256 + part.size], want)


def _e5m2_probe_values(n_random):
    rng = np.random.default_rng(13)
    tab = o.e5m2_value_table()
    mids = ((tab[:-1] + tab[1:]) / 2).astype(np.float32)
    return np.concatenate([
        tab.astype(np.float32), mids,
        np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
        np.array([57344.0, 60000.0, 61439.0], np.float32),
        rng.uniform(0, 61000, n_random // 2).astype(np.float32),
        (2.0 ** rng.uniform(-18, 15.8, n_random // 2)).astype(np.float32),
    ])


def test_e5m2_encode_matches_torch_cast():
    """The E5M2 scale code is torch's float8_e5m2 cast (round to nearest,
    ties to even) wherever that cast is finite; above, it saturates."""
    vals = _e5m2_probe_values(1_000_000)
    vals = vals[vals < 61440.0]                # torch's cast overflows to inf from here
    ours = o.e5m2_encode(vals)
    theirs = torch.from_numpy(vals).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert vals.size > 500_000 and np.array_equal(ours, theirs)
    assert o.e5m2_encode(np.array([61440.0, 1e30], np.float32)).tolist() == [0x7B, 0x7B]


def test_e5m2_decode_matches_torch():
    c = np.arange(0x7C, dtype=np.uint8)
    theirs = torch.from_numpy(c).view(torch.float8_e5m2).to(torch.float32).numpy()
    assert np.array_equal(o.e5m2_decode(c), theirs)
    assert o.e5m2_decode(np.array([0x7B], np.uint8))[0] == 57344.0


def test_u8_scale_code_is_the_nearest_level():
    """Linear 8-bit scale codes: the group's largest scale takes 255, every
    dequantised scale lies within half a step (plus fp32 rounding) of the
    true one, no other of the 256 levels is nearer, and scales that are
    exact multiples of the step come back exactly."""
    rng = np.random.default_rng(14)
    c = np.abs(rng.standard_normal(256 * 40)).astype(np.float32) * np.float32(0.03)
    c[256 * 3:256 * 4] = 0.0                                   # an all-zero group
    step = np.float32(0.001)
    c[256 * 5:256 * 6] = (np.arange(256) % 256).astype(np.float32) * step
    c[256 * 5 + 255] = np.float32(255) * step                  # the group max
    sc, meta = o.double_quantize(c, fmt="u8")
    g = np.arange(c.size) // 256
    for k in range(40):
        part = c[k * 256:(k + 1) * 256]
        if part.max() > 0:
            assert sc[k * 256 + int(np.argmax(part))] == 255
    ct = o.dequantize_scales(sc, meta, fmt="u8").astype(np.float64)
    c2 = meta[g].astype(np.float64)
    err = np.abs(ct - c.astype(np.float64))
    slack = ct * 2.0 ** -23 + c2 * 2.0 ** -18           # fp32 roundings of c / c2 and code * c2
    assert np.all(err <= c2 * 0.5 + slack + 1e-30)
    levels = np.arange(256)[None, :] * c2[:, None]
    best = np.abs(levels - c.astype(np.float64)[:, None]).min(axis=1)
    assert np.all(err <= best + slack + 1e-30)
    exact = slice(256 * 5, 256 * 6)
    assert np.array_equal(sc[exact], np.arange(256, dtype=np.uint8))


def test_scale_formats_cost_on_the_toy():
    """The page's toy (2^20 N(0, 0.02^2) weights, NF4, blocks of 64): fp32
    scales give the printed 0.845 %; a linear 8-bit code of the scales adds
    almost nothing, E4M3 about 0.08 points, E5M2 (two mantissa bits) more
    again; every 8-bit format stays within its scale step of fp32."""
    rng = np.random.default_rng(0)
    w = (rng.standard_normal(2 ** 20) * 0.02).astype(np.float32)
    codes, _ = o.nf4_codebook()
    rel = {}
    for fmt in ("fp32", "u8", "e4m3", "e5m2"):
        p, s_, m = o.quantize_fmt(w, codes, 64, fmt)
        rec = o.bf16_bits_to_float(o.dequantize_fmt_bits(p, s_, m, w.size, codes, 64, fmt))
        rel[fmt] = float(np.sum((rec.astype(np.float64) - w) ** 2) / np.sum(w.astype(np.float64) ** 2))
    assert abs(rel["fp32"] - 0.00845) < 0.00002
    assert rel["fp32"] < rel["u8"] < rel["fp32"] + 0.00002
    assert rel["u8"] < rel["e4m3"] < rel["e5m2"]
    assert 0.0090 < rel["e4m3"] < 0.0095 and 0.0110 < rel["e5m2"] < 0.0120


def test_e4m3_decode_matches_torch():
    c = np.arange(127, dtype=np.uint8)
    theirs = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(o.e4m3_decode(c), theirs)
    assert o.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-30, 100),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]]).astype(np.float32)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.bf16_bits(x), theirs)


def test_double_quant_properties():
    rng = np.random.default_rng(7)
    c = np.abs(rng.normal(0, 0.05, 1000)).astype(np.float32)
    c[512:768] = 0                                    # one all-zero group
    codes, meta = o.double_quantize(c)
    assert codes.size == 1000 and meta.size == 4
    ct = o.dequantize_scales(codes, meta)
    g = np.arange(1000) // 256
    for gi in range(4):
        sel = g == gi
        if meta[gi] == 0:
            assert np.all(codes[sel] == 0) and np.all(ct[sel] == 0)
            continue
        big = c[sel] >= meta[gi] * 2 ** -6           # normal E4M3 range
        rel = np.abs(ct[sel][big] - c[sel][big]) / c[sel][big]
        assert np.all(rel <= 2 ** -4 + 1e-6)
        assert codes[sel].max() == 0x7E               # the group max maps to 448
    assert meta[0] == np.float32(c[:256].max()) / np.float32(448)


def test_dequantize_bits_against_per_element_torch():
    rng = np.random.default_rng(8)
    w = rng.normal(0, 0.02, (2, 256)).astype(np.float32)
    packed, sc, meta = o.quantize(w)
    codes, _ = o.nf4_codebook()
    bits = o.dequantize_bits(packed, sc, meta, w.size)
    idx = o.unpack_nibbles(packed, w.size)
    for e in range(w.size):
        b = e // 64
        cdec = torch.tensor([int(sc[b])], dtype=torch.uint8).view(torch.float8_e4m3fn).float()
        ct = (cdec * torch.tensor([float(meta[b // 256])], dtype=torch.float32))
        v = (torch.tensor([float(codes[idx[e]])], dtype=torch.float32) * ct).to(torch.bfloat16)
        assert int(v.view(torch.int16).item()) & 0xFFFF == int(bits[e])


def test_storage_closed_forms():
    t = _golden_table("toy_statistics.txt")
    assert o.storage_bits_per_param() == 4.126953125
    assert abs(o.storage_bits_per_param() - t["bits_b64_dq"][0]) <= t["bits_b64_dq"][1]
    assert abs(o.storage_bits_per_param(16) - t["bits_b16_dq"][0]) <= t["bits_b16_dq"][1]
    assert o.storage_bits_per_param(16, double_quant=False) == t["bits_b16_nodq"][0]
    saving = o.storage_bits_per_param(64, double_quant=False) - o.storage_bits_per_param()
    assert abs(saving - t["dq_saving_b64"][0]) <= t["dq_saving_b64"][1]
    for n, k in ((4096, 4096), (11008, 4096), (28672, 8192)):
        p, s, m = o.quantized_nbytes(n * k)
        assert p + s + m == n * k // 2 + n * k // 64 + 4 * math.ceil(n * k / 16384)
        assert 8 * (p + s + m) / (n * k) == pytest.approx(4.126953125, abs=1e-4)


# --------------------------------------------------------------------------
# The page's toy statistics
# --------------------------------------------------------------------------
def _relmse(w, cb, B):
    r = o.single_quant_roundtrip(w, cb, B).astype(np.float64)
    return 100 * np.mean((r - w) ** 2) / np.mean(w.astype(np.float64) ** 2)


def test_toy_statistics_reproduce():
    t = _golden_table("toy_statistics.txt")
    rng = np.random.default_rng(0)
    w = rng.normal(0, 0.02, 2 ** 20).astype(np.float32)
    nf4, _ = o.nf4_codebook()
    fp4, int4 = o.fp4_e2m1_codebook(), o.int4_codebook()
    got = {
        "gauss_nf4_b64": _relmse(w, nf4, 64),
        "gauss_fp4_b64": _relmse(w, fp4, 64),
        "gauss_int4_b64": _relmse(w, int4, 64),
        "gauss_nf4_b16": _relmse(w, nf4, 16),
        "gauss_nf4_b4096": _relmse(w, nf4, 4096),
    }
    got["sqnr_nf4_db"] = 10 * math.log10(100 / got["gauss_nf4_b64"])
    got["sqnr_fp4_db"] = 10 * math.log10(100 / got["gauss_fp4_b64"])
    got["sqnr_int4_db"] = 10 * math.log10(100 / got["gauss_int4_b64"])
    s = (rng.standard_t(5, 2 ** 20) * 0.02 / math.sqrt(5 / 3)).astype(np.float32)
    got["student5_nf4_b64"] = _relmse(s, nf4, 64)
    got["student5_fp4_b64"] = _relmse(s, fp4, 64)
    got["student5_int4_b64"] = _relmse(s, int4, 64)
    for k, v in got.items():
        ref, tol = t[k]
        assert abs(v - ref) <= tol, (k, v, ref)


def test_residual_is_close_to_full_rank():
    t = _golden_table("toy_statistics.txt")
    nf4, _ = o.nf4_codebook()
    W = np.random.default_rng(0).normal(0, 0.02, (1024, 1024)).astype(np.float32)
    R = (W - o.single_quant_roundtrip(W, nf4, 64).reshape(W.shape)).astype(np.float64)
    e = np.linalg.svd(R, compute_uv=False) ** 2
    for k in (16, 64, 256):
        ref, tol = t[f"residual_rank{k}"]
        assert abs(100 * e[:k].sum() / e.sum() - ref) <= tol


# --------------------------------------------------------------------------
# The adapted linear layer
# --------------------------------------------------------------------------
def _tiny_linear(seed=9, M=3, N=4, K=5, r=2):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(M, K)), rng.normal(size=(N, K)), rng.normal(size=(r, K)),
            rng.normal(size=(N, r)), rng.normal(size=(M, N)), 1.75)


def test_linear_forward_elementwise_loops():
    X, W, A, B, dY, g = _tiny_linear()
    Y, T = o.linear_forward(X, W, A, B, g)
    M, K = X.shape
    N, r = B.shape
    for m in range(M):
        for j in range(r):
            assert T[m, j] == pytest.approx(sum(X[m, k] * A[j, k] for k in range(K)), abs=1e-12)
        for n in range(N):
            base = sum(X[m, k] * W[n, k] for k in range(K))
            lora = sum(sum(X[m, k] * A[j, k] for k in range(K)) * B[n, j] for j in range(r))
            assert Y[m, n] == pytest.approx(base + g * lora, abs=1e-12)


def test_linear_backward_finite_differences():
    """Gradients of L = <dY, Y> by central differences in fp64."""
    X, W, A, B, dY, g = _tiny_linear()
    dX, dA, dB, _ = o.linear_backward(dY, X, W, A, B, g)

    def loss(X_, A_, B_):
        return float(np.sum(dY * o.linear_forward(X_, W, A_, B_, g)[0]))

    h = 1e-6
    for arr, grad, which in ((X, dX, 0), (A, dA, 1), (B, dB, 2)):
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[i] += h
            m[i] -= h
            args_p = [X, A, B]
            args_m = [X, A, B]
            args_p[which], args_m[which] = p, m
            num[i] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.allclose(num, grad, atol=1e-6), which


def test_no_lora_reduces_to_plain_product():
    X, W, A, B, dY, g = _tiny_linear()
    Y, _ = o.linear_forward(X, W, A, np.zeros_like(B), g)
    assert np.allclose(Y, np.einsum("mk,nk->mn", X, W))
    dX, dA, dB, _ = o.linear_backward(dY, X, W, A, np.zeros_like(B), g)
    assert np.allclose(dX, np.einsum("mn,nk->mk", dY, W)) and np.allclose(dA, 0)


# --------------------------------------------------------------------------
# Merge for export
# --------------------------------------------------------------------------
def _all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    keep = np.isfinite(vals)
    return bits[keep], vals[keep]


def _brute_bf16(x, bits, vals):
    """Nearest finite bf16 by exhaustive search, ties to the even bit pattern;
    beyond the overflow threshold (halfway past the largest finite value) an
    infinity."""
    out = np.empty(x.size, np.uint16)
    pos = np.unique(vals[vals > 0])
    top = float(pos[-1])
    thresh = top + (top - float(pos[-2])) / 2
    for i, xi in enumerate(x):
        if abs(xi) >= thresh:
            out[i] = 0x7F80 if xi > 0 else 0xFF80
            continue
        d = np.abs(vals - xi)
        cand = np.flatnonzero(d == d.min())
        # +0 and -0 are both at distance |x| from a tiny x: keep the sign of x
        cand = [c for c in cand if vals[c] != 0 or np.signbit(vals[c]) == np.signbit(xi)] or list(cand)
        even = [c for c in cand if (bits[c] & 1) == 0]
        out[i] = bits[(even or cand)[0]]
    return out


def test_bf16_rne_f64_against_exhaustive_search():
    bits, vals = _all_finite_bf16()
    rng = np.random.default_rng(21)
    pos = np.unique(vals[vals > 0])
    lo = pos[rng.integers(0, pos.size - 1, 300)]
    hi = np.array([pos[np.searchsorted(pos, v) + 1] for v in lo])
    ties = (lo + hi) / 2                                     # exact in fp64
    x = np.concatenate([
        rng.standard_normal(400) * np.exp(rng.uniform(-60, 60, 400)),
        ties, -ties, np.nextafter(ties, 0), np.nextafter(ties, np.inf),
        [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 1.5 * 2.0 ** -134, 3 * 2.0 ** -135,
         3.3e38, 3.39e38, 3.4e38, -3.4e38, 1e39],
    ])
    assert np.array_equal(o.bf16_rne_f64(x), _brute_bf16(x, bits, vals))


def test_bf16_rne_f64_matches_torch_on_fp32_values():
    """Where the input is already an fp32 value there is no double rounding,
    so torch's fp32 -> bf16 cast (round to nearest even) must agree."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.bf16_rne_f64(x.astype(np.float64)), t)


def test_bf16_rne_f64_rounds_once():
    """1 + 2^-8 + 2^-30 lies just above the tie between 1 and 1 + 2^-7: rounded
    once it goes up; through fp32 first (which lands on the tie) it would go
    to the even neighbour 1."""
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert o.bf16_rne_f64(np.array([x]))[0] == 0x3F81
    assert torch.tensor([x], dtype=torch.float64).float().to(torch.bfloat16).view(torch.int16).item() == 0x3F80


def _merge_case(seed, N, K, r, gamma=0.5):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    A = o.round_to_bf16((rng.standard_normal((r, K)) * 0.05).astype(np.float32)).astype(np.float64)
    B = o.round_to_bf16((rng.standard_normal((N, r)) * 0.05).astype(np.float32)).astype(np.float64)
    return o.quantize(W), A, B, gamma


def test_merge_is_the_model_the_layer_computes():
    """The exact merged weight reproduces the layer: X W_m^T is the oracle's
    forward Y, and dY W_m its input gradient (the page writes dX as
    dY (W~ + gamma B A))."""
    N, K, r = 24, 128, 8
    (p, s, m), A, B, g = _merge_case(31, N, K, r)
    exact, _ = o.merge(p, s, m, N, K, A, B, g)
    Wt = o.dequantize(p, s, m, N, K)
    rng = np.random.default_rng(32)
    X, dY = rng.standard_normal((5, K)), rng.standard_normal((5, N))
    Y, _ = o.linear_forward(X, Wt, A, B, g)
    dX, *_ = o.linear_backward(dY, X, Wt, A, B, g)
    assert np.allclose(X @ exact.T, Y, rtol=1e-12, atol=1e-12)
    assert np.allclose(dY @ exact, dX, rtol=1e-12, atol=1e-12)


def test_merge_elementwise_loop():
    N, K, r = 4, 64, 8
    (p, s, m), A, B, g = _merge_case(33, N, K, r, gamma=1.25)
    exact, bits = o.merge(p, s, m, N, K, A, B, g)
    Wt = o.dequantize(p, s, m, N, K)
    for n in range(N):
        for k in range(0, K, 7):
            v = float(Wt[n, k]) + 1.25 * sum(float(B[n, j]) * float(A[j, k]) for j in range(r))
            assert exact[n, k] == pytest.approx(v, rel=1e-14, abs=1e-18)
    assert np.array_equal(bits, o.bf16_rne_f64(exact))


@pytest.mark.parametrize("zero", ["B", "gamma"])
def test_merge_without_adapter_is_the_dequantised_base(zero):
    N, K, r = 16, 256, 16
    (p, s, m), A, B, g = _merge_case(34, N, K, r)
    if zero == "B":
        B = np.zeros_like(B)
    else:
        g = 0.0
    _, bits = o.merge(p, s, m, N, K, A, B, g)
    ref = o.dequantize_bits(p, s, m, N * K).reshape(N, K)
    unsign0 = lambda b: np.where(b == 0x8000, 0, b)       # -0 + 0 is +0
    assert np.array_equal(unsign0(bits), unsign0(ref))


def test_requantising_the_unmerged_base_keeps_every_index():
    """quantize(W~) keeps each index of a block whose scale is non-zero: the
    block's largest |w~| is bf16(c~), and w~ / bf16(c~) stays within 2^-8 of
    its code, far inside the half-gap to the next code."""
    N, K = 32, 1024
    (p, s, m), _, _, _ = _merge_case(35, N, K, 8)
    Wt = o.dequantize(p, s, m, N, K).astype(np.float32)
    p2, _, _ = o.quantize(Wt)
    idx = o.unpack_nibbles(p, N * K).reshape(-1, o.BLOCK)
    idx2 = o.unpack_nibbles(p2, N * K).reshape(-1, o.BLOCK)
    live = s != 0
    assert live.mean() > 0.99
    assert np.array_equal(idx[live], idx2[live])


# --------------------------------------------------------------------------
# Format variants (codebooks, blocksizes, scale storage)
# --------------------------------------------------------------------------
def test_quantize_fmt_nf4_b64_e4m3_is_quantize():
    rng = np.random.default_rng(41)
    W = (rng.standard_normal(64 * 256 * 3 + 100) * 0.02).astype(np.float32)
    codes, _ = o.nf4_codebook()
    p, s, m = o.quantize_fmt(W, codes, 64, o.SCALES_E4M3)
    p0, s0, m0 = o.quantize(W)
    assert np.array_equal(p, p0) and np.array_equal(s, s0)
    assert np.array_equal(m.view(np.uint32), m0.view(np.uint32))
    assert np.array_equal(o.dequantize_fmt_bits(p, s, m, W.size, codes, 64, o.SCALES_E4M3),
                          o.dequantize_bits(p0, s0, m0, W.size))


@pytest.mark.parametrize("cb", ["nf4", "fp4", "int4"])
@pytest.mark.parametrize("block", [16, 64, 256, 4096])
def test_fp32_scale_variant_matches_brute_force_toy(cb, block):
    """With fp32 scales the variant reconstructs, before its bf16 rounding,
    the brute-force toy of "A toy run ..." (argmin over the codebook)."""
    codes = {"nf4": o.nf4_codebook()[0], "fp4": o.fp4_e2m1_codebook(),
             "int4": o.int4_codebook()}[cb]
    rng = np.random.default_rng(42)
    w = (rng.standard_normal(4096 * 3 + 48) * 0.02).astype(np.float32)
    p, s, _ = o.quantize_fmt(w, codes, block, o.SCALES_FP32)
    idx = o.unpack_nibbles(p, s.size * block).reshape(s.size, block)
    rec = (codes[idx] * s.reshape(-1, 1)).astype(np.float32).reshape(-1)[:w.size]
    toy = o.single_quant_roundtrip(w, codes, block)
    assert np.array_equal(rec, toy)
    bits = o.dequantize_fmt_bits(p, s, None, w.size, codes, block, o.SCALES_FP32)
    assert np.array_equal(bits, o.bf16_bits(rec))


def test_variant_toy_statistics_through_bf16():
    """M1-M3 of "A toy run ..." through the variant quantiser and its bf16
    dequantisation: the bf16 rounding adds at most 2^-18 / 3 of relative
    mean-square error (0.00013 points), so the printed tolerances widen by
    0.0002 points."""
    t = _golden_table("toy_statistics.txt")
    rng = np.random.default_rng(0)
    w = rng.normal(0, 0.02, 2 ** 20).astype(np.float32)
    books = {"nf4": o.nf4_codebook()[0], "fp4": o.fp4_e2m1_codebook(), "int4": o.int4_codebook()}
    cases = {"gauss_nf4_b64": ("nf4", 64), "gauss_fp4_b64": ("fp4", 64),
             "gauss_int4_b64": ("int4", 64), "gauss_nf4_b16": ("nf4", 16),
             "gauss_nf4_b4096": ("nf4", 4096)}
    for key, (cb, block) in cases.items():
        p, s, _ = o.quantize_fmt(w, books[cb], block, o.SCALES_FP32)
        rec = o.bf16_bits_to_float(o.dequantize_fmt_bits(p, s, None, w.size, books[cb], block,
                                                         o.SCALES_FP32)).astype(np.float64)
        rel = 100 * np.mean((rec - w) ** 2) / np.mean(w.astype(np.float64) ** 2)
        ref, tol = t[key]
        assert abs(rel - ref) <= tol + 2e-4, (key, rel, ref)


def test_format_nbytes():
    assert o.format_nbytes(4096 * 4096, 64, o.SCALES_E4M3) == o.quantized_nbytes(4096 * 4096)
    assert o.format_nbytes(100, 16, o.SCALES_FP32) == (56, 28, 0)
    assert o.format_nbytes(2 ** 20, 4096, o.SCALES_E4M3) == (2 ** 19, 256, 4)


# --------------------------------------------------------------------------
# Layer chaining with checkpoint recompute (SwiGLU MLP of adapted layers)
# --------------------------------------------------------------------------
def test_silu_grad_against_central_differences():
    z = np.linspace(-8, 8, 97)
    h = 1e-6
    num = (o.silu(z + h) - o.silu(z - h)) / (2 * h)
    assert np.allclose(o.silu_grad(z), num, atol=1e-8)
    assert o.silu(0.0) == 0.0 and o.silu_grad(0.0) == 0.5


def _tiny_mlp(seed=51, M=3, K=6, F=5, r=2):
    rng = np.random.default_rng(seed)
    mk = lambda n, k: (rng.normal(size=(n, k)), rng.normal(size=(r, k)), rng.normal(size=(n, r)))
    layers = {"gate": mk(F, K), "up": mk(F, K), "down": mk(K, F)}
    return rng.normal(size=(M, K)), layers, rng.normal(size=(M, K)), 0.75


def test_mlp_forward_elementwise():
    X, L, _, g = _tiny_mlp()
    Y, (G, U, H) = o.mlp_forward(X, L, g)
    m, f = 1, 3
    lin = lambda x, name, j: (sum(x[k] * L[name][0][j, k] for k in range(x.size))
                              + g * sum(sum(x[k] * L[name][1][i, k] for k in range(x.size))
                                        * L[name][2][j, i] for i in range(L[name][1].shape[0])))
    gv, uv = lin(X[m], "gate", f), lin(X[m], "up", f)
    assert G[m, f] == pytest.approx(gv, abs=1e-12) and U[m, f] == pytest.approx(uv, abs=1e-12)
    assert H[m, f] == pytest.approx(gv / (1 + math.exp(-gv)) * uv, abs=1e-12)
    assert Y[m, 2] == pytest.approx(lin(H[m], "down", 2), abs=1e-12)


def test_mlp_backward_finite_differences():
    """Gradients of L = <dY, Y> by central differences, for X and every
    adapter matrix of the three chained layers."""
    X, L, dY, g = _tiny_mlp()
    dX, dAB = o.mlp_backward(dY, X, L, g)

    def loss(X_, L_):
        return float(np.sum(dY * o.mlp_forward(X_, L_, g)[0]))

    h = 1e-6
    num = np.zeros_like(X)
    for i in np.ndindex(X.shape):
        p, m = X.copy(), X.copy()
        p[i] += h
        m[i] -= h
        num[i] = (loss(p, L) - loss(m, L)) / (2 * h)
    assert np.allclose(num, dX, atol=1e-5)
    for name in ("gate", "up", "down"):
        for which in (1, 2):                     # A, B
            arr = L[name][which]
            grad = dAB[name][which - 1]
            num = np.zeros_like(arr)
            for i in np.ndindex(arr.shape):
                for sgn, store in ((1, "p"), (-1, "m")):
                    a2 = arr.copy()
                    a2[i] += sgn * h
                    L2 = dict(L)
                    t = list(L[name])
                    t[which] = a2
                    L2[name] = tuple(t)
                    v = loss(X, L2)
                    num[i] += sgn * v / (2 * h)
            assert np.allclose(num, grad, atol=1e-5), (name, which)


def test_checkpointed_backward_equals_stored_activations():
    X, L, dY, g = _tiny_mlp(seed=52, M=4)
    _, saved = o.mlp_forward(X, L, g)
    dX1, d1 = o.mlp_backward(dY, X, L, g, saved=saved)
    dX2, d2 = o.mlp_backward(dY, X, L, g, saved=None)
    assert np.array_equal(dX1, dX2)
    for k in d1:
        assert all(np.array_equal(a, b) for a, b in zip(d1[k], d2[k]))


def test_mlp_bf16_activations():
    """With bf16 activations every activation passed between the steps is a
    bf16 value, equal to bf16_rne of the same step's exact value computed from
    the rounded inputs (checked by redoing one element by hand, with torch's
    bf16 cast as the rounding), and the block's results stay within a few
    bf16 roundings of the exact chain."""
    X, L, dY, g = _tiny_mlp(seed=53, M=5, K=8, F=7)
    Y0, _ = o.mlp_forward(X, L, g)
    Y1, (G, U, H) = o.mlp_forward(X, L, g, bf16_activations=True)
    tb = lambda a: torch.tensor(a, dtype=torch.float64).to(torch.bfloat16).double().item()
    for arr in (G, U, H, Y1):
        assert np.array_equal(o._bf16_of(arr), arr)
    m, f = 2, 4
    gx = float(X[m] @ L["gate"][0][f] + g * (X[m] @ L["gate"][1].T) @ L["gate"][2][f])
    assert G[m, f] == tb(gx)
    assert H[m, f] == tb(G[m, f] / (1 + math.exp(-G[m, f])) * U[m, f])
    assert np.linalg.norm(Y1 - Y0) / np.linalg.norm(Y0) < 2 ** -6
    dX0, d0 = o.mlp_backward(dY, X, L, g)
    dX1, d1 = o.mlp_backward(dY, X, L, g, bf16_activations=True)
    assert np.array_equal(o._bf16_of(dX1), dX1)
    assert np.linalg.norm(dX1 - dX0) / np.linalg.norm(dX0) < 2 ** -5
    for k in d0:
        for a, b in zip(d0[k], d1[k]):
            assert np.linalg.norm(a - b) / np.linalg.norm(a) < 2 ** -5


# --------------------------------------------------------------------------
# Optimiser state for the adapter (AdamW, fp32 and 8-bit blockwise)
# --------------------------------------------------------------------------
def test_adamw_step_matches_torch():
    """Five steps against torch.optim.AdamW (an independent implementation)."""
    rng = np.random.default_rng(61)
    p0 = rng.standard_normal((16, 64)).astype(np.float32)
    grads = [rng.standard_normal((16, 64)).astype(np.float32) for _ in range(5)]
    hp = dict(lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], **hp, foreach=False)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.from_numpy(g.copy())
        opt.step()
        p, m, v = o.adamw_step(p, g, m, v, t, hp["lr"], *hp["betas"], hp["eps"], hp["weight_decay"])
    assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=1e-6)
    st = opt.state[tp]
    # torch blends the moments with lerp, a different fp32 rounding order
    assert np.allclose(m, st["exp_avg"].numpy(), rtol=1e-5, atol=1e-7)
    assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("signed", [True, False])
def test_state8_roundtrip_bounds(signed):
    rng = np.random.default_rng(62)
    x = rng.standard_normal(64 * 9 + 5).astype(np.float32)
    if not signed:
        x = x * x
    x[64:128] = 0.0                                     # an all-zero block
    q, c = o.encode_state8(x, signed, 64)
    y = o.decode_state8(q, c, signed, 64)
    levels = 127 if signed else 255
    per = np.repeat(c, 64)[: x.size]
    assert np.all(np.abs(y - x) <= per / (2 * levels) * (1 + 1e-5) + 1e-30)
    assert np.all(y[64:128] == 0)
    # the block maximum is encoded exactly at full scale
    for b in range(c.size):
        blk = np.abs(x[b * 64:(b + 1) * 64])
        if blk.size and blk.max() > 0:
            i = b * 64 + int(np.argmax(blk))
            assert abs(int(q[i])) == levels
    # values on the grid survive a second round trip unchanged
    q2, c2 = o.encode_state8(y, signed, 64)
    assert np.array_equal(q2, q) and np.array_equal(c2.view(np.uint32), c.view(np.uint32))


def test_adamw8_tracks_fp32_state_on_a_quadratic():
    """Minimising 0.5 |p - p*|^2: the 8-bit state version follows the fp32
    one closely (the moments' quantisation error is < 0.4% of each block's
    absmax) and both converge."""
    rng = np.random.default_rng(63)
    target = rng.standard_normal((8, 128)).astype(np.float32)
    p32 = np.zeros_like(target)
    p8 = np.zeros_like(target)
    m, v = np.zeros_like(target), np.zeros_like(target)
    ms = o.encode_state8(np.zeros(target.size, np.float32), True, 64)
    vs = o.encode_state8(np.zeros(target.size, np.float32), False, 64)
    for t in range(1, 301):
        p32, m, v = o.adamw_step(p32, p32 - target, m, v, t, 0.05, 0.9, 0.999, 1e-8, 0.0)
        p8, ms, vs = o.adamw8_step(p8, p8 - target, ms, vs, t, 0.05, 0.9, 0.999, 1e-8, 0.0)
    e32 = np.abs(p32 - target).max()
    e8 = np.abs(p8 - target).max()
    assert e32 < 0.05 and e8 < 0.1, (e32, e8)
    assert np.abs(p8 - p32).max() < 0.1


def test_linear_code_of_the_second_moment_diverges():
    """The reason the second moment is coded through its square root: with a
    linear code of v itself, small v flush to zero while m does not, and the
    step m / (0 + eps) blows up on the same quadratic."""
    rng = np.random.default_rng(63)
    target = rng.standard_normal((8, 128)).astype(np.float32)
    p = np.zeros_like(target)
    ms = o.encode_state8(np.zeros(target.size, np.float32), True, 64)
    vs = o.encode_state8(np.zeros(target.size, np.float32), False, 64)
    for t in range(1, 301):
        m = o.decode_state8(*ms, True, 64).reshape(p.shape)
        v = o.decode_state8(*vs, False, 64).reshape(p.shape)
        p, m, v = o.adamw_step(p, p - target, m, v, t, 0.05, 0.9, 0.999, 1e-8, 0.0)
        ms, vs = o.encode_state8(m, True, 64), o.encode_state8(v, False, 64)
    assert np.abs(p - target).max() > 1.0
