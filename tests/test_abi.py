"""CPU tests of the C-ABI library: it loads, exports every symbol the header
declares, and its host-only entry points agree with the oracle.  No CUDA
compute call is made here: the validation tests only reach paths that return
before any launch."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("nf4_build_codebook", "qlora_quantize", "qlora_dequantize",
              "qlora_linear_forward", "qlora_linear_backward"):
        assert n in names


def test_library_exports_every_declared_symbol(q):
    L = ctypes.CDLL(q._lib.LIB_PATH)
    for n in _declared():
        assert hasattr(L, n), n
    assert set(_declared()) == set(q.EXPORTED)


def test_host_codebook_bit_exact_with_oracle(q):
    codes, mids = q.nf4_build_codebook()
    oc, om = o.nf4_codebook()
    assert np.array_equal(np.array(codes, np.float32).view(np.uint32), oc.view(np.uint32))
    assert np.array_equal(np.array(mids, np.float32).view(np.uint32), om.view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(4096, 4096), (11008, 4096), (3, 100), (1, 1), (0, 5),
                                       (28672, 8192), (7, 64 * 256 + 3)])
def test_quantized_sizes_match_oracle(q, rows, cols):
    assert q.qlora_quantized_sizes(rows, cols) == o.quantized_nbytes(rows * cols)


def test_status_strings(q):
    for s in range(8):
        assert q.status_string(s)
    assert "unknown" in q.status_string(99)


def test_workspace_size_rules(q):
    L = q.lib()
    b = ctypes.c_size_t()
    assert L.qlora_linear_workspace_size(64, 256, 512, 8, ctypes.byref(b)) == 0 and b.value > 0
    assert L.qlora_linear_workspace_size(64, 256, 500, 8, ctypes.byref(b)) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_linear_workspace_size(64, 250, 512, 8, ctypes.byref(b)) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_linear_workspace_size(64, 256, 512, 12, ctypes.byref(b)) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_linear_workspace_size(64, 256, 512, 136, ctypes.byref(b)) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_linear_workspace_size(-1, 256, 512, 8, ctypes.byref(b)) == q._lib.QLORA_ERR_SHAPE
    assert L.qlora_linear_workspace_size(64, 256, 512, 8, None) == q._lib.QLORA_ERR_NULL


def test_argument_errors_return_before_any_launch(q):
    """Bad arguments are rejected on the host (fake pointers never touched)."""
    L = q.lib()
    T = q._lib._Tensor
    good = T(0x10000, 0x20000, 0x30000, 256, 512)
    fake = 0x40000
    ws_n = ctypes.c_size_t()
    L.qlora_linear_workspace_size(64, 256, 512, 8, ctypes.byref(ws_n))
    # null input
    assert L.qlora_linear_forward(None, 64, ctypes.byref(good), fake, fake, 8, 2.0, fake, None,
                                  fake, ws_n.value, None) == q._lib.QLORA_ERR_NULL
    # misaligned X
    assert L.qlora_linear_forward(fake + 2, 64, ctypes.byref(good), fake, fake, 8, 2.0, fake,
                                  None, fake, ws_n.value, None) == q._lib.QLORA_ERR_ALIGN
    # unsupported rank
    assert L.qlora_linear_forward(fake, 64, ctypes.byref(good), fake, fake, 7, 2.0, fake, None,
                                  fake, ws_n.value, None) == q._lib.QLORA_ERR_UNSUPPORTED
    # workspace too small
    assert L.qlora_linear_forward(fake, 64, ctypes.byref(good), fake, fake, 8, 2.0, fake, None,
                                  fake, ws_n.value - 1, None) == q._lib.QLORA_ERR_WORKSPACE
    # null tensor buffer
    bad = T(0, 0x20000, 0x30000, 256, 512)
    assert L.qlora_dequantize(ctypes.byref(bad), fake, None) == q._lib.QLORA_ERR_NULL
    neg = T(0x10000, 0x20000, 0x30000, -1, 512)
    assert L.qlora_quantize(fake, ctypes.byref(neg), None, None) == q._lib.QLORA_ERR_SHAPE
    mis = T(0x10008, 0x20000, 0x30000, 256, 512)
    assert L.qlora_quantize(fake, ctypes.byref(mis), None, None) == q._lib.QLORA_ERR_ALIGN
    assert L.qlora_linear_backward(fake, fake, 64, ctypes.byref(good), fake, fake, 8, 2.0, None,
                                   fake, None, fake, 0, fake, ws_n.value, None) == q._lib.QLORA_ERR_NULL


def test_merge_and_bf16_quantize_argument_errors(q):
    """qlora_merge / qlora_quantize_bf16 reject bad arguments on the host; an
    empty weight returns before any launch."""
    L = q.lib()
    T = q._lib._Tensor
    fake = 0x40000
    good = T(0x10000, 0x20000, 0x30000, 256, 512)
    E = q._lib
    assert L.qlora_merge(ctypes.byref(good), None, fake, 16, 2.0, fake, None) == E.QLORA_ERR_NULL
    assert L.qlora_merge(ctypes.byref(good), fake, fake, 16, 2.0, None, None) == E.QLORA_ERR_NULL
    assert L.qlora_merge(None, fake, fake, 16, 2.0, fake, None) == E.QLORA_ERR_NULL
    for r in (0, 4, 12, 136):
        assert L.qlora_merge(ctypes.byref(good), fake, fake, r, 2.0, fake, None) == E.QLORA_ERR_UNSUPPORTED
    odd_k = T(0x10000, 0x20000, 0x30000, 256, 500)
    assert L.qlora_merge(ctypes.byref(odd_k), fake, fake, 16, 2.0, fake, None) == E.QLORA_ERR_UNSUPPORTED
    assert L.qlora_merge(ctypes.byref(good), fake + 8, fake, 16, 2.0, fake, None) == E.QLORA_ERR_ALIGN
    assert L.qlora_merge(ctypes.byref(good), fake, fake, 16, 2.0, fake + 2, None) == E.QLORA_ERR_ALIGN
    neg = T(0x10000, 0x20000, 0x30000, -1, 512)
    assert L.qlora_merge(ctypes.byref(neg), fake, fake, 16, 2.0, fake, None) == E.QLORA_ERR_SHAPE
    empty = T(0x10000, 0x20000, 0x30000, 0, 512)
    assert L.qlora_merge(ctypes.byref(empty), fake, fake, 16, 2.0, fake, None) == E.QLORA_OK
    assert L.qlora_quantize_bf16(None, ctypes.byref(good), None, None) == E.QLORA_ERR_NULL
    assert L.qlora_quantize_bf16(fake + 8, ctypes.byref(good), None, None) == E.QLORA_ERR_ALIGN
    assert L.qlora_quantize_bf16(fake, ctypes.byref(neg), None, None) == E.QLORA_ERR_SHAPE
    assert L.qlora_quantize_bf16(fake, ctypes.byref(empty), None, None) == E.QLORA_OK


def _books():
    return {"nf4": tuple(o.nf4_codebook()[0]), "fp4": tuple(o.fp4_e2m1_codebook()),
            "int4": tuple(o.int4_codebook())}


def test_quantize_many_checks_every_job_before_any_launch(q):
    """qlora_quantize_many validates all its jobs on the host first (null or
    misaligned weight, bad stored tensor): the failing job's status, nothing
    launched; an empty list and empty weights (whose W may be NULL) launch
    nothing."""
    L = q.lib()
    E = q._lib
    T, J = q._lib._Tensor, q._lib._QuantJob
    good = T(0x10000, 0x20000, 0x30000, 256, 512)
    empty = T(0x10000, 0x20000, 0x30000, 0, 512)
    nulled = T(0, 0x20000, 0x30000, 256, 512)
    fake = 0x40000
    ok = lambda: J(fake, ctypes.addressof(good))
    assert L.qlora_quantize_many(None, 0, 0, None, None) == E.QLORA_OK
    assert L.qlora_quantize_many(None, 1, 0, None, None) == E.QLORA_ERR_NULL
    assert L.qlora_quantize_many(None, -1, 0, None, None) == E.QLORA_ERR_SHAPE
    for bad, status in ((J(None, ctypes.addressof(good)), E.QLORA_ERR_NULL),
                        (J(fake + 4, ctypes.addressof(good)), E.QLORA_ERR_ALIGN),
                        (J(fake, ctypes.addressof(nulled)), E.QLORA_ERR_NULL),
                        (J(fake, None), E.QLORA_ERR_NULL)):
        arr = (J * 19)(*([ok()] * 17 + [bad] + [ok()]))
        assert L.qlora_quantize_many(arr, 19, 0, None, None) == status
        assert L.qlora_quantize_many(arr, 19, 1, None, None) == status
    bare = T(0, 0, 0, 0, 16384)                 # what torch hands over for an empty tensor
    only_empty = (J * 3)(J(fake, ctypes.addressof(empty)), J(None, ctypes.addressof(empty)),
                         J(None, ctypes.addressof(bare)))
    assert L.qlora_quantize_many(only_empty, 3, 0, None, None) == E.QLORA_OK
    neg = T(0x10000, 0x20000, 0x30000, -1, 64)
    assert L.qlora_quantize_many((J * 1)(J(fake, ctypes.addressof(neg))), 1, 0, None,
                                 None) == E.QLORA_ERR_SHAPE


def test_merge_many_checks_every_job_before_any_launch(q):
    """qlora_merge_many validates all its jobs on the host first: one bad job
    (rank 12, a misaligned output, a null adapter) fails the whole call with
    that job's status and nothing is launched (the fake device pointers are
    never touched); an empty list and empty weights launch nothing."""
    L = q.lib()
    E = q._lib
    T, J = q._lib._Tensor, q._lib._MergeJob
    good = T(0x10000, 0x20000, 0x30000, 256, 512)
    empty = T(0x10000, 0x20000, 0x30000, 0, 512)
    fake = 0x40000
    ok = lambda: J(ctypes.addressof(good), fake, fake, 16, 2.0, fake)
    assert L.qlora_merge_many(None, 0, None) == E.QLORA_OK
    assert L.qlora_merge_many(None, 2, None) == E.QLORA_ERR_NULL
    assert L.qlora_merge_many(None, -1, None) == E.QLORA_ERR_SHAPE
    for bad, status in ((J(ctypes.addressof(good), fake, fake, 12, 2.0, fake), E.QLORA_ERR_UNSUPPORTED),
                        (J(ctypes.addressof(good), fake, fake, 16, 2.0, fake + 2), E.QLORA_ERR_ALIGN),
                        (J(ctypes.addressof(good), None, fake, 16, 2.0, fake), E.QLORA_ERR_NULL),
                        (J(None, fake, fake, 16, 2.0, fake), E.QLORA_ERR_NULL)):
        arr = (J * 20)(*([ok()] * 17 + [bad] + [ok()] * 2))
        assert L.qlora_merge_many(arr, 20, None) == status
    only_empty = (J * 3)(*([J(ctypes.addressof(empty), None, None, 16, 2.0, None)] * 3))
    assert L.qlora_merge_many(only_empty, 3, None) == E.QLORA_OK


@pytest.mark.parametrize("numel", [0, 1, 100, 4096 * 4096, 2 ** 20 + 17])
@pytest.mark.parametrize("block", [16, 64, 4096])
@pytest.mark.parametrize("scales", ["fp32", "e4m3", "e5m2", "u8"])
def test_format_sizes_match_oracle(q, numel, block, scales):
    enum = {"fp32": q.QLORA_SCALES_FP32, "e4m3": q.QLORA_SCALES_E4M3,
            "e5m2": q.QLORA_SCALES_E5M2, "u8": q.QLORA_SCALES_U8}[scales]
    f = q.Format(_books()["fp4"], block, enum)
    assert q.qlora_format_sizes(numel, f) == o.format_nbytes(numel, block, scales)


def test_format_validation_before_any_launch(q):
    L = q.lib()
    E = q._lib
    fake = 0x40000
    p, c, m = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()

    def st(fmt, numel=1000):
        f = fmt.c_struct()
        return L.qlora_format_sizes(numel, ctypes.byref(f), ctypes.byref(p), ctypes.byref(c),
                                    ctypes.byref(m))

    good = q.Format(_books()["nf4"], 64, q.QLORA_SCALES_E4M3)
    assert st(good) == E.QLORA_OK
    for block in (8, 48, 8192, 0):
        assert st(q.Format(good.codes, block)) == E.QLORA_ERR_UNSUPPORTED
    assert st(q.Format((0.5,), 64)) == E.QLORA_ERR_UNSUPPORTED            # one code
    assert st(q.Format((0.0, 0.5, 0.5), 64)) == E.QLORA_ERR_UNSUPPORTED   # not strictly ascending
    assert st(q.Format((0.0, float("nan")), 64)) == E.QLORA_ERR_UNSUPPORTED
    assert st(q.Format(good.codes, 64, 7)) == E.QLORA_ERR_UNSUPPORTED
    assert st(q.Format(good.codes, 64, 4)) == E.QLORA_ERR_UNSUPPORTED
    for enc in (q.QLORA_SCALES_E5M2, q.QLORA_SCALES_U8):
        assert st(q.Format(good.codes, 64, enc)) == E.QLORA_OK
    assert st(good, -1) == E.QLORA_ERR_SHAPE
    assert L.qlora_format_sizes(10, None, ctypes.byref(p), ctypes.byref(c), ctypes.byref(m)) == E.QLORA_ERR_NULL
    f = good.c_struct()
    assert L.qlora_quantize_fmt(None, 1000, ctypes.byref(f), fake, fake, fake, None, None) == E.QLORA_ERR_NULL
    assert L.qlora_quantize_fmt(fake, 1000, ctypes.byref(f), fake, fake, None, None, None) == E.QLORA_ERR_NULL
    assert L.qlora_quantize_fmt(fake + 4, 1000, ctypes.byref(f), fake, fake, fake, None, None) == E.QLORA_ERR_ALIGN
    assert L.qlora_quantize_fmt(None, 0, ctypes.byref(f), None, None, None, None, None) == E.QLORA_OK
    assert L.qlora_dequantize_fmt(fake, fake, fake, 1000, ctypes.byref(f), fake + 2, None) == E.QLORA_ERR_ALIGN
    assert L.qlora_dequantize_fmt(fake, fake, fake, -5, ctypes.byref(f), fake, None) == E.QLORA_ERR_SHAPE
    f32 = q.Format(good.codes, 16, q.QLORA_SCALES_FP32).c_struct()
    assert L.qlora_dequantize_fmt(fake, None, None, 1000, ctypes.byref(f32), fake, None) == E.QLORA_ERR_NULL


def test_adamw8_argument_errors(q):
    L = q.lib()
    E = q._lib
    fake = 0x40000
    cfg = q._lib._AdamConfig(2e-4, 0.9, 0.999, 1e-8, 0.0, 1)
    c, a = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.qlora_adamw8_state_sizes(130, ctypes.byref(c), ctypes.byref(a)) == E.QLORA_OK
    assert (c.value, a.value) == (130, 12)
    assert L.qlora_adamw8_state_sizes(-1, ctypes.byref(c), ctypes.byref(a)) == E.QLORA_ERR_SHAPE
    step = lambda *args: L.qlora_adamw8_step(*args)
    assert step(fake, fake, 100, fake, fake, fake, fake, None, None, None) == E.QLORA_ERR_NULL
    assert step(None, fake, 100, fake, fake, fake, fake, ctypes.byref(cfg), None, None) == E.QLORA_ERR_NULL
    assert step(fake + 4, fake, 100, fake, fake, fake, fake, ctypes.byref(cfg), None, None) == E.QLORA_ERR_ALIGN
    assert step(fake, fake, -1, fake, fake, fake, fake, ctypes.byref(cfg), None, None) == E.QLORA_ERR_SHAPE
    assert step(None, None, 0, None, None, None, None, ctypes.byref(cfg), None, None) == E.QLORA_OK
    C = q._lib._AdamConfig
    for bad in (C(2e-4, 1.0, 0.999, 1e-8, 0.0, 1),
                C(2e-4, 0.9, 0.999, 1e-8, 0.0, 0),
                C(float("nan"), 0.9, 0.999, 1e-8, 0.0, 1),
                C(2e-4, 0.9, 0.999, 0.0, 0.0, 1),          # eps = 0: 0 / 0 on an all-zero block
                C(2e-4, 0.9, 0.999, -1e-8, 0.0, 1),
                C(-2e-4, 0.9, 0.999, 1e-8, 0.0, 1),        # negative learning rate
                C(2e-4, 0.9, 0.999, 1e-8, -0.1, 1),        # negative weight decay
                C(2.0, 0.9, 0.999, 1e-8, 0.5, 1)):         # lr * wd >= 1: decay factor <= 0
        assert step(fake, fake, 100, fake, fake, fake, fake, ctypes.byref(bad), None, None) == E.QLORA_ERR_UNSUPPORTED
    ok = C(2e-4, 0.9, 0.999, 1e-8, 0.01, 1)
    assert step(None, None, 0, None, None, None, None, ctypes.byref(ok), None, None) == E.QLORA_OK


def test_noalloc_error_word_argument_errors(q):
    L = q.lib()
    assert L.qlora_linear_forward_noalloc_error_word(None, None) == q._lib.QLORA_ERR_NULL


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import bit_nf4_quantised_b200._lib as L
    monkeypatch.setattr(L, "_LIB", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        L.lib()


C_CLIENT = r"""
#include <stdio.h>
#include "qlora_nf4.h"
int main(void) {
    float codes[16], mids[15];
    if (nf4_build_codebook(codes, mids) != QLORA_OK) return 2;
    size_t p = 0, c = 0, m = 0;
    if (qlora_quantized_sizes(4096, 4096, &p, &c, &m) != QLORA_OK) return 3;
    qlora_format f = {16, 16, {0}, QLORA_SCALES_FP32};
    for (int i = 0; i < 16; ++i) f.codes[i] = codes[i];
    size_t fp = 0, fs = 0, fm = 0;
    if (qlora_format_sizes(100, &f, &fp, &fs, &fm) != QLORA_OK) return 4;
    for (int i = 0; i < 16; ++i) printf("%a ", codes[i]);
    printf("\n%zu %zu %zu %zu %zu %zu\n%s\n", p, c, m, fp, fs, fm, qlora_status_string(QLORA_ERR_ALIGN));
    return 0;
}
"""


def test_plain_c_client_links_and_runs(q, tmp_path):
    """The boundary is a C ABI: a plain C99 program includes the header, links
    the library and calls its host-only entry points."""
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(q._lib.LIB_PATH)
    import subprocess
    cc = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                         "-L", libdir, "-lqlora_nf4", f"-Wl,-rpath,{libdir}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    lines = run.stdout.strip().splitlines()
    got = np.array([float.fromhex(t) for t in lines[0].split()], np.float32)
    assert np.array_equal(got.view(np.uint32), o.nf4_codebook()[0].view(np.uint32))
    sizes = tuple(int(t) for t in lines[1].split())
    assert sizes[:3] == o.quantized_nbytes(4096 * 4096)
    assert sizes[3:] == o.format_nbytes(100, 16, o.SCALES_FP32)
    assert lines[2] == "misaligned pointer"
