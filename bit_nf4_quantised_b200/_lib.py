"""ctypes binding of libqlora_nf4.so (include/qlora_nf4.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  If the
shared library is missing the import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_NULL = 1
QLORA_ERR_SHAPE = 2
QLORA_ERR_ALIGN = 3
QLORA_ERR_UNSUPPORTED = 4
QLORA_ERR_NONFINITE = 5
QLORA_ERR_CUDA = 6
QLORA_ERR_WORKSPACE = 7

BLOCK = 64
GROUP = 256
MAX_RANK = 128
GEMV_MAX_TOKENS = 16

EXPORTED = (
    "qlora_status_string",
    "nf4_build_codebook",
    "qlora_quantized_sizes",
    "qlora_quantize",
    "qlora_dequantize",
    "qlora_linear_workspace_size",
    "qlora_linear_forward",
    "qlora_linear_backward",
    "qlora_linear_forward_ex",
    "qlora_linear_backward_ex",
    "qlora_linear_forward_noalloc",
    "qlora_linear_forward_noalloc_error_word",
    "qlora_merge",
    "qlora_merge_many",
    "qlora_quantize_bf16",
    "qlora_quantize_many",
    "qlora_format_sizes",
    "qlora_quantize_fmt",
    "qlora_dequantize_fmt",
    "qlora_adamw8_state_sizes",
    "qlora_adamw8_step",
    "qlora_set_gemm_wait_limit_us",
    "qlora_mlp_workspace_size",
    "qlora_mlp_forward",
    "qlora_mlp_backward",
)

QLORA_SCALES_FP32 = 0
QLORA_SCALES_E4M3 = 1
QLORA_SCALES_E5M2 = 2
QLORA_SCALES_U8 = 3


class QloraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class _Events(ctypes.Structure):
    _fields_ = [("gemm_begin", ctypes.c_void_p), ("gemm_end", ctypes.c_void_p)]


def _events(events):
    """(begin, end) torch.cuda.Event pair (timing enabled) -> qlora_events*."""
    if events is None:
        return None
    handles = []
    for ev in events:
        if ev is None:
            handles.append(None)
            continue
        if not ev.cuda_event:          # torch creates the CUDA event on first record
            ev.record()
        handles.append(ev.cuda_event)
    return ctypes.byref(_Events(*handles))


class _QuantJob(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("out", ctypes.c_void_p)]   # const qlora_nf4_tensor*


class _MergeJob(ctypes.Structure):
    _fields_ = [
        ("w", ctypes.c_void_p),          # const qlora_nf4_tensor*
        ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p),
        ("r", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("W_out", ctypes.c_void_p),
    ]


class _Tensor(ctypes.Structure):
    _fields_ = [
        ("packed", ctypes.c_void_p),
        ("scale_codes", ctypes.c_void_p),
        ("meta_scale", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
    ]


class _Format(ctypes.Structure):
    _fields_ = [
        ("block", ctypes.c_int32),
        ("ncodes", ctypes.c_int32),
        ("codes", ctypes.c_float * 16),
        ("scales", ctypes.c_int32),
    ]


class _Mlp(ctypes.Structure):
    _fields_ = [("gate", _Tensor), ("up", _Tensor), ("down", _Tensor),
                ("A_gate", ctypes.c_void_p), ("B_gate", ctypes.c_void_p),
                ("A_up", ctypes.c_void_p), ("B_up", ctypes.c_void_p),
                ("A_down", ctypes.c_void_p), ("B_down", ctypes.c_void_p),
                ("r", ctypes.c_int)]


class _MlpGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dA_gate", "dB_gate", "dA_up", "dB_up", "dA_down", "dB_down")]


class _AdamConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("step", ctypes.c_int64)]


_LIB = None


def lib() -> ctypes.CDLL:
    """Load the library once; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantised_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sz = ctypes.POINTER(ctypes.c_size_t)
        tp = ctypes.POINTER(_Tensor)
        L.qlora_status_string.argtypes = [i32]
        L.qlora_status_string.restype = ctypes.c_char_p
        L.nf4_build_codebook.argtypes = [vp, vp]
        L.qlora_quantized_sizes.argtypes = [i64, i64, sz, sz, sz]
        L.qlora_quantize.argtypes = [vp, tp, vp, vp]
        L.qlora_dequantize.argtypes = [tp, vp, vp]
        L.qlora_quantize_bf16.argtypes = [vp, tp, vp, vp]
        L.qlora_merge.argtypes = [tp, vp, vp, i32, f32, vp, vp]
        L.qlora_merge_many.argtypes = [ctypes.POINTER(_MergeJob), i32, vp]
        L.qlora_quantize_many.argtypes = [ctypes.POINTER(_QuantJob), i32, i32, vp, vp]
        fp = ctypes.POINTER(_Format)
        L.qlora_format_sizes.argtypes = [i64, fp, sz, sz, sz]
        L.qlora_quantize_fmt.argtypes = [vp, i64, fp, vp, vp, vp, vp, vp]
        L.qlora_dequantize_fmt.argtypes = [vp, vp, vp, i64, fp, vp, vp]
        L.qlora_adamw8_state_sizes.argtypes = [i64, sz, sz]
        L.qlora_adamw8_step.argtypes = [vp, vp, i64, vp, vp, vp, vp,
                                        ctypes.POINTER(_AdamConfig), vp, vp]
        L.qlora_linear_workspace_size.argtypes = [i64, i64, i64, i32, sz]
        L.qlora_set_gemm_wait_limit_us.argtypes = [i64]
        mp = ctypes.POINTER(_Mlp)
        L.qlora_mlp_workspace_size.argtypes = [i64, mp, sz]
        L.qlora_mlp_forward.argtypes = [vp, i64, mp, f32, vp, vp, ctypes.c_size_t, vp]
        L.qlora_mlp_backward.argtypes = [vp, vp, i64, mp, f32, vp, ctypes.POINTER(_MlpGrads), i32,
                                         vp, ctypes.c_size_t, vp]
        fwd = [vp, i64, tp, vp, vp, i32, f32, vp, vp, vp, ctypes.c_size_t, vp]
        bwd = [vp, vp, i64, tp, vp, vp, i32, f32, vp, vp, vp, vp, i32, vp, ctypes.c_size_t, vp]
        L.qlora_linear_forward.argtypes = fwd
        L.qlora_linear_backward.argtypes = bwd
        L.qlora_linear_forward_ex.argtypes = fwd + [ctypes.c_void_p]
        L.qlora_linear_backward_ex.argtypes = bwd + [ctypes.c_void_p]
        for name in EXPORTED[1:]:
            getattr(L, name).restype = i32
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    return lib().qlora_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != QLORA_OK:
        raise QloraError(status, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if t.dtype != dtype or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


# --------------------------------------------------------------------------
@dataclass
class NF4Tensor:
    """A stored NF4 weight (three device buffers) of logical shape rows x cols."""
    packed: torch.Tensor        # uint8 [nblocks * 32]
    scale_codes: torch.Tensor   # uint8 [nblocks]
    meta_scale: torch.Tensor    # float32 [ngroups]
    rows: int
    cols: int

    def c_struct(self) -> _Tensor:
        return _Tensor(self.packed.data_ptr(), self.scale_codes.data_ptr(),
                       self.meta_scale.data_ptr(), self.rows, self.cols)

    @property
    def nbytes(self) -> int:
        return self.packed.numel() + self.scale_codes.numel() + 4 * self.meta_scale.numel()


def nf4_build_codebook():
    codes = (ctypes.c_float * 16)()
    mids = (ctypes.c_float * 15)()
    _check(lib().nf4_build_codebook(ctypes.addressof(codes), ctypes.addressof(mids)),
           "nf4_build_codebook")
    return list(codes), list(mids)


def qlora_quantized_sizes(rows: int, cols: int):
    p, c, m = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_quantized_sizes(rows, cols, ctypes.byref(p), ctypes.byref(c),
                                       ctypes.byref(m)), "qlora_quantized_sizes")
    return p.value, c.value, m.value


def empty_nf4(rows: int, cols: int, device="cuda") -> NF4Tensor:
    p, c, m = qlora_quantized_sizes(rows, cols)
    return NF4Tensor(torch.empty(max(p, 16), dtype=torch.uint8, device=device)[:p],
                     torch.empty(max(c, 1), dtype=torch.uint8, device=device)[:c],
                     torch.empty(max(m // 4, 1), dtype=torch.float32, device=device)[: m // 4],
                     rows, cols)


def qlora_quantize(W: torch.Tensor, out: NF4Tensor | None = None, check_finite: bool = True,
                   stream=None) -> NF4Tensor:
    """Quantise a fp32 [rows, cols] CUDA tensor.  With check_finite the
    library synchronises the stream and the call raises
    QloraError(QLORA_ERR_NONFINITE) if the kernel saw a NaN or an infinity."""
    _need(W, torch.float32, "W")
    rows, cols = (W.shape[0], W.shape[1]) if W.dim() == 2 else (1, W.numel())
    out = out if out is not None else empty_nf4(rows, cols, W.device)
    flag = torch.empty(1, dtype=torch.int32, device=W.device) if check_finite else None
    st = out.c_struct()
    _check(lib().qlora_quantize(W.data_ptr(), ctypes.byref(st), _ptr(flag), _stream(stream)),
           "qlora_quantize")
    return out


def qlora_quantize_many(jobs, check_finite: bool = True, stream=None) -> list:
    """Quantise several [rows, cols] CUDA tensors, all fp32 or all bf16, in as
    few launches as the library needs.  jobs: sequence of (W, out) with out
    None or an NF4Tensor; returns the stored tensors in order.  check_finite
    as qlora_quantize, for all of them together."""
    jobs = list(jobs)
    dtypes = {W.dtype for W, _ in jobs}
    if len(dtypes) > 1 or not dtypes <= {torch.float32, torch.bfloat16}:
        raise TypeError(f"qlora_quantize_many: W must be all fp32 or all bf16, got {dtypes}")
    outs, structs = [], []
    for W, out in jobs:
        _need(W, W.dtype, "W")
        rows, cols = (W.shape[0], W.shape[1]) if W.dim() == 2 else (1, W.numel())
        out = out if out is not None else empty_nf4(rows, cols, W.device)
        outs.append(out)
        structs.append((W, out.c_struct()))
    arr = (_QuantJob * max(1, len(structs)))()
    for i, (W, st) in enumerate(structs):
        arr[i] = _QuantJob(W.data_ptr(), ctypes.addressof(st))
    bf16 = bool(jobs) and jobs[0][0].dtype == torch.bfloat16
    flag = (torch.empty(1, dtype=torch.int32, device=jobs[0][0].device)
            if check_finite and jobs else None)
    _check(lib().qlora_quantize_many(arr, len(structs), 1 if bf16 else 0, _ptr(flag),
                                     _stream(stream)), "qlora_quantize_many")
    return outs


def qlora_dequantize(w: NF4Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty(w.rows, w.cols, dtype=torch.bfloat16,
                                                  device=w.packed.device)
    _need(out, torch.bfloat16, "out")
    st = w.c_struct()
    _check(lib().qlora_dequantize(ctypes.byref(st), out.data_ptr(), _stream(stream)),
           "qlora_dequantize")
    return out


def qlora_quantize_bf16(W: torch.Tensor, out: NF4Tensor | None = None, check_finite: bool = True,
                        stream=None) -> NF4Tensor:
    """qlora_quantize of a bf16 [rows, cols] CUDA tensor (values widened
    exactly to fp32): the re-quantisation of a merged weight."""
    _need(W, torch.bfloat16, "W")
    rows, cols = (W.shape[0], W.shape[1]) if W.dim() == 2 else (1, W.numel())
    out = out if out is not None else empty_nf4(rows, cols, W.device)
    flag = torch.empty(1, dtype=torch.int32, device=W.device) if check_finite else None
    st = out.c_struct()
    _check(lib().qlora_quantize_bf16(W.data_ptr(), ctypes.byref(st), _ptr(flag), _stream(stream)),
           "qlora_quantize_bf16")
    return out


def qlora_merge(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor, scale: float,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 [rows, cols] merged weight W~ + scale * B A.  A [r, cols], B [rows, r]."""
    _need(A, torch.bfloat16, "A")
    _need(B, torch.bfloat16, "B")
    r = A.shape[0]
    out = out if out is not None else torch.empty(w.rows, w.cols, dtype=torch.bfloat16,
                                                  device=w.packed.device)
    _need(out, torch.bfloat16, "out")
    st = w.c_struct()
    _check(lib().qlora_merge(ctypes.byref(st), A.data_ptr(), B.data_ptr(), r, float(scale),
                             out.data_ptr(), _stream(stream)), "qlora_merge")
    return out


def qlora_merge_many(jobs, stream=None) -> list:
    """qlora_merge of several weights in as few launches as the library needs.
    jobs: sequence of (w, A, B, scale, out) with out None or a bf16 [rows,
    cols] tensor; returns the outputs in order."""
    outs, structs = [], []
    for w, A, B, scale, out in jobs:
        _need(A, torch.bfloat16, "A")
        _need(B, torch.bfloat16, "B")
        out = out if out is not None else torch.empty(w.rows, w.cols, dtype=torch.bfloat16,
                                                      device=w.packed.device)
        _need(out, torch.bfloat16, "out")
        outs.append(out)
        structs.append((w.c_struct(), A, B, float(scale), out))
    arr = (_MergeJob * max(1, len(structs)))()
    for i, (st, A, B, scale, out) in enumerate(structs):
        arr[i] = _MergeJob(ctypes.addressof(st), A.data_ptr(), B.data_ptr(), A.shape[0], scale,
                           out.data_ptr())
    _check(lib().qlora_merge_many(arr, len(structs), _stream(stream)), "qlora_merge_many")
    return outs


@dataclass
class Format:
    """A quantisation format: codebook (ascending, up to 16 codes), blocksize
    (power of two, 16..4096) and scale storage (QLORA_SCALES_FP32, or an 8-bit
    code: _E4M3, _E5M2 or _U8)."""
    codes: tuple
    block: int = BLOCK
    scales: int = QLORA_SCALES_E4M3

    def c_struct(self) -> _Format:
        f = _Format()
        f.block = int(self.block)
        f.ncodes = len(self.codes)
        for i, c in enumerate(self.codes):
            f.codes[i] = float(c)
        f.scales = int(self.scales)
        return f


def qlora_format_sizes(numel: int, fmt: Format):
    p, c, m = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    f = fmt.c_struct()
    _check(lib().qlora_format_sizes(numel, ctypes.byref(f), ctypes.byref(p), ctypes.byref(c),
                                    ctypes.byref(m)), "qlora_format_sizes")
    return p.value, c.value, m.value


def qlora_quantize_fmt(W: torch.Tensor, fmt: Format, check_finite: bool = True, stream=None):
    """(packed u8, scales (fp32 or u8), meta fp32 or None) of a contiguous fp32
    CUDA tensor in format fmt."""
    _need(W, torch.float32, "W")
    n = W.numel()
    pb, sb, mb = qlora_format_sizes(n, fmt)
    dev = W.device
    packed = torch.empty(max(pb, 16), dtype=torch.uint8, device=dev)[:pb]
    if fmt.scales == QLORA_SCALES_FP32:
        scales = torch.empty(max(sb // 4, 1), dtype=torch.float32, device=dev)[: sb // 4]
        meta = None
    else:
        scales = torch.empty(max(sb, 4), dtype=torch.uint8, device=dev)[:sb]
        meta = torch.empty(max(mb // 4, 1), dtype=torch.float32, device=dev)[: mb // 4]
    flag = torch.empty(1, dtype=torch.int32, device=dev) if check_finite else None
    f = fmt.c_struct()
    _check(lib().qlora_quantize_fmt(W.data_ptr(), n, ctypes.byref(f), _ptr(packed), _ptr(scales),
                                    _ptr(meta), _ptr(flag), _stream(stream)), "qlora_quantize_fmt")
    return packed, scales, meta


def qlora_dequantize_fmt(packed: torch.Tensor, scales: torch.Tensor, meta, numel: int,
                         fmt: Format, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty(numel, dtype=torch.bfloat16, device=packed.device)
    _need(out, torch.bfloat16, "out")
    f = fmt.c_struct()
    _check(lib().qlora_dequantize_fmt(_ptr(packed), _ptr(scales), _ptr(meta), numel,
                                      ctypes.byref(f), out.data_ptr(), _stream(stream)),
           "qlora_dequantize_fmt")
    return out


@dataclass
class Adam8State:
    """8-bit blockwise AdamW state of n parameters (zeros = the initial state)."""
    m_codes: torch.Tensor     # int8 [n]
    m_absmax: torch.Tensor    # float32 [ceil(n/64)]
    v_codes: torch.Tensor     # uint8 [n]
    v_absmax: torch.Tensor    # float32 [ceil(n/64)]
    step: int = 0


def adamw8_state(n: int, device="cuda") -> Adam8State:
    c, a = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_adamw8_state_sizes(n, ctypes.byref(c), ctypes.byref(a)),
           "qlora_adamw8_state_sizes")
    nb = a.value // 4
    z = lambda k, dt: torch.zeros(max(k, 4), dtype=dt, device=device)[:k]
    return Adam8State(z(n, torch.int8), z(nb, torch.float32), z(n, torch.uint8),
                      z(nb, torch.float32))


def qlora_adamw8_step(p: torch.Tensor, g: torch.Tensor, state: Adam8State, lr: float,
                      beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                      weight_decay: float = 0.0, p_bf16: torch.Tensor | None = None,
                      stream=None) -> None:
    """One AdamW step of the fp32 parameters p in place (state.step advances)."""
    _need(p, torch.float32, "p")
    _need(g, torch.float32, "g")
    if p_bf16 is not None:
        _need(p_bf16, torch.bfloat16, "p_bf16")
    state.step += 1
    cfg = _AdamConfig(lr, beta1, beta2, eps, weight_decay, state.step)
    _check(lib().qlora_adamw8_step(p.data_ptr(), g.data_ptr(), p.numel(),
                                   _ptr(state.m_codes), _ptr(state.m_absmax),
                                   _ptr(state.v_codes), _ptr(state.v_absmax), ctypes.byref(cfg),
                                   _ptr(p_bf16), _stream(stream)), "qlora_adamw8_step")


def qlora_linear_workspace_size(M: int, N: int, K: int, r: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().qlora_linear_workspace_size(M, N, K, r, ctypes.byref(b)),
           "qlora_linear_workspace_size")
    return b.value


def workspace(M: int, N: int, K: int, r: int, device="cuda") -> torch.Tensor:
    n = qlora_linear_workspace_size(M, N, K, r)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def qlora_linear_forward(X: torch.Tensor, w: NF4Tensor, A: torch.Tensor, B: torch.Tensor,
                         scale: float, Y: torch.Tensor | None = None,
                         T_save: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                         stream=None, events=None) -> torch.Tensor:
    """Y = X W~^T + scale * (X A^T) B^T.  X [M,K] bf16, A [r,K], B [N,r].
    events: optional (begin, end) torch.cuda.Event pair recorded around the
    main weight kernel."""
    _need(X, torch.bfloat16, "X")
    _need(A, torch.bfloat16, "A")
    _need(B, torch.bfloat16, "B")
    M, K = X.shape
    r = A.shape[0]
    N = w.rows
    Y = Y if Y is not None else torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    _need(Y, torch.bfloat16, "Y")
    if T_save is not None:
        _need(T_save, torch.float32, "T_save")
    ws = ws if ws is not None else workspace(M, N, K, r, X.device)
    st = w.c_struct()
    _check(lib().qlora_linear_forward_ex(X.data_ptr(), M, ctypes.byref(st), A.data_ptr(),
                                         B.data_ptr(), r, float(scale), Y.data_ptr(),
                                         _ptr(T_save), ws.data_ptr(), ws.numel(),
                                         _stream(stream), _events(events)),
           "qlora_linear_forward")
    return Y


def qlora_linear_backward(dY: torch.Tensor, X: torch.Tensor, w: NF4Tensor, A: torch.Tensor,
                          B: torch.Tensor, scale: float, T_saved: torch.Tensor | None = None,
                          dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                          dB: torch.Tensor | None = None, accumulate: bool = False,
                          want_dX: bool = True, ws: torch.Tensor | None = None, stream=None,
                          events=None):
    """(dX, dA, dB) of the adapted layer; dX is None when want_dX is False."""
    for t, n in ((dY, "dY"), (X, "X"), (A, "A"), (B, "B")):
        _need(t, torch.bfloat16, n)
    M, K = X.shape
    r = A.shape[0]
    N = w.rows
    dev = X.device
    if want_dX and dX is None:
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(N, r, dtype=torch.float32, device=dev)
    if T_saved is not None:
        _need(T_saved, torch.float32, "T_saved")
    ws = ws if ws is not None else workspace(M, N, K, r, dev)
    st = w.c_struct()
    _check(lib().qlora_linear_backward_ex(dY.data_ptr(), X.data_ptr(), M, ctypes.byref(st),
                                          A.data_ptr(), B.data_ptr(), r, float(scale),
                                          _ptr(T_saved), _ptr(dX) if want_dX else None,
                                          dA.data_ptr(), dB.data_ptr(), int(bool(accumulate)),
                                          ws.data_ptr(), ws.numel(), _stream(stream),
                                          _events(events)),
           "qlora_linear_backward")
    return (dX if want_dX else None), dA, dB


def device_error_word(ws: torch.Tensor) -> int:
    """The kernels' error word (first 4 bytes of the workspace); 0 = no error,
    bit 0 = a bounded wait inside the GEMM expired."""
    return int(ws[:4].view(torch.int32).item())


# --------------------------------------------------------------------------
@dataclass
class MLP:
    """The SwiGLU MLP of adapted NF4 linears: stored gate, up (F x D) and
    down (D x F) weights and their bf16 adapters (A r x in, B out x r)."""
    gate: NF4Tensor
    up: NF4Tensor
    down: NF4Tensor
    A_gate: torch.Tensor
    B_gate: torch.Tensor
    A_up: torch.Tensor
    B_up: torch.Tensor
    A_down: torch.Tensor
    B_down: torch.Tensor

    @property
    def r(self) -> int:
        return self.A_gate.shape[0]

    def c_struct(self) -> _Mlp:
        for name in ("A_gate", "B_gate", "A_up", "B_up", "A_down", "B_down"):
            _need(getattr(self, name), torch.bfloat16, name)
        return _Mlp(self.gate.c_struct(), self.up.c_struct(), self.down.c_struct(),
                    self.A_gate.data_ptr(), self.B_gate.data_ptr(), self.A_up.data_ptr(),
                    self.B_up.data_ptr(), self.A_down.data_ptr(), self.B_down.data_ptr(), self.r)


def qlora_mlp_workspace_size(M: int, mlp: MLP) -> int:
    b = ctypes.c_size_t()
    st = mlp.c_struct()
    _check(lib().qlora_mlp_workspace_size(M, ctypes.byref(st), ctypes.byref(b)),
           "qlora_mlp_workspace_size")
    return b.value


def mlp_workspace(M: int, mlp: MLP, device="cuda") -> torch.Tensor:
    return torch.empty(max(qlora_mlp_workspace_size(M, mlp), 256), dtype=torch.uint8, device=device)


def qlora_mlp_forward(X: torch.Tensor, mlp: MLP, scale: float, Y: torch.Tensor | None = None,
                      ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = down(silu(gate(X)) * up(X)); X [M, D] bf16."""
    _need(X, torch.bfloat16, "X")
    M, D = X.shape
    Y = Y if Y is not None else torch.empty(M, D, dtype=torch.bfloat16, device=X.device)
    _need(Y, torch.bfloat16, "Y")
    ws = ws if ws is not None else mlp_workspace(M, mlp, X.device)
    st = mlp.c_struct()
    _check(lib().qlora_mlp_forward(X.data_ptr(), M, ctypes.byref(st), float(scale), Y.data_ptr(),
                                   ws.data_ptr(), ws.numel(), _stream(stream)), "qlora_mlp_forward")
    return Y


def qlora_mlp_backward(dY: torch.Tensor, X: torch.Tensor, mlp: MLP, scale: float,
                       dX: torch.Tensor | None = None, grads: dict | None = None,
                       accumulate: bool = False, ws: torch.Tensor | None = None, stream=None):
    """(dX, grads) of the MLP, recomputing its forward (checkpointing); grads
    maps dA_gate, dB_gate, dA_up, dB_up, dA_down, dB_down to fp32 tensors."""
    _need(dY, torch.bfloat16, "dY")
    _need(X, torch.bfloat16, "X")
    M, D = X.shape
    dev = X.device
    dX = dX if dX is not None else torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    if grads is None:
        grads = {}
        for lin, name in ((mlp.gate, "gate"), (mlp.up, "up"), (mlp.down, "down")):
            grads[f"dA_{name}"] = torch.empty(mlp.r, lin.cols, dtype=torch.float32, device=dev)
            grads[f"dB_{name}"] = torch.empty(lin.rows, mlp.r, dtype=torch.float32, device=dev)
    g = _MlpGrads(*(grads[n].data_ptr() for n in
                    ("dA_gate", "dB_gate", "dA_up", "dB_up", "dA_down", "dB_down")))
    ws = ws if ws is not None else mlp_workspace(M, mlp, dev)
    st = mlp.c_struct()
    _check(lib().qlora_mlp_backward(dY.data_ptr(), X.data_ptr(), M, ctypes.byref(st), float(scale),
                                    dX.data_ptr(), ctypes.byref(g), int(bool(accumulate)),
                                    ws.data_ptr(), ws.numel(), _stream(stream)),
           "qlora_mlp_backward")
    return dX, grads
