"""Fine-grained online FP8 (E4M3) quantization and block-scaled FP8 GEMM
for NVIDIA B200 (sm_100a).

Python binding of the C ABI declared in ``include/fp8fg.h``.  Each function
below has the name of the C entry point it calls and only marshals
arguments: it reads pointers, sizes and strides from ``torch.Tensor``
objects (allocating outputs with torch when they are not given) and passes
the current CUDA stream.  All computation happens in the CUDA library;
importing this package fails if that library is not built.

Method (codingmall.com "Kan du förklara rollen för FP8 precision i
träningsprocessen för DeepSeek-V3"): activations are quantized in 1x128
tiles and weights in 128x128 blocks, each with its own scale amax/448
computed on every call, into E4M3; the FP8 GEMM promotes each 128-wide
K chunk's tensor-core partial to FP32 after multiplying it by the two
scales.
"""
import ctypes

import torch

from . import _lib
from ._lib import (FP8_IN_BF16, FP8_IN_FP32, FP8_OUT_BF16, FP8_OUT_FP32, LIB_PATH,
                   STATUS_NAMES, Fp8Error)

__all__ = [
    "fp8_quantize_act_1x128", "fp8_quantize_weight_128x128", "fp8_blockscaled_gemm",
    "fp8_grouped_gemm", "fp8_status_string", "fp8_get_device_error", "Fp8Error",
    "LIB_PATH", "linear_forward", "e2e_linear_forward", "fp8_quantize_act_1x128_gather",
    "fp8_quantize_act_1x128_scatter",
    "fp8_blockscaled_gemm_quant", "fp8_dequantize", "fp8_quantize_act_128x1",
    "fp8_blockscaled_gemm_colscale", "linear_weight_grad", "fp8_set_wait_limit",
    "LinearForwardPipeline",
]

_L = _lib.lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _in_type(t):
    if t.dtype == torch.bfloat16:
        return FP8_IN_BF16
    if t.dtype == torch.float32:
        return FP8_IN_FP32
    raise TypeError("inputs are bfloat16 or float32, got %s" % t.dtype)


def _out_type(dtype):
    if dtype == torch.bfloat16:
        return FP8_OUT_BF16
    if dtype == torch.float32:
        return FP8_OUT_FP32
    raise TypeError("outputs are bfloat16 or float32, got %s" % dtype)


def _rowmajor(t, name):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("%s must be a 2-D tensor with a contiguous last dimension" % name)


def fp8_status_string(status):
    return _L.fp8_status_string(int(status)).decode()


def fp8_get_device_error(stream=None):
    """Synchronize the stream, then read and clear the device error word."""
    code = ctypes.c_int(0)
    _lib.check(_L.fp8_get_device_error(_stream(stream), ctypes.byref(code)),
               "fp8_get_device_error")
    return code.value


def fp8_set_wait_limit(cycles):
    """Set how many SM cycles a wait in this library's kernels may last on
    the current device before the kernel gives up (0 restores the default,
    about one second).  For tests of the timeout path."""
    _lib.check(_L.fp8_set_wait_limit(int(cycles)), "fp8_set_wait_limit")


def fp8_quantize_act_1x128(x, q=None, sa=None, stream=None):
    """x [M, K] (bf16/fp32, CUDA) -> (q uint8 [M, K] E4M3 codes, sa fp32 [M, K/128])."""
    _rowmajor(x, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if sa is None:
        sa = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _rowmajor(q, "q")
    st = _L.fp8_quantize_act_1x128(_ptr(x), _in_type(x), M, K, x.stride(0), _ptr(q), q.stride(0),
                                   _ptr(sa), sa.stride(0), sa.stride(1), _stream(stream))
    _lib.check(st, "fp8_quantize_act_1x128")
    return q, sa


def fp8_quantize_act_1x128_gather(x, rows, q=None, sa=None, stream=None):
    """x [T, K] (bf16/fp32, CUDA), rows int32 [R] (CUDA) -> quantization of
    x[rows]: (q uint8 [R, K], sa fp32 [R, K/128]), without forming x[rows]."""
    _rowmajor(x, "x")
    T, K = x.shape
    if rows.dtype != torch.int32 or not rows.is_contiguous():
        raise ValueError("rows must be a contiguous int32 tensor")
    R = rows.shape[0]
    if q is None:
        q = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    if sa is None:
        sa = torch.empty((R, K // 128), dtype=torch.float32, device=x.device)
    _rowmajor(q, "q")
    st = _L.fp8_quantize_act_1x128_gather(_ptr(x), _in_type(x), T, K, x.stride(0), _ptr(rows), R,
                                          _ptr(q), q.stride(0), _ptr(sa), sa.stride(0),
                                          sa.stride(1), _stream(stream))
    _lib.check(st, "fp8_quantize_act_1x128_gather")
    return q, sa


def fp8_quantize_act_1x128_scatter(x, dest, R, q=None, sa=None, stream=None):
    """x [T, K] (bf16, CUDA), dest int32 [T, topk] (CUDA; -1 = none) ->
    (q uint8 [R, K], sa fp32 [R, K/128]) where every output row
    dest[t, j] holds the 1x128 quantization of x[t].  Each token is read
    and quantized once.  Rows that no dest entry names are left as they
    were (uninitialised when q / sa are allocated here)."""
    _rowmajor(x, "x")
    T, K = x.shape
    if dest.dtype != torch.int32 or dest.dim() != 2 or not dest.is_contiguous() \
            or dest.shape[0] != T:
        raise ValueError("dest must be a contiguous int32 [T, topk] tensor")
    topk = dest.shape[1]
    if q is None:
        q = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    if sa is None:
        sa = torch.empty((R, K // 128), dtype=torch.float32, device=x.device)
    _rowmajor(q, "q")
    st = _L.fp8_quantize_act_1x128_scatter(_ptr(x), _in_type(x), T, K, x.stride(0), _ptr(dest),
                                           topk, _ptr(q), R, q.stride(0), _ptr(sa), sa.stride(0),
                                           sa.stride(1), _stream(stream))
    _lib.check(st, "fp8_quantize_act_1x128_scatter")
    return q, sa


def fp8_quantize_weight_128x128(w, transpose_out=True, q=None, sb=None, stream=None):
    """w [K, N] -> (q uint8 [N, K] if transpose_out else [K, N], sb fp32 [K/128, N/128])."""
    _rowmajor(w, "w")
    K, N = w.shape
    if q is None:
        shape = (N, K) if transpose_out else (K, N)
        q = torch.empty(shape, dtype=torch.uint8, device=w.device)
    if sb is None:
        sb = torch.empty((K // 128, N // 128), dtype=torch.float32, device=w.device)
    _rowmajor(q, "q")
    st = _L.fp8_quantize_weight_128x128(_ptr(w), _in_type(w), K, N, w.stride(0), _ptr(q),
                                        1 if transpose_out else 0, q.stride(0), _ptr(sb),
                                        sb.stride(0), sb.stride(1), _stream(stream))
    _lib.check(st, "fp8_quantize_weight_128x128")
    return q, sb


def fp8_blockscaled_gemm(a, sa, b, sb, out_dtype=torch.bfloat16, c=None, sb_kb_nb=True,
                         stream=None):
    """C [M, N] = block-scaled a [M, K] x b^T, b stored K-major [N, K].

    sa is indexed [m, kb]; sb is indexed [kb, nb] (``sb_kb_nb``) or, when
    False, stored [nb, kb] (the untransposed weight used for dgrad).
    """
    _rowmajor(a, "a")
    _rowmajor(b, "b")
    M, K = a.shape
    N = b.shape[0]
    if c is None:
        c = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _rowmajor(c, "c")
    sb_skb, sb_snb = (sb.stride(0), sb.stride(1)) if sb_kb_nb else (sb.stride(1), sb.stride(0))
    st = _L.fp8_blockscaled_gemm(_ptr(a), a.stride(0), _ptr(sa), sa.stride(0), sa.stride(1),
                                 _ptr(b), b.stride(0), 1, _ptr(sb), sb_skb, sb_snb, _ptr(c),
                                 _out_type(c.dtype), c.stride(0), M, N, K, _stream(stream))
    _lib.check(st, "fp8_blockscaled_gemm")
    return c


def fp8_blockscaled_gemm_quant(a, sa, b, sb, qc=None, sc=None, c=None, want_c=False,
                               stream=None):
    """Block-scaled GEMM with its output quantized for the next layer:
    returns (qc uint8 [M, N] E4M3 codes, sc fp32 [M, N/128]) and, when
    ``want_c`` (or ``c`` is given), the bf16 output [M, N] as a third value.
    Bit-identical to fp8_blockscaled_gemm(..., bf16) + fp8_quantize_act_1x128."""
    _rowmajor(a, "a")
    _rowmajor(b, "b")
    M, K = a.shape
    N = b.shape[0]
    if qc is None:
        qc = torch.empty((M, N), dtype=torch.uint8, device=a.device)
    if sc is None:
        sc = torch.empty((M, N // 128), dtype=torch.float32, device=a.device)
    if c is None and want_c:
        c = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    if c is not None:
        _rowmajor(c, "c")
    st = _L.fp8_blockscaled_gemm_quant(
        _ptr(a), a.stride(0), _ptr(sa), sa.stride(0), sa.stride(1), _ptr(b), b.stride(0), _ptr(sb),
        sb.stride(0), sb.stride(1), _ptr(qc), qc.stride(0), _ptr(sc), sc.stride(0), sc.stride(1),
        _ptr(c) if c is not None else None, c.stride(0) if c is not None else 0, M, N, K,
        _stream(stream))
    _lib.check(st, "fp8_blockscaled_gemm_quant")
    return (qc, sc, c) if c is not None else (qc, sc)


def fp8_quantize_act_128x1(x, qt=None, st=None, st_kb_major=False, stream=None):
    """x [M, K] (bf16, CUDA) -> 1x128 quantization of x^T along M:
    (qt uint8 [K, M] E4M3 codes, st fp32 scales), st [K, M/128] or, with
    ``st_kb_major``, [M/128, K] (the layout of the column-scale GEMM's sb).

    Limits of the CUDA kernel: x must be bfloat16 (float32 raises Fp8Error
    with FP8_ERR_DTYPE) and M a multiple of 128 (a ragged token count such as
    a per-expert MoE batch raises FP8_ERR_SHAPE; pad it with zero rows,
    which change no scale or code of the other rows)."""
    _rowmajor(x, "x")
    M, K = x.shape
    if qt is None:
        qt = torch.empty((K, M), dtype=torch.uint8, device=x.device)
    if st is None:
        shape = (M // 128, K) if st_kb_major else (K, M // 128)
        st = torch.empty(shape, dtype=torch.float32, device=x.device)
    _rowmajor(qt, "qt")
    s_k, s_mb = (st.stride(1), st.stride(0)) if st_kb_major else (st.stride(0), st.stride(1))
    status = _L.fp8_quantize_act_128x1(_ptr(x), _in_type(x), M, K, x.stride(0), _ptr(qt),
                                       qt.stride(0), _ptr(st), s_k, s_mb, _stream(stream))
    _lib.check(status, "fp8_quantize_act_128x1")
    return qt, st


def fp8_blockscaled_gemm_colscale(a, sa, b, sb, out_dtype=torch.bfloat16, c=None, stream=None):
    """C [M, N] = a [M, K] x b^T (b [N, K]) with 1x128 scales on both
    operands: sa [M, K/128] indexed [m, kb], sb [K/128, N] indexed [kb, n]."""
    _rowmajor(a, "a")
    _rowmajor(b, "b")
    _rowmajor(sb, "sb")
    M, K = a.shape
    N = b.shape[0]
    if c is None:
        c = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _rowmajor(c, "c")
    st = _L.fp8_blockscaled_gemm_colscale(_ptr(a), a.stride(0), _ptr(sa), sa.stride(0),
                                          sa.stride(1), _ptr(b), b.stride(0), _ptr(sb),
                                          sb.stride(0), _ptr(c), _out_type(c.dtype), c.stride(0),
                                          M, N, K, _stream(stream))
    _lib.check(st, "fp8_blockscaled_gemm_colscale")
    return c


def linear_weight_grad(x, dy, out_dtype=torch.float32, stream=None):
    """Weight gradient of y = x @ w in FP8: dW [K, N] = x^T dy with x [M, K],
    dy [M, N] (bf16).  Both are quantized in 1x128 tiles along the tokens M
    (scales computed on this call), then multiplied by the column-scale GEMM.
    Three library calls.  Needs bfloat16 x and dy (else FP8_ERR_DTYPE) and
    M a multiple of 128 (else FP8_ERR_SHAPE: pad ragged token counts with
    zero rows, which add nothing to dW)."""
    qxt, sxt = fp8_quantize_act_128x1(x, stream=stream)
    qdt, sdt = fp8_quantize_act_128x1(dy, st_kb_major=True, stream=stream)
    return fp8_blockscaled_gemm_colscale(qxt, sxt, qdt, sdt, out_dtype=out_dtype, stream=stream)


def fp8_grouped_gemm(a, sa, b, sb, offsets, out_dtype=torch.bfloat16, c=None, stream=None):
    """MoE grouped GEMM: a [total_M, K] rows sorted by group, b [G, N, K],
    sb [G, K/128, N/128], offsets int32 [G+1] on the device."""
    _rowmajor(a, "a")
    if b.dim() != 3 or b.stride(2) != 1 or b.stride(0) != b.shape[1] * b.stride(1):
        raise ValueError("b must be [G, N, K] with K contiguous and experts contiguous")
    total, K = a.shape
    G, N, _ = b.shape
    if c is None:
        c = torch.empty((total, N), dtype=out_dtype, device=a.device)
    _rowmajor(c, "c")
    if offsets.dtype != torch.int32 or offsets.numel() != G + 1:
        raise ValueError("offsets must be int32 [G+1]")
    st = _L.fp8_grouped_gemm(_ptr(a), a.stride(0), _ptr(sa), sa.stride(0), sa.stride(1), _ptr(b),
                             b.stride(1), _ptr(sb), sb.stride(0), sb.stride(1), sb.stride(2),
                             _ptr(c), _out_type(c.dtype), c.stride(0), _ptr(offsets), G, total,
                             N, K, _stream(stream))
    _lib.check(st, "fp8_grouped_gemm")
    return c


def fp8_dequantize(q, s, tile_rows, out_dtype=torch.bfloat16, out=None, stream=None):
    """q uint8 [R, C] E4M3 codes with scales s (tile_rows x 128 tiles:
    tile_rows 1 for activations, s [R, C/128]; 128 for weights,
    s [R/128, C/128]) -> E4M3(q) * scale as out_dtype [R, C]."""
    _rowmajor(q, "q")
    R, C = q.shape
    if out is None:
        out = torch.empty((R, C), dtype=out_dtype, device=q.device)
    _rowmajor(out, "out")
    st = _L.fp8_dequantize(_ptr(q), R, C, q.stride(0), _ptr(s), s.stride(0), s.stride(1),
                           tile_rows, _ptr(out), _out_type(out.dtype), out.stride(0),
                           _stream(stream))
    _lib.check(st, "fp8_dequantize")
    return out


def linear_forward(x, w, out_dtype=torch.bfloat16, stream=None):
    """Online-quantized FP8 linear layer: y = x @ w with x [M, K], w [K, N].

    Quantizes x in 1x128 tiles and w in 128x128 blocks (scales computed on
    this call), then runs the block-scaled GEMM.  Three library calls.
    """
    qx, sx = fp8_quantize_act_1x128(x, stream=stream)
    qw, sw = fp8_quantize_weight_128x128(w, transpose_out=True, stream=stream)
    return fp8_blockscaled_gemm(qx, sx, qw, sw, out_dtype=out_dtype, stream=stream)


def e2e_linear_forward(x_host, w_host, out_host=None, device="cuda", stream=None):
    """End-to-end form of ``linear_forward`` on host tensors: copies x and w
    (ideally pinned) to the device, runs the three library calls, and copies
    y back into ``out_host`` (allocated pinned when not given)."""
    x = x_host.to(device, non_blocking=True)
    w = w_host.to(device, non_blocking=True)
    y = linear_forward(x, w, out_dtype=torch.bfloat16, stream=stream)
    if out_host is None:
        out_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    out_host.copy_(y, non_blocking=True)
    return out_host


class LinearForwardPipeline:
    """End-to-end ``linear_forward`` on host tensors, pipelined across calls.

    Each ``submit(x_host, w_host, out_host)`` copies x [M, K] and w [K, N]
    (bf16, pinned host memory) to the device on a host-to-device copy
    stream, quantizes both and runs the block-scaled GEMM on the compute
    stream, and copies y = x @ w [M, N] (bf16) into the pinned ``out_host``
    on a device-to-host copy stream.  ``depth`` sets of device buffers let
    call i+1's inputs travel while call i computes and while its result
    travels back; the two copy directions run on separate streams, so both
    directions of the host link are used at once.  The x quantization starts
    as soon as x has landed, while w is still on its way.

    ``submit`` only enqueues work and returns the event that completes with
    the call's device-to-host copy.  The caller keeps ``x_host`` and
    ``w_host`` unchanged and reads ``out_host`` only after that event (or
    ``join`` / ``synchronize``).  ``join(stream)`` makes ``stream`` wait for
    every submitted call; ``synchronize()`` waits on the host.
    """

    def __init__(self, M, K, N, depth=2, device="cuda", stream=None):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        self.M, self.K, self.N = M, K, N
        self.compute = stream if stream is not None else torch.cuda.current_stream(device)
        self.h2d = torch.cuda.Stream(device)
        self.d2h = torch.cuda.Stream(device)
        self.slots = []
        for _ in range(depth):
            self.slots.append(dict(
                x=torch.empty((M, K), dtype=torch.bfloat16, device=device),
                w=torch.empty((K, N), dtype=torch.bfloat16, device=device),
                qx=torch.empty((M, K), dtype=torch.uint8, device=device),
                sx=torch.empty((M, K // 128), dtype=torch.float32, device=device),
                qw=torch.empty((N, K), dtype=torch.uint8, device=device),
                sw=torch.empty((K // 128, N // 128), dtype=torch.float32, device=device),
                c=torch.empty((M, N), dtype=torch.bfloat16, device=device),
                x_in=torch.cuda.Event(), w_in=torch.cuda.Event(),
                used=torch.cuda.Event(), out=torch.cuda.Event(), busy=False))
        self.n = 0

    def submit(self, x_host, w_host, out_host):
        if (tuple(x_host.shape) != (self.M, self.K) or tuple(w_host.shape) != (self.K, self.N)
                or tuple(out_host.shape) != (self.M, self.N)):
            raise ValueError("shapes differ from the pipeline's [M, K] x [K, N]")
        if x_host.dtype != torch.bfloat16 or w_host.dtype != torch.bfloat16 or \
                out_host.dtype != torch.bfloat16:
            raise TypeError("x, w and out are bfloat16")
        s = self.slots[self.n % len(self.slots)]
        self.n += 1
        if s["busy"]:
            # the slot's inputs were read by its previous call's kernels
            self.h2d.wait_event(s["used"])
        with torch.cuda.stream(self.h2d):
            s["x"].copy_(x_host, non_blocking=True)
            s["x_in"].record(self.h2d)
            s["w"].copy_(w_host, non_blocking=True)
            s["w_in"].record(self.h2d)
        # the caching allocator must not hand these buffers out again while
        # the copy streams still use them (e.g. if the pipeline is dropped
        # without close())
        s["x"].record_stream(self.h2d)
        s["w"].record_stream(self.h2d)
        if s["busy"]:
            # the slot's previous result has left the device
            self.compute.wait_event(s["out"])
        self.compute.wait_event(s["x_in"])
        fp8_quantize_act_1x128(s["x"], q=s["qx"], sa=s["sx"], stream=self.compute)
        self.compute.wait_event(s["w_in"])
        fp8_quantize_weight_128x128(s["w"], transpose_out=True, q=s["qw"], sb=s["sw"],
                                    stream=self.compute)
        fp8_blockscaled_gemm(s["qx"], s["sx"], s["qw"], s["sw"], c=s["c"], stream=self.compute)
        s["used"].record(self.compute)
        self.d2h.wait_event(s["used"])
        with torch.cuda.stream(self.d2h):
            out_host.copy_(s["c"], non_blocking=True)
            s["out"].record(self.d2h)
        s["c"].record_stream(self.d2h)
        s["busy"] = True
        return s["out"]

    def join(self, stream=None):
        """Make `stream` (default: the compute stream) wait for every call."""
        st = stream if stream is not None else self.compute
        st.wait_stream(self.d2h)
        st.wait_stream(self.h2d)

    def synchronize(self):
        self.h2d.synchronize()
        self.compute.synchronize()
        self.d2h.synchronize()

    def close(self):
        """Wait for every call and release the device buffers."""
        self.synchronize()
        self.slots = []
