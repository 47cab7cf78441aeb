"""ctypes binding of libmxq.so: argument marshalling only."""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmxq.so")

_DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
_FORMATS = {"fp8": 0, "mxfp4": 1, "nvfp4": 2}

_lib = None


class MxqError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s failed: %s (%d)" % (what, status_string(status), status))
        self.status = status


# Load another build of the library instead of libmxq.so (the debug variant,
# libmxq_debug.so, built with `python -m nvfp4_quantization_amax_b200.build
# --debug`).
LIB_ENV = "MXQ_LIBRARY"


def lib_path():
    return os.environ.get(LIB_ENV) or _LIB_PATH


def lib():
    """Load libmxq.so (built in-tree by nvfp4_quantization_amax_b200.build)."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError("%s not found; build it with "
                               "`python -m nvfp4_quantization_amax_b200.build`" % path)
        L = ctypes.CDLL(path)
        i, i32, i64, p = ctypes.c_int, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
        L.mx_quantize.restype = i
        L.mx_quantize.argtypes = [p, i, i64, i64, p, p, p]
        L.mx_dequantize.restype = i
        L.mx_dequantize.argtypes = [p, p, i64, i64, p, i, p]
        L.quantize_cache.restype = i
        L.quantize_cache.argtypes = [p, p, i, i64, i64, i, i32, p]
        L.mxfp4_grouped_mm.restype = i
        L.mxfp4_grouped_mm.argtypes = [p, p, p, p, i64, i64, i64, i64, i, p, p, p]
        L.mxq_status_string.restype = ctypes.c_char_p
        L.mxq_status_string.argtypes = [i]
        L.mxq_version.restype = i
        L.mxq_version.argtypes = []
        L.mxq_debug_checks.restype = i
        L.mxq_debug_checks.argtypes = [p]
        L.mxq_debug_selftest.restype = i
        L.mxq_debug_selftest.argtypes = [p, p]
        L.nvfp4_quantize.restype = i
        L.nvfp4_quantize.argtypes = [p, i, i64, i64, p, p, p, p, p]
        L.nvfp4_quantize_mse.restype = i
        L.nvfp4_quantize_mse.argtypes = [p, i, i64, i64, p, p, p, p, p]
        L.nvfp4_quantize_noalloc.restype = i
        L.nvfp4_quantize_noalloc.argtypes = [p, i, i64, i64, p, p, p, p]
        L.nvfp4_dequantize.restype = i
        L.nvfp4_dequantize.argtypes = [p, p, p, i64, i64, p, i, p]
        L.quantize_cache_packed.restype = i
        L.quantize_cache_packed.argtypes = [p, i, i64, i64, i, i32, p, p, p]
        L.dequantize_cache_packed.restype = i
        L.dequantize_cache_packed.argtypes = [p, p, i64, i64, i, i32, p, i, p]
        L.mxfp4_w4a4_grouped_mm.restype = i
        L.mxfp4_w4a4_grouped_mm.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, p, p]
        L.nvfp4_w4a4_grouped_mm.restype = i
        L.nvfp4_w4a4_grouped_mm.argtypes = [p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, p]
        L.mxq_set_wait_limit_ns.restype = ctypes.c_uint64
        L.mxq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        _lib = L
    return _lib


def status_string(status):
    return lib().mxq_status_string(int(status)).decode()


def debug_checks():
    """(check id, index, extent) of the first failed index check since the
    previous call, or None; only the debug variant of the library has checks
    (the normal one raises MxqError with MXQ_ERR_UNSUPPORTED)."""
    rec = (ctypes.c_int64 * 3)()
    _check(lib().mxq_debug_checks(ctypes.cast(rec, ctypes.c_void_p)), "mxq_debug_checks")
    return None if rec[0] == 0 else (int(rec[0]), int(rec[1]), int(rec[2]))


def debug_selftest(words):
    """Launch the debug variant's self-test into `words` (device int32 [2])."""
    if not (words.is_cuda and words.dtype == torch.int32 and words.numel() >= 2):
        raise ValueError("debug_selftest needs a device int32 tensor of 2 words")
    _check(lib().mxq_debug_selftest(_ptr(words), _stream(words.device)), "mxq_debug_selftest")


def set_wait_limit_ns(ns):
    """Set the grouped GEMM's pipeline-wait limit (ns); returns the previous one."""
    return int(lib().mxq_set_wait_limit_ns(int(ns)))


def _check(rc, what):
    if rc != 0:
        raise MxqError(rc, what)


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _to_device(t, dev=None):
    """(device tensor, was_on_host) for an input.  A host tensor is moved to
    `dev` (default: the current CUDA device), a pinned one without blocking
    the host; a CUDA tensor must already be on `dev`."""
    if t.is_cuda:
        if dev is not None and t.device != dev:
            raise ValueError("input on %s, the call runs on %s" % (t.device, dev))
        return t, False
    if not torch.cuda.is_available():
        raise RuntimeError("no CUDA device: libmxq runs only on the GPU")
    if dev is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return t.to(dev, non_blocking=t.is_pinned()), True


def _to_host(t):
    out = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    out.copy_(t, non_blocking=True)
    torch.cuda.current_stream(t.device).synchronize()
    return out


def _out(t, shape, dtype, dev, name):
    """(device buffer, host target) for an output of `shape` and `dtype` of
    a call that runs on `dev`.  None: a new device tensor.  A contiguous
    tensor of that dtype and element count on `dev`: itself.  The same on
    the host: a new device tensor, copied into it by _result.  Anything else
    raises before a launch, so no kernel ever writes outside a buffer."""
    shape = tuple(int(v) for v in shape)
    if t is None:
        return torch.empty(shape, dtype=dtype, device=dev), None
    n = 1
    for v in shape:
        n *= v
    if t.dtype != dtype:
        raise TypeError("%s must be %s, not %s" % (name, dtype, t.dtype))
    if t.numel() != n:
        raise ValueError("%s must hold %d elements (shape %s), not %d"
                         % (name, n, list(shape), t.numel()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.is_cuda:
        if t.device != dev:
            raise ValueError("%s is on %s, the call runs on %s" % (name, t.device, dev))
        return t, None
    return torch.empty(shape, dtype=dtype, device=dev).view(t.shape), t


def _result(buf, target, to_host):
    """What the caller gets back for one output: the host tensor it passed
    (now filled); a pinned host copy when its inputs came from the host;
    else the device buffer."""
    if target is not None:
        target.copy_(buf, non_blocking=target.is_pinned())
        torch.cuda.current_stream(buf.device).synchronize()
        return target
    return _to_host(buf) if to_host else buf


def _device_word(t, dtype, min_numel, dev, name):
    """Pointer of an optional device-side scratch or status buffer."""
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda or t.device != dev:
        raise ValueError("%s must be a tensor on %s" % (name, dev))
    if t.dtype != dtype or t.numel() < min_numel or not t.is_contiguous():
        raise ValueError("%s must be a contiguous %s tensor of at least %d elements"
                         % (name, dtype, min_numel))
    return _ptr(t)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


# A row-wise call on pinned host tensors of at least two chunks streams them
# through the GPU in row ranges of about this many input bytes: the copy of
# chunk i+1 in, the kernels of chunk i and the copy of chunk i-1 out run on
# three streams at once (both copy directions of the bus and the GPU busy
# together).  The results equal one call on the whole tensor: these
# operations treat every row on its own.
HOST_CHUNK_BYTES = 64 << 20
# A tensor of less than two such chunks still streams, in four chunks of at
# least this many bytes (smaller tensors take one round trip).
HOST_MIN_CHUNK_BYTES = 4 << 20
_HOST_DEPTH = 3  # device buffer sets in rotation


def _streamable(inputs, outputs):
    """Every input a pinned contiguous host tensor, every given output on
    the host."""
    return (torch.cuda.is_available()
            and all(not t.is_cuda and t.is_pinned() and t.is_contiguous() for t in inputs)
            and all(o is None or not o.is_cuda for o in outputs))


def _host_target(t, shape, dtype, name):
    """Host output of `shape`: the caller's tensor (checked as _out checks a
    buffer) or a new pinned one."""
    n = 1
    for v in shape:
        n *= v
    if t is None:
        return torch.empty(shape, dtype=dtype, pin_memory=True)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, not %s" % (name, dtype, t.dtype))
    if t.numel() != n or not t.is_contiguous():
        raise ValueError("%s must be a contiguous tensor of %d elements" % (name, n))
    return t


def _stream_rows(inputs, outputs, rows, launch, what):
    """Stream a row-wise call through the GPU in row chunks.

    inputs: pinned host tensors, each viewed [rows, -1]; outputs: host
    tensors to fill, each viewed [rows, -1]; launch(dev_inputs, dev_outputs,
    n_rows, stream) issues one chunk's kernels and returns the status.
    Returns False (nothing done) below two chunks."""
    ins = [t.view(rows, -1) for t in inputs]
    outs = [t.view(rows, -1) for t in outputs]
    in_row = sum(t.shape[1] * t.element_size() for t in ins)
    chunk_bytes = HOST_CHUNK_BYTES
    if rows * in_row < 2 * HOST_CHUNK_BYTES:
        chunk_bytes = max(min(HOST_MIN_CHUNK_BYTES, HOST_CHUNK_BYTES), rows * in_row // 4)
    chunk = max(1, chunk_bytes // max(1, in_row))
    n_chunks = (rows + chunk - 1) // chunk
    if n_chunks < 2:
        return False
    dev = torch.device("cuda", torch.cuda.current_device())
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    depth = min(_HOST_DEPTH, n_chunks)
    d_in = [[torch.empty((chunk, t.shape[1]), dtype=t.dtype, device=dev) for t in ins]
            for _ in range(depth)]
    d_out = [[torch.empty((chunk, t.shape[1]), dtype=t.dtype, device=dev) for t in outs]
             for _ in range(depth)]
    in_free = [None] * depth   # the kernels that last read input set j are done
    out_free = [None] * depth  # the copy that last read output set j is done
    st = ctypes.c_void_p(comp.cuda_stream)
    try:
        for i in range(n_chunks):
            j = i % depth
            r0, r1 = i * chunk, min(rows, (i + 1) * chunk)
            n = r1 - r0
            if in_free[j] is not None:
                s_in.wait_event(in_free[j])
            with torch.cuda.stream(s_in):
                for d, h in zip(d_in[j], ins):
                    d[:n].copy_(h[r0:r1], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
            comp.wait_event(landed)
            if out_free[j] is not None:
                comp.wait_event(out_free[j])
            _check(launch([d[:n] for d in d_in[j]], [d[:n] for d in d_out[j]], n, st), what)
            done = torch.cuda.Event()
            done.record(comp)
            in_free[j] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                for d, h in zip(d_out[j], outs):
                    h[r0:r1].copy_(d[:n], non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(s_out)
            out_free[j] = copied
    finally:
        # every copy out follows its kernels, which follow their copy in
        s_out.synchronize()
        comp.synchronize()
    return True


def mx_quantize(x, packed=None, scales=None):
    """MXFP4 quantize + pack along the last dim.

    x: bf16/f16/f32 [..., K], K % 32 == 0.  Returns (packed uint8 [..., K/2],
    scales uint8 [..., K/32]): two E2M1 codes per byte (low nibble = even
    column) and one E8M0 scale byte (float8_e8m0fnu bits) per 32 columns.
    """
    if x.dtype not in _DTYPES:
        raise TypeError("mx_quantize: unsupported dtype %s" % x.dtype)
    if _streamable([x], [packed, scales]) and x.dim() >= 1 and x.shape[-1] > 0:
        K = x.shape[-1]
        rows, lead = x.numel() // K, tuple(x.shape[:-1])
        hp = _host_target(packed, lead + (K // 2,), torch.uint8, "packed")
        hs = _host_target(scales, lead + (K // 32,), torch.uint8, "scales")
        dt = _DTYPES[x.dtype]
        if _stream_rows([x], [hp, hs], rows,
                        lambda di, do, n, st: lib().mx_quantize(_ptr(di[0]), dt, n, K,
                                                                _ptr(do[0]), _ptr(do[1]), st),
                        "mx_quantize"):
            return hp, hs
    x, host = _to_device(x)
    x = x.contiguous()
    K = x.shape[-1]
    rows = x.numel() // K if K else 0
    lead = tuple(x.shape[:-1])
    packed, hp = _out(packed, lead + (K // 2,), torch.uint8, x.device, "packed")
    scales, hs = _out(scales, lead + (K // 32,), torch.uint8, x.device, "scales")
    rc = lib().mx_quantize(_ptr(x), _DTYPES[x.dtype], rows, K, _ptr(packed), _ptr(scales),
                           _stream(x.device))
    _check(rc, "mx_quantize")
    return _result(packed, hp, host), _result(scales, hs, host)


def mx_dequantize(packed, scales, dtype=torch.bfloat16, out=None):
    """Unpack [..., K/2] E2M1 bytes with [..., K/32] E8M0 scales to dtype [..., K]."""
    if dtype not in _DTYPES:
        raise TypeError("mx_dequantize: unsupported dtype %s" % dtype)
    if (_streamable([packed, scales], [out]) and packed.dim() >= 1 and packed.shape[-1] > 0
            and scales.numel() * 16 == packed.numel()):
        K = 2 * packed.shape[-1]
        rows = packed.numel() // packed.shape[-1]
        ho = _host_target(out, tuple(packed.shape[:-1]) + (K,), dtype, "out")
        dt = _DTYPES[dtype]
        if _stream_rows([packed, scales], [ho], rows,
                        lambda di, do, n, st: lib().mx_dequantize(_ptr(di[0]), _ptr(di[1]), n, K,
                                                                  _ptr(do[0]), dt, st),
                        "mx_dequantize"):
            return ho
    packed, host = _to_device(packed)
    scales, _ = _to_device(scales, packed.device)
    packed = packed.contiguous()
    scales = scales.contiguous()
    Kh = packed.shape[-1]
    K = 2 * Kh
    rows = packed.numel() // Kh if Kh else 0
    if scales.numel() != rows * (K // 32):
        raise ValueError("mx_dequantize: scales must have shape [..., K/32]")
    out, ho = _out(out, tuple(packed.shape[:-1]) + (K,), dtype, packed.device, "out")
    rc = lib().mx_dequantize(_ptr(packed), _ptr(scales), rows, K, _ptr(out), _DTYPES[dtype],
                             _stream(packed.device))
    _check(rc, "mx_dequantize")
    return _result(out, ho, host)


def quantize_cache(values, format, block_size, out=None):
    """Fake quantization of [..., channels] values in fp8 / mxfp4 / nvfp4;
    returns a new tensor of the input dtype."""
    if values.dtype not in _DTYPES:
        raise TypeError("quantize_cache: unsupported dtype %s" % values.dtype)
    if format not in _FORMATS:
        raise ValueError("quantize_cache: format must be one of %s" % sorted(_FORMATS))
    if _streamable([values], [out]) and values.dim() >= 1 and values.shape[-1] > 0:
        C = values.shape[-1]
        rows = values.numel() // C
        ho = _host_target(out, tuple(values.shape), values.dtype, "out")
        dt, fmt, B = _DTYPES[values.dtype], _FORMATS[format], int(block_size)
        if _stream_rows([values], [ho], rows,
                        lambda di, do, n, st: lib().quantize_cache(_ptr(di[0]), _ptr(do[0]), dt, n,
                                                                   C, fmt, B, st),
                        "quantize_cache"):
            return ho
    values, host = _to_device(values)
    values = values.contiguous()
    C = values.shape[-1] if values.dim() else 1
    rows = values.numel() // C if C else 0
    out, ho = _out(out, tuple(values.shape), values.dtype, values.device, "out")
    rc = lib().quantize_cache(_ptr(values), _ptr(out), _DTYPES[values.dtype], rows, C,
                              _FORMATS[format], int(block_size), _stream(values.device))
    _check(rc, "quantize_cache")
    return _result(out, ho, host)


def quantize_cache_packed(values, format, block_size, codes=None, scales=None):
    """Stored form of quantize_cache: returns (codes, scales) uint8.

    codes: fp8 -> [..., C] E4M3 bytes; mxfp4/nvfp4 -> [..., C/2] bytes of two
    E2M1 codes (low nibble = even channel).  scales: [..., C/block_size],
    E8M0 bytes for fp8 and mxfp4, E4M3 bytes for nvfp4.  C % block_size == 0.
    """
    if values.dtype not in _DTYPES:
        raise TypeError("quantize_cache_packed: unsupported dtype %s" % values.dtype)
    if format not in _FORMATS:
        raise ValueError("quantize_cache_packed: format must be one of %s" % sorted(_FORMATS))
    B = int(block_size)
    if (_streamable([values], [codes, scales]) and values.dim() >= 1 and values.shape[-1] > 0
            and B >= 1 and values.shape[-1] % B == 0):
        C = values.shape[-1]
        rows, lead = values.numel() // C, tuple(values.shape[:-1])
        hc = _host_target(codes, lead + (C if format == "fp8" else C // 2,), torch.uint8, "codes")
        hs = _host_target(scales, lead + (C // B,), torch.uint8, "scales")
        dt, fmt = _DTYPES[values.dtype], _FORMATS[format]
        if _stream_rows([values], [hc, hs], rows,
                        lambda di, do, n, st: lib().quantize_cache_packed(
                            _ptr(di[0]), dt, n, C, fmt, B, _ptr(do[0]), _ptr(do[1]), st),
                        "quantize_cache_packed"):
            return hc, hs
    values, host = _to_device(values)
    values = values.contiguous()
    C = values.shape[-1] if values.dim() else 1
    rows = values.numel() // C if C else 0
    lead = tuple(values.shape[:-1])
    dev = values.device
    if B < 1:
        raise ValueError("quantize_cache_packed: block_size must be >= 1")
    codes, hc = _out(codes, lead + (C if format == "fp8" else C // 2,), torch.uint8, dev, "codes")
    scales, hs = _out(scales, lead + (C // B,), torch.uint8, dev, "scales")
    rc = lib().quantize_cache_packed(_ptr(values), _DTYPES[values.dtype], rows, C,
                                     _FORMATS[format], B, _ptr(codes), _ptr(scales), _stream(dev))
    _check(rc, "quantize_cache_packed")
    return _result(codes, hc, host), _result(scales, hs, host)


def dequantize_cache_packed(codes, scales, format, block_size, dtype=torch.bfloat16, out=None):
    """Unpack the stored cache form to dtype [..., C] (C from the scales)."""
    if dtype not in _DTYPES:
        raise TypeError("dequantize_cache_packed: unsupported dtype %s" % dtype)
    if format not in _FORMATS:
        raise ValueError("dequantize_cache_packed: format must be one of %s" % sorted(_FORMATS))
    B = int(block_size)
    if (_streamable([codes, scales], [out]) and scales.dim() >= 1 and scales.shape[-1] > 0
            and B >= 1):
        C = scales.shape[-1] * B
        rows = scales.numel() // scales.shape[-1]
        if codes.numel() == rows * (C if format == "fp8" else C // 2):
            ho = _host_target(out, tuple(scales.shape[:-1]) + (C,), dtype, "out")
            dt, fmt = _DTYPES[dtype], _FORMATS[format]
            if _stream_rows([codes, scales], [ho], rows,
                            lambda di, do, n, st: lib().dequantize_cache_packed(
                                _ptr(di[0]), _ptr(di[1]), n, C, fmt, B, _ptr(do[0]), dt, st),
                            "dequantize_cache_packed"):
                return ho
    codes, host = _to_device(codes)
    scales, _ = _to_device(scales, codes.device)
    codes, scales = codes.contiguous(), scales.contiguous()
    C = scales.shape[-1] * B
    rows = scales.numel() // scales.shape[-1] if scales.shape[-1] else 0
    if codes.numel() != rows * (C if format == "fp8" else C // 2):
        raise ValueError("dequantize_cache_packed: codes do not match the scales' shape")
    out, ho = _out(out, tuple(scales.shape[:-1]) + (C,), dtype, codes.device, "out")
    rc = lib().dequantize_cache_packed(_ptr(codes), _ptr(scales), rows, C, _FORMATS[format], B,
                                       _ptr(out), _DTYPES[dtype], _stream(codes.device))
    _check(rc, "dequantize_cache_packed")
    return _result(out, ho, host)


class CacheQuantization(torch.autograd.Function):
    """quantize_cache in the forward pass, the gradient passed through
    unchanged in the backward pass (straight-through estimator)."""

    @staticmethod
    def forward(ctx, values, block_size, format):
        return quantize_cache(values, format, block_size)

    @staticmethod
    def backward(ctx, gradient):
        return gradient, None, None


def mxfp4_grouped_mm(a, packed, scales, offs, transpose_w=False, out=None, status=None):
    """Grouped GEMM over MXFP4-packed expert weights.

    a: bf16 [T, Kin] grouped by expert; packed uint8 [E, N, K/2]; scales
    uint8 [E, N, K/32]; offs int32 [E] (cumulative row counts).
    transpose_w False: Kin = K, returns a . W_e^T [T, N];
    transpose_w True:  Kin = N, returns a . W_e   [T, K].
    status: optional device int32 [1]; a bad offs or a timed-out pipeline
    wait is reported there (the call itself is asynchronous).
    """
    if a.dtype != torch.bfloat16:
        raise TypeError("mxfp4_grouped_mm: activations must be bf16")
    a, host = _to_device(a)
    packed, _ = _to_device(packed, a.device)
    scales, _ = _to_device(scales, a.device)
    offs, _ = _to_device(offs, a.device)
    a, packed, scales = a.contiguous(), packed.contiguous(), scales.contiguous()
    offs = offs.to(torch.int32).contiguous()
    E, N, Kh = packed.shape
    K = 2 * Kh
    T = a.shape[0]
    kin, nout = (N, K) if transpose_w else (K, N)
    if a.shape[1] != kin:
        raise ValueError("mxfp4_grouped_mm: a must be [T, %d]" % kin)
    if tuple(scales.shape) != (E, N, K // 32) or offs.numel() != E:
        raise ValueError("mxfp4_grouped_mm: scales [E, N, K/32] and offs [E] expected")
    out, ho = _out(out, (T, nout), torch.bfloat16, a.device, "out")
    st = _device_word(status, torch.int32, 1, a.device, "status")
    rc = lib().mxfp4_grouped_mm(_ptr(a), _ptr(packed), _ptr(scales), _ptr(offs), T, E, N, K,
                                1 if transpose_w else 0, _ptr(out), st, _stream(a.device))
    _check(rc, "mxfp4_grouped_mm")
    return _result(out, ho, host)


def _quantized_operand(t, shape, dtype, name, what):
    """A quantized activation operand passed by the caller: a contiguous
    device tensor of the given dtype and shape (checked before any launch)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s: %s must be a CUDA tensor" % (what, name))
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError("%s: %s must be a contiguous %s tensor of shape %s"
                         % (what, name, dtype, list(shape)))
    return t


def w4a4_grouped_mm(x, packed, scales, offs, out=None, status=None, x_packed=None,
                    x_scales=None, x_quantized=None):
    """W4A4 grouped GEMM: the bf16 activations x [T, K] are quantized to
    MXFP4 (mx_quantize) and multiplied with the MXFP4 expert weights on the
    block-scaled tensor cores.  Returns bf16 [T, N] (forward only).
    x_packed / x_scales: optional preallocated [T, K/2] / [T, K/32] buffers
    for the quantized activations.
    x_quantized: optional (x_packed, x_scales) device tensors that already
    hold the activations as mx_quantize writes them; then x is not used (it
    may be None) and no quantization runs: the call is the block-scaled GEMM
    alone (the C entry point mxfp4_w4a4_grouped_mm)."""
    if x_quantized is None:
        if x.dtype != torch.bfloat16:
            raise TypeError("w4a4_grouped_mm: activations must be bf16")
        x, host = _to_device(x)
        dev = x.device
    else:
        host = False
        dev = x_quantized[0].device if isinstance(x_quantized[0], torch.Tensor) else None
        if dev is None or dev.type != "cuda":
            raise ValueError("w4a4_grouped_mm: x_quantized must hold CUDA tensors")
    packed, _ = _to_device(packed, dev)
    scales, _ = _to_device(scales, dev)
    offs, _ = _to_device(offs, dev)
    packed, scales = packed.contiguous(), scales.contiguous()
    offs = offs.to(torch.int32).contiguous()
    E, N, Kh = packed.shape
    K = 2 * Kh
    if tuple(scales.shape) != (E, N, K // 32) or offs.numel() != E:
        raise ValueError("w4a4_grouped_mm: scales [E, N, K/32] and offs [E] expected")
    if x_quantized is None:
        x = x.contiguous()
        T = x.shape[0]
        if x.shape[1] != K:
            raise ValueError("w4a4_grouped_mm: x must be [T, %d]" % K)
        for t, name in ((x_packed, "x_packed"), (x_scales, "x_scales")):
            if t is not None and not (t.is_cuda and t.device == dev):
                raise ValueError("w4a4_grouped_mm: %s must be a tensor on %s" % (name, dev))
        xq, xs = mx_quantize(x, x_packed, x_scales)
    else:
        xq, xs = x_quantized
        T = int(xq.shape[0]) if isinstance(xq, torch.Tensor) and xq.dim() == 2 else -1
        xq = _quantized_operand(xq, (T, K // 2), torch.uint8, "x_quantized[0]", "w4a4_grouped_mm")
        xs = _quantized_operand(xs, (T, K // 32), torch.uint8, "x_quantized[1]",
                                "w4a4_grouped_mm")
        if xs.device != dev:
            raise ValueError("w4a4_grouped_mm: x_quantized tensors must share a device")
    out, ho = _out(out, (T, N), torch.bfloat16, dev, "out")
    st = _device_word(status, torch.int32, 1, dev, "status")
    rc = lib().mxfp4_w4a4_grouped_mm(_ptr(xq), _ptr(xs), _ptr(packed), _ptr(scales), _ptr(offs),
                                     T, E, N, K, _ptr(out), st, _stream(dev))
    _check(rc, "mxfp4_w4a4_grouped_mm")
    return _result(out, ho, host)


def nvfp4_w4a4_grouped_mm(x, packed, block_scales, w_global_scales, offs, out=None,
                          status=None, x_quantized=None):
    """W4A4 grouped GEMM in NVFP4: the bf16 activations x [T, K] are
    quantized to NVFP4 as one tensor (nvfp4_quantize) and multiplied with the
    NVFP4 expert weights (packed [E, N, K/2], E4M3 block scales [E, N, K/16],
    float32 global scales [E]) on the block-scaled tensor cores.  Returns
    bf16 [T, N].
    x_quantized: optional (x_packed [T, K/2] uint8, x_block_scales [T, K/16]
    uint8, x_global_scale float32 [1]) device tensors that already hold the
    activations as nvfp4_quantize writes them; then x is not used (it may be
    None) and the call is the block-scaled GEMM alone."""
    if x_quantized is None:
        if x.dtype != torch.bfloat16:
            raise TypeError("nvfp4_w4a4_grouped_mm: activations must be bf16")
        x, host = _to_device(x)
        dev = x.device
    else:
        host = False
        dev = x_quantized[0].device if isinstance(x_quantized[0], torch.Tensor) else None
        if dev is None or dev.type != "cuda":
            raise ValueError("nvfp4_w4a4_grouped_mm: x_quantized must hold CUDA tensors")
    packed, _ = _to_device(packed, dev)
    block_scales, _ = _to_device(block_scales, dev)
    w_global_scales, _ = _to_device(w_global_scales, dev)
    offs, _ = _to_device(offs, dev)
    packed, block_scales = packed.contiguous(), block_scales.contiguous()
    w_global_scales = w_global_scales.to(torch.float32).contiguous()
    offs = offs.to(torch.int32).contiguous()
    E, N, Kh = packed.shape
    K = 2 * Kh
    if (tuple(block_scales.shape) != (E, N, K // 16) or offs.numel() != E or
            w_global_scales.numel() != E):
        raise ValueError("nvfp4_w4a4_grouped_mm: block_scales [E, N, K/16], global scales [E] "
                         "and offs [E] expected")
    if x_quantized is None:
        x = x.contiguous()
        T = x.shape[0]
        if x.shape[1] != K:
            raise ValueError("nvfp4_w4a4_grouped_mm: x must be [T, %d]" % K)
        xq, xs, xg = nvfp4_quantize(x)
    else:
        xq, xs, xg = x_quantized
        T = int(xq.shape[0]) if isinstance(xq, torch.Tensor) and xq.dim() == 2 else -1
        what = "nvfp4_w4a4_grouped_mm"
        xq = _quantized_operand(xq, (T, K // 2), torch.uint8, "x_quantized[0]", what)
        xs = _quantized_operand(xs, (T, K // 16), torch.uint8, "x_quantized[1]", what)
        if isinstance(xg, torch.Tensor) and xg.numel() == 1:
            xg = xg.reshape(1)
        xg = _quantized_operand(xg, (1,), torch.float32, "x_quantized[2]", what)
        if xs.device != dev or xg.device != dev:
            raise ValueError("%s: x_quantized tensors must share a device" % what)
    out, ho = _out(out, (T, N), torch.bfloat16, dev, "out")
    st = _device_word(status, torch.int32, 1, dev, "status")
    rc = lib().nvfp4_w4a4_grouped_mm(_ptr(xq), _ptr(xs), _ptr(xg), _ptr(packed),
                                     _ptr(block_scales), _ptr(w_global_scales), _ptr(offs),
                                     T, E, N, K, _ptr(out), st, _stream(dev))
    _check(rc, "nvfp4_w4a4_grouped_mm")
    return _result(out, ho, host)


NVFP4_WORKSPACE_BYTES = 16


def nvfp4_quantize(x, packed=None, block_scales=None, global_scale=None, workspace=None,
                   rule="max"):
    """NVFP4 two-level quantize + pack along the last dim (K % 16 == 0).

    Returns (packed uint8 [..., K/2], E4M3 block scales uint8 [..., K/16],
    global scale float32 [1]); the per-tensor scale is g = max|x| / 2688.
    rule "max": s_b = E4M3(amax_b / (6 g)); rule "mse": the E4M3 code with
    the least squared weight error per block.
    `workspace` (device uint8, at least NVFP4_WORKSPACE_BYTES) is scratch.
    """
    if x.dtype not in _DTYPES:
        raise TypeError("nvfp4_quantize: unsupported dtype %s" % x.dtype)
    if rule not in ("max", "mse"):
        raise ValueError("nvfp4_quantize: rule must be 'max' or 'mse'")
    x, host = _to_device(x)
    x = x.contiguous()
    K = x.shape[-1]
    rows = x.numel() // K if K else 0
    dev = x.device
    lead = tuple(x.shape[:-1])
    packed, hp = _out(packed, lead + (K // 2,), torch.uint8, dev, "packed")
    block_scales, hb = _out(block_scales, lead + (K // 16,), torch.uint8, dev, "block_scales")
    global_scale, hg = _out(global_scale, (1,), torch.float32, dev, "global_scale")
    if workspace is None:
        workspace = torch.empty(NVFP4_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)
    ws = _device_word(workspace, torch.uint8, NVFP4_WORKSPACE_BYTES, dev, "workspace")
    fn = lib().nvfp4_quantize if rule == "max" else lib().nvfp4_quantize_mse
    rc = fn(_ptr(x), _DTYPES[x.dtype], rows, K, _ptr(packed), _ptr(block_scales),
            _ptr(global_scale), ws, _stream(dev))
    _check(rc, "nvfp4_quantize" if rule == "max" else "nvfp4_quantize_mse")
    return (_result(packed, hp, host), _result(block_scales, hb, host),
            _result(global_scale, hg, host))


def nvfp4_dequantize(packed, block_scales, global_scale, dtype=torch.bfloat16, out=None):
    """Unpack NVFP4 storage: E2M1 code * E4M3 block scale * global scale."""
    if dtype not in _DTYPES:
        raise TypeError("nvfp4_dequantize: unsupported dtype %s" % dtype)
    if (_streamable([packed, block_scales], [out]) and packed.dim() >= 1 and packed.shape[-1] > 0
            and block_scales.numel() * 8 == packed.numel() and global_scale.numel() >= 1):
        K = 2 * packed.shape[-1]
        rows = packed.numel() // packed.shape[-1]
        ho = _host_target(out, tuple(packed.shape[:-1]) + (K,), dtype, "out")
        dev = torch.device("cuda", torch.cuda.current_device())
        gs = global_scale.reshape(-1)[:1].to(device=dev, dtype=torch.float32)
        dt = _DTYPES[dtype]
        if _stream_rows([packed, block_scales], [ho], rows,
                        lambda di, do, n, st: lib().nvfp4_dequantize(
                            _ptr(di[0]), _ptr(di[1]), _ptr(gs), n, K, _ptr(do[0]), dt, st),
                        "nvfp4_dequantize"):
            return ho
    packed, host = _to_device(packed)
    block_scales, _ = _to_device(block_scales, packed.device)
    global_scale, _ = _to_device(global_scale, packed.device)
    packed, block_scales = packed.contiguous(), block_scales.contiguous()
    global_scale = global_scale.to(torch.float32).contiguous()
    Kh = packed.shape[-1]
    K = 2 * Kh
    rows = packed.numel() // Kh if Kh else 0
    if block_scales.numel() != rows * (K // 16):
        raise ValueError("nvfp4_dequantize: block_scales must have shape [..., K/16]")
    if global_scale.numel() < 1:
        raise ValueError("nvfp4_dequantize: global_scale must hold one float32")
    out, ho = _out(out, tuple(packed.shape[:-1]) + (K,), dtype, packed.device, "out")
    rc = lib().nvfp4_dequantize(_ptr(packed), _ptr(block_scales), _ptr(global_scale), rows, K,
                                _ptr(out), _DTYPES[dtype], _stream(packed.device))
    _check(rc, "nvfp4_dequantize")
    return _result(out, ho, host)
