"""B200-native KV-cache format conversion (FP16 <-> FP8 E5M2, FP16 <-> Q4 / Q6).

Thin Python binding over ``libkvq.so`` (C ABI in ``include/kvq.h``).  It only
marshals arguments: it checks dtypes, devices, shapes and contiguity the way
the original extension's host wrappers did (page "Implementation: Turboderp
org Exllamav2 Ext Cache", Description: input kHalf / output kUInt8, scales
kHalf, cache_seqlens and block_table kInt), makes the tensors' device current
and passes torch's current stream.  Every conversion runs in the library's
CUDA kernels; there is no fallback of any kind.  If ``libkvq.so`` is missing,
importing this package raises ``ImportError``.

Names and argument order follow the page's Signature section::

    fp16_to_fp8(in_tensor, out_tensor, batch_size, offset, width)
    fp8_to_fp16(in_tensor, out_tensor, batch_size, offset, width)
    fp16_to_q_kv(k_in, k_out, k_scales, v_in, v_out, v_scales,
                 batch_size, offset, width, page_size, cache_seqlens, block_table, wbits)
    q_to_fp16_kv(k_in, k_out, k_scales, v_in, v_out, v_scales,
                 batch_size, offset, width, page_size, cache_seqlens, block_table, wbits)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["fp16_to_fp8", "fp8_to_fp16", "fp16_to_fp8_kv", "fp8_to_fp16_kv", "fp16_to_q_kv", "q_to_fp16_kv",
           "poll_device_error", "decode_attention_q", "decode_attention_q_noalloc", "decode_attention_fp8",
           "ATTENTION_SCRATCH_BYTES", "count_match", "selfcheck_code_rounding", "selfcheck_wait_timeout",
           "selfcheck_attention_numerics",
           "attention_workspace_bytes", "q_shapes", "set_engine", "get_engine", "engine", "set_attention_path",
           "get_attention_path", "attention_path", "ATTENTION_PATHS", "KVQError",
           "LIB_PATH", "library"]

ENGINES = {"auto": 0, "ldg": 1, "bulk": 2, "ldg_tiled": 3}
ATTENTION_PATHS = {"auto": 0, "mma": 1, "tcgen05": 2}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python __graft_entry__.py` "
                      "or kv_cache_quantization_fp16_b200/_build.py (nvcc, sm_100a)")


class _Desc(ctypes.Structure):
    _fields_ = [("dim0", ctypes.c_int32), ("dim1", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_table_stride", ctypes.c_int32)]


def _i32(x, name: str) -> int:
    """An int argument of the C ABI, refused when it does not fit (ctypes would wrap it)."""
    x = int(x)
    if not -0x80000000 <= x <= 0x7FFFFFFF:
        raise ValueError(f"{name} = {x} does not fit the library's int32 argument")
    return x


def _i32s(**args) -> tuple:
    """_i32 of each keyword argument, in order."""
    return tuple(_i32(v, k) for k, v in args.items())


def _desc(d0, d1, H, D, stride) -> _Desc:
    """The cache descriptor, after checking that every field fits its int32 (ctypes would
    wrap a larger value silently into a different geometry)."""
    for name, x in (("dim0", d0), ("dim1", d1), ("kv_heads", H), ("head_dim", D), ("block_table_stride", stride)):
        if not 0 <= int(x) <= 0x7FFFFFFF:
            raise ValueError(f"{name} = {int(x)} does not fit the library's int32 cache descriptor")
    return _Desc(int(d0), int(d1), int(H), int(D), int(stride))


_STATUS = {0: "ok", 1: "null pointer", 2: "bad shape", 3: "wbits must be 4, 6 or 8",
           4: "window, batch or page geometry out of range", 5: "buffer not 16-byte aligned",
           6: "CUDA runtime error", 7: "device recorded bad paging metadata"}


class KVQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: kvq status {status} ({_STATUS.get(status, 'unknown')})")


def _load() -> ctypes.CDLL:
    L = ctypes.CDLL(LIB_PATH)
    vp, I = ctypes.c_void_p, ctypes.c_int
    dp = ctypes.POINTER(_Desc)
    L.kvq_fp16_to_fp8.argtypes = [vp, vp, dp, I, I, I, vp]
    L.kvq_fp8_to_fp16.argtypes = [vp, vp, dp, I, I, I, vp]
    L.kvq_fp16_to_fp8_kv.argtypes = [vp, vp, vp, vp, dp, I, I, I, I, vp, vp, vp]
    L.kvq_fp8_to_fp16_kv.argtypes = [vp, vp, vp, vp, dp, I, I, I, I, vp, vp, vp]
    L.kvq_fp16_to_q_kv.argtypes = [vp, vp, vp, vp, vp, vp, dp, I, I, I, I, vp, vp, I, vp]
    L.kvq_q_to_fp16_kv.argtypes = [vp, vp, vp, vp, vp, vp, dp, I, I, I, I, vp, vp, I, vp]
    L.kvq_status_string.argtypes = [I]
    L.kvq_status_string.restype = ctypes.c_char_p
    L.kvq_poll_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    L.kvq_selfcheck_code_rounding.argtypes = [I, vp, vp]
    L.kvq_selfcheck_wait_timeout.argtypes = [vp, vp]
    L.kvq_selfcheck_attention_numerics.argtypes = [vp, vp]
    LL = ctypes.c_longlong
    L.kvq_decode_attention_q.argtypes = [vp, vp, vp, vp, vp, vp, dp, I, I, I, vp, vp, I, ctypes.c_float, vp,
                                         ctypes.c_size_t, vp]
    L.kvq_decode_attention_q.restype = I
    L.kvq_decode_attention_fp8.argtypes = [vp, vp, vp, vp, dp, I, I, I, vp, vp, ctypes.c_float, vp, ctypes.c_size_t,
                                           vp]
    L.kvq_decode_attention_fp8.restype = I
    L.kvq_decode_attention_q_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, dp, I, I, I, vp, vp, I, ctypes.c_float,
                                                 vp]
    L.kvq_decode_attention_q_noalloc.restype = I
    L.kvq_decode_attention_workspace_size.argtypes = [dp, I, I, I]
    L.kvq_decode_attention_workspace_size.restype = ctypes.c_size_t
    L.kvq_count_match.argtypes = [vp, LL, vp, LL, LL]
    L.kvq_count_match.restype = LL
    L.kvq_set_engine.argtypes = [I]
    L.kvq_get_engine.argtypes = []
    L.kvq_get_engine.restype = I
    L.kvq_set_attention_path.argtypes = [I]
    L.kvq_set_attention_path.restype = I
    L.kvq_get_attention_path.argtypes = []
    L.kvq_get_attention_path.restype = I
    for f in ("kvq_fp16_to_fp8", "kvq_fp8_to_fp16", "kvq_fp16_to_fp8_kv", "kvq_fp8_to_fp16_kv",
              "kvq_fp16_to_q_kv", "kvq_q_to_fp16_kv",
              "kvq_poll_device_error", "kvq_selfcheck_code_rounding", "kvq_selfcheck_wait_timeout",
              "kvq_selfcheck_attention_numerics", "kvq_set_engine"):
        getattr(L, f).restype = I
    return L


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def _check(st: int, where: str) -> None:
    if st != 0:
        raise KVQError(st, where)


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _cuda4(t: torch.Tensor, dtype, name: str) -> None:
    _require(isinstance(t, torch.Tensor), f"{name} must be a tensor")
    _require(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    _require(t.is_cuda, f"{name} must be a CUDA tensor")
    _require(t.dim() == 4, f"{name} must be 4-D, got shape {tuple(t.shape)}")
    _require(t.is_contiguous(), f"{name} must be contiguous")


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def q_shapes(shape, wbits: int):
    """Shapes of the code and scale tensors for an FP16 cache of shape [d0, d1, H, D]."""
    d0, d1, H, D = shape
    return (d0, d1, H, D * wbits // 8), (d0, d1, H, D // 32)


def _fp8(fn, in_tensor, out_tensor, batch_size, offset, width, in_dtype, out_dtype, where):
    batch_size, offset, width = _i32s(batch_size=batch_size, offset=offset, width=width)
    _cuda4(in_tensor, in_dtype, "in_tensor")
    _cuda4(out_tensor, out_dtype, "out_tensor")
    _require(in_tensor.shape == out_tensor.shape, "in_tensor and out_tensor must have the same shape")
    _require(in_tensor.device == out_tensor.device, "tensors must be on one device")
    d0, d1, H, D = in_tensor.shape
    desc = _desc(d0, d1, H, D, 0)
    with torch.cuda.device(in_tensor.device):
        st = fn(in_tensor.data_ptr(), out_tensor.data_ptr(), ctypes.byref(desc), int(batch_size),
                int(offset), int(width), _stream(in_tensor.device))
    _check(st, where)


def fp16_to_fp8(in_tensor: torch.Tensor, out_tensor: torch.Tensor, batch_size: int, offset: int,
                width: int) -> None:
    """Encode the FP16 cache window into E5M2 bytes (out_tensor: uint8, same shape)."""
    _fp8(_lib.kvq_fp16_to_fp8, in_tensor, out_tensor, batch_size, offset, width, torch.float16,
         torch.uint8, "fp16_to_fp8")


def fp8_to_fp16(in_tensor: torch.Tensor, out_tensor: torch.Tensor, batch_size: int, offset: int,
                width: int) -> None:
    """Decode the E5M2 cache window back into FP16 (out_tensor: float16, same shape)."""
    _fp8(_lib.kvq_fp8_to_fp16, in_tensor, out_tensor, batch_size, offset, width, torch.uint8,
         torch.float16, "fp8_to_fp16")


def _paging(page_size, cache_seqlens, block_table, batch_size, dev):
    """Checks of the paged-mode metadata (kInt tensors on the caches' device)."""
    if not page_size:
        return 0, None, None
    _require(cache_seqlens is not None and block_table is not None,
             "paged mode needs cache_seqlens and block_table")
    _require(cache_seqlens.dtype == torch.int32 and block_table.dtype == torch.int32,
             "cache_seqlens and block_table must be int32")
    _require(cache_seqlens.device == dev and block_table.device == dev, "tensors must be on one device")
    _require(block_table.dim() == 2 and block_table.is_contiguous() and cache_seqlens.is_contiguous(),
             "block_table must be a contiguous [batch, max_pages] tensor")
    _require(cache_seqlens.numel() >= batch_size and block_table.shape[0] >= batch_size,
             "cache_seqlens / block_table have fewer rows than batch_size")
    return block_table.shape[1], cache_seqlens.data_ptr(), block_table.data_ptr()


def _fp8_kv(fn, k_in, k_out, v_in, v_out, batch_size, offset, width, page_size, cache_seqlens, block_table,
            in_dtype, out_dtype, where):
    batch_size, offset, width, page_size = _i32s(batch_size=batch_size, offset=offset, width=width, page_size=page_size)
    for t, n in ((k_in, "k_in"), (v_in, "v_in")):
        _cuda4(t, in_dtype, n)
    for t, n in ((k_out, "k_out"), (v_out, "v_out")):
        _cuda4(t, out_dtype, n)
    _require(k_in.shape == k_out.shape == v_in.shape == v_out.shape, "K and V caches must share one shape")
    dev = k_in.device
    for t in (k_out, v_in, v_out):
        _require(t.device == dev, "tensors must be on one device")
    stride, sl_ptr, bt_ptr = _paging(page_size, cache_seqlens, block_table, batch_size, dev)
    d0, d1, H, D = k_in.shape
    desc = _desc(d0, d1, H, D, stride)
    with torch.cuda.device(dev):
        st = fn(k_in.data_ptr(), k_out.data_ptr(), v_in.data_ptr(), v_out.data_ptr(), ctypes.byref(desc),
                int(batch_size), int(offset), int(width), int(page_size), sl_ptr, bt_ptr, _stream(dev))
    _check(st, where)


def fp16_to_fp8_kv(k_in, k_out, v_in, v_out, batch_size, offset, width, page_size=0, cache_seqlens=None,
                   block_table=None) -> None:
    """E5M2-encode the K and V FP16 cache windows in one launch, contiguous or paged
    (an extension of fp16_to_fp8 with the window and page rules of fp16_to_q_kv)."""
    _fp8_kv(_lib.kvq_fp16_to_fp8_kv, k_in, k_out, v_in, v_out, batch_size, offset, width, page_size,
            cache_seqlens, block_table, torch.float16, torch.uint8, "fp16_to_fp8_kv")


def fp8_to_fp16_kv(k_in, k_out, v_in, v_out, batch_size, offset, width, page_size=0, cache_seqlens=None,
                   block_table=None) -> None:
    """Decode the K and V E5M2 cache windows into FP16 in one launch, contiguous or paged."""
    _fp8_kv(_lib.kvq_fp8_to_fp16_kv, k_in, k_out, v_in, v_out, batch_size, offset, width, page_size,
            cache_seqlens, block_table, torch.uint8, torch.float16, "fp8_to_fp16_kv")


def _q(fn, fp16_is_input, k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset, width,
       page_size, cache_seqlens, block_table, wbits, where):
    batch_size, offset, width, page_size, wbits = _i32s(
        batch_size=batch_size, offset=offset, width=width, page_size=page_size, wbits=wbits)
    k16, kq = (k_in, k_out) if fp16_is_input else (k_out, k_in)
    v16, vq = (v_in, v_out) if fp16_is_input else (v_out, v_in)
    for t, n in ((k16, "FP16 K"), (v16, "FP16 V")):
        _cuda4(t, torch.float16, n)
    for t, n in ((kq, "K codes"), (vq, "V codes")):
        _cuda4(t, torch.uint8, n)
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _cuda4(t, torch.float16, n)
    _require(k16.shape == v16.shape, "K and V caches must have the same shape")
    _require(wbits in (4, 6, 8), f"wbits must be 4, 6 or 8, got {wbits}")
    _require(k16.shape[3] % 32 == 0, "head_dim must be a multiple of 32")
    cshape, sshape = q_shapes(tuple(k16.shape), wbits)
    for t, n in ((kq, "K codes"), (vq, "V codes")):
        _require(tuple(t.shape) == cshape, f"{n} must have shape {cshape}, got {tuple(t.shape)}")
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _require(tuple(t.shape) == sshape, f"{n} must have shape {sshape}, got {tuple(t.shape)}")
    dev = k16.device
    for t in (kq, v16, vq, k_scales, v_scales):
        _require(t.device == dev, "tensors must be on one device")
    stride, sl_ptr, bt_ptr = _paging(page_size, cache_seqlens, block_table, batch_size, dev)
    d0, d1, H, D = k16.shape
    desc = _desc(d0, d1, H, D, stride)
    with torch.cuda.device(dev):
        st = fn(k_in.data_ptr(), k_out.data_ptr(), k_scales.data_ptr(), v_in.data_ptr(), v_out.data_ptr(),
                v_scales.data_ptr(), ctypes.byref(desc), int(batch_size), int(offset), int(width),
                int(page_size), sl_ptr, bt_ptr, int(wbits), _stream(dev))
    _check(st, where)


def fp16_to_q_kv(k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset, width,
                 page_size=0, cache_seqlens=None, block_table=None, wbits=4) -> None:
    """Quantize the K and V FP16 cache windows to wbits-bit codes + FP16 scales (one launch)."""
    _q(_lib.kvq_fp16_to_q_kv, True, k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset,
       width, page_size, cache_seqlens, block_table, wbits, "fp16_to_q_kv")


def q_to_fp16_kv(k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset, width,
                 page_size=0, cache_seqlens=None, block_table=None, wbits=4) -> None:
    """Dequantize the K and V code windows back into the FP16 caches (one launch)."""
    _q(_lib.kvq_q_to_fp16_kv, False, k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset,
       width, page_size, cache_seqlens, block_table, wbits, "q_to_fp16_kv")


def poll_device_error(device=None) -> int:
    """Synchronize the current stream and return (and clear) the device error code (0 = none)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        st = _lib.kvq_poll_device_error(ctypes.byref(code), _stream(dev))
    if st not in (0, 7):
        raise KVQError(st, "poll_device_error")
    return int(code.value)


def selfcheck_code_rounding(wbits: int, device=None) -> int:
    """Number of (x, s) binary16 pairs where the kernels' fast code rounding differs from
    IEEE division + rint + clamp (0 expected)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.zeros(1, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        st = _lib.kvq_selfcheck_code_rounding(int(wbits), out.data_ptr(), _stream(dev))
    _check(st, "selfcheck_code_rounding")
    return int(out.item())


def selfcheck_attention_numerics(device=None) -> dict:
    """The arithmetic constants the decode-attention error bound rests on, measured on the
    device: the largest relative error of the softmax's hardware 2^x approximation over
    [-126, 8] (``ex2_rel``), of exp2f over [-126, 0] (``exp2f_rel``), and the largest
    error of one mma.sync accumulation step in units of 2^-23 times its largest term
    (``mma_step_ulps``)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.zeros(3, dtype=torch.float64, device=dev)
    with torch.cuda.device(dev):
        st = _lib.kvq_selfcheck_attention_numerics(out.data_ptr(), _stream(dev))
    _check(st, "selfcheck_attention_numerics")
    r = out.cpu().tolist()
    return {"ex2_rel": r[0], "exp2f_rel": r[1], "mma_step_ulps": r[2]}


def selfcheck_wait_timeout(device=None) -> int:
    """Run the bulk engine's bounded wait against an mbarrier nothing arrives on (about
    1 s).  Returns 1 when the wait gave up as designed; the device error word then holds
    KVQ_DEV_TIMEOUT (read it with poll_device_error)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.full((1,), -1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.kvq_selfcheck_wait_timeout(out.data_ptr(), _stream(dev))
    _check(st, "selfcheck_wait_timeout")
    return int(out.item())


def set_engine(name: str) -> None:
    """Select the load engine for all later conversions: "auto" (default: the engine
    measured faster for each operation), "ldg" (plain 16-byte loads; contiguous: one tile
    per CTA, paged: one wave of CTAs over equal shares of all windows), "bulk" (TMA bulk
    copies into a shared-memory pipeline) or "ldg_tiled" (plain loads, per-sequence tiles
    in paged mode too)."""
    _check(_lib.kvq_set_engine(ENGINES[name]), "set_engine")


def get_engine() -> str:
    code = _lib.kvq_get_engine()
    return {v: k for k, v in ENGINES.items()}[code]


class engine:
    """Context manager: ``with engine("bulk"): ...`` selects an engine temporarily."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        self.prev = get_engine()
        set_engine(self.name)
        return self

    def __exit__(self, *exc):
        set_engine(self.prev)
        return False


def set_attention_path(name: str) -> None:
    """Select the decode-attention kernel for all later calls: "auto" (default), "mma"
    (warp-level mma.sync tiles) or "tcgen05" (fifth-generation tensor cores with
    tensor-memory accumulators, for head_dim 128 and batches of up to 256 sequences;
    other geometries run the mma.sync kernel)."""
    _check(_lib.kvq_set_attention_path(ATTENTION_PATHS[name]), "set_attention_path")


def get_attention_path() -> str:
    return {v: k for k, v in ATTENTION_PATHS.items()}[_lib.kvq_get_attention_path()]


class attention_path:
    """Context manager: ``with attention_path("mma"): ...`` selects a decode-attention
    kernel temporarily."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        self.prev = get_attention_path()
        set_attention_path(self.name)
        return self

    def __exit__(self, *exc):
        set_attention_path(self.prev)
        return False


def count_match(a: torch.Tensor, b: torch.Tensor, max_a: int) -> int:
    """Length of the matching prefix of two 1-D int64 CPU tensors (e.g. token ids),
    comparing at most max_a elements (page Description: count_match)."""
    for t, n in ((a, "a"), (b, "b")):
        _require(isinstance(t, torch.Tensor) and t.dtype == torch.int64 and t.dim() == 1,
                 f"{n} must be a 1-D int64 tensor")
        _require(t.device.type == "cpu", f"{n} must be a CPU tensor")
    a, b = a.contiguous(), b.contiguous()
    n = _lib.kvq_count_match(a.data_ptr() if a.numel() else None, a.numel(),
                             b.data_ptr() if b.numel() else None, b.numel(), int(max_a))
    if n < 0:
        raise KVQError(1, "count_match")
    return int(n)


_SIZE_MAX = (1 << (8 * ctypes.sizeof(ctypes.c_size_t))) - 1  # the workspace size query's overflow value


def attention_workspace_bytes(cache_shape, batch_size: int, n_heads: int, page_size: int = 0,
                              block_table_stride: int = 0) -> int:
    """Workspace bytes decode_attention_q needs: cache_shape is the FP16 cache shape
    [d0, d1, kv_heads, head_dim] the codes were made from."""
    batch_size, n_heads, page_size = _i32s(batch_size=batch_size, n_heads=n_heads, page_size=page_size)
    d0, d1, H, D = cache_shape
    desc = _desc(d0, d1, H, D, block_table_stride if page_size else 0)
    return int(_lib.kvq_decode_attention_workspace_size(ctypes.byref(desc), int(batch_size), int(n_heads),
                                                        int(page_size)))


def decode_attention_q(q, k_codes, k_scales, v_codes, v_scales, out, batch_size, cache_seqlens, wbits,
                       softmax_scale, page_size=0, block_table=None, workspace=None) -> None:
    """Decode attention reading the quantized cache directly (no FP16 cache is written).

    q, out: [batch, n_heads, head_dim] float16 CUDA tensors; codes / scales as written by
    fp16_to_q_kv ([d0, d1, kv_heads, head_dim * wbits / 8] uint8, [d0, d1, kv_heads,
    head_dim / 32] float16); cache_seqlens [batch] int32 (positions [0, len) are attended);
    paged mode with page_size > 0 and block_table.  ``workspace`` is a CUDA uint8 tensor of at
    least attention_workspace_bytes(...) bytes; when omitted one is allocated with torch."""
    batch_size, page_size, wbits = _i32s(batch_size=batch_size, page_size=page_size, wbits=wbits)
    _require(isinstance(q, torch.Tensor) and q.dtype == torch.float16 and q.is_cuda and q.dim() == 3
             and q.is_contiguous(), "q must be a contiguous [batch, n_heads, head_dim] float16 CUDA tensor")
    _require(out.shape == q.shape and out.dtype == torch.float16 and out.is_contiguous() and out.device == q.device,
             "out must match q")
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _cuda4(t, torch.uint8, n)
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _cuda4(t, torch.float16, n)
    _require(wbits in (4, 6, 8), f"wbits must be 4, 6 or 8, got {wbits}")
    D = q.shape[2]
    cshape, sshape = q_shapes((*k_codes.shape[:3], D), wbits)
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _require(tuple(t.shape) == cshape, f"{n} must have shape {cshape}, got {tuple(t.shape)}")
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _require(tuple(t.shape) == sshape, f"{n} must have shape {sshape}, got {tuple(t.shape)}")
    dev = q.device
    for t in (k_codes, k_scales, v_codes, v_scales):
        _require(t.device == dev, "tensors must be on one device")
    _require(cache_seqlens is not None and cache_seqlens.dtype == torch.int32 and cache_seqlens.device == dev
             and cache_seqlens.is_contiguous() and cache_seqlens.numel() >= batch_size,
             "cache_seqlens must be a contiguous int32 tensor on the caches' device with batch_size entries")
    stride, _, bt_ptr = _paging(page_size, cache_seqlens, block_table, batch_size, dev)
    d0, d1, H, _ = k_codes.shape
    desc = _desc(d0, d1, H, D, stride)
    n_heads = q.shape[1]
    need = int(_lib.kvq_decode_attention_workspace_size(ctypes.byref(desc), int(batch_size), int(n_heads),
                                                        int(page_size)))
    _require(need < _SIZE_MAX, "the workspace this geometry needs does not fit in size_t")
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _require(workspace.is_cuda and workspace.device == dev and workspace.numel() >= need,
             f"workspace must hold at least {need} bytes on the caches' device")
    with torch.cuda.device(dev):
        st = _lib.kvq_decode_attention_q(q.data_ptr(), k_codes.data_ptr(), k_scales.data_ptr(), v_codes.data_ptr(),
                                         v_scales.data_ptr(), out.data_ptr(), ctypes.byref(desc), int(batch_size),
                                         int(n_heads), int(page_size), cache_seqlens.data_ptr(), bt_ptr, int(wbits),
                                         float(softmax_scale), workspace.data_ptr(), workspace.numel(), _stream(dev))
    _check(st, "decode_attention_q")


def decode_attention_fp8(q, k_fp8, v_fp8, out, batch_size, cache_seqlens, softmax_scale, page_size=0,
                         block_table=None, workspace=None) -> None:
    """Decode attention reading an FP8 (E5M2) cache directly, the bytes decoded exactly as
    fp8_to_fp16 does (no FP16 cache is written).

    q, out: [batch, n_heads, head_dim] float16 CUDA tensors; k_fp8, v_fp8: [d0, d1, kv_heads,
    head_dim] uint8 as written by fp16_to_fp8 / fp16_to_fp8_kv; cache_seqlens, paging and
    ``workspace`` as for decode_attention_q."""
    batch_size, page_size = _i32s(batch_size=batch_size, page_size=page_size)
    _require(isinstance(q, torch.Tensor) and q.dtype == torch.float16 and q.is_cuda and q.dim() == 3
             and q.is_contiguous(), "q must be a contiguous [batch, n_heads, head_dim] float16 CUDA tensor")
    _require(out.shape == q.shape and out.dtype == torch.float16 and out.is_contiguous() and out.device == q.device,
             "out must match q")
    D = q.shape[2]
    for t, n in ((k_fp8, "k_fp8"), (v_fp8, "v_fp8")):
        _cuda4(t, torch.uint8, n)
        _require(t.shape[3] == D and t.device == q.device, f"{n} must be [d0, d1, kv_heads, {D}] on q's device")
    _require(k_fp8.shape == v_fp8.shape, "k_fp8 and v_fp8 must have one shape")
    dev = q.device
    _require(cache_seqlens is not None and cache_seqlens.dtype == torch.int32 and cache_seqlens.device == dev
             and cache_seqlens.is_contiguous() and cache_seqlens.numel() >= batch_size,
             "cache_seqlens must be a contiguous int32 tensor on the caches' device with batch_size entries")
    stride, _, bt_ptr = _paging(page_size, cache_seqlens, block_table, batch_size, dev)
    d0, d1, H, _ = k_fp8.shape
    desc = _desc(d0, d1, H, D, stride)
    n_heads = q.shape[1]
    need = int(_lib.kvq_decode_attention_workspace_size(ctypes.byref(desc), int(batch_size), int(n_heads),
                                                        int(page_size)))
    _require(need < _SIZE_MAX, "the workspace this geometry needs does not fit in size_t")
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _require(workspace.is_cuda and workspace.device == dev and workspace.numel() >= need,
             f"workspace must hold at least {need} bytes on the caches' device")
    with torch.cuda.device(dev):
        st = _lib.kvq_decode_attention_fp8(q.data_ptr(), k_fp8.data_ptr(), v_fp8.data_ptr(), out.data_ptr(),
                                           ctypes.byref(desc), int(batch_size), int(n_heads), int(page_size),
                                           cache_seqlens.data_ptr(), bt_ptr, float(softmax_scale),
                                           workspace.data_ptr(), workspace.numel(), _stream(dev))
    _check(st, "decode_attention_fp8")


ATTENTION_SCRATCH_BYTES = 32 << 20  # KVQ_ATTENTION_SCRATCH_BYTES


def decode_attention_q_noalloc(q, k_codes, k_scales, v_codes, v_scales, out, batch_size, cache_seqlens, wbits,
                               softmax_scale, page_size=0, block_table=None) -> None:
    """decode_attention_q for callers that cannot allocate device memory at the call
    site: the workspace is the library's own 32 MiB array (one per device), so nothing is
    allocated, by torch or by CUDA.  Geometries needing more workspace than
    ATTENTION_SCRATCH_BYTES are rejected.  Calls that overlap on the GPU share the array
    and race; make the first call on a device before any stream capture."""
    batch_size, page_size, wbits = _i32s(batch_size=batch_size, page_size=page_size, wbits=wbits)
    _require(isinstance(q, torch.Tensor) and q.dtype == torch.float16 and q.is_cuda and q.dim() == 3
             and q.is_contiguous(), "q must be a contiguous [batch, n_heads, head_dim] float16 CUDA tensor")
    _require(out.shape == q.shape and out.dtype == torch.float16 and out.is_contiguous() and out.device == q.device,
             "out must match q")
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _cuda4(t, torch.uint8, n)
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _cuda4(t, torch.float16, n)
    _require(wbits in (4, 6, 8), f"wbits must be 4, 6 or 8, got {wbits}")
    D = q.shape[2]
    cshape, sshape = q_shapes((*k_codes.shape[:3], D), wbits)
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _require(tuple(t.shape) == cshape, f"{n} must have shape {cshape}, got {tuple(t.shape)}")
    for t, n in ((k_scales, "k_scales"), (v_scales, "v_scales")):
        _require(tuple(t.shape) == sshape, f"{n} must have shape {sshape}, got {tuple(t.shape)}")
    dev = q.device
    for t in (k_codes, k_scales, v_codes, v_scales):
        _require(t.device == dev, "tensors must be on one device")
    _require(cache_seqlens is not None and cache_seqlens.dtype == torch.int32 and cache_seqlens.device == dev
             and cache_seqlens.is_contiguous() and cache_seqlens.numel() >= batch_size,
             "cache_seqlens must be a contiguous int32 tensor on the caches' device with batch_size entries")
    stride, _, bt_ptr = _paging(page_size, cache_seqlens, block_table, batch_size, dev)
    d0, d1, H, _ = k_codes.shape
    desc = _desc(d0, d1, H, D, stride)
    n_heads = q.shape[1]
    need = int(_lib.kvq_decode_attention_workspace_size(ctypes.byref(desc), int(batch_size), int(n_heads),
                                                        int(page_size)))
    _require(need <= ATTENTION_SCRATCH_BYTES,
             f"this geometry needs {need} bytes of workspace, above the {ATTENTION_SCRATCH_BYTES}-byte scratch array")
    with torch.cuda.device(dev):
        st = _lib.kvq_decode_attention_q_noalloc(q.data_ptr(), k_codes.data_ptr(), k_scales.data_ptr(),
                                                 v_codes.data_ptr(), v_scales.data_ptr(), out.data_ptr(),
                                                 ctypes.byref(desc), int(batch_size), int(n_heads), int(page_size),
                                                 cache_seqlens.data_ptr(), bt_ptr, int(wbits), float(softmax_scale),
                                                 _stream(dev))
    _check(st, "decode_attention_q_noalloc")
