"""Thin Python binding of the C-ABI library libtq.so (include/tq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory (``tensor.data_ptr()``) and the
stream (``torch.cuda.current_stream().cuda_stream``).  Function names match
the C entry points.  There is no fallback: if libtq.so is missing, loading
raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK = 0
STATUS = {0: "TQ_OK", 1: "TQ_ERR_INVALID_ARGUMENT", 2: "TQ_ERR_UNSUPPORTED",
          3: "TQ_ERR_CAPACITY", 4: "TQ_ERR_WORKSPACE", 5: "TQ_ERR_CUDA",
          6: "TQ_ERR_INTERNAL"}
TQ_F32, TQ_BF16 = 0, 1
TQ_VALUES_GROUP, TQ_VALUES_MSE = 0, 1
TILE_TOKENS = 128
MAX_BATCH = 1024

# Every function include/tq.h declares.
EXPORTS = ("tq_status_string", "tq_make_codebook", "tq_record_bytes", "tq_cache_bytes",
           "tq_quantize_append", "tq_decode_workspace_size", "tq_decode_attention",
           "tq_dequantize", "tq_decode_attention_noalloc", "tq_decode_attention_window",
           "tq_prefill_workspace_size", "tq_prefill_attention", "tq_prefill_tokens_per_pass",
           "tq_set_wait_limit_ns", "tq_device_errors", "tq_test_withhold_handoffs",
           "tq_test_sign_refine_threshold", "tq_test_refine_count", "tq_sketch_product", "tq_prepare_operands")
ERRF_DECODE_WAIT, ERRF_QUANTIZE_WAIT = 1, 2
NOALLOC_SCRATCH_BYTES = 8 << 20


class TQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("key_bits", ctypes.c_int),
                ("value_bits", ctypes.c_int), ("group", ctypes.c_int),
                ("pi", ctypes.c_void_p), ("s", ctypes.c_void_p),
                ("centroids", ctypes.c_void_p), ("boundaries", ctypes.c_void_p),
                ("value_mode", ctypes.c_int), ("v_centroids", ctypes.c_void_p),
                ("v_boundaries", ctypes.c_void_p), ("s_pit", ctypes.c_void_p),
                ("tc_operands", ctypes.c_void_p)]

TQ_TC_OPERAND_BYTES = 5 * 128 * 128 * 2


class Cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("h_kv", ctypes.c_int),
                ("capacity", ctypes.c_int), ("data", ctypes.c_void_p)]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libtq.so (once) and declare its prototypes."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} not built; run python -m kv_cache_quantization_turboquantprod_b200.build")
    lib = ctypes.CDLL(p)
    P, C = ctypes.POINTER(Params), ctypes.POINTER(Cache)
    i32p = ctypes.POINTER(ctypes.c_int32)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.tq_status_string.restype = ctypes.c_char_p
    lib.tq_status_string.argtypes = [ci]
    lib.tq_make_codebook.restype = ci
    lib.tq_make_codebook.argtypes = [ci, ci, ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_double)]
    lib.tq_record_bytes.restype = sz
    lib.tq_record_bytes.argtypes = [P]
    lib.tq_sketch_product.restype = ci
    lib.tq_sketch_product.argtypes = [P, vp, vp]
    lib.tq_prepare_operands.restype = ci
    lib.tq_prepare_operands.argtypes = [P, vp, vp]
    lib.tq_cache_bytes.restype = sz
    lib.tq_cache_bytes.argtypes = [P, ci, ci, ci]
    lib.tq_quantize_append.restype = ci
    lib.tq_quantize_append.argtypes = [P, C, vp, vp, ci, ci, i32p, i32p, vp]
    lib.tq_decode_workspace_size.restype = sz
    lib.tq_decode_workspace_size.argtypes = [P, C, ci, ci]
    lib.tq_decode_attention.restype = ci
    lib.tq_decode_attention.argtypes = [P, C, vp, ci, ci, vp, ci, ctypes.c_float, vp, vp, sz, vp]
    lib.tq_decode_attention_noalloc.restype = ci
    lib.tq_decode_attention_noalloc.argtypes = [P, C, vp, ci, ci, vp, ci, ctypes.c_float, vp, vp]
    lib.tq_decode_attention_window.restype = ci
    lib.tq_decode_attention_window.argtypes = [P, C, vp, ci, ci, vp, ci, vp, vp, ci, vp, ci,
                                               ctypes.c_float, vp, vp, sz, vp]
    lib.tq_prefill_workspace_size.restype = sz
    lib.tq_prefill_workspace_size.argtypes = [P, C, ci, ci, ci]
    lib.tq_prefill_tokens_per_pass.restype = ci
    lib.tq_prefill_tokens_per_pass.argtypes = [P, ci, ci, ci]
    lib.tq_prefill_attention.restype = ci
    lib.tq_prefill_attention.argtypes = [P, C, vp, ci, ci, ci, vp, ci, ctypes.c_float, vp, vp, sz, vp]
    lib.tq_dequantize.restype = ci
    lib.tq_dequantize.argtypes = [P, C, ci, ci, ci, vp, vp, vp]
    lib.tq_set_wait_limit_ns.restype = ci
    lib.tq_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.tq_test_withhold_handoffs.restype = ci
    lib.tq_test_withhold_handoffs.argtypes = [ci]
    lib.tq_test_sign_refine_threshold.restype = ci
    lib.tq_test_sign_refine_threshold.argtypes = [ctypes.c_double]
    lib.tq_test_refine_count.restype = ci
    lib.tq_test_refine_count.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ci]
    lib.tq_device_errors.restype = ci
    lib.tq_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), ci]
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, st: int) -> None:
    if st != TQ_OK:
        raise TQError(fn, st)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_rows(name: str, t: torch.Tensor, shape, dtypes, device=None) -> None:
    """Shape, dtype, contiguity and device of a tensor handed to the C ABI,
    which cannot check buffer sizes itself."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda or (device is not None and t.device != device):
        raise ValueError(f"{name} must be a CUDA tensor on the cache's device")


def _check_decode_io(cache, q: torch.Tensor, len_dev: torch.Tensor, out: torch.Tensor) -> int:
    """q [B, H_q, d] fp32/bf16, len_dev [B] int32, out [B, H_q, d] fp32, all
    contiguous on the cache's device; returns H_q."""
    if q.dim() != 3:
        raise ValueError("q must be [B, H_q, d]")
    dev = cache.buffer.device
    B, hq, d = cache.batch, int(q.shape[1]), int(q.shape[2])
    _check_rows("q", q, (B, hq, d), (torch.float32, torch.bfloat16), dev)
    _check_rows("len_dev", len_dev, (B,), (torch.int32,), dev)
    _check_rows("out", out, (B, hq, d), (torch.float32,), dev)
    return hq


def _i32_array(xs):
    arr = (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])
    return arr


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def tq_status_string(status: int) -> str:
    return load().tq_status_string(int(status)).decode()


def tq_make_codebook(mse_bits: int, d: int):
    """Host-only Lloyd-Max codebook: (centroids [2^b], boundaries [2^b - 1]) as
    Python float lists."""
    n = 1 << mse_bits if 1 <= mse_bits <= 4 else 1
    c = (ctypes.c_double * n)()
    b = (ctypes.c_double * max(n - 1, 1))()
    _check("tq_make_codebook", load().tq_make_codebook(mse_bits, d, c, b))
    return list(c), list(b)[: n - 1]


class Layer:
    """Device-resident constants of one layer (Pi, S, codebooks) packaged as
    the C struct tq_params.  Holds references to the tensors it points to.
    value_mode "group" (min/max groups of 32) or "mse" (TurboQuant-MSE values
    with the value_bits Lloyd-Max codebook)."""

    def __init__(self, pi, s, key_bits: int, value_bits: int, group: int = 32,
                 device="cuda", value_mode: str = "group"):
        d = int(pi.shape[0])
        cent, bnd = tq_make_codebook(key_bits - 1, d)
        self.pi = torch.as_tensor(pi, dtype=torch.float32).contiguous().to(device)
        self.s = torch.as_tensor(s, dtype=torch.float32).contiguous().to(device)
        self.centroids = torch.tensor(cent, dtype=torch.float32, device=device)
        self.boundaries = torch.tensor(bnd if bnd else [0.0], dtype=torch.float32, device=device)
        self.codebook = (cent, bnd)
        self.value_mode = value_mode
        mode = {"group": TQ_VALUES_GROUP, "mse": TQ_VALUES_MSE}[value_mode]
        vc_ptr = vb_ptr = None
        if mode == TQ_VALUES_MSE:
            vcent, vbnd = tq_make_codebook(value_bits, d)
            self.v_centroids = torch.tensor(vcent, dtype=torch.float32, device=device)
            self.v_boundaries = torch.tensor(vbnd, dtype=torch.float32, device=device)
            self.value_codebook = (vcent, vbnd)
            vc_ptr, vb_ptr = self.v_centroids.data_ptr(), self.v_boundaries.data_ptr()
        # W = S Pi^T in float64, for the append kernels' sign refinement and
        # sketch; at d = 128 also the tensor-core append's operand images
        self.s_pit = torch.empty((d, d), dtype=torch.float64, device=device)
        on_gpu = self.s_pit.is_cuda
        self.tc_operands = (torch.empty(TQ_TC_OPERAND_BYTES, dtype=torch.uint8, device=device)
                            if on_gpu and d == 128 else None)
        self.params = Params(d, key_bits, value_bits, group, self.pi.data_ptr(),
                             self.s.data_ptr(), self.centroids.data_ptr(),
                             self.boundaries.data_ptr(), mode, vc_ptr, vb_ptr,
                             self.s_pit.data_ptr(),
                             self.tc_operands.data_ptr() if self.tc_operands is not None else None)
        if on_gpu:
            tq_sketch_product(self)
            if self.tc_operands is not None:
                tq_prepare_operands(self)

    @property
    def d(self):
        return self.params.d

    def record_bytes(self) -> int:
        return int(load().tq_record_bytes(ctypes.byref(self.params)))


class CompressedCache:
    """A caller-owned cache buffer (torch uint8 tensor) as the C struct
    tq_cache."""

    def __init__(self, layer: Layer, batch: int, h_kv: int, capacity: int,
                 device="cuda", zero: bool = False):
        n = tq_cache_bytes(layer, batch, h_kv, capacity)
        if n == 0:
            raise TQError("tq_cache_bytes", 1)
        alloc = torch.zeros if zero else torch.empty
        self.buffer = alloc(n, dtype=torch.uint8, device=device)
        self.cache = Cache(batch, h_kv, capacity, self.buffer.data_ptr())
        self.batch, self.h_kv, self.capacity = batch, h_kv, capacity


def tq_sketch_product(layer: Layer, stream=None) -> None:
    """Write W = S Pi^T (float64) into layer.s_pit from the layer's Pi and S."""
    st = load().tq_sketch_product(ctypes.byref(layer.params), layer.s_pit.data_ptr(), _stream(stream))
    _check("tq_sketch_product", st)


def tq_prepare_operands(layer: Layer, stream=None) -> None:
    """Write the tensor-core append's operand images of the layer's Pi and
    W into layer.tc_operands (after tq_sketch_product)."""
    st = load().tq_prepare_operands(ctypes.byref(layer.params), layer.tc_operands.data_ptr(), _stream(stream))
    _check("tq_prepare_operands", st)


def tq_record_bytes(layer: Layer) -> int:
    return int(load().tq_record_bytes(ctypes.byref(layer.params)))


def tq_cache_bytes(layer: Layer, batch: int, h_kv: int, capacity: int) -> int:
    return int(load().tq_cache_bytes(ctypes.byref(layer.params), batch, h_kv, capacity))


def tq_quantize_append(layer: Layer, cache: CompressedCache, k: torch.Tensor,
                       v: torch.Tensor, len_host, n_new_host=None, stream=None) -> None:
    """k, v: [B, T, H_kv, d] device tensors (fp32 or bf16, contiguous)."""
    if k.dtype != v.dtype:
        raise TypeError("k and v must share a dtype")
    if not (k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous")
    T = int(k.shape[1]) if k.dim() == 4 else 0
    lens = _i32_array(len_host)
    nn = _i32_array(n_new_host) if n_new_host is not None else None
    st = load().tq_quantize_append(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                   k.data_ptr(), v.data_ptr(), _dtype_code(k), T, lens,
                                   nn, _stream(stream))
    _check("tq_quantize_append", st)


def tq_decode_workspace_size(layer: Layer, cache: CompressedCache, h_q: int, max_len: int) -> int:
    return int(load().tq_decode_workspace_size(ctypes.byref(layer.params),
                                               ctypes.byref(cache.cache), h_q, max_len))


def tq_decode_attention(layer: Layer, cache: CompressedCache, q: torch.Tensor,
                        len_dev: torch.Tensor, max_len: int, out: torch.Tensor,
                        workspace: torch.Tensor, softmax_scale: float | None = None,
                        stream=None) -> None:
    """q [B, H_q, d] (fp32/bf16), len_dev [B] int32 device, out [B, H_q, d]
    fp32, workspace a uint8 device tensor."""
    hq = _check_decode_io(cache, q, len_dev, out)
    scale = (1.0 / layer.d ** 0.5) if softmax_scale is None else float(softmax_scale)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor")
    st = load().tq_decode_attention(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                    q.data_ptr(), _dtype_code(q), hq,
                                    len_dev.data_ptr(), int(max_len), scale, out.data_ptr(),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    _check("tq_decode_attention", st)


def tq_decode_attention_window(layer: Layer, cache: CompressedCache, q: torch.Tensor,
                               len_dev: torch.Tensor, max_len: int, win_k: torch.Tensor,
                               win_v: torch.Tensor, win_len_dev: torch.Tensor, out: torch.Tensor,
                               workspace: torch.Tensor, softmax_scale: float | None = None,
                               stream=None) -> None:
    """Decode over the compressed cache plus a window of recent tokens kept
    exactly: win_k, win_v [B, H_kv, win_cap, d] (fp32/bf16, contiguous),
    win_len_dev [B] int32 device (valid slots per sequence)."""
    hq = _check_decode_io(cache, q, len_dev, out)
    if win_k.dim() != 4:
        raise ValueError("win_k must be [B, H_kv, win_cap, d]")
    wshape = (cache.batch, cache.h_kv, int(win_k.shape[2]), int(q.shape[2]))
    _check_rows("win_k", win_k, wshape, (torch.float32, torch.bfloat16), cache.buffer.device)
    _check_rows("win_v", win_v, wshape, (win_k.dtype,), cache.buffer.device)
    _check_rows("win_len_dev", win_len_dev, (cache.batch,), (torch.int32,), cache.buffer.device)
    scale = (1.0 / layer.d ** 0.5) if softmax_scale is None else float(softmax_scale)
    st = load().tq_decode_attention_window(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                           q.data_ptr(), _dtype_code(q), hq,
                                           len_dev.data_ptr(), int(max_len), win_k.data_ptr(),
                                           win_v.data_ptr(), _dtype_code(win_k), win_len_dev.data_ptr(),
                                           int(win_k.shape[2]), scale, out.data_ptr(),
                                           workspace.data_ptr(),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream))
    _check("tq_decode_attention_window", st)


def tq_decode_attention_noalloc(layer: Layer, cache: CompressedCache, q: torch.Tensor,
                                len_dev: torch.Tensor, max_len: int, out: torch.Tensor,
                                softmax_scale: float | None = None, stream=None) -> None:
    """Decode attention for callers that cannot allocate a workspace: the
    scratch is the library's fixed 8 MiB device array (see include/tq.h)."""
    hq = _check_decode_io(cache, q, len_dev, out)
    scale = (1.0 / layer.d ** 0.5) if softmax_scale is None else float(softmax_scale)
    st = load().tq_decode_attention_noalloc(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                            q.data_ptr(), _dtype_code(q), hq,
                                            len_dev.data_ptr(), int(max_len), scale,
                                            out.data_ptr(), _stream(stream))
    _check("tq_decode_attention_noalloc", st)


def tq_prefill_workspace_size(layer: Layer, cache: CompressedCache, h_q: int, t_chunk: int,
                              max_len: int) -> int:
    return int(load().tq_prefill_workspace_size(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                                h_q, t_chunk, max_len))


def tq_prefill_attention(layer: Layer, cache: CompressedCache, q: torch.Tensor,
                         len_dev: torch.Tensor, max_len: int, out: torch.Tensor,
                         workspace: torch.Tensor, softmax_scale: float | None = None,
                         stream=None) -> None:
    """Causal attention of a chunk over the compressed cache (the chunk already
    appended): q [B, T, H_q, d] (fp32/bf16, contiguous), len_dev [B] int32
    device (cached tokens, the chunk included), out [B, T, H_q, d] fp32."""
    if q.dim() != 4:
        raise ValueError("q must be a contiguous [B, T, H_q, d] tensor")
    dev = cache.buffer.device
    _check_rows("q", q, (cache.batch,) + tuple(q.shape[1:]), (torch.float32, torch.bfloat16), dev)
    _check_rows("len_dev", len_dev, (cache.batch,), (torch.int32,), dev)
    _check_rows("out", out, tuple(q.shape), (torch.float32,), dev)
    scale = (1.0 / layer.d ** 0.5) if softmax_scale is None else float(softmax_scale)
    st = load().tq_prefill_attention(ctypes.byref(layer.params), ctypes.byref(cache.cache),
                                     q.data_ptr(), _dtype_code(q), int(q.shape[2]), int(q.shape[1]),
                                     len_dev.data_ptr(), int(max_len), scale, out.data_ptr(),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check("tq_prefill_attention", st)


def tq_prefill_tokens_per_pass(layer: Layer, h_q: int, h_kv: int, t_chunk: int) -> int:
    return int(load().tq_prefill_tokens_per_pass(ctypes.byref(layer.params), h_q, h_kv, t_chunk))


def prefill_workspace_for(layer: Layer, cache: CompressedCache, h_q: int, t_chunk: int,
                          max_len: int, device="cuda") -> torch.Tensor:
    n = tq_prefill_workspace_size(layer, cache, h_q, t_chunk, max_len)
    if n == 0:
        raise TQError("tq_prefill_workspace_size", 1)
    return torch.empty(n, dtype=torch.uint8, device=device)


def tq_set_wait_limit_ns(ns: int) -> None:
    """Time limit of the kernels' bounded waits for later calls (0: the
    default, 2 s).  For tests of the timeout path."""
    _check("tq_set_wait_limit_ns", load().tq_set_wait_limit_ns(int(ns)))


def tq_test_withhold_handoffs(on: bool) -> None:
    """Tests of the timeout path: make later calls' tensor-core kernels
    withhold one hand-off so that their bounded waits run out."""
    _check("tq_test_withhold_handoffs", load().tq_test_withhold_handoffs(int(bool(on))))


def tq_test_sign_refine_threshold(z: float) -> None:
    """Tests of the float64 sign refinement: later appends re-decide every
    QJL sign with |(S r)_j| < z in float64 (0: the default, 1e-5)."""
    _check("tq_test_sign_refine_threshold", load().tq_test_sign_refine_threshold(float(z)))


def tq_test_refine_count(clear: bool = False) -> int:
    """Synchronise the device; QJL sign bits re-decided in float64 by the
    append kernels since the last reset (reset it when ``clear``)."""
    n = ctypes.c_ulonglong(0)
    _check("tq_test_refine_count", load().tq_test_refine_count(ctypes.byref(n), int(bool(clear))))
    return int(n.value)


def tq_device_errors(clear: bool = False) -> int:
    """Synchronise the current device and return its sticky error word
    (ERRF_* bits of kernels that gave up on a bounded wait); optionally
    reset it."""
    v = ctypes.c_uint32(0)
    _check("tq_device_errors", load().tq_device_errors(ctypes.byref(v), int(bool(clear))))
    return int(v.value)


def decode_status(workspace: torch.Tensor) -> int:
    """The status word a decode call left in its workspace (first int32):
    nonzero if a kernel of that call gave up on a bounded wait."""
    return int(workspace[:4].view(torch.int32).item())


def tq_dequantize(layer: Layer, cache: CompressedCache, b: int, start: int, count: int,
                  k_out: torch.Tensor, v_out: torch.Tensor, stream=None) -> None:
    st = load().tq_dequantize(ctypes.byref(layer.params), ctypes.byref(cache.cache), b, start,
                              count, k_out.data_ptr(), v_out.data_ptr(), _stream(stream))
    _check("tq_dequantize", st)


def workspace_for(layer: Layer, cache: CompressedCache, h_q: int, max_len: int,
                  device="cuda") -> torch.Tensor:
    n = tq_decode_workspace_size(layer, cache, h_q, max_len)
    if n == 0:
        raise TQError("tq_decode_workspace_size", 1)
    return torch.empty(n, dtype=torch.uint8, device=device)
