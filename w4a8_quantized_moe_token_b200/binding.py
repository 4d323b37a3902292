"""ctypes binding of libw4a8.so (the C ABI declared in include/w4a8.h).

Argument marshalling only: every function checks tensor devices / dtypes /
shapes, passes raw pointers and the current CUDA stream, and raises W4A8Error
on a non-zero status.  All computation happens in the CUDA library; if the
library is missing the first call raises -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a8.so")

W4A8_LAYOUT_PLAIN = 0
W4A8_LAYOUT_GATEUP = 1
W4A8_PACK_SYMMETRIC = 0x100  # OR into the layout: symmetric INT4 (scale = max|w|/7, codes q + 8, zero point 8)
W4A8_PACK_CLIP999 = 0x200  # OR into the layout: asymmetric INT4 over the 0.1th..99.9th percentile range
W4A8_PACK_GROUP64 = 0x400  # OR into the layout: one scale and zero point per 64 weights along K
W4A8_PACK_GROUP256 = 0x800  # OR into the layout: one scale and zero point per 256 weights along K
GROUP_FLAG = {64: W4A8_PACK_GROUP64, 128: 0, 256: W4A8_PACK_GROUP256}

DUMP = {
    "counts": 0, "offs": 1, "perm": 2, "inv": 3, "poffs": 4, "act1": 5, "s1": 6,
    "h": 7, "act2": 8, "s2": 9, "y2": 10, "err": 11,
}
W4A8_DUMP_W4A16 = 0x100  # OR into a dump id: the region of a w4a16_moe_forward workspace
DUMP_GROUP = {64: 0x400, 128: 0, 256: 0x800}  # OR into a dump id: a w4a8_moe_forward_g workspace

_c_int, _c_size, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "w4a8_version": ([], _c_int),
    "w4a8_status_string": ([_c_int], ctypes.c_char_p),
    "w4a8_packed_bytes": ([_c_int, _c_int, _c_int, _c_int], _c_size),
    "w4a8_pack_weights": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp, _vp, _vp, _vp], _c_int),
    "w4a8_quant_act": ([_vp, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "w4a8_kv_calibrate": ([_vp, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "w4a8_kv_quant": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "w4a8_kv_dequant": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "w4a8_route_topk": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "w4a8_moe_workspace_bytes": ([_c_int] * 5, _c_size),
    "w4a8_moe_host_workspace_bytes": ([_c_int] * 5, _c_size),
    "w4a8_moe_rows_capacity": ([_c_int] * 3, _c_int),
    "w4a8_moe_act_block_rows": ([_c_int] * 3, _c_int),
    "w4a8_moe_forward": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _c_int, _vp, _vp, _c_size, _vp],
                         _c_int),
    "w4a8_moe_forward_host": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _c_int, _vp, _vp, _c_size,
                               _vp], _c_int),
    "w4a8_gemm_workspace_bytes": ([_c_int] * 3, _c_size),
    "w4a8_gemm": ([_vp, _vp, _c_int, _vp, _c_int, _c_int, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "w4a8_gemm_noalloc": ([_vp, _vp, _c_int, _vp, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "w4a8_gemm_workspace_bytes_g": ([_c_int] * 4, _c_size),
    "w4a8_gemm_g": ([_vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "w4a8_moe_workspace_bytes_g": ([_c_int] * 6, _c_size),
    "w4a8_moe_forward_g": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _c_int, _vp, _vp, _c_size,
                            _vp], _c_int),
    "w4a8_gemm_noalloc_last_error": ([_vp], _c_int),
    "w4a8_moe_forward_logits_host": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _c_int, _vp, _vp,
                                      _c_size, _vp], _c_int),
    "w4a16_gemm_workspace_bytes": ([_c_int] * 3, _c_size),
    "w4a16_gemm": ([_vp, _c_int, _vp, _c_int, _c_int, _vp, _vp, _c_size, _vp], _c_int),
    "w4a16_moe_workspace_bytes": ([_c_int] * 5, _c_size),
    "w4a16_moe_forward": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _c_int, _vp, _vp, _c_size, _vp],
                          _c_int),
    "w4a8_debug_inject": ([ctypes.c_uint, ctypes.c_longlong], _c_int),
    "w4a8_debug_region": ([_c_int] * 6 + [ctypes.POINTER(_c_size), ctypes.POINTER(_c_size)], _c_int),
    "w4a8_debug_dump": ([_vp] + [_c_int] * 6 + [_vp, _c_size, _vp], _c_int),
    "w4a8_last_device_error": ([_vp, _vp], _c_int),
    "w4a8_profile_start": ([], _c_int),
    "w4a8_profile_stop": ([ctypes.POINTER(_c_int), ctypes.POINTER(ctypes.c_float), _c_int], _c_int),
}

KERNEL_KINDS = ["perm", "act_quant", "gemm_up", "requant", "gemm_down", "combine", "gemm_dense", "route"]
W4A8_DEBUG_SKIP_FIRST_COPY = 1

_lib = None


class W4A8Error(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """Load libw4a8.so (built in-tree by w4a8_quantized_moe_token_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise W4A8Error(f"{LIB_PATH} is missing: build it with `python -m w4a8_quantized_moe_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(status: int, what: str):
    if status != 0:
        msg = lib().w4a8_status_string(status).decode()
        raise W4A8Error(f"{what}: {msg} ({status})")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise W4A8Error("tensors passed to libw4a8 must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dev(t, dtype, name):
    if not t.is_cuda:
        raise W4A8Error(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise W4A8Error(f"{name} is on {t.device}, not on the current device cuda:{torch.cuda.current_device()}")
    if t.dtype != dtype:
        raise W4A8Error(f"{name} must be {dtype}, got {t.dtype}")


def _need(cond, msg):
    if not cond:
        raise W4A8Error(msg)


def padded_k(K: int, group: int = 128) -> int:
    """K rounded up to a whole number of 128-wide planes and of groups (the layout's
    row length)."""
    m = max(128, group)
    return (K + m - 1) // m * m


# --------------------------------------------------------------------------- #
def w4a8_version() -> int:
    return lib().w4a8_version()


def w4a8_packed_bytes(E: int, N: int, K: int, layout: int) -> int:
    return lib().w4a8_packed_bytes(E, N, K, layout)


def w4a8_pack_weights(w: torch.Tensor, layout: int, packed: torch.Tensor, codes=None, scale=None, zp=None):
    """w: bf16 [E][N][K] (cuda).  packed: uint8 cuda tensor of w4a8_packed_bytes bytes."""
    _dev(w, torch.bfloat16, "w")
    if w.dim() == 2:
        w = w.unsqueeze(0)
    E, N, K = w.shape
    _dev(packed, torch.uint8, "packed")
    for t, dt, nm in ((codes, torch.uint8, "codes"), (scale, torch.float16, "scale"), (zp, torch.float16, "zp")):
        if t is not None:
            _dev(t, dt, nm)
    _check(lib().w4a8_pack_weights(_ptr(w), E, N, K, layout, _ptr(packed), packed.numel(), _ptr(codes),
                                   _ptr(scale), _ptr(zp), _stream()), "w4a8_pack_weights")


def w4a8_quant_act(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor):
    """x: bf16 [T][K]; q: int8 [T][Kp]; s: float32 [T]."""
    _dev(x, torch.bfloat16, "x")
    _dev(q, torch.int8, "q")
    _dev(s, torch.float32, "s")
    T, K = x.shape
    _check(lib().w4a8_quant_act(_ptr(x), T, K, _ptr(q), _ptr(s), _stream()), "w4a8_quant_act")


def w4a8_kv_calibrate(x: torch.Tensor, scale: torch.Tensor):
    """x: bf16 [T][H][D] calibration values; scale: float32 [H] (written)."""
    _dev(x, torch.bfloat16, "x")
    _dev(scale, torch.float32, "scale")
    T, H, D = x.shape
    _check(lib().w4a8_kv_calibrate(_ptr(x), T, H, D, _ptr(scale), _stream()), "w4a8_kv_calibrate")


def w4a8_kv_quant(x: torch.Tensor, scale: torch.Tensor, q: torch.Tensor):
    """x: bf16 [T][H][D]; scale: float32 [H]; q: int8 [T][H][D] (written)."""
    _dev(x, torch.bfloat16, "x")
    _dev(scale, torch.float32, "scale")
    _dev(q, torch.int8, "q")
    T, H, D = x.shape
    _check(lib().w4a8_kv_quant(_ptr(x), T, H, D, _ptr(scale), _ptr(q), _stream()), "w4a8_kv_quant")


def w4a8_kv_dequant(q: torch.Tensor, scale: torch.Tensor, x: torch.Tensor):
    """q: int8 [T][H][D]; scale: float32 [H]; x: bf16 [T][H][D] (written)."""
    _dev(q, torch.int8, "q")
    _dev(scale, torch.float32, "scale")
    _dev(x, torch.bfloat16, "x")
    T, H, D = q.shape
    _check(lib().w4a8_kv_dequant(_ptr(q), T, H, D, _ptr(scale), _ptr(x), _stream()), "w4a8_kv_dequant")


def w4a8_route_topk(logits: torch.Tensor, k: int, ids: torch.Tensor, w: torch.Tensor):
    _dev(logits, torch.bfloat16, "logits")
    _dev(ids, torch.int32, "ids")
    _dev(w, torch.float32, "w")
    T, E = logits.shape
    _check(lib().w4a8_route_topk(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _stream()), "w4a8_route_topk")


def w4a8_moe_workspace_bytes(T, E, k, H, F) -> int:
    return lib().w4a8_moe_workspace_bytes(T, E, k, H, F)


def w4a8_moe_host_workspace_bytes(T, E, k, H, F) -> int:
    return lib().w4a8_moe_host_workspace_bytes(T, E, k, H, F)


def w4a8_moe_rows_capacity(T, E, k) -> int:
    return lib().w4a8_moe_rows_capacity(T, E, k)


def w4a8_moe_act_block_rows(T, E, k) -> int:
    return lib().w4a8_moe_act_block_rows(T, E, k)


def _moe_buffers(packed_up, packed_down, E, H, F, ws, host_ws=False, group=128):
    _dev(packed_up, torch.uint8, "packed_up")
    _dev(packed_down, torch.uint8, "packed_down")
    _dev(ws, torch.uint8, "ws")
    _need(group in GROUP_FLAG, f"group must be 64, 128 or 256, got {group}")
    _need(packed_up.numel() >= w4a8_packed_bytes(E, 2 * F, H, W4A8_LAYOUT_GATEUP | GROUP_FLAG[group]),
          "packed_up is smaller than the packed gate|up weights of this layer")
    _need(packed_down.numel() >= w4a8_packed_bytes(E, H, F, W4A8_LAYOUT_PLAIN | GROUP_FLAG[group]),
          "packed_down is smaller than the packed down weights of this layer")


def w4a8_moe_forward(packed_up, packed_down, E, H, F, x, ids, w, out, ws):
    """x bf16 [T][H], ids int32 [T][k], w float32 [T][k], out bf16 [T][H], ws uint8 (cuda)."""
    _dev(x, torch.bfloat16, "x")
    _dev(ids, torch.int32, "ids")
    _dev(w, torch.float32, "w")
    _dev(out, torch.bfloat16, "out")
    _moe_buffers(packed_up, packed_down, E, H, F, ws)
    T, k = ids.shape
    _need(tuple(x.shape) == (T, H), f"x must be [T={T}][H={H}], got {tuple(x.shape)}")
    _need(tuple(w.shape) == (T, k), f"w must be [T={T}][k={k}], got {tuple(w.shape)}")
    _need(tuple(out.shape) == (T, H), f"out must be [T={T}][H={H}], got {tuple(out.shape)}")
    _check(lib().w4a8_moe_forward(_ptr(packed_up), _ptr(packed_down), E, H, F, _ptr(x), T, _ptr(ids), _ptr(w), k,
                                  _ptr(out), _ptr(ws), ws.numel(), _stream()), "w4a8_moe_forward")


def w4a8_moe_workspace_bytes_g(T, E, k, H, F, group) -> int:
    return lib().w4a8_moe_workspace_bytes_g(T, E, k, H, F, group)


def w4a8_moe_forward_g(packed_up, packed_down, E, H, F, group, x, ids, w, out, ws):
    """w4a8_moe_forward for experts packed with group size 64, 128 or 256."""
    _dev(x, torch.bfloat16, "x")
    _dev(ids, torch.int32, "ids")
    _dev(w, torch.float32, "w")
    _dev(out, torch.bfloat16, "out")
    _moe_buffers(packed_up, packed_down, E, H, F, ws, group=group)
    T, k = ids.shape
    _need(tuple(x.shape) == (T, H), f"x must be [T={T}][H={H}], got {tuple(x.shape)}")
    _need(tuple(w.shape) == (T, k), f"w must be [T={T}][k={k}], got {tuple(w.shape)}")
    _need(tuple(out.shape) == (T, H), f"out must be [T={T}][H={H}], got {tuple(out.shape)}")
    _check(lib().w4a8_moe_forward_g(_ptr(packed_up), _ptr(packed_down), E, H, F, group, _ptr(x), T, _ptr(ids),
                                    _ptr(w), k, _ptr(out), _ptr(ws), ws.numel(), _stream()), "w4a8_moe_forward_g")


def w4a16_moe_workspace_bytes(T, E, k, H, F) -> int:
    return lib().w4a16_moe_workspace_bytes(T, E, k, H, F)


def w4a16_moe_forward(packed_up, packed_down, E, H, F, x, ids, w, out, ws):
    """The W4A16 comparison layer: same arguments as w4a8_moe_forward, bf16 token rows
    into both projections; ws sized by w4a16_moe_workspace_bytes."""
    _dev(x, torch.bfloat16, "x")
    _dev(ids, torch.int32, "ids")
    _dev(w, torch.float32, "w")
    _dev(out, torch.bfloat16, "out")
    _moe_buffers(packed_up, packed_down, E, H, F, ws)
    T, k = ids.shape
    _need(tuple(x.shape) == (T, H), f"x must be [T={T}][H={H}], got {tuple(x.shape)}")
    _need(tuple(w.shape) == (T, k), f"w must be [T={T}][k={k}], got {tuple(w.shape)}")
    _need(tuple(out.shape) == (T, H), f"out must be [T={T}][H={H}], got {tuple(out.shape)}")
    _check(lib().w4a16_moe_forward(_ptr(packed_up), _ptr(packed_down), E, H, F, _ptr(x), T, _ptr(ids), _ptr(w), k,
                                   _ptr(out), _ptr(ws), ws.numel(), _stream()), "w4a16_moe_forward")


def w4a8_moe_forward_host(packed_up, packed_down, E, H, F, x, ids, w, out, ws):
    """Same as w4a8_moe_forward with x / ids / w / out in (pinned) HOST memory."""
    for t, nm in ((x, "x"), (ids, "ids"), (w, "w"), (out, "out")):
        if t.is_cuda:
            raise W4A8Error(f"{nm} must be a host tensor")
    _moe_buffers(packed_up, packed_down, E, H, F, ws)
    T, k = ids.shape
    _need(x.dtype == torch.bfloat16 and tuple(x.shape) == (T, H), "x must be bf16 [T][H]")
    _need(ids.dtype == torch.int32, "ids must be int32")
    _need(w.dtype == torch.float32 and tuple(w.shape) == (T, k), "w must be float32 [T][k]")
    _need(out.dtype == torch.bfloat16 and tuple(out.shape) == (T, H), "out must be bf16 [T][H]")
    _check(lib().w4a8_moe_forward_host(_ptr(packed_up), _ptr(packed_down), E, H, F, _ptr(x), T, _ptr(ids), _ptr(w),
                                       k, _ptr(out), _ptr(ws), ws.numel(), _stream()), "w4a8_moe_forward_host")


def w4a8_moe_forward_logits_host(packed_up, packed_down, E, H, F, x, logits, k, out, ws):
    """The layer routed on the device from bf16 router logits [T][E]; x, logits and
    out are (pinned) HOST tensors; ws as for w4a8_moe_forward_host."""
    for t, nm in ((x, "x"), (logits, "logits"), (out, "out")):
        if t.is_cuda:
            raise W4A8Error(f"{nm} must be a host tensor")
    _moe_buffers(packed_up, packed_down, E, H, F, ws)
    T = x.shape[0]
    _need(x.dtype == torch.bfloat16 and tuple(x.shape) == (T, H), "x must be bf16 [T][H]")
    _need(logits.dtype == torch.bfloat16 and tuple(logits.shape) == (T, E), "logits must be bf16 [T][E]")
    _need(out.dtype == torch.bfloat16 and tuple(out.shape) == (T, H), "out must be bf16 [T][H]")
    _check(lib().w4a8_moe_forward_logits_host(_ptr(packed_up), _ptr(packed_down), E, H, F, _ptr(x), T,
                                              _ptr(logits), k, _ptr(out), _ptr(ws), ws.numel(), _stream()),
           "w4a8_moe_forward_logits_host")


def w4a8_gemm_workspace_bytes(M, N, K) -> int:
    return lib().w4a8_gemm_workspace_bytes(M, N, K)


def _gemm_buffers(qa, sa, packed, N, K, y, partials, group=128):
    """Check every buffer of a dense GEMM against its shape before the call: the
    kernels trust the sizes they are given."""
    _need(group in GROUP_FLAG, f"group must be 64, 128 or 256, got {group}")
    _dev(qa, torch.int8, "qa")
    _dev(sa, torch.float32, "sa")
    _dev(y, torch.float32, "y")
    _dev(packed, torch.uint8, "packed")
    _need(qa.dim() == 2, "qa must be [M][Kp]")
    M = qa.shape[0]
    Kp = padded_k(K)
    _need(tuple(qa.shape) == (M, Kp), f"qa must be [M][{Kp}] for K = {K}, got {tuple(qa.shape)}")
    _need(sa.numel() >= M, f"sa needs {M} entries, has {sa.numel()}")
    _need(y.numel() >= M * N, f"y needs {M * N} elements, has {y.numel()}")
    _need(packed.numel() >= w4a8_packed_bytes(1, N, K, W4A8_LAYOUT_PLAIN | GROUP_FLAG[group]),
          "packed is smaller than the packed weights of an N x K matrix")
    if partials is not None:
        _dev(partials, torch.int32, "partials")
        ng = padded_k(K, group) // group
        _need(partials.numel() >= M * N * ng, f"partials needs {M * N * ng} elements")
    return M


def w4a8_gemm(qa, sa, packed, N, K, y, ws, partials=None):
    """qa int8 [M][Kp], sa float32 [M], y float32 [M][N], partials int32 [M][N][Kp/128] or None."""
    M = _gemm_buffers(qa, sa, packed, N, K, y, partials)
    _dev(ws, torch.uint8, "ws")
    _check(lib().w4a8_gemm(_ptr(qa), _ptr(sa), M, _ptr(packed), N, K, _ptr(y), _ptr(partials), _ptr(ws), ws.numel(),
                           _stream()), "w4a8_gemm")


def w4a8_gemm_workspace_bytes_g(M, N, K, group) -> int:
    return lib().w4a8_gemm_workspace_bytes_g(M, N, K, group)


def w4a8_gemm_g(qa, sa, packed, N, K, group, y, ws, partials=None):
    """w4a8_gemm for weights packed with group size 64, 128 or 256; partials int32
    [M][N][padded_k(K, group) / group] or None."""
    M = _gemm_buffers(qa, sa, packed, N, K, y, partials, group)
    _dev(ws, torch.uint8, "ws")
    _check(lib().w4a8_gemm_g(_ptr(qa), _ptr(sa), M, _ptr(packed), N, K, group, _ptr(y), _ptr(partials), _ptr(ws),
                             ws.numel(), _stream()), "w4a8_gemm_g")


def w4a8_gemm_noalloc(qa, sa, packed, N, K, y, partials=None):
    """w4a8_gemm without a caller workspace: the library's own fixed scratch array
    is used (for callers that cannot allocate; concurrent calls race)."""
    M = _gemm_buffers(qa, sa, packed, N, K, y, partials)
    _check(lib().w4a8_gemm_noalloc(_ptr(qa), _ptr(sa), M, _ptr(packed), N, K, _ptr(y), _ptr(partials), _stream()),
           "w4a8_gemm_noalloc")


def w4a8_gemm_noalloc_last_error() -> int:
    """Device error word of the last w4a8_gemm_noalloc call on the current device."""
    r = lib().w4a8_gemm_noalloc_last_error(_stream())
    if r < 0:
        _check(r, "w4a8_gemm_noalloc_last_error")
    return r


def w4a16_gemm_workspace_bytes(M, N, K) -> int:
    return lib().w4a16_gemm_workspace_bytes(M, N, K)


def w4a16_gemm(x, packed, N, K, y, ws):
    """x bf16 [M][K] (16-bit activations, not quantised), y float32 [M][N]."""
    _dev(x, torch.bfloat16, "x")
    _dev(y, torch.float32, "y")
    _dev(packed, torch.uint8, "packed")
    _dev(ws, torch.uint8, "ws")
    _need(x.dim() == 2 and x.shape[1] == K, f"x must be [M][K={K}], got {tuple(x.shape)}")
    M = x.shape[0]
    _need(y.numel() >= M * N, f"y needs {M * N} elements, has {y.numel()}")
    _need(packed.numel() >= w4a8_packed_bytes(1, N, K, W4A8_LAYOUT_PLAIN),
          "packed is smaller than the packed weights of an N x K matrix")
    _check(lib().w4a16_gemm(_ptr(x), M, _ptr(packed), N, K, _ptr(y), _ptr(ws), ws.numel(), _stream()), "w4a16_gemm")


def w4a8_debug_inject(flags: int = 0, wait_limit_cycles: int = 0):
    """Test hook: bounded-wait limit and skipped-copy flag for the GEMM launches of
    this host thread (0, 0 restores normal operation)."""
    _check(lib().w4a8_debug_inject(flags, wait_limit_cycles), "w4a8_debug_inject")


def w4a8_debug_region(T, E, k, H, F, what) -> tuple[int, int]:
    off, nb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().w4a8_debug_region(T, E, k, H, F, DUMP.get(what, what), ctypes.byref(off), ctypes.byref(nb)),
           "w4a8_debug_region")
    return off.value, nb.value


def w4a8_debug_dump(ws, T, E, k, H, F, what) -> torch.Tensor:
    """Copy one workspace region to a new uint8 cuda tensor."""
    _, nb = w4a8_debug_region(T, E, k, H, F, what)
    dst = torch.empty(nb, dtype=torch.uint8, device=ws.device)
    _check(lib().w4a8_debug_dump(_ptr(ws), T, E, k, H, F, DUMP.get(what, what), _ptr(dst), nb, _stream()),
           "w4a8_debug_dump")
    return dst


def w4a8_last_device_error(ws) -> int:
    r = lib().w4a8_last_device_error(_ptr(ws), _stream())
    if r < 0:
        _check(r, "w4a8_last_device_error")
    return r


def empty_aligned(nbytes: int, device="cuda") -> torch.Tensor:
    """A uint8 device buffer whose start is 256-byte aligned (torch's caching
    allocator returns at least 512-byte aligned blocks)."""
    t = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)
    if t.data_ptr() % 256:
        raise W4A8Error("allocator returned a buffer that is not 256-byte aligned")
    return t


def w4a8_profile_start():
    _check(lib().w4a8_profile_start(), "w4a8_profile_start")


def w4a8_profile_stop() -> dict:
    """{kernel kind: (launches, total device ms)} since w4a8_profile_start()."""
    n = len(KERNEL_KINDS)
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_float * n)()
    _check(lib().w4a8_profile_stop(launches, ms, n), "w4a8_profile_stop")
    return {k: (launches[i], ms[i]) for i, k in enumerate(KERNEL_KINDS)}
