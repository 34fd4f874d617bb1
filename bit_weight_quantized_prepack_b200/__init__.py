"""Python binding of ``libwq.so``, the C ABI declared in ``include/wq.h``.

Argument marshalling only: every computation runs in the library's CUDA kernels. The
functions keep the C names; shapes are read from the tensors where the tensors carry them.
torch provides device memory and streams. The binding raises ``ImportError`` when the
library is not built and ``WqError`` when a call returns an error status: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import sys

import torch

__all__ = [
    "WqError", "lib", "LIB_PATH", "status_string", "wq_version",
    "wq_prepacked_bytes", "wq_prepacked_bytes_w4a8", "wq_prepack", "wq_prepack_w4a8",
    "wq_unpack", "wq_unpack_w4a8", "wq_gemm_w4a16", "wq_gemm_w4a16_noalloc", "wq_gemm_w4a8",
    "wq_quantize_act", "wq_gemm_w4a8_fp16act",
    "wq_prepacked_bytes_zp", "wq_prepack_zp", "wq_unpack_zp", "wq_gemm_w4a16_zp",
    "wq_prepack_act_order", "wq_permute_act", "wq_gemm_w4a16_act_order",
    "wq_prepacked_bytes_sparse24", "wq_prepack_sparse24", "wq_unpack_sparse24", "wq_gemm_w4a16_sparse24",
    "wq_prepacked_bytes_mixed", "wq_prepack_mixed", "wq_unpack_mixed", "wq_gemm_w4a16_mixed",
    "wq_workspace_bytes", "wq_workspace_reserve", "wq_get_device_status", "wq_plan", "wq_plan_for",
    "wq_debug_set_wait_timeout_ns", "wq_debug_skip_publish",
    "WQ_OK", "WQ_ERR_INVALID_ARG", "WQ_ERR_UNSUPPORTED_SHAPE", "WQ_ERR_MISALIGNED",
    "WQ_ERR_UNSUPPORTED_DEVICE", "WQ_ERR_CUDA", "WQ_ERR_TIMEOUT", "WQ_ERR_NO_MEMORY", "WQ_ERR_CAPTURING",
    "WQ_ERR_SCRATCH_LIMIT", "WQ_ERR_NOT_SPARSE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwq.so")

(WQ_OK, WQ_ERR_INVALID_ARG, WQ_ERR_UNSUPPORTED_SHAPE, WQ_ERR_MISALIGNED, WQ_ERR_UNSUPPORTED_DEVICE,
 WQ_ERR_CUDA, WQ_ERR_TIMEOUT, WQ_ERR_NO_MEMORY, WQ_ERR_CAPTURING, WQ_ERR_SCRATCH_LIMIT,
 WQ_ERR_NOT_SPARSE) = range(11)


class WqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)}")
        self.status = status


class _Plan(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int), ("tile_m", ctypes.c_int), ("m_tiles", ctypes.c_int),
                ("n_tiles", ctypes.c_int), ("k_blocks", ctypes.c_int), ("stages", ctypes.c_int),
                ("smem_bytes", ctypes.c_int), ("threads", ctypes.c_int), ("units", ctypes.c_longlong)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m bit_weight_quantized_prepack_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, Z, V = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, None
    sigs = {
        "wq_status_string": (ctypes.c_char_p, [I]),
        "wq_version": (I, []),
        "wq_prepacked_bytes": (Z, [I, I, I]),
        "wq_prepacked_bytes_w4a8": (Z, [I, I]),
        "wq_prepack": (I, [P, P, I, I, I, P, P]),
        "wq_prepack_w4a8": (I, [P, I, I, P, P]),
        "wq_unpack": (I, [P, I, I, I, P, P, P]),
        "wq_unpack_w4a8": (I, [P, I, I, P, P]),
        "wq_gemm_w4a16": (I, [P, P, P, I, I, I, I, P]),
        "wq_gemm_w4a16_noalloc": (I, [P, P, P, I, I, I, I, P]),
        "wq_gemm_w4a8": (I, [P, P, P, P, P, P, I, I, I, P]),
        "wq_quantize_act": (I, [P, I, I, I, P, P, P]),
        "wq_prepacked_bytes_zp": (Z, [I, I, I]),
        "wq_prepack_zp": (I, [P, P, P, I, I, I, P, P]),
        "wq_unpack_zp": (I, [P, I, I, I, P, P, P, P]),
        "wq_gemm_w4a16_zp": (I, [P, P, P, I, I, I, I, P]),
        "wq_prepack_act_order": (I, [P, P, P, P, I, I, I, P, P]),
        "wq_permute_act": (I, [P, P, I, I, P, P]),
        "wq_gemm_w4a16_act_order": (I, [P, P, P, P, I, I, I, I, I, P]),
        "wq_gemm_w4a8_fp16act": (I, [P, P, P, P, P, P, I, I, I, I, P]),
        "wq_prepacked_bytes_sparse24": (Z, [I, I, I]),
        "wq_prepack_sparse24": (I, [P, P, I, I, I, P, P]),
        "wq_unpack_sparse24": (I, [P, I, I, I, P, P, P]),
        "wq_gemm_w4a16_sparse24": (I, [P, P, P, I, I, I, I, P]),
        "wq_prepacked_bytes_mixed": (Z, [I, I, I, ctypes.c_longlong]),
        "wq_prepack_mixed": (I, [P, P, P, I, I, I, P, Z, P]),
        "wq_unpack_mixed": (I, [P, I, I, I, P, P, P, P]),
        "wq_gemm_w4a16_mixed": (I, [P, P, Z, P, I, I, I, I, P]),
        "wq_workspace_bytes": (Z, [I, I, I, I]),
        "wq_workspace_reserve": (I, [Z, P]),
        "wq_get_device_status": (I, [P]),
        "wq_plan": (I, [I, I, I, I, I, ctypes.POINTER(_Plan)]),
        "wq_plan_for": (I, [I, I, I, I, I, I, I, ctypes.POINTER(_Plan)]),
        "wq_debug_set_wait_timeout_ns": (I, [ctypes.c_ulonglong]),
        "wq_debug_skip_publish": (I, [I]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    del V
    return L


try:
    lib = _load()
except (ImportError, OSError, AttributeError) as _err:  # missing, unloadable or older than the header
    # `python -m bit_weight_quantized_prepack_b200.build` imports this package before it runs the
    # build (sys.argv[0] is "-m" while Python locates the module): let that command proceed.
    if sys.argv[:1] != ["-m"]:
        raise ImportError(f"libwq.so is missing or older than include/wq.h ({_err})") from _err
    lib = None


def status_string(status: int) -> str:
    return lib.wq_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != WQ_OK:
        raise WqError(rc, where)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _tensor(t, dtype, name, shape=None, min_numel=None):
    """Type, dtype, contiguity and size of one argument; raises before anything reaches the library.

    ``shape`` is the exact shape the call implies; ``min_numel`` the least number of elements
    (for the flat prepacked buffer). A wrongly sized buffer would otherwise become an
    out-of-bounds copy or store on the device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, the call needs at least {min_numel}")
    return t


def _on_one_cuda_device(**tensors):
    """Every given tensor on the same CUDA device (checked after the sizes)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {dev}")


def _matrix(t, name):
    if not isinstance(t, torch.Tensor) or t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor")
    return t.shape


def _prepacked_size(K, N, g, name):
    n = wq_prepacked_bytes(K, N, g) if g is not None else wq_prepacked_bytes_w4a8(K, N)
    if n == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE if K % 128 == 0 or g is None else WQ_ERR_INVALID_ARG, name)
    return n


def wq_version() -> int:
    return lib.wq_version()


def wq_prepacked_bytes(K: int, N: int, g: int) -> int:
    return lib.wq_prepacked_bytes(K, N, g)


def wq_prepacked_bytes_w4a8(K: int, N: int) -> int:
    return lib.wq_prepacked_bytes_w4a8(K, N)


def wq_prepack(Q: torch.Tensor, s: torch.Tensor, g: int, Wp: torch.Tensor | None = None, stream=None):
    """Q int32 [K/8, N], s fp16 [K/g, N] -> Wp uint8 [wq_prepacked_bytes(K, N, g)]."""
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    if g <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_prepack")
    _tensor(s, torch.float16, "s", shape=(K // g, N))
    nbytes = _prepacked_size(K, N, g, "wq_prepack")
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Q=Q, s=s, Wp=Wp)
    if Wp is None:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack(_ptr(Q), _ptr(s), K, N, g, _ptr(Wp), _stream(stream)), "wq_prepack")
    return Wp


def wq_prepack_w4a8(Q: torch.Tensor, Wp: torch.Tensor | None = None, stream=None):
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    nbytes = _prepacked_size(K, N, None, "wq_prepack_w4a8")
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Q=Q, Wp=Wp)
    if Wp is None:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack_w4a8(_ptr(Q), K, N, _ptr(Wp), _stream(stream)), "wq_prepack_w4a8")
    return Wp


def wq_unpack(Wp: torch.Tensor, K: int, N: int, g: int, stream=None):
    """Inverse of wq_prepack: (Q int32 [K/8, N], s fp16 [K/g, N])."""
    if g <= 0 or K <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_unpack")
    _tensor(Wp, torch.uint8, "Wp", min_numel=_prepacked_size(K, N, g, "wq_unpack"))
    _on_one_cuda_device(Wp=Wp)
    Q = torch.empty((K // 8, N), dtype=torch.int32, device=Wp.device)
    s = torch.empty((K // g, N), dtype=torch.float16, device=Wp.device)
    _check(lib.wq_unpack(_ptr(Wp), K, N, g, _ptr(Q), _ptr(s), _stream(stream)), "wq_unpack")
    return Q, s


def wq_unpack_w4a8(Wp: torch.Tensor, K: int, N: int, stream=None):
    _tensor(Wp, torch.uint8, "Wp", min_numel=_prepacked_size(K, N, None, "wq_unpack_w4a8"))
    _on_one_cuda_device(Wp=Wp)
    Q = torch.empty((K // 8, N), dtype=torch.int32, device=Wp.device)
    _check(lib.wq_unpack_w4a8(_ptr(Wp), K, N, _ptr(Q), _stream(stream)), "wq_unpack_w4a8")
    return Q


def _gemm_w4a16_args(A, Wp, N, g, Y, where):
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    if g <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, where)
    _tensor(Wp, torch.uint8, "Wp", min_numel=_prepacked_size(K, N, g, where))
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    _on_one_cuda_device(A=A, Wp=Wp, Y=Y)
    return M, K


def wq_gemm_w4a16(A: torch.Tensor, Wp: torch.Tensor, N: int, g: int, Y: torch.Tensor | None = None, stream=None):
    """Y fp16 [M, N] = A fp16 [M, K] . dequant(Wp)."""
    M, K = _gemm_w4a16_args(A, Wp, N, g, Y, "wq_gemm_w4a16")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a16(_ptr(A), _ptr(Wp), _ptr(Y), M, N, K, g, _stream(stream)), "wq_gemm_w4a16")
    return Y


def wq_gemm_w4a16_noalloc(A: torch.Tensor, Wp: torch.Tensor, N: int, g: int, Y: torch.Tensor, stream=None):
    """wq_gemm_w4a16 for callers that must not allocate: the library's stream-K scratch is a
    fixed 8 MiB device array (M <= 64 on a 148-SM B200) and Y must be given. Calls whose
    kernels overlap on the GPU race on that array."""
    if Y is None:
        raise ValueError("wq_gemm_w4a16_noalloc: Y must be given (the call allocates nothing)")
    M, K = _gemm_w4a16_args(A, Wp, N, g, Y, "wq_gemm_w4a16_noalloc")
    _check(lib.wq_gemm_w4a16_noalloc(_ptr(A), _ptr(Wp), _ptr(Y), M, N, K, g, _stream(stream)),
           "wq_gemm_w4a16_noalloc")
    return Y


def wq_gemm_w4a8(A: torch.Tensor, sa: torch.Tensor, Wp: torch.Tensor, sw: torch.Tensor, N: int,
                 Y: torch.Tensor | None = None, acc_out: torch.Tensor | None = None, stream=None):
    """Y fp16 [M, N] = (A int8 [M, K] . (q - 8)) * sa[m] * sw[n]; acc_out (optional) gets the int32 sums."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.int8, "A")
    _tensor(sa, torch.float32, "sa", shape=(M,))
    _tensor(sw, torch.float32, "sw", shape=(N,))
    _tensor(Wp, torch.uint8, "Wp", min_numel=_prepacked_size(K, N, None, "wq_gemm_w4a8"))
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    if acc_out is not None:
        _tensor(acc_out, torch.int32, "acc_out", shape=(M, N))
    _on_one_cuda_device(A=A, sa=sa, sw=sw, Wp=Wp, Y=Y, acc_out=acc_out)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a8(_ptr(A), _ptr(sa), _ptr(Wp), _ptr(sw), _ptr(Y), _ptr(acc_out), M, N, K,
                            _stream(stream)), "wq_gemm_w4a8")
    return Y


def wq_prepacked_bytes_zp(K: int, N: int, g: int) -> int:
    return lib.wq_prepacked_bytes_zp(K, N, g)


def wq_prepack_zp(Q: torch.Tensor, s: torch.Tensor, z: torch.Tensor, g: int, Wp: torch.Tensor | None = None,
                  stream=None):
    """Q int32 [K/8, N], s fp16 [K/g, N], zero points z uint8 [K/g, N] (0..15) -> the zero-point buffer."""
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    if g <= 0 or K % g or g == K:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_prepack_zp")
    _tensor(s, torch.float16, "s", shape=(K // g, N))
    _tensor(z, torch.uint8, "z", shape=(K // g, N))
    nbytes = wq_prepacked_bytes_zp(K, N, g)
    if nbytes == 0:
        raise WqError(WQ_ERR_INVALID_ARG if K % 128 == 0 else WQ_ERR_UNSUPPORTED_SHAPE, "wq_prepack_zp")
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Q=Q, s=s, z=z, Wp=Wp)
    if Wp is None:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack_zp(_ptr(Q), _ptr(s), _ptr(z), K, N, g, _ptr(Wp), _stream(stream)), "wq_prepack_zp")
    return Wp


def wq_unpack_zp(Wp: torch.Tensor, K: int, N: int, g: int, stream=None):
    """Inverse of wq_prepack_zp: (Q int32 [K/8, N], s fp16 [K/g, N], z uint8 [K/g, N])."""
    if g <= 0 or K <= 0 or K % g or g == K:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_unpack_zp")
    nbytes = wq_prepacked_bytes_zp(K, N, g)
    if nbytes == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_unpack_zp")
    _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Wp=Wp)
    Q = torch.empty((K // 8, N), dtype=torch.int32, device=Wp.device)
    s = torch.empty((K // g, N), dtype=torch.float16, device=Wp.device)
    z = torch.empty((K // g, N), dtype=torch.uint8, device=Wp.device)
    _check(lib.wq_unpack_zp(_ptr(Wp), K, N, g, _ptr(Q), _ptr(s), _ptr(z), _stream(stream)), "wq_unpack_zp")
    return Q, s, z


def wq_gemm_w4a16_zp(A: torch.Tensor, Wp: torch.Tensor, N: int, g: int, Y: torch.Tensor | None = None, stream=None):
    """Y fp16 [M, N] = A fp16 [M, K] . ((q - z) * s), from the zero-point buffer."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    if g <= 0 or K % g or g == K:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_gemm_w4a16_zp")
    nbytes = wq_prepacked_bytes_zp(K, N, g)
    if nbytes == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_gemm_w4a16_zp")
    _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    _on_one_cuda_device(A=A, Wp=Wp, Y=Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a16_zp(_ptr(A), _ptr(Wp), _ptr(Y), M, N, K, g, _stream(stream)), "wq_gemm_w4a16_zp")
    return Y


def wq_prepack_act_order(Q: torch.Tensor, s: torch.Tensor, perm: torch.Tensor, g: int, z: torch.Tensor | None = None,
                         Wp: torch.Tensor | None = None, stream=None):
    """Act order: Q int32 [K/8, N] in the checkpoint's row order, s fp16 [K/g, N] and optional zero
    points z uint8 [K/g, N] by group, perm int32 [K] with g_idx[perm[i]] == i // g (for example
    ``torch.argsort(g_idx, stable=True)``) -> the buffer of the reordered weight (the zero-point
    layout when z is given). Synchronises the stream (perm is checked on the host)."""
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    if g <= 0 or K % g or (z is not None and g == K):
        raise WqError(WQ_ERR_INVALID_ARG, "wq_prepack_act_order")
    _tensor(s, torch.float16, "s", shape=(K // g, N))
    _tensor(perm, torch.int32, "perm", shape=(K,))
    if z is not None:
        _tensor(z, torch.uint8, "z", shape=(K // g, N))
        nbytes = wq_prepacked_bytes_zp(K, N, g)
        if nbytes == 0:
            raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_prepack_act_order")
    else:
        nbytes = _prepacked_size(K, N, g, "wq_prepack_act_order")
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Q=Q, s=s, z=z, perm=perm, Wp=Wp)
    if Wp is None:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack_act_order(_ptr(Q), _ptr(s), _ptr(z), _ptr(perm), K, N, g, _ptr(Wp), _stream(stream)),
           "wq_prepack_act_order")
    return Wp


def wq_permute_act(A: torch.Tensor, perm: torch.Tensor, A_out: torch.Tensor | None = None, stream=None):
    """A_out fp16 [M, K] = A[:, perm] (perm int32 [K]); an index outside [0, K) gives 0 and is
    reported by wq_get_device_status."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    _tensor(perm, torch.int32, "perm", shape=(K,))
    if A_out is not None:
        _tensor(A_out, torch.float16, "A_out", shape=(M, K))
    _on_one_cuda_device(A=A, perm=perm, A_out=A_out)
    if A_out is None:
        A_out = torch.empty((M, K), dtype=torch.float16, device=A.device)
    _check(lib.wq_permute_act(_ptr(A), _ptr(perm), M, K, _ptr(A_out), _stream(stream)), "wq_permute_act")
    return A_out


def wq_gemm_w4a16_act_order(A: torch.Tensor, perm: torch.Tensor, Wp: torch.Tensor, N: int, g: int,
                            zero_points: bool = False, Y: torch.Tensor | None = None, stream=None):
    """Y fp16 [M, N] = A[:, perm] . W_reordered from a wq_prepack_act_order buffer (with zero
    points when ``zero_points``): the activations are gathered and the layer run in one call."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    _tensor(perm, torch.int32, "perm", shape=(K,))
    if g <= 0 or K % g or (zero_points and g == K):
        raise WqError(WQ_ERR_INVALID_ARG, "wq_gemm_w4a16_act_order")
    if zero_points:
        nbytes = wq_prepacked_bytes_zp(K, N, g)
        if nbytes == 0:
            raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_gemm_w4a16_act_order")
    else:
        nbytes = _prepacked_size(K, N, g, "wq_gemm_w4a16_act_order")
    _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    _on_one_cuda_device(A=A, perm=perm, Wp=Wp, Y=Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a16_act_order(_ptr(A), _ptr(perm), _ptr(Wp), _ptr(Y), M, N, K, g, int(bool(zero_points)),
                                       _stream(stream)), "wq_gemm_w4a16_act_order")
    return Y


def wq_prepacked_bytes_sparse24(K: int, N: int, g: int) -> int:
    return lib.wq_prepacked_bytes_sparse24(K, N, g)


def _sparse_size(K, N, g, where):
    if g <= 0 or K <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, where)
    n = wq_prepacked_bytes_sparse24(K, N, g)
    if n == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE if K % 128 == 0 else WQ_ERR_INVALID_ARG, where)
    return n


def wq_prepack_sparse24(Q: torch.Tensor, s: torch.Tensor, g: int, Wp: torch.Tensor | None = None, stream=None):
    """Q int32 [K/8, N] of 2:4 sparse codes (at most 2 of every 4 rows 4i..4i+3 differ from 8),
    s fp16 [K/g, N] -> the sparse buffer. Raises WqError(WQ_ERR_NOT_SPARSE) otherwise; the
    call synchronises the stream."""
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    nbytes = _sparse_size(K, N, g, "wq_prepack_sparse24")
    _tensor(s, torch.float16, "s", shape=(K // g, N))
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    _on_one_cuda_device(Q=Q, s=s, Wp=Wp)
    if Wp is None:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack_sparse24(_ptr(Q), _ptr(s), K, N, g, _ptr(Wp), _stream(stream)), "wq_prepack_sparse24")
    return Wp


def wq_unpack_sparse24(Wp: torch.Tensor, K: int, N: int, g: int, stream=None):
    """Inverse of wq_prepack_sparse24: (Q int32 [K/8, N] with pruned codes 8, s fp16 [K/g, N])."""
    _tensor(Wp, torch.uint8, "Wp", min_numel=_sparse_size(K, N, g, "wq_unpack_sparse24"))
    _on_one_cuda_device(Wp=Wp)
    Q = torch.empty((K // 8, N), dtype=torch.int32, device=Wp.device)
    s = torch.empty((K // g, N), dtype=torch.float16, device=Wp.device)
    _check(lib.wq_unpack_sparse24(_ptr(Wp), K, N, g, _ptr(Q), _ptr(s), _stream(stream)), "wq_unpack_sparse24")
    return Q, s


def wq_gemm_w4a16_sparse24(A: torch.Tensor, Wp: torch.Tensor, N: int, g: int, Y: torch.Tensor | None = None,
                           stream=None):
    """Y fp16 [M, N] = A fp16 [M, K] . dequant(Wp) for a 2:4 sparse buffer, M <= 16."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    _tensor(Wp, torch.uint8, "Wp", min_numel=_sparse_size(K, N, g, "wq_gemm_w4a16_sparse24"))
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    _on_one_cuda_device(A=A, Wp=Wp, Y=Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a16_sparse24(_ptr(A), _ptr(Wp), _ptr(Y), M, N, K, g, _stream(stream)),
           "wq_gemm_w4a16_sparse24")
    return Y


def wq_prepacked_bytes_mixed(K: int, N: int, g: int, n4: int) -> int:
    return lib.wq_prepacked_bytes_mixed(K, N, g, n4)


def wq_prepack_mixed(Q: torch.Tensor, s: torch.Tensor, widths: torch.Tensor, g: int, Wp: torch.Tensor | None = None,
                     stream=None):
    """Mixed 2/4-bit weights: Q int32 [K/8, N] (codes of 2-bit blocks 0..3), s fp16 [K/g, N],
    widths uint8 [K/32, ceil(N/128)] of 2 or 4 -> the mixed buffer. Synchronises the stream."""
    K8, N = _matrix(Q, "Q")
    K = K8 * 8
    _tensor(Q, torch.int32, "Q")
    if g <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_prepack_mixed")
    _tensor(s, torch.float16, "s", shape=(K // g, N))
    _tensor(widths, torch.uint8, "widths", shape=(K // 32, -(-N // 128)))
    _on_one_cuda_device(Q=Q, s=s, widths=widths, Wp=Wp)
    nbytes = wq_prepacked_bytes_mixed(K, N, g, int((widths == 4).sum().item()))
    if nbytes == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE if K % 128 == 0 else WQ_ERR_INVALID_ARG, "wq_prepack_mixed")
    if Wp is not None:
        _tensor(Wp, torch.uint8, "Wp", min_numel=nbytes)
    else:
        Wp = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    _check(lib.wq_prepack_mixed(_ptr(Q), _ptr(s), _ptr(widths), K, N, g, _ptr(Wp), Wp.numel(), _stream(stream)),
           "wq_prepack_mixed")
    return Wp


def wq_unpack_mixed(Wp: torch.Tensor, K: int, N: int, g: int, stream=None):
    """Inverse of wq_prepack_mixed: (Q int32 [K/8, N], s fp16 [K/g, N], widths uint8 [K/32, ceil(N/128)]).
    A test aid: it reads the blobs where Wp's table points, so Wp must come from wq_prepack_mixed."""
    if g <= 0 or K <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_unpack_mixed")
    least = wq_prepacked_bytes_mixed(K, N, g, 0)
    if least == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_unpack_mixed")
    _tensor(Wp, torch.uint8, "Wp", min_numel=least)
    _on_one_cuda_device(Wp=Wp)
    Q = torch.empty((K // 8, N), dtype=torch.int32, device=Wp.device)
    s = torch.empty((K // g, N), dtype=torch.float16, device=Wp.device)
    widths = torch.empty((K // 32, -(-N // 128)), dtype=torch.uint8, device=Wp.device)
    _check(lib.wq_unpack_mixed(_ptr(Wp), K, N, g, _ptr(Q), _ptr(s), _ptr(widths), _stream(stream)), "wq_unpack_mixed")
    return Q, s, widths


def wq_gemm_w4a16_mixed(A: torch.Tensor, Wp: torch.Tensor, N: int, g: int, Y: torch.Tensor | None = None,
                        stream=None):
    """Y fp16 [M, N] = A fp16 [M, K] . dequant(Wp) for a mixed 2/4-bit buffer, M <= 16."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    if g <= 0 or K % g:
        raise WqError(WQ_ERR_INVALID_ARG, "wq_gemm_w4a16_mixed")
    least = wq_prepacked_bytes_mixed(K, N, g, 0)
    if least == 0:
        raise WqError(WQ_ERR_UNSUPPORTED_SHAPE, "wq_gemm_w4a16_mixed")
    _tensor(Wp, torch.uint8, "Wp", min_numel=least)
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    _on_one_cuda_device(A=A, Wp=Wp, Y=Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a16_mixed(_ptr(A), _ptr(Wp), Wp.numel(), _ptr(Y), M, N, K, g, _stream(stream)),
           "wq_gemm_w4a16_mixed")
    return Y


def wq_quantize_act(A: torch.Tensor, A_q: torch.Tensor | None = None, sa: torch.Tensor | None = None, stream=None,
                    bits: int = 8):
    """fp16 A [M, K] -> (int8 codes [M, K], fp32 per-token scales [M]): symmetric, 127 levels
    each side for bits = 8, 7 for bits = 4 (codes held one per int8)."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    if A_q is not None:
        _tensor(A_q, torch.int8, "A_q", shape=(M, K))
    if sa is not None:
        _tensor(sa, torch.float32, "sa", shape=(M,))
    _on_one_cuda_device(A=A, A_q=A_q, sa=sa)
    if A_q is None:
        A_q = torch.empty((M, K), dtype=torch.int8, device=A.device)
    if sa is None:
        sa = torch.empty((M,), dtype=torch.float32, device=A.device)
    _check(lib.wq_quantize_act(_ptr(A), M, K, bits, _ptr(A_q), _ptr(sa), _stream(stream)), "wq_quantize_act")
    return A_q, sa


def wq_gemm_w4a8_fp16act(A: torch.Tensor, Wp: torch.Tensor, sw: torch.Tensor, N: int,
                         Y: torch.Tensor | None = None, acc_out: torch.Tensor | None = None,
                         sa_out: torch.Tensor | None = None, stream=None, act_bits: int = 8):
    """The layer on fp16 activations: per-token quantisation of A [M, K] to act_bits (8: W4A8,
    4: W4A4) then the layer on the int8 tensor cores, one call."""
    M, K = _matrix(A, "A")
    _tensor(A, torch.float16, "A")
    _tensor(sw, torch.float32, "sw", shape=(N,))
    _tensor(Wp, torch.uint8, "Wp", min_numel=_prepacked_size(K, N, None, "wq_gemm_w4a8_fp16act"))
    if Y is not None:
        _tensor(Y, torch.float16, "Y", shape=(M, N))
    if acc_out is not None:
        _tensor(acc_out, torch.int32, "acc_out", shape=(M, N))
    if sa_out is not None:
        _tensor(sa_out, torch.float32, "sa_out", shape=(M,))
    _on_one_cuda_device(A=A, sw=sw, Wp=Wp, Y=Y, acc_out=acc_out, sa_out=sa_out)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib.wq_gemm_w4a8_fp16act(_ptr(A), _ptr(Wp), _ptr(sw), _ptr(Y), _ptr(acc_out), _ptr(sa_out), M, N, K,
                                    act_bits, _stream(stream)), "wq_gemm_w4a8_fp16act")
    return Y


def wq_workspace_bytes(kind: int, M: int, N: int, K: int) -> int:
    return lib.wq_workspace_bytes(kind, M, N, K)


def wq_workspace_reserve(nbytes: int, stream=None) -> None:
    _check(lib.wq_workspace_reserve(nbytes, _stream(stream)), "wq_workspace_reserve")


def wq_get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status: WQ_OK or WQ_ERR_TIMEOUT."""
    return lib.wq_get_device_status(_stream(stream))


def wq_plan(kind: int, M: int, N: int, K: int, g: int) -> dict:
    p = _Plan()
    _check(lib.wq_plan(kind, M, N, K, g, ctypes.byref(p)), "wq_plan")
    return {f: getattr(p, f) for f, _ in _Plan._fields_}


def wq_plan_for(kind: int, M: int, N: int, K: int, g: int, num_sms: int, smem_optin: int) -> dict:
    """The plan on a device with num_sms SMs and smem_optin bytes of opt-in shared memory (no GPU needed)."""
    p = _Plan()
    _check(lib.wq_plan_for(kind, M, N, K, g, num_sms, smem_optin, ctypes.byref(p)), "wq_plan_for")
    return {f: getattr(p, f) for f, _ in _Plan._fields_}


def wq_debug_set_wait_timeout_ns(ns: int) -> None:
    _check(lib.wq_debug_set_wait_timeout_ns(ns), "wq_debug_set_wait_timeout_ns")


def wq_debug_skip_publish(cta: int) -> None:
    _check(lib.wq_debug_skip_publish(cta), "wq_debug_skip_publish")
