"""Python binding of the B200 Muon-step library (``libdmuon_b200.so``).

Argument marshalling only: every function below takes torch tensors (for
device memory) and an optional CUDA stream, turns them into the plain
pointers and sizes of the C ABI declared in ``include/dmuon.h`` and calls the
function of the same name.  All computation happens in the library's CUDA
kernels; there is no CPU or PyTorch fallback.  If the shared library is
missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DMUON_LIBRARY may name another build of the same library (e.g. a debug build)
LIB_PATH = os.environ.get("DMUON_LIBRARY") or os.path.join(_HERE, "libdmuon_b200.so")

DMUON_OK = 0
DMUON_ERR_INVALID_ARG = 1
DMUON_ERR_UNSUPPORTED = 2
DMUON_ERR_CUDA = 3
DMUON_ERR_OOM = 4
DMUON_ERR_TIMEOUT = 5
DMUON_ERR_BOUNDS = 6
STATUS_NAMES = {0: "DMUON_OK", 1: "DMUON_ERR_INVALID_ARG", 2: "DMUON_ERR_UNSUPPORTED",
                3: "DMUON_ERR_CUDA", 4: "DMUON_ERR_OOM", 5: "DMUON_ERR_TIMEOUT",
                6: "DMUON_ERR_BOUNDS"}
DMUON_F32 = 0
DMUON_BF16 = 1
DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)

EXPORTED = ("dmuon_ns", "dmuon_ns_ex", "dmuon_step", "dmuon_plan_groups", "dmuon_gram",
            "dmuon_gram_poly", "dmuon_poly_apply", "dmuon_momentum", "dmuon_update",
            "dmuon_get_last_error", "dmuon_stream_status", "dmuon_release_workspace",
            "dmuon_workspace_bytes", "dmuon_step_launches", "dmuon_build_info",
            "dmuon_profile_start", "dmuon_profile_stop", "dmuon_ns_noalloc", "dmuon_selftest_timeout",
            "dmuon_clip_grad_norm", "dmuon_step_clipped", "dmuon_selftest_bounds",
            "dmuon_profile_stop_launches", "dmuon_assign_owners", "dmuon_clip_grad_norm_buckets")


class DmuonError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


class LaunchRecord(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("start_ms", ctypes.c_double), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class Shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python newton_schulz_grad_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    fp = ctypes.POINTER(ctypes.c_float)
    sig = {
        "dmuon_ns": ([vp, vp, i64, i64, i32, fp, vp], i32),
        "dmuon_ns_ex": ([vp, vp, i64, i64, i32, fp, i32, vp], i32),
        "dmuon_step": ([ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                        ctypes.POINTER(Shape), i32, f32, f32, i32, i32, fp, f32, vp], i32),
        "dmuon_step_clipped": ([ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                ctypes.POINTER(Shape), i32, f32, f32, i32, i32, fp, f32, f32, f32, vp, vp], i32),
        "dmuon_plan_groups": ([ctypes.POINTER(Shape), i32, ctypes.POINTER(i32),
                               ctypes.POINTER(i32), ctypes.POINTER(i32)], i32),
        "dmuon_gram": ([vp, vp, i64, i64, i64, i64, i64, f32, i32, vp], i32),
        "dmuon_gram_poly": ([vp, vp, i64, i64, i64, i64, f32, f32, i32, vp], i32),
        "dmuon_poly_apply": ([vp, vp, vp, i64, i64, i64, i64, i64, i64, f32, f32, i32, vp], i32),
        "dmuon_momentum": ([vp, vp, vp, i64, i64, f32, i32, i32, vp, vp], i32),
        "dmuon_update": ([vp, vp, i64, i64, f32, f32, i32, vp], i32),
        "dmuon_get_last_error": ([], ctypes.c_char_p),
        "dmuon_stream_status": ([vp], i32),
        "dmuon_release_workspace": ([], None),
        "dmuon_workspace_bytes": ([ctypes.POINTER(Shape), i32, i32], i64),
        "dmuon_step_launches": ([ctypes.POINTER(Shape), i32, i32], i64),
        "dmuon_build_info": ([], ctypes.c_char_p),
        "dmuon_profile_start": ([], i32),
        "dmuon_profile_stop": ([ctypes.POINTER(KernelStat), i32], i32),
        "dmuon_profile_stop_launches": ([ctypes.POINTER(LaunchRecord), i32], i32),
        "dmuon_assign_owners": ([ctypes.POINTER(Shape), i32, i32, ctypes.POINTER(i32),
                                 ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)], i32),
        "dmuon_ns_noalloc": ([vp, vp, i64, i64, i32, fp, i32, vp, vp], i32),
        "dmuon_selftest_timeout": ([i32, vp], i32),
        "dmuon_clip_grad_norm": ([ctypes.POINTER(vp), ctypes.POINTER(Shape), i32, f32, f32, vp, vp], i32),
        "dmuon_clip_grad_norm_buckets": ([ctypes.POINTER(vp), ctypes.POINTER(Shape), i32, ctypes.POINTER(i32), i32,
                                          ctypes.POINTER(f32), ctypes.POINTER(f32), vp, vp], i32),
        "dmuon_selftest_bounds": ([vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


# ------------------------------------------------------------------ helpers
def _check(status: int) -> None:
    if status != DMUON_OK:
        raise DmuonError(status, _lib.dmuon_get_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DMUON_BF16
    if t.dtype == torch.float32:
        return DMUON_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _stream(stream, dev: Optional[torch.device] = None) -> ctypes.c_void_p:
    """The cudaStream_t of `stream` (default: the current stream of `dev`)."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    if dev is not None and getattr(stream, "device", dev) != dev:
        raise ValueError(f"the stream belongs to {stream.device}, the tensors to {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _device_of(*ts: Optional[torch.Tensor]) -> torch.device:
    """The one CUDA device that every given tensor (None skipped) lives on.

    The library launches on the calling thread's current device, so a call
    whose tensors sit on another device (or on several) is refused here, and
    the wrappers make the tensors' device current around the call."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"all tensors of one call must be on one device ({dev} and {t.device})")
    if dev is None:
        raise ValueError("no tensor given")
    return dev


def _out_word(t: Optional[torch.Tensor], dtype: torch.dtype, name: str) -> None:
    """Checks an optional one-element device output (status word, norm)."""
    if t is None:
        return
    if t.dtype != dtype or not t.is_cuda or t.numel() < 1 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of at least one element")


def _coeffs(steps: int, coeffs):
    """None -> NULL (library default); one triple -> repeated; else 3*steps floats."""
    if coeffs is None or steps == 0:
        return None
    flat = [float(v) for trip in (coeffs if isinstance(coeffs[0], (tuple, list)) else [coeffs])
            for v in trip]
    if len(flat) == 3 and steps != 1:
        flat = flat * steps
    if len(flat) != 3 * steps:
        raise ValueError("coeffs must hold one triple or one triple per step")
    arr = (ctypes.c_float * max(1, len(flat)))(*flat)
    return arr


def _shape_array(shapes: Sequence[Tuple[int, int, int]]):
    arr = (Shape * max(1, len(shapes)))()
    for i, (r, c, d) in enumerate(shapes):
        arr[i].rows, arr[i].cols, arr[i].dtype, arr[i].reserved = int(r), int(c), int(d), 0
    return arr


def _rows_ld(t: torch.Tensor):
    """(batch, rows, cols, ld) of a 2D or 3D tensor with unit column stride."""
    if t.dim() == 2:
        t3 = t.unsqueeze(0)
    elif t.dim() == 3:
        t3 = t
    else:
        raise ValueError("expected a 2D or 3D tensor")
    b, r, c = t3.shape
    if t3.stride(2) != 1:
        raise ValueError("last dimension must be contiguous")
    ld = t3.stride(1)
    if b > 1 and t3.stride(0) != r * ld:
        raise ValueError("matrices of a batch must follow one another (stride rows*ld)")
    return b, r, c, ld


# ------------------------------------------------------------- whole path
def dmuon_ns(X: torch.Tensor, out: torch.Tensor, steps: int = 5, coeffs=None, stream=None) -> None:
    """out = Gram Newton-Schulz(X / (||X|| + eps)); bf16 or fp32 (``dmuon_ns_ex``)."""
    dev = _device_of(X, out)
    if X.shape != out.shape or X.dim() != 2 or X.dtype != out.dtype:
        raise ValueError("X and out must be 2D tensors of equal shape and dtype")
    if not (X.is_contiguous() and out.is_contiguous()):
        raise ValueError("X and out must be contiguous")
    c = _coeffs(steps, coeffs)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_ns_ex(_ptr(X), _ptr(out), X.shape[0], X.shape[1], steps, c,
                                _dtype_code(X), st))


def dmuon_ns_noalloc(X: torch.Tensor, out: torch.Tensor, steps: int = 5, coeffs=None,
                     status: Optional[torch.Tensor] = None, stream=None) -> None:
    """dmuon_ns for callers that cannot allocate device memory.

    The library keeps a fixed scratch array (``DMUON_NOALLOC_SCRATCH_BYTES``)
    on each device and runs the same kernels as ``dmuon_ns`` in it, so this
    call never allocates.  Matrices too large for the array are rejected.
    ``status`` (a CUDA int32 tensor of one element, optional) receives
    DMUON_ERR_TIMEOUT if a bounded device wait ran out.  Calls share the
    array: calls that could overlap on the GPU must be serialised.
    """
    _out_word(status, torch.int32, "status")
    dev = _device_of(X, out, status)
    if X.shape != out.shape or X.dim() != 2 or X.dtype != out.dtype:
        raise ValueError("X and out must be 2D tensors of equal shape and dtype")
    if not (X.is_contiguous() and out.is_contiguous()):
        raise ValueError("X and out must be contiguous")
    c = _coeffs(steps, coeffs)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_ns_noalloc(_ptr(X), _ptr(out), X.shape[0], X.shape[1], steps, c,
                                     _dtype_code(X), _ptr(status), st))


def dmuon_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
               mom_bufs: Sequence[torch.Tensor], lr: float = 0.02, momentum: float = 0.95,
               nesterov: bool = True, ns_steps: int = 5, coeffs=None, wd: float = 0.0,
               stream=None, max_norm: Optional[float] = None, norm_type: float = 2.0,
               total_norm: Optional[torch.Tensor] = None) -> None:
    """One Muon step over lists of 2D tensors; params and mom_bufs updated in place.

    With ``max_norm`` set, the call is dmuon_step_clipped: the gradients are
    clipped by their global ``norm_type`` norm inside the step (not in memory).
    """
    n = len(params)
    if len(grads) != n or len(mom_bufs) != n:
        raise ValueError("params, grads and mom_bufs must have the same length")
    if max_norm is not None:
        _out_word(total_norm, torch.float64, "total_norm")
    if n == 0:
        return
    dev = _device_of(*params, *grads, *mom_bufs, total_norm if max_norm is not None else None)
    shapes = []
    for p, g, b in zip(params, grads, mom_bufs):
        if p.dim() != 2 or p.shape != g.shape or p.shape != b.shape:
            raise ValueError("each param, grad and buffer must be 2D with one shape")
        if not (p.dtype == g.dtype == b.dtype):
            raise ValueError("param, grad and buffer must share a dtype")
        if not (p.is_contiguous() and g.is_contiguous() and b.is_contiguous()):
            raise ValueError("tensors must be contiguous")
        shapes.append((p.shape[0], p.shape[1], _dtype_code(p)))
    vp = ctypes.c_void_p
    pa = (vp * max(1, n))(*[t.data_ptr() for t in params])
    ga = (vp * max(1, n))(*[t.data_ptr() for t in grads])
    ba = (vp * max(1, n))(*[t.data_ptr() for t in mom_bufs])
    c = _coeffs(ns_steps, coeffs)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if max_norm is None:
            _check(_lib.dmuon_step(pa, ga, ba, _shape_array(shapes), n, lr, momentum, int(bool(nesterov)),
                                   ns_steps, c, wd, st))
        else:
            _check(_lib.dmuon_step_clipped(pa, ga, ba, _shape_array(shapes), n, lr, momentum,
                                           int(bool(nesterov)), ns_steps, c, wd, float(max_norm),
                                           float(norm_type), _ptr(total_norm), st))


def dmuon_step_ptrs(params: Sequence[int], grads: Sequence[int], mom_bufs: Sequence[int],
                    shapes: Sequence[Tuple[int, int, int]], lr: float = 0.02,
                    momentum: float = 0.95, nesterov: bool = True, ns_steps: int = 5,
                    coeffs=None, wd: float = 0.0, stream=None, max_norm: Optional[float] = None,
                    norm_type: float = 2.0) -> None:
    """dmuon_step (dmuon_step_clipped with ``max_norm``) on raw device addresses."""
    n = len(params)
    vp = ctypes.c_void_p
    pa = (vp * max(1, n))(*params)
    ga = (vp * max(1, n))(*grads)
    ba = (vp * max(1, n))(*mom_bufs)
    if max_norm is None:
        _check(_lib.dmuon_step(pa, ga, ba, _shape_array(shapes), n, lr, momentum, int(bool(nesterov)),
                               ns_steps, _coeffs(ns_steps, coeffs), wd, _stream(stream)))
    else:
        _check(_lib.dmuon_step_clipped(pa, ga, ba, _shape_array(shapes), n, lr, momentum,
                                       int(bool(nesterov)), ns_steps, _coeffs(ns_steps, coeffs), wd,
                                       float(max_norm), float(norm_type), None, _stream(stream)))


def dmuon_clip_grad_norm(grads: Sequence[torch.Tensor], max_norm: float, norm_type: float = 2.0,
                         total_norm: Optional[torch.Tensor] = None, stream=None) -> None:
    """Global p-norm clipping of the gradients, in place (see dmuon.h)."""
    _out_word(total_norm, torch.float64, "total_norm")
    n = len(grads)
    if n == 0:
        return
    dev = _device_of(*grads, total_norm)
    shapes = []
    for g in grads:
        if g.dim() != 2 or not g.is_contiguous():
            raise ValueError("gradients must be contiguous 2D tensors")
        shapes.append((g.shape[0], g.shape[1], _dtype_code(g)))
    ga = (ctypes.c_void_p * max(1, n))(*[g.data_ptr() for g in grads])
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_clip_grad_norm(ga, _shape_array(shapes), n, float(max_norm), float(norm_type),
                                         _ptr(total_norm), st))


_MAX_SIDE = 1 << 20


def _flat_shape(t: torch.Tensor) -> Tuple[int, int]:
    # the clip reads a gradient as one flat array: any rank, as rows x cols
    n = t.numel()
    if n == 0:
        raise ValueError("empty gradient")
    cols = t.shape[-1] if t.dim() >= 2 else n
    if cols > _MAX_SIDE or n // cols > _MAX_SIDE:
        cols = next((c for c in range(min(n, _MAX_SIDE), 0, -1) if n % c == 0 and n // c <= _MAX_SIDE), 0)
        if cols == 0:
            raise ValueError(f"a gradient of {n} elements cannot be described as rows x cols <= 2^20")
    return n // cols, cols


def dmuon_clip_grad_norm_buckets(buckets: Sequence[Sequence[torch.Tensor]], max_norms: Sequence[float],
                                 norm_types=2.0, total_norms: Optional[torch.Tensor] = None, stream=None) -> None:
    """Independent global-norm clips of several gradient buckets, in place (see dmuon.h).

    ``buckets[k]`` is a list of contiguous CUDA gradients of any rank, clipped
    by its own ``max_norms[k]`` and ``norm_types[k]`` (one value for all
    buckets, or one per bucket); ``total_norms`` (float64, one per bucket)
    receives the totals.
    """
    nb = len(buckets)
    if isinstance(norm_types, (int, float)):
        norm_types = [float(norm_types)] * nb
    if len(max_norms) != nb or len(norm_types) != nb:
        raise ValueError("one max_norm and one norm_type per bucket")
    if total_norms is not None and (total_norms.dtype != torch.float64 or not total_norms.is_cuda
                                    or not total_norms.is_contiguous() or total_norms.numel() < nb):
        raise ValueError("total_norms must be a contiguous CUDA float64 tensor with one entry per bucket")
    grads, bucket_of = [], []
    for k, b in enumerate(buckets):
        for g in b:
            if not g.is_contiguous():
                raise ValueError("gradients must be contiguous")
            grads.append(g)
            bucket_of.append(k)
    n = len(grads)
    dev = _device_of(*grads, total_norms) if (n or total_norms is not None) else torch.device(
        "cuda", torch.cuda.current_device())
    shapes = [_flat_shape(g) + (_dtype_code(g),) for g in grads]
    ga = (ctypes.c_void_p * max(1, n))(*[g.data_ptr() for g in grads])
    bo = (ctypes.c_int32 * max(1, n))(*bucket_of)
    mx = (ctypes.c_float * max(1, nb))(*[float(v) for v in max_norms])
    nt = (ctypes.c_float * max(1, nb))(*[float(v) for v in norm_types])
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_clip_grad_norm_buckets(ga, _shape_array(shapes), n, bo, nb, mx, nt, _ptr(total_norms),
                                                 st))


def dmuon_plan_groups(shapes: Sequence[Tuple[int, int, int]]):
    """(group_of, order, num_groups) for (rows, cols, dtype_code) shapes (host only)."""
    n = len(shapes)
    g = (ctypes.c_int32 * max(1, n))()
    o = (ctypes.c_int32 * max(1, n))()
    k = ctypes.c_int32(0)
    _check(_lib.dmuon_plan_groups(_shape_array(shapes), n, g, o, ctypes.byref(k)))
    return list(g)[:n], list(o)[:n], k.value


def dmuon_assign_owners(shapes: Sequence[Tuple[int, int, int]], world: int):
    """(owner_of, loads, imbalance): dedicated ownership over `world` ranks (host only)."""
    n = len(shapes)
    own = (ctypes.c_int32 * max(1, n))()
    loads = (ctypes.c_double * max(1, world))()
    imb = ctypes.c_double(0.0)
    _check(_lib.dmuon_assign_owners(_shape_array(shapes), n, int(world), own, loads, ctypes.byref(imb)))
    return list(own)[:n], list(loads)[:world], imb.value


def dmuon_workspace_bytes(shapes, ns_steps: int = 5) -> int:
    return int(_lib.dmuon_workspace_bytes(_shape_array(shapes), len(shapes), ns_steps))


def dmuon_step_launches(shapes, ns_steps: int = 5) -> int:
    return int(_lib.dmuon_step_launches(_shape_array(shapes), len(shapes), ns_steps))


# ------------------------------------------------------------- stage calls
def dmuon_gram(X: torch.Tensor, G: torch.Tensor, alpha: float = 1.0, stream=None) -> None:
    """G = alpha X X^T over a batch ([B,] m x n -> [B,] m x m)."""
    dev = _device_of(X, G)
    b, m, n, ldx = _rows_ld(X)
    b2, m2, m3, ldg = _rows_ld(G)
    if (b2, m2, m3) != (b, m, m) or X.dtype != G.dtype:
        raise ValueError("G must be [B,] m x m with X's dtype")
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_gram(_ptr(X), _ptr(G), b, m, n, ldx, ldg, alpha, _dtype_code(X), st))


def dmuon_gram_poly(G: torch.Tensor, P: torch.Tensor, b: float, c: float, stream=None) -> None:
    """P = b G + c G G for symmetric G ([B,] m x m)."""
    dev = _device_of(G, P)
    bb, m, m2, ldg = _rows_ld(G)
    b2, p1, p2, ldp = _rows_ld(P)
    if m != m2 or (b2, p1, p2) != (bb, m, m) or G.dtype != P.dtype:
        raise ValueError("G and P must be [B,] m x m of one dtype")
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_gram_poly(_ptr(G), _ptr(P), bb, m, ldg, ldp, b, c, _dtype_code(G), st))


def dmuon_poly_apply(P: torch.Tensor, X: torch.Tensor, Y: torch.Tensor, a: float,
                     alpha: float = 1.0, stream=None) -> None:
    """Y = alpha (a X + P X) ([B,] m x m, [B,] m x n -> [B,] m x n)."""
    dev = _device_of(P, X, Y)
    bp, m, m2, ldp = _rows_ld(P)
    bx, mx, n, ldx = _rows_ld(X)
    by, my, ny, ldy = _rows_ld(Y)
    if not (bp == bx == by and m == m2 == mx == my and n == ny) or not (P.dtype == X.dtype == Y.dtype):
        raise ValueError("shape or dtype mismatch")
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_poly_apply(_ptr(P), _ptr(X), _ptr(Y), bx, m, n, ldp, ldx, ldy, a, alpha,
                                     _dtype_code(X), st))


def dmuon_momentum(buf: torch.Tensor, grad: torch.Tensor, x0: torch.Tensor, momentum: float = 0.95,
                   nesterov: bool = True, sumsq: Optional[torch.Tensor] = None, stream=None) -> None:
    """buf <- mu buf + g ; x0 = g + mu buf (or buf); optional fp64 sum of squares of x0."""
    _out_word(sumsq, torch.float64, "sumsq")
    dev = _device_of(buf, grad, x0, sumsq)
    if not (buf.shape == grad.shape == x0.shape) or buf.dim() != 2:
        raise ValueError("buf, grad and x0 must be 2D of one shape")
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_momentum(_ptr(buf), _ptr(grad), _ptr(x0), buf.shape[0], buf.shape[1],
                                   momentum, int(bool(nesterov)), _dtype_code(buf), _ptr(sumsq), st))


def dmuon_update(param: torch.Tensor, O: torch.Tensor, lr: float, wd: float = 0.0,
                 stream=None) -> None:
    """param <- param (1 - lr wd) - lr 0.2 sqrt(max(m,n)) O."""
    dev = _device_of(param, O)
    if param.shape != O.shape or param.dim() != 2 or param.dtype != O.dtype:
        raise ValueError("param and O must be 2D of one shape and dtype")
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(_lib.dmuon_update(_ptr(param), _ptr(O), param.shape[0], param.shape[1], lr, wd,
                                 _dtype_code(param), st))


# ---------------------------------------------------------- status / misc
def dmuon_stream_status(stream=None) -> int:
    """Synchronise the stream and return (without raising) the library status."""
    return int(_lib.dmuon_stream_status(_stream(stream)))


def dmuon_selftest_timeout(limit_us: int = 50000, stream=None) -> None:
    """Launch a kernel whose bounded device wait is made to run out (see dmuon.h)."""
    _check(_lib.dmuon_selftest_timeout(int(limit_us), _stream(stream)))


def dmuon_selftest_bounds(stream=None) -> None:
    """Evaluate one deliberately failing bounds check (see dmuon.h); touches no memory."""
    _check(_lib.dmuon_selftest_bounds(_stream(stream)))


def dmuon_get_last_error() -> str:
    return _lib.dmuon_get_last_error().decode()


def dmuon_release_workspace() -> None:
    _lib.dmuon_release_workspace()


def dmuon_profile_start() -> None:
    _check(_lib.dmuon_profile_start())


def dmuon_profile_stop() -> dict:
    """{kind: {launches, total_ms, flops, bytes}} for the launches since start."""
    arr = (KernelStat * 32)()
    n = _lib.dmuon_profile_stop(arr, 32)
    if n < 0:
        raise DmuonError(DMUON_ERR_CUDA, dmuon_get_last_error())
    return {arr[i].name.decode(): {"launches": int(arr[i].launches), "total_ms": arr[i].total_ms,
                                   "flops": arr[i].flops, "bytes": arr[i].bytes}
            for i in range(min(n, 32))}


def dmuon_profile_stop_launches(max_records: int = 100000) -> list:
    """[{name, start_ms, ms, flops, bytes}] for every launch since start, in enqueue order."""
    arr = (LaunchRecord * max_records)()
    n = _lib.dmuon_profile_stop_launches(arr, max_records)
    if n < 0:
        raise DmuonError(DMUON_ERR_CUDA, dmuon_get_last_error())
    return [{"name": arr[i].name.decode(), "start_ms": arr[i].start_ms, "ms": arr[i].ms,
             "flops": arr[i].flops, "bytes": arr[i].bytes} for i in range(min(n, max_records))]


def dmuon_build_info() -> str:
    return _lib.dmuon_build_info().decode()


def coeff_list(steps: int, coeffs=None) -> List[Tuple[float, float, float]]:
    """The per-iteration coefficient triples the library will use."""
    if coeffs is None:
        return [DEFAULT_COEFFS] * steps
    if not isinstance(coeffs[0], (tuple, list)):
        return [tuple(coeffs)] * steps
    return [tuple(c) for c in coeffs]
