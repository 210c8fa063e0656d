"""AWQ activation-aware per-layer scale search on NVIDIA B200 (sm_100a).

Python binding of ``libawqsearch.so`` (C ABI in ``include/awq_search.h``). This module
only marshals arguments: torch provides device memory and the stream, and every step
of the search runs in the library's CUDA kernels. There is no CPU fallback: if the
library is missing or cannot load, every call raises.

    import torch, post_quantization_column_b200 as awq
    out = awq.search(X, W, group=128, n_grid=20)   # X: (M, K) bf16/fp32 CUDA, W: (K, N)
    out.scales, out.codes, out.steps, out.zeros, out.losses, out.best   # best: the library's chosen index
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

__all__ = [
    "AwqError", "SearchOutput", "search", "search_async", "alloc_outputs", "PendingSearch", "search_host", "search_host_batch", "library", "library_path", "header_path",
    "tile_shape", "workspace_bytes", "release_cached", "profile_enable", "profile_last",
    "last_launch_count", "debug_set_fault", "status_string", "exported_functions",
    "activation_statistic", "candidate_scales", "qdq_candidates", "ClipOutput", "clip_search",
    "clip_token_count", "clip_profile_last", "fp64_mma_peak", "w4a16_matmul", "w4a16_dequant", "w4a16_profile_last", "search_mlp", "QUANTIZERS", "w4a16_repack", "w4a16_matmul_packed", "loss_gemm_variant", "loss_gemm_launches", "qdq_in_loss_gemm",
    "search_attn", "attn_profile_last", "ATTN_HEAD_DIM",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libawqsearch.so")
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "awq_search.h")

DTYPE_BF16, DTYPE_F32 = 0, 1
_STATUS = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_NONFINITE",
           4: "AWQ_ERR_OOM", 5: "AWQ_ERR_CUDA", 6: "AWQ_ERR_TIMEOUT", 7: "AWQ_ERR_UNSUPPORTED_DEVICE"}

_lib = None


class AwqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def header_path() -> str:
    return _HEADER


def library() -> ctypes.CDLL:
    """Load libawqsearch.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m post_quantization_column_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, f32p, f64p = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
    lib.awq_search.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.awq_search_f32.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.awq_search_ex.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, vp, vp, vp, vp, f32p, vp, f64p, i64, vp]
    lib.awq_search_host.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_host_batch.argtypes = [i32, vp, vp, i32, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_async.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_noalloc.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_noalloc.restype = ctypes.c_int
    lib.awq_search_async.restype = ctypes.c_int
    lib.awq_search_status.argtypes = [ctypes.c_int32]
    lib.awq_search_status.restype = ctypes.c_int
    lib.awq_profile_last_ticket.argtypes = []
    lib.awq_profile_last_ticket.restype = ctypes.c_int64
    lib.awq_profile_collect.argtypes = [ctypes.c_int64, ctypes.POINTER(ctypes.c_float), i32]
    lib.awq_profile_collect.restype = ctypes.c_int
    for name in ("awq_search", "awq_search_f32", "awq_search_ex", "awq_search_host", "awq_search_host_batch",
                 "awq_release_cached",
                 "awq_profile_enable", "awq_profile_last", "awq_last_launch_count", "awq_debug_set_fault",
                 "awq_version"):
        getattr(lib, name).restype = ctypes.c_int
    lib.awq_tile_shape.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.awq_tile_shape.restype = None
    lib.awq_workspace_bytes.argtypes = [i32, i64, i64, i64, i32, i32]
    lib.awq_workspace_bytes.restype = ctypes.c_int64
    lib.awq_status_string.argtypes = [i32]
    lib.awq_status_string.restype = ctypes.c_char_p
    lib.awq_last_error_message.argtypes = []
    lib.awq_last_error_message.restype = ctypes.c_char_p
    lib.awq_profile_enable.argtypes = [i32]
    lib.awq_profile_last.argtypes = [ctypes.POINTER(ctypes.c_float), i32]
    lib.awq_profile_phase_name.argtypes = [i32]
    lib.awq_profile_phase_name.restype = ctypes.c_char_p
    lib.awq_debug_set_fault.argtypes = [i32, i64]
    lib.awq_activation_statistic.argtypes = [vp, i32, i64, i64, vp, vp]
    lib.awq_candidate_scales.argtypes = [vp, i64, i32, vp, vp]
    lib.awq_qdq_candidates.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp, vp]
    lib.awq_clip_search.argtypes = [vp, vp, i32, vp, i64, i64, i64, i32, i32, i64, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_quant.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_mlp.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_attn.argtypes = [vp, vp, i32, i64, i64, i64, i32, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.awq_search_attn.restype = ctypes.c_int
    lib.awq_attn_profile_last.argtypes = [ctypes.POINTER(ctypes.c_float), i32]
    lib.awq_attn_profile_last.restype = ctypes.c_int
    lib.awq_clip_profile_last.argtypes = [ctypes.POINTER(ctypes.c_float), i32]
    lib.awq_clip_profile_last.restype = ctypes.c_int
    lib.awq_fp64_mma_peak.argtypes = [ctypes.POINTER(ctypes.c_double), vp]
    lib.awq_fp64_mma_peak.restype = ctypes.c_int
    lib.awq_w4a16_matmul.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp]
    lib.awq_w4a16_dequant.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp]
    lib.awq_w4a16_repack.argtypes = [vp, i64, i64, vp, vp]
    lib.awq_w4a16_matmul_packed.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp]
    lib.awq_w4a16_profile_last.argtypes = []
    lib.awq_w4a16_profile_last.restype = ctypes.c_float
    lib.awq_loss_gemm_variant.argtypes = [i64, i64, i64, i32]
    lib.awq_loss_gemm_variant.restype = ctypes.c_int
    lib.awq_loss_gemm_launches.argtypes = [i32, i64, i64, i64, i32, i32]
    lib.awq_loss_gemm_launches.restype = ctypes.c_int
    lib.awq_qdq_in_loss_gemm.argtypes = [i32, i64, i64, i64, i32, i32]
    lib.awq_qdq_in_loss_gemm.restype = ctypes.c_int
    lib.awq_clip_token_count.argtypes = [i64, i64]
    lib.awq_clip_token_count.restype = ctypes.c_int64
    for name in ("awq_activation_statistic", "awq_candidate_scales", "awq_qdq_candidates", "awq_clip_search",
                 "awq_search_quant", "awq_search_mlp",
                 "awq_w4a16_matmul", "awq_w4a16_dequant", "awq_w4a16_repack", "awq_w4a16_matmul_packed"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def exported_functions() -> list[str]:
    """Function names `include/awq_search.h` declares."""
    with open(_HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return library().awq_status_string(status).decode()


def _check(status: int):
    if status != 0:
        msg = library().awq_last_error_message().decode()
        raise AwqError(status, msg)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_handle(stream, device) -> ctypes.c_void_p:
    """The stream a call runs on (default: the current stream of ``device``). A stream
    other than the current one first waits for the work already enqueued on the current
    stream, which is where the inputs (and their contiguous copies) were produced."""
    current = torch.cuda.current_stream(device)
    if stream is None:
        stream = current
    elif stream.cuda_stream != current.cuda_stream:
        stream.wait_stream(current)
    return ctypes.c_void_p(stream.cuda_stream)


def tile_shape() -> tuple[int, int]:
    m, n = ctypes.c_int(), ctypes.c_int()
    library().awq_tile_shape(ctypes.byref(m), ctypes.byref(n))
    return m.value, n.value


def workspace_bytes(M: int, K: int, N: int, group: int = 128, n_grid: int = 20, dtype=torch.bfloat16) -> int:
    return int(library().awq_workspace_bytes(DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32,
                                             M, K, N, group, n_grid))


def release_cached() -> None:
    _check(library().awq_release_cached())


def profile_enable(on: bool = True) -> None:
    library().awq_profile_enable(1 if on else 0)


def profile_last() -> dict:
    lib = library()
    buf = (ctypes.c_float * 16)()
    n = lib.awq_profile_last(buf, 16)
    return {lib.awq_profile_phase_name(i).decode(): float(buf[i]) for i in range(n)}


def last_launch_count() -> int:
    return int(library().awq_last_launch_count())


def debug_set_fault(mode: int, timeout_ns: int = 0) -> None:
    _check(library().awq_debug_set_fault(mode, timeout_ns))


@dataclass
class SearchOutput:
    scales: torch.Tensor        # (K,) fp32: the chosen s
    codes: torch.Tensor         # (K, N/8) int32: eight 4-bit codes per word along N
    steps: torch.Tensor         # (K/group, N) fp16
    zeros: torch.Tensor         # (K/group, N) fp16
    losses: torch.Tensor        # (n_grid,) fp32
    best_index: torch.Tensor    # (1,) int32: the index the library chose (out_best of the C ABI)
    tile_sq_err: torch.Tensor | None = None  # (n_grid, tiles_m, tiles_n) fp64

    @property
    def best(self) -> int:
        """Index of the chosen alpha (alpha = best / n_grid), as the library returned it."""
        return int(self.best_index[0])


def _dtype_code_of(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return DTYPE_BF16
    if dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"X and W must be bfloat16 or float32, got {dtype}")


def _dtype_code(t: torch.Tensor) -> int:
    return _dtype_code_of(t.dtype)


def _alloc_outputs(K, N, group, n_grid, device, pin=False):
    """scales, codes, steps, zeros, losses and the chosen index of one layer."""
    kw = dict(device=device) if not pin else dict(pin_memory=True)
    return (torch.empty(K, dtype=torch.float32, **kw),
            torch.empty(K, N // 8, dtype=torch.int32, **kw),
            torch.empty(K // group, N, dtype=torch.float16, **kw),
            torch.empty(K // group, N, dtype=torch.float16, **kw),
            torch.empty(n_grid, dtype=torch.float32, **kw),
            torch.full((1,), -1, dtype=torch.int32, **kw))


def alloc_outputs(K: int, N: int, group: int = 128, n_grid: int = 20, device=None, pin: bool = False) -> tuple:
    """The six output tensors of one layer's search (scales, codes, steps, zeros, losses,
    chosen index), on ``device`` or in pinned host memory."""
    return _alloc_outputs(K, N, group, n_grid, device, pin)


def _with_best(out: tuple) -> tuple:
    """A caller's 5-tuple of host outputs plus a pinned word for the chosen index."""
    return tuple(out) if len(out) == 6 else tuple(out) + (torch.full((1,), -1, dtype=torch.int32, pin_memory=True),)


QUANTIZERS = {"asym": 0, "sym": 1}


def search(X: torch.Tensor, W: torch.Tensor, group: int = 128, n_grid: int = 20, *,
           stream: torch.cuda.Stream | None = None, tile_sq_err: bool = False,
           quantizer: str = "asym") -> SearchOutput:
    """Run the search on device tensors X (M, K) and W (K, N) of the same dtype.

    ``quantizer`` "asym" (the search's zero-point quantizer) or "sym" (the symmetric
    [-7, 7] teaching quantizer, artifact codes q + 7 with zero point 7)."""
    if X.dim() != 2 or W.dim() != 2 or X.shape[1] != W.shape[0]:
        raise ValueError("X must be (M, K) and W must be (K, N)")
    if X.dtype != W.dtype:
        raise TypeError("X and W must share a dtype")
    if not (X.is_cuda and W.is_cuda):
        raise ValueError("search() takes CUDA tensors; use search_host() for host tensors")
    lib = library()
    X = X.contiguous()
    W = W.contiguous()
    M, K = X.shape
    N = W.shape[1]
    if group <= 0 or K % group or N % 8:
        raise ValueError("group must divide K and N must be a multiple of 8")
    scales, codes, steps, zeros, losses, best = _alloc_outputs(K, N, group, n_grid, X.device)
    tiles = None
    if tile_sq_err:
        tm, tn = tile_shape()
        tiles = torch.empty(n_grid, -(-M // tm), -(-N // tn), dtype=torch.float64, device=X.device)
    if quantizer not in QUANTIZERS:
        raise ValueError(f"quantizer must be one of {sorted(QUANTIZERS)}")
    if quantizer != "asym":
        if tile_sq_err:
            raise ValueError("tile partials are available for the asymmetric quantizer only")
        st = lib.awq_search_quant(_ptr(X), _ptr(W), _dtype_code(X), M, K, N, group, n_grid, QUANTIZERS[quantizer],
                                  _ptr(scales), _ptr(codes), _ptr(steps), _ptr(zeros), _ptr(losses), _ptr(best),
                                  _stream_handle(stream, X.device))
        _check(st)
        return SearchOutput(scales, codes, steps, zeros, losses, best, None)
    st = lib.awq_search_ex(_ptr(X), _ptr(W), _dtype_code(X), M, K, N, group, n_grid, _ptr(scales), _ptr(codes),
                           _ptr(steps), _ptr(zeros), _ptr(losses), _ptr(best), _ptr(tiles),
                           tiles.numel() if tiles is not None else 0, _stream_handle(stream, X.device))
    _check(st)
    return SearchOutput(scales, codes, steps, zeros, losses, best, tiles)


class PendingSearch:
    """A search enqueued by search_async(): ``wait()`` synchronizes its stream, raises
    AwqError if the kernels reported an error, and returns the SearchOutput;
    ``profile()`` (after wait, with profiling on) gives the call's phase times in ms."""

    def __init__(self, out: SearchOutput, status: torch.Tensor, stream, device, ticket: int):
        self.out, self._status, self._stream, self._device, self._ticket = out, status, stream, device, ticket
        self._done = False

    def wait(self) -> SearchOutput:
        if not self._done:
            self._stream.synchronize()
            self._done = True
        _check(library().awq_search_status(int(self._status[0])))
        return self.out

    def profile(self) -> dict:
        lib = library()
        buf = (ctypes.c_float * 16)()
        n = lib.awq_profile_collect(self._ticket, buf, 16) if self._ticket >= 0 else -1
        if n < 0:
            raise RuntimeError("no phase times for this call (profiling off, still running, or reused)")
        return {lib.awq_profile_phase_name(i).decode(): float(buf[i]) for i in range(n)}


def search_async(X: torch.Tensor, W: torch.Tensor, group: int = 128, n_grid: int = 20, *,
                 stream: torch.cuda.Stream | None = None, out: tuple | None = None,
                 status: torch.Tensor | None = None) -> PendingSearch:
    """search() without waiting: the whole search is enqueued on ``stream`` and the call
    returns at once, so consecutive layers run back to back on the device. Argument
    errors raise here; errors the kernels detect raise from ``wait()``. ``out`` (the six
    device outputs of _alloc_outputs) and ``status`` (one pinned int32) may be given to
    enqueue without allocating."""
    if X.dim() != 2 or W.dim() != 2 or X.shape[1] != W.shape[0]:
        raise ValueError("X must be (M, K) and W must be (K, N)")
    if X.dtype != W.dtype:
        raise TypeError("X and W must share a dtype")
    if not (X.is_cuda and W.is_cuda):
        raise ValueError("search_async() takes CUDA tensors")
    lib = library()
    X = X.contiguous()
    W = W.contiguous()
    M, K = X.shape
    N = W.shape[1]
    if group <= 0 or K % group or N % 8:
        raise ValueError("group must divide K and N must be a multiple of 8")
    outs = _alloc_outputs(K, N, group, n_grid, X.device) if out is None else tuple(out)
    scales, codes, steps, zeros, losses, best = outs
    if status is None:
        status = torch.full((1,), -1, dtype=torch.int32, pin_memory=True)
    elif not status.is_pinned():
        raise ValueError("status must be pinned host memory")
    if stream is None:  # the stream current now is the one wait() synchronizes later
        stream = torch.cuda.current_stream(X.device)
    handle = _stream_handle(stream, X.device)   # a side stream waits for the current one
    _check(lib.awq_search_async(_ptr(X), _ptr(W), _dtype_code(X), M, K, N, group, n_grid, _ptr(scales), _ptr(codes),
                                _ptr(steps), _ptr(zeros), _ptr(losses), _ptr(best), status.data_ptr(), handle))
    if stream.cuda_stream != torch.cuda.current_stream(X.device).cuda_stream:
        # the caching allocator must not hand these blocks out again before `stream` is done
        for t in (X, W) + outs:
            t.record_stream(stream)
    ticket = int(lib.awq_profile_last_ticket())
    out = SearchOutput(scales, codes, steps, zeros, losses, best, None)
    # keep the inputs alive until the stream has passed the call
    pending = PendingSearch(out, status, stream, X.device, ticket)
    pending._inputs = (X, W)
    return pending


def activation_statistic(X: torch.Tensor, *, stream=None) -> torch.Tensor:
    """Step 1 alone: a_j = mean_m |X[m, j]| (fp32, shape (K,))."""
    M, K = X.shape
    X = X.contiguous()
    a = torch.empty(K, dtype=torch.float32, device=X.device)
    _check(library().awq_activation_statistic(_ptr(X), _dtype_code(X), M, K, _ptr(a),
                                              _stream_handle(stream, X.device)))
    return a


def candidate_scales(a: torch.Tensor, n_grid: int = 20, *, stream=None) -> torch.Tensor:
    """Step 2 alone: the (n_grid, K) candidate scale vectors."""
    a = a.contiguous()
    S = torch.empty(n_grid, a.numel(), dtype=torch.float32, device=a.device)
    _check(library().awq_candidate_scales(_ptr(a), a.numel(), n_grid, _ptr(S), _stream_handle(stream, a.device)))
    return S


def qdq_candidates(W: torch.Tensor, S: torch.Tensor, group: int = 128, *, stream=None) -> torch.Tensor:
    """Steps 3-4 alone: (n_grid + 1, N, K) bf16 operands; slot 0 is bf16(W)^T."""
    K, N = W.shape
    W = W.contiguous()
    S = S.contiguous()
    n_grid = S.shape[0]
    out = torch.empty(n_grid + 1, N, K, dtype=torch.bfloat16, device=W.device)
    _check(library().awq_qdq_candidates(_ptr(W), _dtype_code(W), K, N, group, n_grid, _ptr(S), _ptr(out),
                                        _stream_handle(stream, W.device)))
    return out


def search_host(X: torch.Tensor, W: torch.Tensor, group: int = 128, n_grid: int = 20, *,
                stream: torch.cuda.Stream | None = None, out: tuple | None = None,
                device: int | torch.device | None = None) -> SearchOutput:
    """End-to-end form: host tensors in (pinned for asynchronous copies), host tensors out.

    The library copies X and W to the device, runs the search and copies the artifact
    back, all on `stream` (default: the current stream of `device`).
    """
    if X.is_cuda or W.is_cuda:
        raise ValueError("search_host() takes host tensors")
    if X.dtype != W.dtype:
        raise TypeError("X and W must share a dtype")
    lib = library()
    X = X.contiguous()
    W = W.contiguous()
    M, K = X.shape
    N = W.shape[1]
    out = _alloc_outputs(K, N, group, n_grid, None, pin=True) if out is None else _with_best(out)
    scales, codes, steps, zeros, losses, best = out
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = lib.awq_search_host(_ptr(X), _ptr(W), _dtype_code(X), M, K, N, group, n_grid, _ptr(scales), _ptr(codes),
                             _ptr(steps), _ptr(zeros), _ptr(losses), _ptr(best), _stream_handle(stream, dev))
    _check(st)
    return SearchOutput(scales, codes, steps, zeros, losses, best)


def search_host_batch(Xs: list, Ws: list, group: int = 128, n_grid: int = 20, *,
                      stream: torch.cuda.Stream | None = None, outs: list | None = None,
                      device: int | torch.device | None = None) -> list:
    """search_host() for several layers of one shape: layer i + 1's inputs are copied while
    layer i is searched and layer i's artifact is copied back while layer i + 1 runs."""
    if len(Xs) != len(Ws) or not Xs:
        raise ValueError("Xs and Ws must be equally long, non-empty lists")
    X0, W0 = Xs[0], Ws[0]
    for X, W in zip(Xs, Ws):
        if X.is_cuda or W.is_cuda:
            raise ValueError("search_host_batch() takes host tensors")
        if X.dtype != X0.dtype or W.dtype != X0.dtype or X.shape != X0.shape or W.shape != W0.shape:
            raise TypeError("every layer needs the same shapes and dtype")
    Xs = [X.contiguous() for X in Xs]
    Ws = [W.contiguous() for W in Ws]
    M, K = X0.shape
    N = W0.shape[1]
    if outs is None:
        outs = [_alloc_outputs(K, N, group, n_grid, None, pin=True) for _ in Xs]
    if len(outs) != len(Xs):
        raise ValueError("outs needs one output tuple per layer")
    outs = [_with_best(o) for o in outs]
    n = len(Xs)

    def arr(ptrs):
        return (ctypes.c_void_p * n)(*ptrs)

    keep = [arr([_ptr(x) for x in Xs]), arr([_ptr(w) for w in Ws])] + [arr([_ptr(o[k]) for o in outs])
                                                                        for k in range(6)]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = library().awq_search_host_batch(n, keep[0], keep[1], _dtype_code(X0), M, K, N, group, n_grid, keep[2],
                                         keep[3], keep[4], keep[5], keep[6], keep[7], _stream_handle(stream, dev))
    _check(st)
    return [SearchOutput(*o) for o in outs]


@dataclass
class ClipOutput:
    max_val: torch.Tensor              # (K/group, N) fp32: the chosen clamp threshold
    best: torch.Tensor                 # (K/group, N) int32: index of the chosen shrink factor
    codes: torch.Tensor                # (K, N/8) int32: the clipped group's codes
    steps: torch.Tensor                # (K/group, N) fp16
    zeros: torch.Tensor                # (K/group, N) fp16
    errors: torch.Tensor | None = None  # (n_shrink, K/group, N) fp64


def clip_token_count(M: int, max_tokens: int = 512) -> int:
    """Number of rows of X the clipping search samples."""
    return int(library().awq_clip_token_count(M, max_tokens))


def clip_search(X: torch.Tensor, W: torch.Tensor, scales: torch.Tensor, group: int = 128, n_shrink: int = 10,
                max_tokens: int = 512, *, errors: bool = False, quantizer: str = "asym",
                stream: torch.cuda.Stream | None = None) -> ClipOutput:
    """Clipping search after the scaling on device tensors X (M, K), W (K, N) and the
    chosen scales (K,) fp32: per (group, column) threshold, its index, and the artifact
    of the clipped, scaled weights."""
    if X.dim() != 2 or W.dim() != 2 or X.shape[1] != W.shape[0] or scales.shape != (X.shape[1],):
        raise ValueError("X must be (M, K), W (K, N) and scales (K,)")
    if X.dtype != W.dtype:
        raise TypeError("X and W must share a dtype")
    if scales.dtype != torch.float32:
        raise TypeError("scales must be float32")
    if not (X.is_cuda and W.is_cuda and scales.is_cuda):
        raise ValueError("clip_search() takes CUDA tensors")
    lib = library()
    X, W, scales = X.contiguous(), W.contiguous(), scales.contiguous()
    M, K = X.shape
    N = W.shape[1]
    if group <= 0 or K % group or N % 8:
        raise ValueError("group must divide K and N must be a multiple of 8")
    dev = X.device
    G = K // group
    max_val = torch.empty(G, N, dtype=torch.float32, device=dev)
    best = torch.empty(G, N, dtype=torch.int32, device=dev)
    codes = torch.empty(K, N // 8, dtype=torch.int32, device=dev)
    steps = torch.empty(G, N, dtype=torch.float16, device=dev)
    zeros = torch.empty(G, N, dtype=torch.float16, device=dev)
    errs = torch.empty(n_shrink, G, N, dtype=torch.float64, device=dev) if errors else None
    if quantizer not in QUANTIZERS:
        raise ValueError(f"quantizer must be one of {sorted(QUANTIZERS)}")
    st = lib.awq_clip_search(_ptr(X), _ptr(W), _dtype_code(X), _ptr(scales), M, K, N, group, n_shrink, max_tokens,
                             QUANTIZERS[quantizer], _ptr(max_val), _ptr(best), _ptr(errs), _ptr(codes), _ptr(steps), _ptr(zeros),
                             _stream_handle(stream, dev))
    _check(st)
    return ClipOutput(max_val, best, codes, steps, zeros, errs)


def clip_profile_last() -> dict:
    """Device times (ms) of the last clipping search's kernels (profiling on)."""
    ms = (ctypes.c_float * 2)()
    library().awq_clip_profile_last(ms, 2)
    return {"gram": ms[0], "clip_search": ms[1]}


def fp64_mma_peak(device=None, stream=None) -> float:
    """Measured fp64 tensor-core MMA throughput of the device, TFLOP/s."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = ctypes.c_double(0.0)
    _check(library().awq_fp64_mma_peak(ctypes.byref(out), _stream_handle(stream, dev)))
    return out.value


def _artifact_args(codes, steps, zeros, group):
    if not (codes.is_cuda and steps.is_cuda and zeros.is_cuda):
        raise ValueError("the artifact must be on the device")
    if codes.dtype != torch.int32 or steps.dtype != torch.float16 or zeros.dtype != torch.float16:
        raise TypeError("codes int32, steps and zeros float16")
    K = codes.shape[0]
    N = steps.shape[1]
    if codes.shape != (K, N // 8) or steps.shape != (K // group, N) or zeros.shape != steps.shape:
        raise ValueError("codes (K, N/8), steps and zeros (K/group, N)")
    return codes.contiguous(), steps.contiguous(), zeros.contiguous(), K, N


def w4a16_matmul(A: torch.Tensor, codes: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor, group: int = 128,
                 *, stream=None) -> torch.Tensor:
    """Y = A w16 with w16 = fp16((q - z) step) from the packed artifact; A (M, K) fp16 on the
    device, already divided by the scales. Returns (M, N) fp32 (for M <= 16 the call is
    asynchronous on `stream`)."""
    codes, steps, zeros, K, N = _artifact_args(codes, steps, zeros, group)
    if A.dtype != torch.float16 or not A.is_cuda or A.dim() != 2 or A.shape[1] != K:
        raise ValueError("A must be a (M, K) float16 CUDA tensor")
    A = A.contiguous()
    Y = torch.empty(A.shape[0], N, dtype=torch.float32, device=A.device)
    _check(library().awq_w4a16_matmul(_ptr(A), _ptr(codes), _ptr(steps), _ptr(zeros), A.shape[0], K, N, group,
                                      _ptr(Y), _stream_handle(stream, A.device)))
    return Y


def w4a16_dequant(codes: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor, group: int = 128, *,
                  stream=None) -> torch.Tensor:
    """The dequantized operand, transposed: (N, K) fp16, K contiguous."""
    codes, steps, zeros, K, N = _artifact_args(codes, steps, zeros, group)
    out = torch.empty(N, K, dtype=torch.float16, device=codes.device)
    _check(library().awq_w4a16_dequant(_ptr(codes), _ptr(steps), _ptr(zeros), K, N, group, _ptr(out),
                                       _stream_handle(stream, codes.device)))
    return out


def w4a16_profile_last() -> float:
    """Device time (ms) of the last W4A16 call's kernels when profiling is on, else -1."""
    return float(library().awq_w4a16_profile_last())


def search_mlp(X: torch.Tensor, W_gu: torch.Tensor, W_down: torch.Tensor, group: int = 128, n_grid: int = 20, *,
               stream: torch.cuda.Stream | None = None) -> SearchOutput:
    """Scale search of the gate and up projections W_gu = [W_gate | W_up] (K, 2F) scored on
    the MLP block output down(silu(X W_gate) * (X W_up)) with W_down (F, K_out)."""
    if not (X.is_cuda and W_gu.is_cuda and W_down.is_cuda):
        raise ValueError("search_mlp() takes CUDA tensors")
    if not (X.dtype == W_gu.dtype == W_down.dtype):
        raise TypeError("X, W_gu and W_down must share a dtype")
    X, W_gu, W_down = X.contiguous(), W_gu.contiguous(), W_down.contiguous()
    M, K = X.shape
    N = W_gu.shape[1]
    F, K_out = W_down.shape
    if W_gu.shape[0] != K or N != 2 * F:
        raise ValueError("W_gu must be (K, 2F) and W_down (F, K_out)")
    scales, codes, steps, zeros, losses, best = _alloc_outputs(K, N, group, n_grid, X.device)
    _check(library().awq_search_mlp(_ptr(X), _ptr(W_gu), _ptr(W_down), _dtype_code(X), M, K, F, K_out, group, n_grid,
                                    _ptr(scales), _ptr(codes), _ptr(steps), _ptr(zeros), _ptr(losses), _ptr(best),
                                    _stream_handle(stream, X.device)))
    return SearchOutput(scales, codes, steps, zeros, losses, best)


ATTN_HEAD_DIM = 128   # head dimension of the attention-block objective


def search_attn(X: torch.Tensor, W_qkv: torch.Tensor, n_heads: int, seq_len: int, group: int = 128,
                n_grid: int = 20, *, stream: torch.cuda.Stream | None = None) -> SearchOutput:
    """Scale search of the query, key and value projections W_qkv = [W_q | W_k | W_v]
    (K, 3D), D = n_heads * 128, scored on the causal multi-head attention output of the
    calibration sequences (seq_len consecutive rows of X (M, K) each)."""
    if not (X.is_cuda and W_qkv.is_cuda):
        raise ValueError("search_attn() takes CUDA tensors")
    if X.dtype != W_qkv.dtype:
        raise TypeError("X and W_qkv must share a dtype")
    X, W_qkv = X.contiguous(), W_qkv.contiguous()
    M, K = X.shape
    N = W_qkv.shape[1]
    if W_qkv.shape[0] != K or N % 3:
        raise ValueError("W_qkv must be (K, 3D)")
    scales, codes, steps, zeros, losses, best = _alloc_outputs(K, N, group, n_grid, X.device)
    _check(library().awq_search_attn(_ptr(X), _ptr(W_qkv), _dtype_code(X), M, K, N // 3, n_heads, seq_len, group,
                                     n_grid, _ptr(scales), _ptr(codes), _ptr(steps), _ptr(zeros), _ptr(losses),
                                     _ptr(best), _stream_handle(stream, X.device)))
    return SearchOutput(scales, codes, steps, zeros, losses, best)


def attn_profile_last() -> dict:
    """Device times (ms) of the last attention-block search's phases (profiling on)."""
    ms = (ctypes.c_float * 6)()
    n = library().awq_attn_profile_last(ms, 6)
    names = ("qdq", "gemm_qk", "gemm_vt", "attention_reference", "attention_loss", "reduce_pack")
    return {names[i]: float(ms[i]) for i in range(n)}


def w4a16_repack(codes: torch.Tensor, *, stream=None) -> torch.Tensor:
    """The artifact's codes (K, N/8) int32 rewritten in the decode kernel's order (same size)."""
    if not codes.is_cuda or codes.dtype != torch.int32 or codes.dim() != 2:
        raise ValueError("codes must be a (K, N/8) int32 CUDA tensor")
    codes = codes.contiguous()
    K, N = codes.shape[0], codes.shape[1] * 8
    out = torch.empty_like(codes)
    _check(library().awq_w4a16_repack(_ptr(codes), K, N, _ptr(out), _stream_handle(stream, codes.device)))
    return out


def w4a16_matmul_packed(A: torch.Tensor, packed: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor,
                        group: int = 128, *, stream=None) -> torch.Tensor:
    """w4a16_matmul for at most 16 tokens on repacked codes (asynchronous on `stream`)."""
    packed, steps, zeros, K, N = _artifact_args(packed, steps, zeros, group)
    if A.dtype != torch.float16 or not A.is_cuda or A.dim() != 2 or A.shape[1] != K:
        raise ValueError("A must be a (M, K) float16 CUDA tensor")
    A = A.contiguous()
    Y = torch.empty(A.shape[0], N, dtype=torch.float32, device=A.device)
    _check(library().awq_w4a16_matmul_packed(_ptr(A), _ptr(packed), _ptr(steps), _ptr(zeros), A.shape[0], K, N,
                                             group, _ptr(Y), _stream_handle(stream, A.device)))
    return Y


def loss_gemm_variant(M: int, K: int, N: int, n_grid: int = 20) -> int:
    """Which loss-GEMM kernel a search of this size runs (1 one-SM, 2 two-SM)."""
    return int(library().awq_loss_gemm_variant(M, K, N, n_grid))


def loss_gemm_launches(M: int, K: int, N: int, n_grid: int = 20, group: int = 128,
                       dtype: torch.dtype = torch.bfloat16) -> int:
    """How many loss-GEMM launches a search of this form runs on the current device: 1
    (reference and candidates in one launch) or 2 (the reference output in its own launch)."""
    n = int(library().awq_loss_gemm_launches(_dtype_code_of(dtype), M, K, N, group, n_grid))
    if n < 0:
        _check(-n)
    return n


def qdq_in_loss_gemm(M: int, K: int, N: int, n_grid: int = 20, group: int = 128,
                     dtype: torch.dtype = torch.bfloat16) -> bool:
    """Whether a search of this form makes its candidate operands with the loss GEMM's own
    QDQ warps (else a QDQ kernel runs before the GEMM)."""
    return bool(library().awq_qdq_in_loss_gemm(_dtype_code_of(dtype), M, K, N, group, n_grid))
