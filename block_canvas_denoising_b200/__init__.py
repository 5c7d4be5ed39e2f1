"""B200 (sm_100a) denoising step of block discrete-diffusion text generation.

A thin ctypes binding of ``libdg.so`` (C ABI in ``include/dg.h``): argument
marshalling only.  Every step of the path runs in the library's CUDA
kernels; PyTorch supplies device memory and streams.  There is no CPU
fallback: if the library is missing or no sm_100 device is present, calls
raise ``DGError``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

__all__ = ["DGError", "Params", "lib", "workspace_size", "Workspace", "denoise_step",
           "debug_logits", "device_status", "denoise_loop", "debug_gumbel",
           "selftest_bounded_wait", "set_head_events", "denoise_step_noalloc", "noalloc_status",
           "noalloc_selftest_bounded_wait", "STATUS", "E_BF16", "E_FP8_E4M3",
           "SELECT_CUMSUM", "SELECT_MI", "SELECT_TOPK", "partials_count", "head_partials", "merge_partials",
           "gather_partials", "init_canvas", "generate_blocks", "loop_state_bytes", "LoopState",
           "denoise_loop_graph", "selfcond_workspace_size", "embedder_transpose", "denoise_step_selfcond"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

E_BF16 = 0
E_FP8_E4M3 = 1

STATUS = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_UNSUPPORTED_SHAPE", 3: "DG_ERR_WORKSPACE",
          4: "DG_ERR_RANGE", 5: "DG_ERR_CUDA", 6: "DG_ERR_TIMEOUT", 7: "DG_ERR_CALLBACK",
          8: "DG_ERR_NO_DEVICE", 9: "DG_ERR_VALUE"}


class DGError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, self.code)}")


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("d", ctypes.c_int32),
                ("V", ctypes.c_int32), ("e_dtype", ctypes.c_int32)]


class _Params(ctypes.Structure):
    _fields_ = [("tau0", ctypes.c_double), ("tau1", ctypes.c_double), ("max_steps", ctypes.c_int32),
                ("entropy_bound", ctypes.c_double), ("stop_entropy", ctypes.c_double),
                ("seed", ctypes.c_uint64), ("selection_rule", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("block", ctypes.c_int32)]


SELECT_CUMSUM = 0
SELECT_MI = 1
SELECT_TOPK = 2


_HIDDEN_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_void_p, ctypes.c_void_p)
_BLOCK_HIDDEN_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p)


@dataclass
class Params:
    """Sampler parameters (defaults: the serving configuration of the docs)."""
    tau0: float = 0.8
    tau1: float = 0.4
    max_steps: int = 48
    entropy_bound: float = 0.1
    stop_entropy: float = 0.005
    seed: int = 1234
    selection_rule: int = SELECT_CUMSUM
    top_k: int = 1
    block: int = 0

    def c(self) -> _Params:
        return _Params(self.tau0, self.tau1, self.max_steps, self.entropy_bound,
                       self.stop_entropy, int(self.seed) & 0xFFFFFFFFFFFFFFFF,
                       int(self.selection_rule), int(self.top_k), int(self.block))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdg.so (built in-tree by ``block_canvas_denoising_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DGError(5, f"libdg.so not built at {LIB_PATH}")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        L.dg_default_params.restype = _Params
        L.dg_error_string.restype = ctypes.c_char_p
        L.dg_error_string.argtypes = [ctypes.c_int]
        L.dg_workspace_size.restype = ctypes.c_size_t
        L.dg_workspace_size.argtypes = [ctypes.POINTER(_Shape)]
        L.dg_workspace_init.argtypes = [P, ctypes.c_size_t, P]
        step_args = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P, P, P, P, P,
                     P, P, P, P, P, P, P]
        L.dg_denoise_step.argtypes = step_args + [P, ctypes.c_size_t, P]
        L.dg_debug_logits.argtypes = step_args + [P, P, ctypes.c_size_t, P]
        L.dg_device_status.argtypes = [P, ctypes.c_size_t, P]
        L.dg_denoise_loop.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P,
                                      _HIDDEN_FN, P, ctypes.c_int32, P, P, P, P, P,
                                      P, P, P, P, P, P, ctypes.c_size_t, P]
        L.dg_selftest_bounded_wait.argtypes = [ctypes.c_uint64, P, ctypes.c_size_t, P]
        L.dg_debug_gumbel.argtypes = [P, ctypes.c_int32, P, P, P]
        L.dg_set_head_events.argtypes = [P, P]
        L.dg_denoise_step_noalloc.argtypes = step_args + [P]
        L.dg_denoise_step_noalloc.restype = ctypes.c_int
        L.dg_noalloc_status.argtypes = [P]
        L.dg_noalloc_status.restype = ctypes.c_int
        L.dg_noalloc_selftest_bounded_wait.argtypes = [ctypes.c_uint64, P]
        L.dg_noalloc_selftest_bounded_wait.restype = ctypes.c_int
        L.dg_last_error_message.restype = ctypes.c_char_p
        L.dg_selfcond_workspace_size.argtypes = [ctypes.POINTER(_Shape)]
        L.dg_selfcond_workspace_size.restype = ctypes.c_size_t
        L.dg_embedder_transpose.argtypes = [ctypes.POINTER(_Shape), P, P, P]
        L.dg_embedder_transpose.restype = ctypes.c_int
        L.dg_denoise_step_selfcond.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P, P, P, P, P,
                                               P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.dg_denoise_step_selfcond.restype = ctypes.c_int
        L.dg_loop_state_bytes.argtypes = [ctypes.c_int32]
        L.dg_loop_state_bytes.restype = ctypes.c_size_t
        L.dg_denoise_loop_graph.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P, P,
                                            ctypes.c_int32, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P,
                                            ctypes.c_size_t, P]
        L.dg_denoise_loop_graph.restype = ctypes.c_int
        L.dg_loop_graph_create.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P, P, P, P, P,
                                           P, P, P, P, P, P, ctypes.c_size_t, P, ctypes.c_size_t,
                                           ctypes.POINTER(ctypes.c_void_p)]
        L.dg_loop_graph_create.restype = ctypes.c_int
        L.dg_loop_graph_run.argtypes = [P, ctypes.c_int32, P, P, P]
        L.dg_loop_graph_run.restype = ctypes.c_int
        L.dg_loop_graph_destroy.argtypes = [P]
        L.dg_loop_graph_destroy.restype = None
        L.dg_init_canvas.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P]
        L.dg_init_canvas.restype = ctypes.c_int
        L.dg_generate_blocks.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, P, ctypes.c_int32,
                                         _BLOCK_HIDDEN_FN, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.dg_generate_blocks.restype = ctypes.c_int
        L.dg_partials_count.restype = ctypes.c_int32
        L.dg_partials_count.argtypes = [ctypes.POINTER(_Shape)]
        L.dg_head_partials.restype = ctypes.c_int
        L.dg_head_partials.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), ctypes.c_int32,
                                       P, P, P, P, P, P, ctypes.c_size_t, P]
        L.dg_merge_partials.restype = ctypes.c_int
        L.dg_merge_partials.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Params), P, ctypes.c_int32,
                                        ctypes.c_int32, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        for name in ("dg_workspace_init", "dg_denoise_step", "dg_debug_logits", "dg_device_status",
                     "dg_denoise_loop", "dg_selftest_bounded_wait", "dg_debug_gumbel",
                     "dg_set_head_events"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(code: int, where: str) -> None:
    if code != 0:
        msg = lib().dg_last_error_message().decode(errors="replace")
        raise DGError(code, where + (f" [{msg}]" if msg else ""))


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _host(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def _shape(B: int, d: int, V: int, e_dtype: int = E_BF16, L: int = 256) -> _Shape:
    return _Shape(B, L, d, V, e_dtype)


def workspace_size(B: int, d: int, V: int, e_dtype: int = E_BF16, L: int = 256) -> int:
    """Bytes of workspace one step needs on the current device (0 if invalid)."""
    return int(lib().dg_workspace_size(ctypes.byref(_shape(B, d, V, e_dtype, L))))


def selfcond_workspace_size(B: int, d: int, V: int, e_dtype: int = E_BF16, L: int = 256) -> int:
    """Bytes of workspace a step with the self-conditioning signal needs."""
    return int(lib().dg_selfcond_workspace_size(ctypes.byref(_shape(B, d, V, e_dtype, L))))


class Workspace:
    """Device scratch for steps of one shape (a zeroed torch uint8 buffer);
    ``selfcond=True`` sizes it for ``denoise_step_selfcond``."""

    def __init__(self, B: int, d: int, V: int, e_dtype: int = E_BF16, device=None, stream=None,
                 selfcond: bool = False):
        import torch
        n = selfcond_workspace_size(B, d, V, e_dtype) if selfcond else workspace_size(B, d, V, e_dtype)
        if n == 0:
            raise DGError(2, "workspace_size")
        self.nbytes = n
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
        _check(lib().dg_workspace_init(_ptr(self.buf), ctypes.c_size_t(n), _stream(stream)),
               "dg_workspace_init")


def _step_call(fn_name, h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled,
               argmax, stop, ws: Workspace, params: Params, e_scale=None, active=None, logits=None,
               stream=None):
    B = int(len(step_idx))
    R, d = h.shape
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // max(B, 1))
    prm = params.c()
    ks = _host(step_idx, np.int32)
    hp = _host(has_prev, np.uint8)
    act = None if active is None else _host(active, np.uint8)
    args = [ctypes.byref(shp), ctypes.byref(prm), _ptr(h), _ptr(E), _ptr(e_scale),
            ks.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p),
            None if act is None else act.ctypes.data_as(ctypes.c_void_p),
            _ptr(canvas), _ptr(prev_argmax), _ptr(accept), _ptr(entropy), _ptr(sampled),
            _ptr(argmax), _ptr(stop)]
    if fn_name == "dg_debug_logits":
        args.append(_ptr(logits))
    args += [_ptr(ws.buf), ctypes.c_size_t(ws.nbytes), _stream(stream)]
    _check(getattr(lib(), fn_name)(*args), fn_name)


def denoise_step(h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled, argmax,
                 stop, ws: Workspace, params: Params = Params(), e_scale=None, active=None,
                 stream=None) -> None:
    """Enqueue one step (see ``dg_denoise_step`` in include/dg.h).

    Tensors are CUDA tensors: h bf16 [B*256, d], E bf16 [V, d] (or uint8
    E4M3 codes with ``e_scale`` float [V]), canvas / prev_argmax / sampled /
    argmax int32 [B*256], accept uint8 [B*256], entropy float32 [B*256],
    stop int32 [B].  ``step_idx``, ``has_prev`` and ``active`` are host
    sequences of length B."""
    _step_call("dg_denoise_step", h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy,
               sampled, argmax, stop, ws, params, e_scale, active, None, stream)


def denoise_step_noalloc(h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled,
                         argmax, stop, params: Params = Params(), e_scale=None, active=None,
                         stream=None) -> None:
    """``dg_denoise_step_noalloc``: the same step without a caller workspace,
    for callers that cannot allocate device memory (the scratch is a fixed
    8 MiB array inside the library; calls must not overlap on the GPU; a
    device-side fault is reported by ``noalloc_status``)."""
    B = int(len(step_idx))
    R, d = h.shape
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // max(B, 1))
    prm = params.c()
    ks = _host(step_idx, np.int32)
    hp = _host(has_prev, np.uint8)
    act = None if active is None else _host(active, np.uint8)
    _check(lib().dg_denoise_step_noalloc(
        ctypes.byref(shp), ctypes.byref(prm), _ptr(h), _ptr(E), _ptr(e_scale),
        ks.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p),
        None if act is None else act.ctypes.data_as(ctypes.c_void_p),
        _ptr(canvas), _ptr(prev_argmax), _ptr(accept), _ptr(entropy), _ptr(sampled),
        _ptr(argmax), _ptr(stop), _stream(stream)), "dg_denoise_step_noalloc")


def noalloc_status(stream=None) -> int:
    """Synchronise and read/clear the fault latch of the allocation-free
    step's scratch array on the current device (0 = no fault)."""
    return int(lib().dg_noalloc_status(_stream(stream)))


def noalloc_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """The bounded-wait self test against the allocation-free step's latch;
    returns the status it leaves (6 = timed out as designed)."""
    return int(lib().dg_noalloc_selftest_bounded_wait(ctypes.c_uint64(limit_ns), _stream(stream)))


def debug_logits(h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled, argmax,
                 stop, logits, ws: Workspace, params: Params = Params(), e_scale=None, active=None,
                 stream=None) -> None:
    """The same step, also writing the float32 logits [B*256, V] it consumed."""
    _step_call("dg_debug_logits", h, E, step_idx, has_prev, canvas, prev_argmax, accept, entropy,
               sampled, argmax, stop, ws, params, e_scale, active, logits, stream)


def device_status(ws: Workspace, stream=None) -> int:
    """Synchronise and read/clear the device fault latch (0 = clean)."""
    return int(lib().dg_device_status(_ptr(ws.buf), ctypes.c_size_t(ws.nbytes), _stream(stream)))


def denoise_loop(E, hidden_fn, h_buf, canvas, prev_argmax, has_prev, accept, entropy, sampled,
                 argmax, stop, ws: Workspace, params: Params = Params(), k_start: int = 0,
                 e_scale=None, stream=None):
    """Run the adaptive loop (``dg_denoise_loop``).

    ``hidden_fn(k, canvas_tensor, h_buf)`` must fill ``h_buf`` for step k on
    the current stream and return None.  ``has_prev`` is a host uint8 numpy
    array [B] updated in place.  Returns the host int32 array of steps taken.
    """
    B = int(len(has_prev))
    R, d = h_buf.shape
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // B)
    prm = params.c()
    steps = np.zeros(B, np.int32)
    assert isinstance(has_prev, np.ndarray) and has_prev.dtype == np.uint8
    errors = []

    def cb(k, canvas_ptr, h_ptr, user, stream_ptr):
        try:
            hidden_fn(int(k), canvas, h_buf)
            return 0
        except Exception as exc:  # reported as DG_ERR_CALLBACK
            errors.append(exc)
            return 1

    cfn = _HIDDEN_FN(cb)
    code = lib().dg_denoise_loop(
        ctypes.byref(shp), ctypes.byref(prm), _ptr(E), _ptr(e_scale), cfn, None,
        ctypes.c_int32(k_start), _ptr(h_buf), _ptr(canvas), _ptr(prev_argmax),
        has_prev.ctypes.data_as(ctypes.c_void_p), steps.ctypes.data_as(ctypes.c_void_p),
        _ptr(accept), _ptr(entropy), _ptr(sampled), _ptr(argmax), _ptr(stop), _ptr(ws.buf),
        ctypes.c_size_t(ws.nbytes), _stream(stream))
    if code != 0:
        err = DGError(code, "dg_denoise_loop")
        if errors:
            raise err from errors[0]
        raise err
    return steps


def loop_state_bytes(B: int) -> int:
    """Bytes of device loop state ``dg_denoise_loop_graph`` needs for B canvases."""
    return int(lib().dg_loop_state_bytes(ctypes.c_int32(B)))


class LoopState:
    """Device loop state of the device-side loop (a torch uint8 buffer);
    ``k`` is a one-element int32 view of the step index the loop's graph
    body is about to run, for a hidden-state graph to read."""

    def __init__(self, B: int, device=None):
        import torch
        n = loop_state_bytes(B)
        if n == 0:
            raise DGError(1, "loop_state_bytes")
        self.nbytes = n
        self.buf = torch.zeros(n, dtype=torch.uint8, device=device or "cuda")
        self.k = self.buf[:4].view(torch.int32)


def denoise_loop_graph(E, hidden_graph, h_buf, canvas, prev_argmax, has_prev, accept, entropy, sampled,
                       argmax, stop, ws: Workspace, state: LoopState, params: Params = Params(),
                       k_start: int = 0, e_scale=None, stream=None):
    """The adaptive loop run on the device (``dg_denoise_loop_graph``).

    ``hidden_graph`` is a ``torch.cuda.CUDAGraph`` captured with
    ``keep_graph=True`` that writes step ``state.k``'s hidden states into
    ``h_buf`` (or None: ``h_buf`` stays as it is).  ``has_prev`` is a host
    uint8 numpy array [B] updated in place.  Returns the host int32 array of
    steps taken."""
    B = int(len(has_prev))
    R, d = h_buf.shape
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // B)
    prm = params.c()
    steps = np.zeros(B, np.int32)
    assert isinstance(has_prev, np.ndarray) and has_prev.dtype == np.uint8
    g = None if hidden_graph is None else ctypes.c_void_p(int(hidden_graph.raw_cuda_graph()))
    _check(lib().dg_denoise_loop_graph(
        ctypes.byref(shp), ctypes.byref(prm), _ptr(E), _ptr(e_scale), g, ctypes.c_int32(k_start), _ptr(h_buf),
        _ptr(canvas), _ptr(prev_argmax), has_prev.ctypes.data_as(ctypes.c_void_p),
        steps.ctypes.data_as(ctypes.c_void_p), _ptr(accept), _ptr(entropy), _ptr(sampled), _ptr(argmax),
        _ptr(stop), _ptr(state.buf), ctypes.c_size_t(state.nbytes), _ptr(ws.buf), ctypes.c_size_t(ws.nbytes),
        _stream(stream)), "dg_denoise_loop_graph")
    return steps


class LoopGraph:
    """The device-side loop built once and run many times
    (``dg_loop_graph_create`` / ``_run`` / ``_destroy``): the buffers are
    fixed at construction (they must outlive the object); ``run`` takes the
    first step, the host uint8 ``has_prev`` array (updated in place) and
    returns the host int32 array of steps taken."""

    def __init__(self, E, hidden_graph, h_buf, canvas, prev_argmax, accept, entropy, sampled, argmax, stop,
                 ws: Workspace, state: LoopState, params: Params = Params(), e_scale=None):
        B = int(stop.shape[0])
        R, d = h_buf.shape
        V = E.shape[0]
        e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
        self.B = B
        shp = _shape(B, d, V, e_dtype, L=R // B)
        prm = params.c()
        g = None if hidden_graph is None else ctypes.c_void_p(int(hidden_graph.raw_cuda_graph()))
        handle = ctypes.c_void_p()
        # the buffers stay referenced for the handle's lifetime
        self._keep = (E, e_scale, h_buf, canvas, prev_argmax, accept, entropy, sampled, argmax, stop, ws, state)
        self._h = None
        _check(lib().dg_loop_graph_create(
            ctypes.byref(shp), ctypes.byref(prm), _ptr(E), _ptr(e_scale), g, _ptr(h_buf), _ptr(canvas),
            _ptr(prev_argmax), _ptr(accept), _ptr(entropy), _ptr(sampled), _ptr(argmax), _ptr(stop),
            _ptr(state.buf), ctypes.c_size_t(state.nbytes), _ptr(ws.buf), ctypes.c_size_t(ws.nbytes),
            ctypes.byref(handle)), "dg_loop_graph_create")
        self._h = handle

    def run(self, has_prev, k_start: int = 0, stream=None):
        assert isinstance(has_prev, np.ndarray) and has_prev.dtype == np.uint8 and len(has_prev) == self.B
        steps = np.zeros(self.B, np.int32)
        _check(lib().dg_loop_graph_run(self._h, ctypes.c_int32(k_start), has_prev.ctypes.data_as(ctypes.c_void_p),
                                       steps.ctypes.data_as(ctypes.c_void_p), _stream(stream)), "dg_loop_graph_run")
        return steps

    def close(self) -> None:
        if self._h is not None:
            lib().dg_loop_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def embedder_transpose(E, E_t, e_fp8: bool = False, stream=None) -> None:
    """E_t [d, V] bf16 = E^T (``dg_embedder_transpose``); E bf16 [V, d], or
    E4M3 codes (uint8) with ``e_fp8``."""
    V, d = E.shape
    shp = _shape(1, d, V, E_FP8_E4M3 if e_fp8 else E_BF16)
    _check(lib().dg_embedder_transpose(ctypes.byref(shp), _ptr(E), _ptr(E_t), _stream(stream)),
           "dg_embedder_transpose")


def denoise_step_selfcond(h, E, E_t, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled, argmax,
                          stop, signal, ws: Workspace, params: Params = Params(), e_scale=None,
                          stream=None) -> None:
    """One step plus the self-conditioning signal (``dg_denoise_step_selfcond``):
    ``signal`` float32 [B*256, d]; ``ws`` made with ``selfcond=True``."""
    B = int(len(step_idx))
    R, d = h.shape
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // max(B, 1))
    prm = params.c()
    ks = _host(step_idx, np.int32)
    hp = _host(has_prev, np.uint8)
    _check(lib().dg_denoise_step_selfcond(
        ctypes.byref(shp), ctypes.byref(prm), _ptr(h), _ptr(E), _ptr(e_scale), _ptr(E_t),
        ks.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p), _ptr(canvas), _ptr(prev_argmax),
        _ptr(accept), _ptr(entropy), _ptr(sampled), _ptr(argmax), _ptr(stop), _ptr(signal), _ptr(ws.buf),
        ctypes.c_size_t(ws.nbytes), _stream(stream)), "dg_denoise_step_selfcond")


def init_canvas(canvas, B: int, V: int, params: Params = Params(), d: int = 64, stream=None) -> None:
    """Fill ``canvas`` (int32 CUDA tensor [B*256]) with the uniform noise
    block ``params.block`` starts from (``dg_init_canvas``)."""
    shp = _shape(B, d, V, E_BF16, L=int(canvas.numel()) // max(B, 1))
    prm = params.c()
    _check(lib().dg_init_canvas(ctypes.byref(shp), ctypes.byref(prm), _ptr(canvas), _stream(stream)),
           "dg_init_canvas")


def generate_blocks(E, hidden_fn, n_blocks: int, h_buf, blocks, canvas, prev_argmax, accept, entropy, sampled,
                    argmax, stop, ws: Workspace, params: Params = Params(), e_scale=None, stream=None):
    """Block-by-block generation (``dg_generate_blocks``).

    ``hidden_fn(j, k, canvas_tensor, committed, h_buf)`` fills ``h_buf``
    for step k of block j on the current stream; ``committed`` is the view
    ``blocks[:j]`` of the blocks committed so far.  ``blocks`` is an int32
    CUDA tensor [n_blocks, B*256].  Returns the host int32 array of steps
    taken, [n_blocks, B]."""
    R, d = h_buf.shape
    B = int(len(stop))
    V = E.shape[0]
    e_dtype = E_BF16 if e_scale is None else E_FP8_E4M3
    shp = _shape(B, d, V, e_dtype, L=R // B)
    prm = params.c()
    steps = np.zeros((n_blocks, B), np.int32)
    errors = []

    def cb(j, k, canvas_ptr, committed_ptr, h_ptr, user, stream_ptr):
        try:
            hidden_fn(int(j), int(k), canvas, blocks[:int(j)], h_buf)
            return 0
        except Exception as exc:  # reported as DG_ERR_CALLBACK
            errors.append(exc)
            return 1

    cfn = _BLOCK_HIDDEN_FN(cb)
    code = lib().dg_generate_blocks(
        ctypes.byref(shp), ctypes.byref(prm), _ptr(E), _ptr(e_scale), ctypes.c_int32(n_blocks), cfn, None,
        _ptr(h_buf), _ptr(blocks), steps.ctypes.data_as(ctypes.c_void_p), _ptr(canvas), _ptr(prev_argmax),
        _ptr(accept), _ptr(entropy), _ptr(sampled), _ptr(argmax), _ptr(stop), _ptr(ws.buf),
        ctypes.c_size_t(ws.nbytes), _stream(stream))
    if code != 0:
        err = DGError(code, "dg_generate_blocks")
        if errors:
            raise err from errors[0]
        raise err
    return steps


def debug_gumbel(words, stream=None):
    """Device g32 and the screening pass's approximate lg2(E / ln 2), E = -ln u,
    for uint32 words (torch int32 CUDA tensor)."""
    import torch
    n = int(words.numel())
    g = torch.empty(n, dtype=torch.float32, device=words.device)
    a = torch.empty(n, dtype=torch.float32, device=words.device)
    _check(lib().dg_debug_gumbel(_ptr(words), ctypes.c_int32(n), _ptr(g), _ptr(a), _stream(stream)),
           "dg_debug_gumbel")
    return g, a


def set_head_events(ev_start=None, ev_stop=None) -> None:
    """Record torch.cuda.Events around the fused head kernel of later steps
    on this thread (None, None clears)."""
    a = None if ev_start is None else ctypes.c_void_p(ev_start.cuda_event)
    b = None if ev_stop is None else ctypes.c_void_p(ev_stop.cuda_event)
    _check(lib().dg_set_head_events(a, b), "dg_set_head_events")


def selftest_bounded_wait(limit_ns: int, ws: Workspace, stream=None) -> int:
    """Run the bounded-wait self test; returns the status code (6 = timed out as designed)."""
    return int(lib().dg_selftest_bounded_wait(ctypes.c_uint64(limit_ns), _ptr(ws.buf),
                                              ctypes.c_size_t(ws.nbytes), _stream(stream)))


# ---------------------------------------------------------------------------
# vocabulary-sharded step (dg_head_partials / dg_merge_partials)
# ---------------------------------------------------------------------------

def partials_count(B: int, d: int, V_shard: int, e_dtype: int = E_BF16, L: int = 256) -> int:
    """Records per row that one shard's head writes (``dg_partials_count``)."""
    return int(lib().dg_partials_count(ctypes.byref(_shape(B, d, V_shard, e_dtype, L))))


def head_partials(h, E_shard, v_offset: int, step_idx, partials, ws: Workspace, params: Params = Params(),
                  e_scale=None, stream=None) -> None:
    """Head and sampler over vocabulary rows v_offset .. v_offset + len(E_shard) - 1,
    writing the float32 records [7, B*256, count] into ``partials``."""
    B = int(len(step_idx))
    R, d = h.shape
    shp = _shape(B, d, E_shard.shape[0], E_BF16 if e_scale is None else E_FP8_E4M3, L=R // max(B, 1))
    prm = params.c()
    ks = _host(step_idx, np.int32)
    _check(lib().dg_head_partials(ctypes.byref(shp), ctypes.byref(prm), ctypes.c_int32(v_offset), _ptr(h),
                                  _ptr(E_shard), _ptr(e_scale), ks.ctypes.data_as(ctypes.c_void_p),
                                  _ptr(partials), _ptr(ws.buf), ctypes.c_size_t(ws.nbytes), _stream(stream)),
           "dg_head_partials")


def merge_partials(partials, V: int, d: int, step_idx, has_prev, canvas, prev_argmax, accept, entropy, sampled,
                   argmax, stop, ws: Workspace, params: Params = Params(), active=None, stream=None) -> None:
    """Merge the gathered records ``partials`` [S, 7, B*256, count] over the
    whole vocabulary V, then selection, renoise and stop."""
    B = int(len(step_idx))
    S, _, R, count = partials.shape
    shp = _shape(B, d, V, E_BF16, L=R // max(B, 1))
    prm = params.c()
    ks = _host(step_idx, np.int32)
    hp = _host(has_prev, np.uint8)
    act = None if active is None else _host(active, np.uint8)
    _check(lib().dg_merge_partials(ctypes.byref(shp), ctypes.byref(prm), _ptr(partials), ctypes.c_int32(S),
                                   ctypes.c_int32(count), ks.ctypes.data_as(ctypes.c_void_p),
                                   hp.ctypes.data_as(ctypes.c_void_p),
                                   None if act is None else act.ctypes.data_as(ctypes.c_void_p),
                                   _ptr(canvas), _ptr(prev_argmax), _ptr(accept), _ptr(entropy), _ptr(sampled),
                                   _ptr(argmax), _ptr(stop), _ptr(ws.buf), ctypes.c_size_t(ws.nbytes),
                                   _stream(stream)), "dg_merge_partials")


def gather_partials(local, group=None):
    """All-gather one rank's records [7, R, count] into [world, 7, R, count]
    (torch.distributed over the default or given process group; NCCL for
    CUDA tensors).  The only collective of the sharded step."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    local = local.contiguous()
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, local, group=group)
    return out.view((world,) + tuple(local.shape))
