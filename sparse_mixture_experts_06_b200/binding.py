"""ctypes binding of libmoe.so: one Python function per C entry point, same
names, argument marshalling only (torch tensors -> device pointers, the
current CUDA stream -> cudaStream_t).  Every step of the layer runs in the
library's kernels; if the library is missing, importing this module fails."""

from __future__ import annotations

import ctypes
import os

MOE_BF16, MOE_F32 = 0, 1
MOE_HOST_X_READY, MOE_HOST_Y_ASYNC = 1, 2
_STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
           4: "MOE_ERR_CUDA"}

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")
if not os.path.exists(lib_path):
    raise ImportError("libmoe.so is not built at %s; run python sparse_mixture_experts_06_b200/build.py"
                      % lib_path)
lib = ctypes.CDLL(lib_path)

_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "moe_workspace_size": ([_I, _I, _I, _I, _I, _I], ctypes.c_size_t),
    "moe_router_topk": ([_P, _P, _I, _I, _I, _I, _I, _P, _P, _P], _I),
    "moe_permute": ([_P, _I, _I, _I, _P, _P, _P, _P], _I),
    "moe_routing_stats": ([_P, _I, _I, _I, _I, _P, _P], _I),
    "moe_expert_ffn": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z, _P, _P], _I),
    "moe_layer_forward": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P], _I),
    "moe_layer_forward_ex": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z, _P, _P], _I),
    "moe_layer_forward_host": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P], _I),
    "moe_layer_forward_host_wait": ([_P], _I),
    "moe_layer_forward_noalloc": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P], _I),
    "moe_stack_forward": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P, _P], _I),
    "moe_release_workspace": ([_P], _I),
    "moe_device_errors": ([], ctypes.c_uint),
    "moe_profile_enable": ([_I], _I),
    "moe_profile_read": ([_P, _P, _I], _I),
    "moe_profile_stage_name": ([_I], ctypes.c_char_p),
    "moe_profile_select": ([ctypes.c_uint], _I),
    "moe_set_gemm_variant": ([_I, _I, _I, _I], _I),
    "moe_set_wait_test": ([ctypes.c_ulonglong, _I], _I),
    "moe_last_error_string": ([], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_char_p),
}
for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _ret


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%s)" % (where, _STATUS.get(code, code), moe_last_error_string()))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, ref=None):
    import torch
    if stream is None:
        dev = ref.device if ref is not None else torch.device("cuda", torch.cuda.current_device())
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError("tensors must be bfloat16 or float32, got %s" % t.dtype)


def _check(rc, where):
    if rc != 0:
        raise MoEError(rc, where)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


def moe_last_error_string() -> str:
    return lib.moe_last_error_string().decode()


def moe_version() -> str:
    return lib.moe_version().decode()


def moe_device_errors() -> int:
    return int(lib.moe_device_errors())


MOE_PROFILE_STAGES = 7


def moe_profile_enable(on: bool = True):
    _check(lib.moe_profile_enable(1 if on else 0), "moe_profile_enable")


def moe_profile_read() -> dict:
    """{stage name: (total ms, launches)} since moe_profile_enable(True); clears."""
    ms = (ctypes.c_double * MOE_PROFILE_STAGES)()
    n = (ctypes.c_int * MOE_PROFILE_STAGES)()
    rc = lib.moe_profile_read(ms, n, MOE_PROFILE_STAGES)
    if rc < 0:
        raise MoEError(4, "moe_profile_read")
    return {moe_profile_stage_name(i): (ms[i], n[i]) for i in range(MOE_PROFILE_STAGES)}


def moe_profile_stage_name(i: int) -> str:
    return lib.moe_profile_stage_name(i).decode()


def moe_profile_select(stages=None):
    """Record only the named stages (None: all)."""
    mask = 0xFFFFFFFF
    if stages is not None:
        names = [moe_profile_stage_name(i) for i in range(MOE_PROFILE_STAGES)]
        mask = 0
        for st in stages:
            mask |= 1 << names.index(st)
    _check(lib.moe_profile_select(mask), "moe_profile_select")


def moe_set_gemm_variant(cta_group=0, up_bn=0, token_rows=0, pair_cols=0):
    """Force the expert GEMMs' tile variant (0 = automatic); test and measurement hook."""
    _check(lib.moe_set_gemm_variant(cta_group, up_bn, token_rows, pair_cols), "moe_set_gemm_variant")


def moe_set_wait_test(wait_limit_ns=0, stall_epilogue=False):
    """Bound of the GEMM pipeline waits (0 = default 4 s) and the epilogue stall
    of the failure-detection test."""
    _check(lib.moe_set_wait_test(int(wait_limit_ns), 1 if stall_epilogue else 0), "moe_set_wait_test")


def moe_workspace_size(T, d, f, E, k, dtype=MOE_BF16) -> int:
    return int(lib.moe_workspace_size(T, d, f, E, k, dtype))


def moe_router_topk(x, Wg, k, topk_idx=None, topk_w=None, stream=None):
    """Router + top-k gate; returns (topk_idx [T,k] int32, topk_w [T,k] fp32)."""
    import torch
    _dev(x, Wg)
    T, d = x.shape
    E = Wg.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib.moe_router_topk(_ptr(x), _ptr(Wg), T, d, E, k, _dtype_code(x), _ptr(topk_idx), _ptr(topk_w),
                               _stream(stream, x)), "moe_router_topk")
    return topk_idx, topk_w


def moe_permute(topk_idx, E, offsets=None, perm=None, inv=None, stream=None):
    """Expert-grouped stable permutation; returns (offsets [E+1], perm [T*k], inv [T*k])."""
    import torch
    _dev(topk_idx)
    T, k = topk_idx.shape
    dv = topk_idx.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dv) if offsets is None else offsets
    perm = torch.empty(T * k, dtype=torch.int32, device=dv) if perm is None else perm
    inv = torch.empty(T * k, dtype=torch.int32, device=dv) if inv is None else inv
    _check(lib.moe_permute(_ptr(topk_idx), T, E, k, _ptr(offsets), _ptr(perm), _ptr(inv), _stream(stream, topk_idx)),
           "moe_permute")
    return offsets, perm, inv


def moe_routing_stats(topk_idx, E, seq_len=0, out=None, stream=None):
    """Expert loads and consecutive-token repetition counts (uint32 [E + 3]):
    loads[0:E], first-choice repeats, kept-set overlaps, pairs counted."""
    import torch
    _dev(topk_idx)
    T, k = topk_idx.shape
    out = torch.empty(E + 3, dtype=torch.int32, device=topk_idx.device) if out is None else out
    _check(lib.moe_routing_stats(_ptr(topk_idx), T, E, k, seq_len, _ptr(out), _stream(stream, topk_idx)),
           "moe_routing_stats")
    return out


def _workspace(T, d, f, E, k, dt, device, workspace):
    import torch
    need = moe_workspace_size(T, d, f, E, k, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def moe_expert_ffn(x, W1, W3, W2, offsets, perm, inv, topk_w, y=None, workspace=None, stream=None):
    """SwiGLU experts + gate-weighted combine from a given routing; returns y."""
    import torch
    _dev(x, W1, W3, W2, offsets, perm, inv, topk_w)
    T, d = x.shape
    E, f, _ = W1.shape
    k = topk_w.shape[-1] if topk_w.dim() == 2 else topk_w.numel() // max(T, 1)
    dt = _dtype_code(x)
    y = torch.empty_like(x) if y is None else y
    ws, nb = _workspace(T, d, f, E, k, dt, x.device, workspace)
    _check(lib.moe_expert_ffn(_ptr(x), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(offsets), _ptr(perm), _ptr(inv),
                              _ptr(topk_w), T, d, f, E, k, dt, _ptr(ws), nb, _ptr(y), _stream(stream, x)),
           "moe_expert_ffn")
    return y


def moe_layer_forward(x, Wg, W1, W3, W2, k, y=None, stream=None):
    """The whole bf16 layer with the library-owned workspace; returns y."""
    import torch
    _dev(x, Wg, W1, W3, W2)
    T, d = x.shape
    E, f, _ = W1.shape
    y = torch.empty_like(x) if y is None else y
    _check(lib.moe_layer_forward(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, f, E, k, _ptr(y),
                                 _stream(stream, x)), "moe_layer_forward")
    return y


def moe_layer_forward_host(x, Wg, W1, W3, W2, k, y=None, chunks=1, x_ready=False, y_async=False, stream=None):
    """The bf16 layer on host x / y (CPU tensors; page-locked for overlap),
    pipelined in `chunks` pieces; returns y (a pinned CPU tensor unless given).
    x_ready=True passes MOE_HOST_X_READY (x's copies may start before work
    already queued on the stream ends); y_async=True passes MOE_HOST_Y_ASYNC
    (call moe_layer_forward_host_wait before reading y).  Asynchronous:
    synchronise `stream` (default: the current stream of W1's device) before
    reading y."""
    import torch
    _dev(Wg, W1, W3, W2)
    if x.is_cuda or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bfloat16 CPU tensor")
    T, d = x.shape
    E, f, _ = W1.shape
    y = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True) if y is None else y
    if y.is_cuda or not y.is_contiguous() or y.dtype != torch.bfloat16 or tuple(y.shape) != (T, d):
        raise ValueError("y must be a contiguous bfloat16 CPU tensor of shape [T, d]")
    _check(lib.moe_layer_forward_host(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, f, E, k, _ptr(y),
                                      chunks, (MOE_HOST_X_READY if x_ready else 0) | (MOE_HOST_Y_ASYNC if y_async else 0),
                                      _stream(stream, W1)), "moe_layer_forward_host")
    return y


def moe_layer_forward_host_wait(stream=None):
    """Orders `stream` (default: the current stream) after every copy out of
    earlier moe_layer_forward_host calls on the current device."""
    _check(lib.moe_layer_forward_host_wait(_stream(stream)), "moe_layer_forward_host_wait")


def moe_layer_forward_noalloc(x, Wg, W1, W3, W2, k, y, stream=None):
    """The whole bf16 layer using the library's static scratch instead of any
    allocation (for callers that cannot allocate device memory while they
    run).  `y` must be given: this wrapper allocates nothing either."""
    _dev(x, Wg, W1, W3, W2, y)
    T, d = x.shape
    E, f, _ = W1.shape
    _check(lib.moe_layer_forward_noalloc(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, f, E, k, _ptr(y),
                                         _stream(stream, x)), "moe_layer_forward_noalloc")
    return y


def moe_layer_forward_ex(x, Wg, W1, W3, W2, k, residual=None, y=None, workspace=None, stream=None):
    """The whole layer (bf16 or fp32) with a caller workspace and optional residual; returns y."""
    import torch
    _dev(x, Wg, W1, W3, W2, residual)
    T, d = x.shape
    E, f, _ = W1.shape
    dt = _dtype_code(x)
    y = torch.empty_like(x) if y is None else y
    ws, nb = _workspace(T, d, f, E, k, dt, x.device, workspace)
    _check(lib.moe_layer_forward_ex(_ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(residual), T, d, f, E, k,
                                    dt, _ptr(ws), nb, _ptr(y), _stream(stream, x)), "moe_layer_forward_ex")
    return y


def moe_stack_forward(x, layers, k, y=None, scratch=None, workspace=None, stream=None):
    """L layers with the residual between them: `layers` is a list of
    (Wg, W1, W3, W2) device tensors; returns y = x_L."""
    import torch
    L = len(layers)
    _dev(x, *[w for lay in layers for w in lay])
    T, d = x.shape
    E, f, _ = layers[0][1].shape
    dt = _dtype_code(x)
    y = torch.empty_like(x) if y is None else y
    scratch = torch.empty_like(x) if (scratch is None and L > 1) else scratch
    ws, nb = _workspace(T, d, f, E, k, dt, x.device, workspace)
    arr = [(ctypes.c_void_p * L)(*[lay[i].data_ptr() for lay in layers]) for i in range(4)]
    _check(lib.moe_stack_forward(_ptr(x), arr[0], arr[1], arr[2], arr[3], L, T, d, f, E, k, dt, _ptr(scratch),
                                 _ptr(ws), nb, _ptr(y), _stream(stream, x)), "moe_stack_forward")
    return y


def moe_release_workspace(stream=None):
    _check(lib.moe_release_workspace(_stream(stream)), "moe_release_workspace")
