"""Device-resident inputs from the same generator (libsynth.so), as torch tensors.

Only input generation: x, Wg, W1, W3, W2 of one layer on a CUDA device, bit
identical to synth.host_inputs (checked by the GPU tests)."""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import gen

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth.so")
        if not os.path.exists(path):
            raise ImportError("synth/libsynth.so is not built (run python synth/build.py)")
        lib = ctypes.CDLL(path)
        lib.synth_normal_fill.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
        lib.synth_normal_fill.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def normal_tensor(shape, seed, tid, sigma, dtype, device="cuda", start=0):
    """A torch tensor of `shape` holding elements [start, start+numel) of the stream."""
    import torch
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty(shape, dtype=tdt, device=device)
    n = out.numel()
    rc = _lib().synth_normal_fill(ctypes.c_void_p(out.data_ptr()), n, start, seed, tid, float(np.float32(sigma)),
                                  1 if dtype == "bf16" else 0,
                                  ctypes.c_void_p(torch.cuda.current_stream(out.device).cuda_stream))
    if rc != 0:
        raise RuntimeError("synth_normal_fill failed with cudaError %d" % rc)
    return out


def device_inputs(shape: gen.MoEShape, seed: int = 0, layer: int = 0, device="cuda",
                  with_x: bool = True, skew_beta: float | None = None) -> dict:
    """Inputs of one layer on `device` (layouts as synth.host_inputs)."""
    import torch
    T, d, f, E, dt = shape.T, shape.d, shape.f, shape.E, shape.dtype
    out = {}
    if with_x:
        out["x"] = normal_tensor((T, d), seed, gen.tensor_id(gen.TENSOR_X, layer), gen.sigma_of(gen.TENSOR_X, d, f), dt, device)
    out["Wg"] = normal_tensor((E, d), seed, gen.tensor_id(gen.TENSOR_WG, layer), gen.sigma_of(gen.TENSOR_WG, d, f), dt, device)
    out["W1"] = normal_tensor((E, f, d), seed, gen.tensor_id(gen.TENSOR_W1, layer), gen.sigma_of(gen.TENSOR_W1, d, f), dt, device)
    out["W3"] = normal_tensor((E, f, d), seed, gen.tensor_id(gen.TENSOR_W3, layer), gen.sigma_of(gen.TENSOR_W3, d, f), dt, device)
    out["W2"] = normal_tensor((E, d, f), seed, gen.tensor_id(gen.TENSOR_W2, layer),
                              gen.sigma_of(gen.TENSOR_W2, d, f, shape.w2_scale), dt, device)
    if shape.skew:
        beta = gen.SKEW_BETA if skew_beta is None else skew_beta
        b = gen.skew_biases(E, beta, dt)
        if dt == "bf16":
            bias = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(device)
        else:
            bias = torch.from_numpy(b).to(device)
        if with_x:
            out["x"][:, -1] = 1.0
        out["Wg"][:, -1] = bias
    return out


def to_host_bits(t):
    """A device tensor as numpy (bf16 as uint16 bit patterns, fp32 as float32)."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
