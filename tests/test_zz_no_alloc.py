"""moe_layer_forward_noalloc: the layer for callers that cannot allocate
device memory while they run (a plug-in whose host framework owns the
device memory, a server that allows no allocation on its serving path).
It works out of a fixed scratch array inside the library, so it must give
the same result as the regular entry point, call after call, and refuse
shapes that do not fit the scratch.  This file is collected last on
purpose, so that a run stopping at its first failure has already run every
other test."""

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

import sparse_mixture_experts_06_b200 as moe  # noqa: E402


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [
    synth.MoEShape("small", 200, 512, 1024, 8, 2, "bf16"),
    synth.CONFIGS["decode"],
], ids=["small", "mixtral-decode"])
def test_noalloc_matches_the_regular_entry_point_twice(shape):
    """Two calls in a row (different tokens and weights): each equals the
    regular entry point within the bf16 bound, and the first is also checked
    on its own against the fp64 oracle (every token, expert indices exact)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.gpu_util import assert_close, check_routing, f64, host_copy, oracle_rows
    from synth.device import device_inputs
    for call, seed in enumerate((11, 12)):   # two calls in a row, different tokens and weights
        t = device_inputs(shape, seed)
        y_ref = moe.moe_layer_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], shape.k)
        y = torch.full_like(y_ref, float("nan"))
        moe.moe_layer_forward_noalloc(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], shape.k, y)
        torch.cuda.synchronize()
        a = y.float().double().cpu().numpy()
        b = y_ref.float().double().cpu().numpy()
        assert np.isfinite(a).all(), "call %d left unwritten outputs" % call
        assert np.abs(a - b).max() <= 1e-2 * np.abs(b).max(), "call %d differs" % call
        if call == 0:
            idx, w = moe.moe_router_topk(t["x"], t["Wg"], shape.k)
            h = host_copy(t)
            check_routing(idx.cpu().numpy(), w.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), shape.k)
            y_o, _, _ = oracle_rows(h, shape.k, np.arange(shape.T))
            assert_close(a, y_o, "bf16", "noalloc y")
    assert moe.moe_device_errors() == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    """Checked on the host before anything is looked up or launched."""
    import ctypes
    P = ctypes.c_void_p
    rc = moe.lib.moe_layer_forward_noalloc(P(16), P(16), P(16), P(16), P(16), 4096, 4096, 14336, 8, 2, P(512),
                                           None)
    assert rc == 3  # MOE_ERR_WORKSPACE
    msg = moe.moe_last_error_string()
    assert "static scratch" in msg and str(32 << 20) in msg
