"""moe_layer_forward_host: the layer on host x / y, pipelined in pieces.

Tokens are independent, so the pipelined call must give exactly the bits
of the device entry point run piece by piece on the same split, and match
the oracle within the bf16 bound."""

import numpy as np
import pytest

import synth
from tests.gpu_util import assert_close, device_inputs, host_copy, oracle_rows

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert moe.moe_device_errors() == 0


def piecewise_device(t, k, chunks):
    T = t["x"].shape[0]
    C = min(chunks, T)
    Tc = -(-T // C)
    outs = []
    for t0 in range(0, T, Tc):
        outs.append(moe.moe_layer_forward(t["x"][t0:t0 + Tc].contiguous(), t["Wg"], t["W1"], t["W3"], t["W2"], k))
    return torch.cat(outs)


@pytest.mark.parametrize("chunks", [1, 2, 3, 7])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_layer_matches_device_pieces_and_oracle(chunks, pinned):
    s = synth.MoEShape("host", 1000, 256, 512, 8, 2, "bf16")
    t = device_inputs(s, 21)
    x_h = t["x"].cpu()
    if pinned:
        x_h = x_h.pin_memory()
    y_h = torch.empty_like(x_h).pin_memory() if pinned else torch.empty_like(x_h)
    moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], 2, y=y_h, chunks=chunks)
    torch.cuda.current_stream().synchronize()
    ref = piecewise_device(t, 2, chunks).cpu()
    assert torch.equal(y_h.view(torch.int16), ref.view(torch.int16))
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(s.T))
    assert_close(y_h.float().double().numpy(), y_ref, "bf16")


def test_host_layer_more_chunks_than_tokens_and_repeat_calls():
    """chunks > T runs one token per piece; back-to-back calls reuse the
    staging buffers and events without a host synchronisation between them."""
    s = synth.MoEShape("host-small", 5, 64, 128, 8, 2, "bf16")
    t = device_inputs(s, 22)
    x_h = t["x"].cpu().pin_memory()
    ys = [moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], 2, chunks=c) for c in (8, 2, 8)]
    torch.cuda.current_stream().synchronize()
    ref = moe.moe_layer_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 2).cpu()
    one = piecewise_device(t, 2, 5).cpu()
    assert torch.equal(ys[0].view(torch.int16), one.view(torch.int16))
    assert torch.equal(ys[2].view(torch.int16), one.view(torch.int16))
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(s.T))
    for y in ys + [ref]:
        assert_close(y.float().double().numpy(), y_ref, "bf16")


def test_host_layer_prefill_shape_two_chunks():
    s = synth.CONFIGS["prefill"]
    t = device_inputs(s, 0)
    x_h = t["x"].cpu().pin_memory()
    y_h = moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], s.k, chunks=2)
    torch.cuda.current_stream().synchronize()
    ref = piecewise_device(t, s.k, 2).cpu()
    assert torch.equal(y_h.view(torch.int16), ref.view(torch.int16))
    moe.moe_release_workspace()
