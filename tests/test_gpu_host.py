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


@pytest.mark.parametrize("x_ready,y_async", [(False, False), (True, False), (True, True)])
def test_host_layer_back_to_back_calls_alternate_buffers(x_ready, y_async):
    """Many calls in a row without a host synchronisation, piece sizes
    changing between calls (the staging layout changes) and host inputs
    that differ per call: every call's y matches the device path on its own
    x.  With x_ready the copies of a call may start while the previous call
    still computes; with y_async its copies out may overlap the next call,
    and moe_layer_forward_host_wait orders the stream after them."""
    s = synth.MoEShape("host-b2b", 600, 128, 256, 8, 2, "bf16")
    t = device_inputs(s, 23)
    xs = [(t["x"] * (1.0 + 0.25 * i)).to(torch.bfloat16) for i in range(6)]
    xs_h = [x.cpu().pin_memory() for x in xs]
    plan = [1, 1, 2, 2, 3, 1]
    ys = [moe.moe_layer_forward_host(xh, t["Wg"], t["W1"], t["W3"], t["W2"], 2, chunks=c, x_ready=x_ready,
                                     y_async=y_async)
          for xh, c in zip(xs_h, plan)]
    if y_async:
        moe.moe_layer_forward_host_wait()
    torch.cuda.current_stream().synchronize()
    for x, c, y in zip(xs, plan, ys):
        tt = dict(t, x=x)
        ref = piecewise_device(tt, 2, c).cpu()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_host_layer_chained_through_host_memory():
    """Without x_ready, a call whose x_host is the y_host of the call before
    (written by that call's copy out, still queued on the stream) reads the
    finished values: two layers chained through pinned host memory equal two
    device layers."""
    s = synth.MoEShape("host-chain", 300, 128, 256, 8, 2, "bf16")
    t = device_inputs(s, 24)
    x_h = t["x"].cpu().pin_memory()
    mid = torch.empty_like(x_h).pin_memory()
    out = torch.empty_like(x_h).pin_memory()
    moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], 2, y=mid, chunks=2)
    moe.moe_layer_forward_host(mid, t["Wg"], t["W1"], t["W3"], t["W2"], 2, y=out, chunks=3)
    torch.cuda.current_stream().synchronize()
    ref1 = piecewise_device(t, 2, 2)
    assert torch.equal(mid.view(torch.int16), ref1.cpu().view(torch.int16))
    y2 = piecewise_device(dict(t, x=ref1), 2, 3)
    assert torch.equal(out.view(torch.int16), y2.cpu().view(torch.int16))


@pytest.mark.parametrize("chunks", [1, 2])
def test_host_layer_prefill_shape(chunks):
    """The serving entry at the bench's end-to-end size (T = 4096, Mixtral
    dimensions, pinned host buffers; the bench uses one piece): the bits of
    the device entry point on the same split, which the full-shape tests
    check against the oracle."""
    s = synth.CONFIGS["prefill"]
    t = device_inputs(s, 0)
    x_h = t["x"].cpu().pin_memory()
    y_h = moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], s.k, chunks=chunks)
    torch.cuda.current_stream().synchronize()
    ref = piecewise_device(t, s.k, chunks).cpu()
    assert torch.equal(y_h.view(torch.int16), ref.view(torch.int16))
    moe.moe_release_workspace()

