"""Two layers in flight at once on two streams, each with its own
workspace: the results equal the same calls made one after the other (the
GEMM tile counters, the permutation's chunk bases and every buffer a call
writes live in its own workspace; the kernels carry no other state)."""

import pytest

import synth
from tests.gpu_util import device_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402


@pytest.mark.parametrize("shapes", [
    (synth.MoEShape("st-a", 2304, 256, 512, 8, 2, "bf16"), synth.MoEShape("st-b", 700, 128, 384, 8, 2, "bf16")),
    (synth.MoEShape("st-c", 4100, 128, 256, 8, 2, "bf16"), synth.MoEShape("st-d", 4100, 128, 256, 8, 2, "bf16")),
], ids=["pairs+single", "pairs+pairs"])
def test_concurrent_layers_on_two_streams_match_sequential(shapes):
    ins = [device_inputs(s, 51 + i) for i, s in enumerate(shapes)]
    wss = [torch.empty(moe.moe_workspace_size(s.T, s.d, s.f, s.E, s.k, 0), dtype=torch.uint8, device="cuda")
           for s in shapes]
    ref = [moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, workspace=ws)
           for s, t, ws in zip(shapes, ins, wss)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(t["x"]) for t in ins]
    for rep in range(5):  # enqueue interleaved, so the two streams' kernels overlap
        for s, t, ws, y, st in zip(shapes, ins, wss, outs, streams):
            moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y, workspace=ws, stream=st)
    torch.cuda.synchronize()
    for r, y in zip(ref, outs):
        assert torch.equal(r.view(torch.int16), y.view(torch.int16))
    assert moe.moe_device_errors() == 0


def test_library_workspace_grows_safely_across_streams():
    """moe_layer_forward shares one library workspace per device.  A larger
    shape that arrives on another stream while a call is still queued grows
    it: the old workspace must be freed only after the queued call's work
    (the library orders the free after an event recorded at the end of its
    last user's work).  The first call's result must equal the same layer
    run alone; the second call must be correct too."""
    small = synth.MoEShape("grow-a", 2304, 256, 512, 8, 2, "bf16")
    big = synth.MoEShape("grow-b", 6000, 256, 512, 8, 2, "bf16")
    ta, tb = device_inputs(small, 61), device_inputs(big, 62)
    ref_a = moe.moe_layer_forward_ex(ta["x"], ta["Wg"], ta["W1"], ta["W3"], ta["W2"], 2)
    ref_b = moe.moe_layer_forward_ex(tb["x"], tb["Wg"], tb["W1"], tb["W3"], tb["W2"], 2)
    torch.cuda.synchronize()
    for _ in range(3):
        moe.moe_release_workspace()  # start from a pool sized for nothing
        torch.cuda.synchronize()
        sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
        ya, yb = torch.empty_like(ta["x"]), torch.empty_like(tb["x"])
        # a long kernel first on stream a, so its layer is still queued when b grows the pool
        busy = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
        with torch.cuda.stream(sa):
            busy.fill_(1)
        moe.moe_layer_forward(ta["x"], ta["Wg"], ta["W1"], ta["W3"], ta["W2"], 2, y=ya, stream=sa)
        moe.moe_layer_forward(tb["x"], tb["Wg"], tb["W1"], tb["W3"], tb["W2"], 2, y=yb, stream=sb)
        torch.cuda.synchronize()
        assert torch.equal(ref_a.view(torch.int16), ya.view(torch.int16))
        assert torch.equal(ref_b.view(torch.int16), yb.view(torch.int16))
    moe.moe_release_workspace()
    assert moe.moe_device_errors() == 0
