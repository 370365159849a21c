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
