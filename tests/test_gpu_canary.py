"""Out-of-bounds writes, without a sanitizer: every output the library
writes (y, the caller's workspace, the router's indices and weights, the
permutation arrays, the host output of the serving entry) is a view into a
larger buffer whose padding holds a canary pattern; after the call the
padding must be unchanged.  Shapes cover ragged tiles, both permutation
paths, pair and single-CTA GEMM tiles, E = 64, fp32 and bf16."""

import pytest

import synth
from tests.gpu_util import device_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402

CANARY = 0x5A
PAD = 4096  # bytes of padding on each side


def padded(nbytes, device="cuda"):
    """A canary-filled byte buffer and the 256-byte aligned window of nbytes inside it."""
    buf = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device=device)
    return buf, buf[PAD:PAD + nbytes]


def untouched(buf, nbytes):
    return bool((buf[:PAD] == CANARY).all()) and bool((buf[PAD + nbytes:] == CANARY).all())


SHAPES = [
    synth.MoEShape("cn-ragged", 37, 72, 136, 8, 2, "bf16"),
    synth.MoEShape("cn-tiles", 1000, 128, 384, 4, 2, "bf16"),
    synth.MoEShape("cn-chunked-pairs", 2304, 256, 320, 8, 2, "bf16"),   # chunked permutation, pair tiles, ragged f
    synth.MoEShape("cn-E64k8", 256, 128, 128, 64, 8, "bf16"),
    synth.MoEShape("cn-f32", 37, 72, 136, 8, 2, "f32"),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_layer_writes_stay_inside_their_buffers(shape):
    t = device_inputs(shape, 41)
    dt = 0 if shape.dtype == "bf16" else 1
    esz = 2 if shape.dtype == "bf16" else 4
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    ny = shape.T * shape.d * esz
    ybuf, ywin = padded(ny)
    y = ywin.view(tdt).view(shape.T, shape.d)
    nws = moe.moe_workspace_size(shape.T, shape.d, shape.f, shape.E, shape.k, dt)
    wsbuf, ws = padded(nws)
    moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], shape.k, y=y, workspace=ws)
    torch.cuda.synchronize()
    assert untouched(ybuf, ny), "the layer wrote outside y"
    assert untouched(wsbuf, nws), "the layer wrote outside its workspace"
    # the router and the permutation on their own
    n = shape.T * shape.k
    ib, iw = padded(4 * n)
    wb, ww = padded(4 * n)
    idx = iw.view(torch.int32).view(shape.T, shape.k)
    w = ww.view(torch.float32).view(shape.T, shape.k)
    moe.moe_router_topk(t["x"], t["Wg"], shape.k, topk_idx=idx, topk_w=w)
    ob, ow = padded(4 * (shape.E + 1))
    pb, pw = padded(4 * n)
    vb, vw = padded(4 * n)
    moe.moe_permute(idx, shape.E, offsets=ow.view(torch.int32), perm=pw.view(torch.int32), inv=vw.view(torch.int32))
    torch.cuda.synchronize()
    for b, nb_, what in ((ib, 4 * n, "topk_idx"), (wb, 4 * n, "topk_w"), (ob, 4 * (shape.E + 1), "offsets"),
                         (pb, 4 * n, "perm"), (vb, 4 * n, "inv")):
        assert untouched(b, nb_), "wrote outside " + what
    assert moe.moe_device_errors() == 0


def test_host_entry_writes_stay_inside_y_host():
    s = synth.MoEShape("cn-host", 600, 128, 256, 8, 2, "bf16")
    t = device_inputs(s, 42)
    x_h = t["x"].cpu().pin_memory()
    ny = s.T * s.d * 2
    ybuf = torch.full((ny + 2 * PAD,), CANARY, dtype=torch.uint8).pin_memory()
    y_h = ybuf[PAD:PAD + ny].view(torch.bfloat16).view(s.T, s.d)
    for chunks in (1, 3):
        moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], 2, y=y_h, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert untouched(ybuf, ny), "the host entry wrote outside y_host"
    moe.moe_release_workspace()
