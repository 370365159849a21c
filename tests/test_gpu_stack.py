"""The layer stack (residual between layers) through moe_stack_forward.

Checked per layer with teacher forcing: the oracle takes the GPU's own bf16
x_l for the sampled tokens, so 32 layers of bf16 rounding do not create
near-ties that an fp64 chain would resolve differently."""

import numpy as np
import pytest

import synth
from tests.gpu_util import assert_close, assert_residual_close, device_inputs, f64, host_copy, oracle_rows

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert moe.moe_device_errors() == 0


def layer_weights(shape, L, seed=0):
    return [device_inputs(shape, seed, layer=l, with_x=False) for l in range(L)]


def chain(x, layers, k):
    """Layer by layer with moe_layer_forward_ex (residual = input); returns all x_l."""
    xs = [x]
    for w in layers:
        xs.append(moe.moe_layer_forward_ex(xs[-1], w["Wg"], w["W1"], w["W3"], w["W2"], k, residual=xs[-1]))
    return xs


def as_tuple(w):
    return (w["Wg"], w["W1"], w["W3"], w["W2"])


@pytest.mark.parametrize("L", [1, 2, 3])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_small_stack_matches_chain_and_oracle(L, dt):
    s = synth.MoEShape("stk", 300, 128, 256, 8, 2, dt, w2_scale=0.25)
    ws = layer_weights(s, L, seed=9)
    x = device_inputs(s, 9)["x"]
    y = moe.moe_stack_forward(x, [as_tuple(w) for w in ws], 2)
    xs = chain(x, ws, 2)
    assert torch.equal(y.view(torch.int16) if dt == "bf16" else y, xs[-1].view(torch.int16) if dt == "bf16" else xs[-1])
    for l, w in enumerate(ws):
        h = host_copy(dict(w, x=xs[l]))
        moe_ref, _, _ = oracle_rows(h, 2, np.arange(s.T))
        got = xs[l + 1].float().double().cpu().numpy()
        if dt == "f32":
            assert_close(got - f64(h["x"]), moe_ref, "f32")
        else:
            assert_residual_close(got, f64(h["x"]), moe_ref)


def test_mixtral_stack_32_layers_T8192():
    """Config: 32 Mixtral-shaped layers (90 GB of weights), T = 8192, residual
    between layers; teacher-forced checks of layers 0, 1, 15 and 31 on 64
    sampled tokens, and moe_stack_forward equal bit for bit to the chain."""
    import dataclasses
    s = synth.CONFIGS["stack"]
    one = dataclasses.replace(s, name="stack-layer", layers=1)
    ws = layer_weights(one, s.layers)
    x = device_inputs(synth.MoEShape("x", s.T, s.d, 8, s.E, s.k, s.dtype), 0)["x"]
    y = moe.moe_stack_forward(x, [as_tuple(w) for w in ws], s.k)
    xs = chain(x, ws, s.k)
    assert torch.equal(y.view(torch.int16), xs[-1].view(torch.int16))
    toks = np.sort(np.random.default_rng(0).choice(s.T, 64, replace=False))
    for l in (0, 1, 15, 31):
        w = ws[l]
        h = host_copy({"x": xs[l][torch.from_numpy(toks).cuda()], "Wg": w["Wg"], "W1": w["W1"], "W3": w["W3"],
                       "W2": w["W2"]})
        moe_ref, _, _ = oracle_rows(h, s.k, np.arange(len(toks)))
        got = xs[l + 1][torch.from_numpy(toks).cuda()].float().double().cpu().numpy()
        assert_residual_close(got, f64(h["x"]), moe_ref, "layer %d" % l)
