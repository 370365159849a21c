"""Failure detection of the expert GEMM pipelines, without a GPU fault.

Every wait of the GEMM pipelines (ring stages, accumulators, tile numbers)
is bounded; when a bound runs out the kernel raises
MOE_DEVERR_PIPELINE_TIMEOUT, stops the other roles of its CTA and of its CTA
pair, lets what it already issued finish, frees its tensor memory and
returns.  The test makes a wait run out in the allowed way: with
moe_set_wait_test the epilogue waits on a barrier that nothing completes,
under a short bound.  It checks that the call returns, that the flag is
raised, and that the next call at the default bound matches the oracle."""

import time

import numpy as np
import pytest

import synth
from tests.gpu_util import assert_close, device_inputs, host_copy, oracle_rows

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402

PIPELINE_TIMEOUT = 1


@pytest.fixture(autouse=True)
def restore_defaults():
    yield
    moe.moe_set_wait_test(0, False)
    moe.moe_set_gemm_variant()


@pytest.mark.parametrize("variant", [(1, 0, 128, 0), (1, 0, 32, 0), (2, 0, 0, 512), (2, 0, 0, 256)],
                         ids=["single-cta", "single-cta-32-rows", "pair-256x512", "pair-256x256"])
def test_pipeline_wait_bound_aborts_cleanly(variant):
    # one expert (E = k = 1), 1024 rows: 4 pair row blocks, or 8 (32) single-CTA
    # ones of 128 (32) rows, several column tiles each; the 32-row tiles issue
    # their first weight loads before the dependency wait
    s = synth.MoEShape("abort", 1024, 256, 1024, 1, 1, "bf16")
    t = device_inputs(s, 21)
    moe.moe_set_gemm_variant(*variant)
    assert moe.moe_device_errors() == 0
    moe.moe_set_wait_test(200_000, True)  # 200 us bound, epilogue stalled
    y = torch.full_like(t["x"], float("nan"))
    t0 = time.monotonic()
    moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 1, y=y)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert moe.moe_device_errors() & PIPELINE_TIMEOUT
    assert elapsed < 30.0
    # the context is usable and the next call, at the default bound, is exact
    moe.moe_set_wait_test(0, False)
    y = moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 1)
    torch.cuda.synchronize()
    assert moe.moe_device_errors() == 0
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 1, np.arange(s.T))
    assert_close(y.float().double().cpu().numpy(), y_ref, "bf16")

