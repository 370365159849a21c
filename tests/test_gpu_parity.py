"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Indices and the permutation must match bit for bit; gate weights to 1e-6;
outputs within max|y - y_ref| <= 1e-2 max|y_ref| (bf16) or 1e-5 (fp32).
Small shapes are checked on every token and span several 128-row tiles
with ragged tails; the full Mixtral shapes (decode T = 32, prefill
T = 4096, skewed T = 16384) are checked on every token's routing and on a
stratified sample of tokens for the outputs, in the launch configuration
the benchmark times."""

import numpy as np
import pytest

import synth
from tests.gpu_util import (assert_close, check_permutation, check_routing, device_inputs, f64,
                            host_copy, oracle_rows, stratified_tokens)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import sparse_mixture_experts_06_b200 as moe  # noqa: E402


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    moe.moe_set_gemm_variant()  # back to the automatic choice
    assert moe.moe_device_errors() == 0


def force_variant(cta_group, bn="0", rb="0", wide=None):
    """Tile variant by the test's labels: cta_group 1 / 2 / h (hybrid), up
    tile width, token rows, and pair tiles 512 (wide = "1") or 256 columns."""
    cg = {"1": 1, "2": 2, "h": 3}[cta_group]
    cols = 0 if wide is None else (512 if wide == "1" else 256)
    moe.moe_set_gemm_variant(cg, int(bn), int(rb), cols)


def run_layer(t, k, residual=None):
    return moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], k, residual=residual)


def to64(y):
    return y.float().double().cpu().numpy()


def full_check(shape: synth.MoEShape, seed: int = 0):
    """Every token: routing, permutation and outputs against the oracle."""
    t = device_inputs(shape, seed)
    y = run_layer(t, shape.k)
    idx_g, w_g = moe.moe_router_topk(t["x"], t["Wg"], shape.k)
    off_g, perm_g, inv_g = moe.moe_permute(idx_g, shape.E)
    torch.cuda.synchronize()
    h = host_copy(t)
    idx_o, _, _ = check_routing(idx_g.cpu().numpy(), w_g.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), shape.k)
    check_permutation(off_g.cpu().numpy(), perm_g.cpu().numpy(), inv_g.cpu().numpy(), idx_o, shape.E)
    y_ref, _, _ = oracle_rows(h, shape.k, np.arange(shape.T))
    return assert_close(to64(y), y_ref, shape.dtype), idx_o


# ---------------------------------------------------------------- generator

@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_device_generator_matches_host(dt):
    from synth.device import normal_tensor, to_host_bits
    start, n = 987654321, 1 << 20
    dev = to_host_bits(normal_tensor((n,), 5, 11, 0.0125, dt, start=start))
    host = synth.normal_values(5, 11, n, 0.0125, dt, start=start)
    np.testing.assert_array_equal(dev, host)


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("T,d,E,k,dt", [
    (16, 64, 8, 2, "f32"), (37, 72, 8, 2, "bf16"), (1, 8, 1, 1, "bf16"), (300, 256, 64, 8, "bf16"),
    (129, 4096, 8, 2, "bf16"), (250, 96, 5, 3, "f32"), (100, 128, 8, 8, "bf16"), (70, 64, 64, 64, "f32"),
    (64, 256, 16, 12, "bf16"),
    # many tokens: several token groups per cluster (2, 4, and 3 for E = 64), ragged last group
    (4100, 256, 8, 2, "bf16"), (8229, 512, 8, 2, "bf16"), (8200, 128, 64, 8, "bf16"), (9000, 64, 8, 2, "f32"),
])
def test_router_parity(T, d, E, k, dt):
    t = device_inputs(synth.MoEShape("r", T, d, 8, E, k, dt), seed=T + E)
    idx, w = moe.moe_router_topk(t["x"], t["Wg"], k)
    h = host_copy({"x": t["x"], "Wg": t["Wg"]})
    _, _, near = check_routing(idx.cpu().numpy(), w.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), k)
    assert near == 0


def test_router_ties_go_to_lower_index():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    Wg = torch.randn((8, 64), device="cuda").to(torch.bfloat16)
    idx, w = moe.moe_router_topk(x, Wg, 2)
    assert idx.cpu().tolist() == [[0, 1]] * 4
    assert (w.cpu() == 0.5).all()
    x = torch.ones((2, 64), dtype=torch.bfloat16, device="cuda")
    Wg = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    Wg[6] = 0.25
    Wg[2] = 0.25
    idx, w = moe.moe_router_topk(x, Wg, 2)
    assert idx.cpu().tolist() == [[2, 6]] * 2
    assert (w.cpu() == 0.5).all()


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (511, 8, 2), (512, 8, 2), (1500, 8, 2), (3000, 64, 8),
                                   (777, 3, 1), (20000, 8, 2), (16384, 8, 2), (5000, 16, 4), (2000, 17, 3),
                                   (0, 8, 2),
                                   # the one-pass kernel (E <= 16, 4096..16384 assignments)
                                   (4096, 8, 2), (2049, 8, 2), (8192, 8, 2), (2048, 16, 4), (4100, 5, 3)])
def test_permute_parity(T, E, k):
    rng = np.random.default_rng(T)
    # a skewed draw that leaves some experts empty
    p = rng.dirichlet(np.ones(E) * 0.3)
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32) if T else \
        np.zeros((0, k), dtype=np.int32)
    off, perm, inv = moe.moe_permute(torch.from_numpy(idx).cuda(), E)
    check_permutation(off.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), idx, E)


@pytest.mark.parametrize("E,T", [(8, 3), (20, 3), (8, 3000)])  # the general and the one-pass kernel
def test_permute_flags_bad_expert_ids(E, T):
    rows = [[0, 1], [E + 1, 2], [-3, 4]] + [[5, 6]] * (T - 3)
    idx = torch.tensor(rows, dtype=torch.int32, device="cuda")
    off, perm, inv = moe.moe_permute(idx, E)
    assert moe.moe_device_errors() == 2
    assert off.cpu().tolist()[-1] == 2 * T - 2 and inv.cpu().tolist()[2] == -1 and inv.cpu().tolist()[4] == -1
    assert sorted(perm.cpu().tolist()[:4]) == [0, 1, 3, 5]


# ---------------------------------------------------------------- routing statistics

@pytest.mark.parametrize("T,E,k,seq_len", [(1, 8, 2, 0), (5000, 8, 2, 0), (4096, 8, 2, 512), (3000, 64, 8, 0),
                                           (777, 16, 3, 100)])
def test_routing_stats_parity(T, E, k, seq_len):
    import oracle
    rng = np.random.default_rng(T + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx[1::7] = idx[0::7][: len(idx[1::7])]          # plant some repeats
    out = moe.moe_routing_stats(torch.from_numpy(idx).cuda(), E, seq_len)
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.int64), oracle.routing_stats(idx, E, seq_len))


def test_routing_stats_of_the_synthetic_router():
    """The seeded near-uniform router shows the uniform baselines quoted with
    tab. 5 (first choice ~1/8, first or second ~13/28)."""
    import math
    s = synth.CONFIGS["prefill"]
    t = device_inputs(synth.MoEShape("st", s.T, s.d, 8, s.E, s.k, "bf16"), 0)
    idx, _ = moe.moe_router_topk(t["x"], t["Wg"], 2)
    st = moe.moe_routing_stats(idx, 8).cpu().numpy().astype(np.int64)
    n = st[10]
    assert n == s.T - 1 and st[:8].sum() == 2 * s.T
    assert abs(st[8] / n - 1 / 8) < 4 * math.sqrt(1 / 8 * 7 / 8 / n)
    assert abs(st[9] / n - 13 / 28) < 4 * math.sqrt(13 / 28 * 15 / 28 / n)


# ---------------------------------------------------------------- the layer's own permutation

def workspace_routing_views(ws, T, E, k):
    """offsets, perm, inv as the layer leaves them in its workspace (the
    carve order of the C library: topk_idx, topk_w, offsets, perm, inv, each
    at a 256-byte boundary)."""
    n = T * k
    a = lambda b: (b + 255) // 256 * 256  # noqa: E731
    o_off = 2 * a(4 * n)
    p_off = o_off + a(4 * (E + 1))
    i_off = p_off + a(4 * n)
    as_i32 = lambda off, cnt: ws[off: off + 4 * cnt].view(torch.int32)  # noqa: E731
    return as_i32(o_off, E + 1), as_i32(p_off, n), as_i32(i_off, n)


@pytest.mark.parametrize("shape", [
    synth.MoEShape("perm-decode", 32, 256, 256, 8, 2, "bf16"),      # the router permutes (one cluster)
    synth.MoEShape("perm-router-256", 64, 128, 128, 16, 4, "bf16"),  # the router's largest: 256 assignments
    synth.MoEShape("perm-router-T1", 1, 64, 128, 8, 2, "bf16"),
    synth.MoEShape("perm-one-block", 65, 128, 128, 8, 2, "bf16"),    # one-block permutation kernel
    synth.MoEShape("perm-ragged", 1100, 128, 128, 8, 2, "bf16"),     # 2200 assignments: ragged last chunk
    synth.MoEShape("perm-4100", 4100, 128, 128, 8, 2, "bf16"),
    synth.MoEShape("perm-E64k8", 300, 128, 128, 64, 8, "bf16"),
    synth.MoEShape("perm-f32", 1200, 64, 128, 8, 2, "f32"),
    synth.MoEShape("perm-fallback", 50000, 64, 64, 64, 1, "bf16"),  # E x chunks above the scan's shared memory
], ids=lambda s: s.name)
def test_layer_permutation_matches_the_stable_sort(shape):
    """The permutation the layer builds for itself (in the router's cluster
    up to 64 tokens and 256 assignments; from 2048 assignments from the
    router's per-chunk counts in the scatter; else, or when E x chunks is
    too large, the one-block kernel) equals
    the oracle's stable counting sort of the router's choices, bit for bit,
    and the layer's output on sampled tokens matches the oracle."""
    t = device_inputs(shape, 31)
    ws = torch.empty(moe.moe_workspace_size(shape.T, shape.d, shape.f, shape.E, shape.k,
                                            0 if shape.dtype == "bf16" else 1), dtype=torch.uint8, device="cuda")
    y = moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], shape.k, workspace=ws)
    idx, _ = moe.moe_router_topk(t["x"], t["Wg"], shape.k)
    off, perm, inv = workspace_routing_views(ws, shape.T, shape.E, shape.k)
    torch.cuda.synchronize()
    check_permutation(off.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), idx.cpu().numpy(), shape.E)
    h = host_copy(t)
    toks = np.random.default_rng(1).choice(shape.T, size=min(shape.T, 64), replace=False)
    y_ref, _, _ = oracle_rows(h, shape.k, np.sort(toks), routing=None)
    assert_close(to64(y)[np.sort(toks)], y_ref, shape.dtype)


# ---------------------------------------------------------------- whole layer, every token

F32_SHAPES = [
    synth.CONFIGS["tiny"],
    synth.MoEShape("f32-ragged", 37, 72, 136, 8, 2, "f32"),
    synth.MoEShape("f32-mid", 200, 256, 512, 8, 2, "f32"),
]
BF16_SHAPES = [
    synth.MoEShape("bf16-tiles", 1000, 128, 384, 4, 2, "bf16"),     # 500 rows/expert: several tiles + tail
    synth.MoEShape("bf16-ragged", 37, 72, 136, 8, 2, "bf16"),       # every tile ragged, K tails
    synth.MoEShape("bf16-wide", 700, 512, 1024, 8, 2, "bf16"),
    synth.MoEShape("bf16-k1", 300, 256, 256, 8, 1, "bf16"),
    synth.MoEShape("bf16-E64k8", 256, 128, 128, 64, 8, "bf16"),
    synth.MoEShape("bf16-T1", 1, 64, 128, 8, 2, "bf16"),
    synth.MoEShape("bf16-many-tiles", 2500, 256, 768, 8, 2, "bf16"),  # 625 rows/expert, 2-3 pair tiles
    synth.MoEShape("bf16-k-eq-E", 150, 128, 256, 8, 8, "bf16"),       # K = E: dense softmax mixture
    synth.MoEShape("bf16-E16k12", 120, 128, 256, 16, 12, "bf16"),
    synth.MoEShape("bf16-wide-d", 200, 8192, 512, 8, 2, "bf16"),      # up K = 8192, down 16+ column tiles
    synth.MoEShape("bf16-deep-f", 200, 128, 28672, 8, 2, "bf16"),     # down K = 28672 (448 k blocks)
]


@pytest.mark.parametrize("shape", F32_SHAPES, ids=lambda s: s.name)
def test_layer_parity_every_token_f32(shape):
    rel, _ = full_check(shape)
    assert rel <= 1e-5


GEMM_VARIANTS = [("1", "256", "128", "0"), ("1", "128", "128", "0"), ("1", "256", "32", "0"),
                 ("1", "128", "32", "0"), ("2", "256", "128", "0"), ("2", "256", "128", "1"),
                 ("h", "256", "128", "0")]


@pytest.mark.parametrize("variant", GEMM_VARIANTS, ids=lambda v: "cg%s-bn%s-rb%s-wide%s" % v)
@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: s.name)
def test_layer_parity_every_token_bf16(shape, variant):
    """Every GEMM variant: single-CTA tiles of 128 or 32 token rows, CTA-pair
    tiles (256 rows, or 128 for an expert's short last block) 256 or 512
    columns wide, the hybrid (pairs on whole 256-row blocks, single CTAs on
    the rest), and 256- or 128-column up-projection tiles (pairs always use
    256-column MMAs)."""
    force_variant(*variant)
    rel, _ = full_check(shape)
    assert rel <= 1e-2


# Expert block sizes around every tile edge: pair tiles are 256 rows, or 128
# (an M = 128 pair MMA, 64 rows per CTA) when an expert's last block holds at
# most 128 rows; in the up projection's 256 x 512 pair tiles such a tail after
# a whole block is merged with it (257, 320, 321, 384, 640: tails of 1, 64,
# 65 and 128 rows); single-CTA tiles are 128 rows.
BLOCK_SIZES = [1, 64, 65, 128, 129, 200, 257, 320, 321, 384, 385, 640]


@pytest.mark.parametrize("cta_group,wide", [("1", "0"), ("2", "0"), ("2", "1"), ("h", "0")])
def test_expert_blocks_at_tile_edges(cta_group, wide):
    """moe_expert_ffn on a routing built to give the experts the block sizes
    above (k = 1, tokens shuffled, arbitrary gate weights), ragged in both
    output widths (f = 320, d = 384), against the oracle on every token."""
    force_variant(cta_group, wide=wide)
    E, d, f = len(BLOCK_SIZES), 384, 320
    T = sum(BLOCK_SIZES)
    s = synth.MoEShape("blocks", T, d, f, E, 1, "bf16")
    t = device_inputs(s, 11)
    rng = np.random.default_rng(5)
    idx = rng.permutation(np.repeat(np.arange(E), BLOCK_SIZES)).astype(np.int32).reshape(T, 1)
    w = rng.uniform(0.25, 1.0, size=(T, 1)).astype(np.float32)
    idx_d = torch.from_numpy(idx).cuda()
    w_d = torch.from_numpy(w).cuda()
    off, perm, inv = moe.moe_permute(idx_d, E)
    assert np.diff(off.cpu().numpy()).tolist() == BLOCK_SIZES
    y = moe.moe_expert_ffn(t["x"], t["W1"], t["W3"], t["W2"], off, perm, inv, w_d)
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 1, np.arange(T), routing=(idx, w.astype(np.float64)))
    assert_close(to64(y), y_ref, "bf16")


@pytest.mark.parametrize("variant", [("2", "256", "128", "1"), ("1", "256", "128", "0"), ("1", "256", "32", "0")],
                         ids=["pairs-512", "single-128", "single-32"])
def test_large_expert_in_grouped_tile_order(variant):
    """An expert whose rows span many more row blocks than one group of the
    GEMMs' tile order (groups of about sqrt(2 x CTA pairs) 256-row blocks for
    pairs, more for single-CTA tiles; 6000 rows = 23 pair blocks + a short
    one, 47 + 1 single-CTA blocks of 128, 188 of 32), next to small and
    ragged experts: moe_expert_ffn against the oracle on every token."""
    force_variant(*variant)
    sizes = [6000, 100, 333, 900]
    E, d, f = len(sizes), 256, 512
    T = sum(sizes)
    s = synth.MoEShape("grouped", T, d, f, E, 1, "bf16")
    t = device_inputs(s, 12)
    rng = np.random.default_rng(6)
    idx = rng.permutation(np.repeat(np.arange(E), sizes)).astype(np.int32).reshape(T, 1)
    w = rng.uniform(0.25, 1.0, size=(T, 1)).astype(np.float32)
    off, perm, inv = moe.moe_permute(torch.from_numpy(idx).cuda(), E)
    y = moe.moe_expert_ffn(t["x"], t["W1"], t["W3"], t["W2"], off, perm, inv, torch.from_numpy(w).cuda())
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 1, np.arange(T), routing=(idx, w.astype(np.float64)))
    assert_close(to64(y), y_ref, "bf16")


@pytest.mark.parametrize("seed", range(1, 101))
def test_tiny_fp32_many_seeds(seed):
    full_check(synth.CONFIGS["tiny"], seed)


def test_dense_special_case_E1_k1():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN."""
    full_check(synth.MoEShape("dense", 64, 128, 256, 1, 1, "bf16"))
    full_check(synth.MoEShape("dense32", 64, 128, 256, 1, 1, "f32"))


def test_identical_experts_give_single_expert_output():
    s = synth.MoEShape("ident", 300, 128, 256, 8, 2, "bf16")
    t = device_inputs(s, 3)
    for name in ("W1", "W3", "W2"):
        t[name][:] = t[name][0:1].clone()
    y = run_layer(t, 2)
    h = host_copy(t)
    import oracle
    ref = oracle.swiglu_expert(f64(h["x"]), f64(h["W1"][0]), f64(h["W3"][0]), f64(h["W2"][0]))
    assert_close(to64(y), ref, "bf16")


def test_empty_experts():
    """A router that only ever picks experts 5 and 2 leaves six experts empty."""
    s = synth.MoEShape("empty", 400, 128, 256, 8, 2, "bf16")
    t = device_inputs(s, 4)
    t["x"][:, -1] = 4.0
    t["Wg"][:, -1] = 0.0
    t["Wg"][5, -1] = 8.0
    t["Wg"][2, -1] = 6.0
    y = run_layer(t, 2)
    idx, _ = moe.moe_router_topk(t["x"], t["Wg"], 2)
    assert set(np.unique(idx.cpu().numpy()).tolist()) == {2, 5}
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(s.T))
    assert_close(to64(y), y_ref, "bf16")


def test_worked_example_through_the_gpu():
    """The hand-worked closed-form instance (tests/golden/worked_example.json),
    zero-padded to d = f = 8 (padding adds exact zeros)."""
    import json
    import math
    import os
    ex = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))  # noqa: E731
    y_ref = [eval(s, {"sigma": sig}) for s in ex["y_closed_form"]]
    for dt, torch_dt, tol in (("f32", torch.float32, 1e-6), ("bf16", torch.bfloat16, 1e-2)):
        x = torch.zeros((1, 8)); x[0, :2] = torch.tensor(ex["x"])
        Wg = torch.zeros((3, 8)); Wg[:, :2] = torch.tensor(ex["Wg"])
        W1 = torch.zeros((3, 8, 8)); W1[:, :1, :2] = torch.tensor(ex["W1"])
        W3 = torch.zeros((3, 8, 8)); W3[:, :1, :2] = torch.tensor(ex["W3"])
        W2 = torch.zeros((3, 8, 8)); W2[:, :2, :1] = torch.tensor(ex["W2"])
        args = [a.to(torch_dt).cuda() for a in (x, Wg, W1, W3, W2)]
        y = moe.moe_layer_forward_ex(*args, 2)
        idx, _ = moe.moe_router_topk(args[0], args[1], 2)
        assert idx.cpu().tolist() == [ex["idx"]]
        got = y.float().cpu().numpy()[0]
        np.testing.assert_allclose(got[:2], y_ref, rtol=tol, atol=0)
        assert (got[2:] == 0).all()


def test_residual_add():
    s = synth.MoEShape("res", 300, 256, 512, 8, 2, "bf16")
    t = device_inputs(s, 6)
    y = run_layer(t, 2, residual=t["x"])
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(s.T))
    assert_close(to64(y), f64(h["x"]) + y_ref, "bf16")
    s32 = synth.MoEShape("res32", 40, 64, 128, 8, 2, "f32")
    t = device_inputs(s32, 6)
    y = run_layer(t, 2, residual=t["x"])
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(s32.T))
    assert_close(to64(y), f64(h["x"]) + y_ref, "f32")


def test_entry_points_agree_and_are_deterministic():
    """moe_layer_forward (library workspace), moe_layer_forward_ex and the
    three-call path router -> permute -> expert_ffn give identical bits, run
    after run."""
    s = synth.MoEShape("api", 900, 256, 512, 8, 2, "bf16")
    t = device_inputs(s, 7)
    a = moe.moe_layer_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 2)
    b = run_layer(t, 2)
    idx, w = moe.moe_router_topk(t["x"], t["Wg"], 2)
    off, perm, inv = moe.moe_permute(idx, 8)
    c = moe.moe_expert_ffn(t["x"], t["W1"], t["W3"], t["W2"], off, perm, inv, w)
    d_ = moe.moe_layer_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 2)
    for o in (b, c, d_):
        assert torch.equal(a.view(torch.int16), o.view(torch.int16))
    moe.moe_release_workspace()


@pytest.mark.parametrize("T,kernels", [(32, 4), (100, 5), (2304, 4)],
                         ids=["router-permutes", "one-block-permutation", "chunked-permutation"])
def test_bf16_layer_kernels(T, kernels):
    """The bf16 layer is router, one-block permutation and row gather, up-
    projection GEMM and down-projection GEMM: the combine runs in the down
    GEMM's epilogue, with no kernel of its own.  Up to 64 tokens (one router
    cluster) the router writes the permutation, and from 2048 assignments
    the per-chunk counts for the row scatter: four kernels."""
    s = synth.MoEShape("launches", T, 256, 512, 8, 2, "bf16")
    t = device_inputs(s, 3)
    ws = torch.empty(moe.moe_workspace_size(T, s.d, s.f, s.E, s.k, 0), dtype=torch.uint8, device="cuda")
    run_layer(t, 2)  # set-up outside the record
    torch.cuda.synchronize()
    moe.moe_profile_select(None)
    moe.moe_profile_enable(True)
    y = moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], 2, workspace=ws)
    torch.cuda.synchronize()
    prof = moe.moe_profile_read()
    moe.moe_profile_enable(False)
    n = {name: cnt for name, (_, cnt) in prof.items()}
    assert n["combine"] == 0 and n["down_combine_gemm"] == 1 and n["up_swiglu_gemm"] == 1
    assert sum(n.values()) == kernels, n
    assert n["permute"] == (0 if kernels == 4 else 1) and n["gather_rows"] == 1
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, np.arange(T))
    assert_close(to64(y), y_ref, "bf16")


def test_unrouted_and_repeated_slots():
    """moe_expert_ffn on a caller's routing with slots the permutation skips
    (expert id -1: inv = -1, flagged) and tokens that name one expert twice.
    Skipped slots add nothing, a token with no routed slot gets y = 0, and a
    repeated expert adds both weighted copies; the oracle reads the same
    routing (a slot with an id outside [0, E) contributes nothing there)."""
    s = synth.MoEShape("unrouted", 300, 256, 384, 8, 2, "bf16")
    t = device_inputs(s, 12)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(8, size=2, replace=False) for _ in range(s.T)]).astype(np.int32)
    tok = np.arange(s.T)
    idx[tok % 3 == 0, 1] = -1
    idx[tok % 5 == 0, 0] = -1          # tokens 0, 15, 30, ...: no routed slot at all
    idx[tok % 7 == 1, 1] = idx[tok % 7 == 1, 0]
    w = rng.uniform(0.1, 0.9, size=(s.T, 2)).astype(np.float32)
    idx_d, w_d = torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda()
    off, perm, inv = moe.moe_permute(idx_d, s.E)
    y = torch.full_like(t["x"], float("nan"))
    moe.moe_expert_ffn(t["x"], t["W1"], t["W3"], t["W2"], off, perm, inv, w_d, y=y)
    torch.cuda.synchronize()
    assert moe.moe_device_errors() == 2  # MOE_DEVERR_BAD_EXPERT, from the permutation
    h = host_copy(t)
    y_ref, _, _ = oracle_rows(h, 2, tok, routing=(idx, w.astype(np.float64)))
    got = to64(y)
    assert_close(got, y_ref, "bf16")
    assert (got[tok % 15 == 0] == 0).all()


def test_zero_tokens_is_a_no_op():
    s = synth.MoEShape("z", 4, 64, 128, 8, 2, "bf16")
    t = device_inputs(s, 8)
    y = torch.full((0, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    out = moe.moe_layer_forward_ex(t["x"][:0], t["Wg"], t["W1"], t["W3"], t["W2"], 2, y=y)
    assert out.shape == (0, 64)


# ---------------------------------------------------------------- full Mixtral shapes

@pytest.fixture(scope="module")
def mixtral_weights():
    """Layer-0 expert weights of seed 0 (shared by the decode, prefill and
    skewed workloads), on the device and as host bf16 bits."""
    s = synth.CONFIGS["prefill"]
    t = device_inputs(s, 0, with_x=False)
    return t, host_copy({k: t[k] for k in ("W1", "W3", "W2")})


def big_check(name, mixtral_weights, sample):
    s = synth.CONFIGS[name]
    tw, hw = mixtral_weights
    t = device_inputs(synth.MoEShape(s.name, s.T, s.d, 8, s.E, s.k, s.dtype, skew=s.skew), 0)
    t = {"x": t["x"], "Wg": t["Wg"], "W1": tw["W1"], "W3": tw["W3"], "W2": tw["W2"]}
    y = run_layer(t, s.k)
    idx_g, w_g = moe.moe_router_topk(t["x"], t["Wg"], s.k)
    off_g, perm_g, inv_g = moe.moe_permute(idx_g, s.E)
    torch.cuda.synchronize()
    h = dict(hw, x=to_bits(t["x"]), Wg=to_bits(t["Wg"]))
    idx_o, _, _ = check_routing(idx_g.cpu().numpy(), w_g.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), s.k)
    off, perm, _ = check_permutation(off_g.cpu().numpy(), perm_g.cpu().numpy(), inv_g.cpu().numpy(), idx_o, s.E)
    toks = np.arange(s.T) if sample is None else stratified_tokens(off, perm, s.k, sample)
    y_ref, _, _ = oracle_rows(h, s.k, toks)
    rel = assert_close(to64(y)[toks], y_ref, "bf16")
    return rel, np.diff(off)


def to_bits(t):
    from synth.device import to_host_bits
    return to_host_bits(t)


def test_decode_full_shape_every_token(mixtral_weights):
    big_check("decode", mixtral_weights, None)


def test_decode_full_shape_f32_every_token():
    """The fp32 layer (router, permutation, fp32 expert kernels, combine) at
    Mixtral dimensions (T = 32, d = 4096, f = 14336: 5.6 GB of fp32 expert
    weights), every token within the fp32 bound."""
    full_check(synth.MoEShape("decode-f32", 32, 4096, 14336, 8, 2, "f32"), 3)


def test_prefill_full_shape_every_token(mixtral_weights):
    """The headline workload (T = 4096, Mixtral dimensions, the default
    256 x 512 pair tiles) against the oracle on all 4096 tokens."""
    big_check("prefill", mixtral_weights, None)


@pytest.mark.parametrize("name,cta_group,bn,rb,wide", [
    ("decode", "2", "256", "128", "0"), ("decode", "2", "256", "128", "1"), ("decode", "1", "256", "128", "0"),
    ("decode", "h", "256", "128", "0"),
    ("prefill", "1", "128", "128", "0"), ("prefill", "2", "256", "128", "0"), ("prefill", "2", "256", "128", "1"),
    ("prefill", "1", "256", "128", "0"), ("prefill", "1", "256", "32", "0")])
def test_full_shapes_other_gemm_variant(name, cta_group, bn, rb, wide, mixtral_weights):
    """Variants the size heuristics do not pick, at the full shapes, on
    every token."""
    force_variant(cta_group, bn, rb, wide)
    big_check(name, mixtral_weights, None)


def test_top4_at_mixtral_dimensions_every_token(mixtral_weights):
    """k = 4 of E = 8 at d = 4096, f = 14336 (the Mixtral expert weights),
    T = 1024: 4096 assignments, so the chunked permutation and CTA-pair tiles
    run, and the combine adds slots 2 and 3 through inv; routing, permutation
    and outputs against the oracle on every token."""
    s = synth.MoEShape("top4", 1024, 4096, 14336, 8, 4, "bf16")
    tw, hw = mixtral_weights
    t = device_inputs(synth.MoEShape(s.name, s.T, s.d, 8, s.E, s.k, s.dtype), 5)
    t = {"x": t["x"], "Wg": t["Wg"], "W1": tw["W1"], "W3": tw["W3"], "W2": tw["W2"]}
    y = run_layer(t, s.k)
    idx_g, w_g = moe.moe_router_topk(t["x"], t["Wg"], s.k)
    off_g, perm_g, inv_g = moe.moe_permute(idx_g, s.E)
    torch.cuda.synchronize()
    h = dict(hw, x=to_bits(t["x"]), Wg=to_bits(t["Wg"]))
    idx_o, _, _ = check_routing(idx_g.cpu().numpy(), w_g.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), s.k)
    check_permutation(off_g.cpu().numpy(), perm_g.cpu().numpy(), inv_g.cpu().numpy(), idx_o, s.E)
    y_ref, _, _ = oracle_rows(h, s.k, np.arange(s.T))
    assert_close(to64(y), y_ref, "bf16")


def test_skewed_full_shape_every_token(mixtral_weights):
    """T = 16384 with the skewed router (hottest expert 35 %, 45 pair row
    blocks, several groups of the tile order) on every token."""
    _, counts = big_check("skewed", mixtral_weights, None)
    share = counts / counts.sum()
    assert abs(share[0] - 0.35) < 0.005 and (np.diff(share) < 0).all()


def test_many_tokens_small_widths():
    """65536 tokens with the skewed router (hottest expert ~35 %: ~45 000
    rows, 180 pair row blocks, several groups of the tile order) at small
    widths: 2048 permutation chunks, 1024 router clusters, the combine's
    arrival counters for every token; routing and permutation checked on
    every token, outputs on a stratified sample."""
    s = synth.MoEShape("many", 65536, 128, 256, 8, 2, "bf16", skew=True)
    t = device_inputs(s, 41)
    y = run_layer(t, s.k)
    idx_g, w_g = moe.moe_router_topk(t["x"], t["Wg"], s.k)
    off_g, perm_g, inv_g = moe.moe_permute(idx_g, s.E)
    torch.cuda.synchronize()
    h = host_copy(t)
    idx_o, _, _ = check_routing(idx_g.cpu().numpy(), w_g.cpu().numpy(), f64(h["x"]), f64(h["Wg"]), s.k)
    off, perm, _ = check_permutation(off_g.cpu().numpy(), perm_g.cpu().numpy(), inv_g.cpu().numpy(), idx_o, s.E)
    assert np.diff(off).max() > 12 * 256 * 2  # the hottest expert spans several groups of row blocks
    toks = stratified_tokens(off, perm, s.k, 512)
    y_ref, _, _ = oracle_rows(h, s.k, toks)
    assert_close(to64(y)[toks], y_ref, "bf16")
