"""Helpers for the GPU parity tests: inputs, the oracle on the same inputs,
and the comparisons (indices bit-exact, gate weights to 1e-6, outputs to
the relative bound of the dtype)."""

from __future__ import annotations

import numpy as np

import oracle
import synth
from synth.device import device_inputs, to_host_bits

TOL = {"bf16": 1e-2, "f32": 1e-5}   # max|y - y_ref| <= TOL * max|y_ref|
W_ATOL = 1e-6                       # |w - w_ref|, fp32 softmax of the kept logits
NEAR_TIE_FRACTION = 1e-3            # at most this share of tokens may be genuine near-ties


def f64(bits_or_f32: np.ndarray) -> np.ndarray:
    a = np.asarray(bits_or_f32)
    return synth.bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def host_copy(t: dict) -> dict:
    return {k: to_host_bits(v) for k, v in t.items()}


def check_routing(idx_gpu: np.ndarray, w_gpu: np.ndarray, x64: np.ndarray, wg64: np.ndarray, k: int):
    """Indices must equal the oracle's.  A differing token is accepted only if
    the oracle's competing logits are closer than twice the fp64 summation
    bound (a genuine near-tie that any summation order may resolve either
    way); such tokens are counted and capped.  Gate weights to W_ATOL where
    the indices agree.  Returns (oracle idx, oracle w, number of near-ties)."""
    idx_o, w_o, lg = oracle.route(x64, wg64, k)
    bound = 2.0 * oracle.logit_sum_bound(x64, wg64)
    bad = np.nonzero((idx_gpu != idx_o).any(axis=1))[0]
    near = 0
    for t in bad:
        chosen_g = lg[t, idx_gpu[t]]
        chosen_o = lg[t, idx_o[t]]
        slack = bound[t].max()
        assert len(set(idx_gpu[t].tolist())) == k, ("duplicate expert", t, idx_gpu[t])
        assert np.all(np.abs(np.sort(chosen_g)[::-1] - np.sort(chosen_o)[::-1]) <= slack), \
            ("index mismatch that is not a near-tie", t, idx_gpu[t], idx_o[t], lg[t])
        near += 1
    assert near <= max(1, NEAR_TIE_FRACTION * len(idx_o)), near
    ok = ~np.isin(np.arange(len(idx_o)), bad)
    if ok.any():
        err = np.abs(w_gpu[ok].astype(np.float64) - w_o[ok]).max()
        assert err <= W_ATOL, err
    return idx_o, w_o, near


def check_permutation(off_g, perm_g, inv_g, idx: np.ndarray, E: int):
    off_o, perm_o, inv_o = oracle.permute(idx, E)
    np.testing.assert_array_equal(off_g, off_o)
    np.testing.assert_array_equal(perm_g, perm_o)
    np.testing.assert_array_equal(inv_g, inv_o)
    return off_o, perm_o, inv_o


def assert_close(y_gpu64: np.ndarray, y_ref: np.ndarray, dtype: str, what: str = "y"):
    scale = np.abs(y_ref).max()
    err = np.abs(y_gpu64 - y_ref).max()
    assert np.isfinite(y_gpu64).all(), what + " has non-finite values"
    assert err <= TOL[dtype] * scale, "%s: max|dy| = %.3e > %.0e * max|y_ref| = %.3e" % (
        what, err, TOL[dtype], TOL[dtype] * scale)
    return err / scale


def stratified_tokens(off: np.ndarray, perm: np.ndarray, k: int, n: int, seed: int = 0) -> np.ndarray:
    """Tokens whose rows sit at each expert's first and last permuted rows and
    at the 128-row tile edges (127, 128, 255, 256 into the block), topped up
    with random tokens to n.  Tokens are independent, so checking a sample is
    exact for the sampled rows."""
    rows = []
    E = len(off) - 1
    for e in range(E):
        b, t = int(off[e]), int(off[e + 1])
        if t == b:
            continue
        for r in (b, t - 1, b + 127, b + 128, b + 255, b + 256):
            if b <= r < t:
                rows.append(r)
    toks = set(int(perm[r]) // k for r in rows)
    T = len(perm) // k
    rng = np.random.default_rng(seed)
    for t in rng.permutation(T):
        if len(toks) >= n:
            break
        toks.add(int(t))
    return np.array(sorted(toks))


def oracle_rows(h: dict, k: int, tokens, routing=None):
    """Oracle outputs for `tokens` from host copies `h` (bf16 bits or fp32)."""
    x64 = f64(h["x"][tokens])
    y, idx, w = oracle.moe_forward(x64, f64(h["Wg"]), h["W1"], h["W3"], h["W2"], k, to_f64=f64,
                                   routing=routing)
    return y, idx, w


__all__ = ["device_inputs", "host_copy", "check_routing", "check_permutation", "assert_close",
           "stratified_tokens", "oracle_rows", "f64", "TOL"]


def assert_residual_close(gpu64, x64, moe_ref, what="x_{l+1}"):
    """Residual layers: gpu = round_bf16(x + MoE(x)).  Bound: the bf16 layer
    tolerance on the MoE part, 1e-2 * max|MoE_ref|, plus the final bf16
    rounding of the sum, 2^-8 |x + MoE_ref| (twice the half-ulp)."""
    ref = x64 + moe_ref
    bound = 1e-2 * np.abs(moe_ref).max() + 2.0 ** -8 * np.abs(ref)
    err = np.abs(gpu64 - ref)
    assert np.isfinite(gpu64).all(), what + " has non-finite values"
    assert (err <= bound).all(), "%s: worst excess %.3e" % (what, (err - bound).max())
    return float((err / np.abs(moe_ref).max()).max())
