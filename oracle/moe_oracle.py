"""fp64 CPU oracle of the sparse mixture-of-experts feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with
it.

What it computes: the layer of "Mixtral of Experts", §2.1, written out as its
definition, in float64, one token at a time (plain numpy; a matrix product is
the only library routine used, for the expert's three projections):

  * router logits l = x . W_g, bias-free and linear (Method, step 2; the
    hyper-parameter table: "router: linear, no bias");
  * TopK keeps the K largest logits (§2.1, display 2; K = 2 for Mixtral);
  * the gate weights are a softmax over the kept K logits only, so they sum
    to 1 over the chosen experts (§2.1 display 2; Pitfalls, "Renormalised
    top-2 weights": the softmax is not over all eight);
  * each chosen expert is a SwiGLU block, w2 (SiLU(w1 x) * (w3 x))
    (Method, "SwiGLU expert"; §2.1);
  * y = sum over the kept experts of weight * expert output (§2.1, displays
    1 and 3; Method, step 4).

Readings taken where the pages are silent (each is listed in the design
notes): ties in TopK go to the lower expert index and slot 0 holds the larger
logit; logits are summed in increasing feature order; no capacity limit and
no token dropping (hyper-parameter table: "Code has no capacity limit");
SiLU(a) = a / (1 + exp(-a)); the expert-grouped permutation is a stable
counting sort of the assignment ids t*K + j by expert (Method: the batch is
processed "grouped by expert").

All inputs are bf16 or fp32 values; both are exact in fp64, and so is every
product x_i * w_i of two of them (at most 48 significant bits), so the only
rounding in the logits is that of the running sum.

Every function here is pinned by a CPU test against something other than
itself (closed forms, brute force, special cases, invariants); see
tests/test_oracle_pins.py.
"""

from __future__ import annotations

import numpy as np

F64_UNIT_ROUNDOFF = 2.0 ** -53


def router_logits(x: np.ndarray, Wg: np.ndarray) -> np.ndarray:
    """l[t, e] = sum_i x[t, i] * Wg[e, i], accumulated in fp64 in increasing i.

    x: [T, d]; Wg: [E, d] (the router weight stored as (n_experts, dim), as
    in the Method pseudocode).  Returns [T, E] float64.
    Mixtral of Experts, Method step 2 and §2.1 (linear, bias-free router).
    """
    x = np.asarray(x, dtype=np.float64)
    Wg = np.asarray(Wg, dtype=np.float64)
    T, d = x.shape
    acc = np.zeros((T, Wg.shape[0]), dtype=np.float64)
    for i in range(d):
        acc += np.multiply.outer(x[:, i], Wg[:, i])
    return acc


def logit_sum_bound(x: np.ndarray, Wg: np.ndarray) -> np.ndarray:
    """Upper bound on |computed - exact| logit for ANY summation order of the
    d exact fp64 products: gamma_{d-1} * sum_i |x_i * Wg[e, i]|, with
    gamma_n = n u / (1 - n u) (Higham, Accuracy and Stability of Numerical
    Algorithms, 2nd ed., §4.2).  Two implementations that each meet it
    differ by at most twice this."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    Wg = np.abs(np.asarray(Wg, dtype=np.float64))
    n = x.shape[1] - 1
    gamma = n * F64_UNIT_ROUNDOFF / (1.0 - n * F64_UNIT_ROUNDOFF)
    return gamma * (x @ Wg.T)


def topk_lower_index(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first; an exact tie
    goes to the lower expert index.  Mixtral of Experts §2.1 display 2 (TopK).

    Written as k rounds of "take the arg-max of what is left"; np.argmax
    returns the first (lowest-index) maximum, which is the tie rule.
    """
    lg = np.array(logits, dtype=np.float64, copy=True)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), dtype=np.int32)
    rows = np.arange(T)
    for j in range(k):
        a = np.argmax(lg, axis=1)
        idx[:, j] = a
        lg[rows, a] = -np.inf
    return idx


def kept_softmax(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Gate weights: softmax over the kept logits only (max-subtracted, fp64).
    Mixtral of Experts §2.1 display 2; Pitfalls, renormalised top-2 weights."""
    kept = np.take_along_axis(np.asarray(logits, dtype=np.float64), idx.astype(np.int64), axis=1)
    z = np.exp(kept - kept[:, :1])
    return z / z.sum(axis=1, keepdims=True)


def route(x: np.ndarray, Wg: np.ndarray, k: int):
    """Router + TopK + kept softmax for every row of x.
    Returns (idx [T, k] int32, w [T, k] float64, logits [T, E] float64)."""
    lg = router_logits(x, Wg)
    idx = topk_lower_index(lg, k)
    return idx, kept_softmax(lg, idx), lg


def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a))."""
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu_expert(X: np.ndarray, W1e: np.ndarray, W3e: np.ndarray, W2e: np.ndarray) -> np.ndarray:
    """One SwiGLU expert applied to each row of X (fp64, no intermediate
    rounding): w2 (SiLU(w1 x) * (w3 x)).  W1e, W3e: [f, d]; W2e: [d, f].
    Mixtral of Experts, Method: SwiGLU expert; §2.1."""
    X = np.asarray(X, dtype=np.float64)
    a = X @ np.asarray(W1e, dtype=np.float64).T
    b = X @ np.asarray(W3e, dtype=np.float64).T
    return (silu(a) * b) @ np.asarray(W2e, dtype=np.float64).T


def moe_forward(x, Wg, W1, W3, W2, k: int, tokens=None, to_f64=None, routing=None):
    """y for the rows `tokens` of x (all rows if None), fp64.

    x: [T, d]; Wg: [E, d]; W1, W3: [E, f, d]; W2: [E, d, f].  `to_f64` turns
    one expert's stored weight slice into float64 (identity by default; the
    tests pass the exact bf16 -> fp64 widening).  `routing` may supply
    (idx, w) for the selected rows, else they are computed here.

    For each selected token t: y[t] = sum_{j < k} w[t, j] * Expert_{idx[t, j]}(x[t]),
    summed in slot order j = 0, 1, ...  Mixtral of Experts §2.1 displays 1-3;
    Method steps 2-4 and the layer pseudocode.
    Returns (y [n, d], idx [n, k], w [n, k]).
    """
    conv = (lambda a: np.asarray(a, dtype=np.float64)) if to_f64 is None else to_f64
    x = np.asarray(x)
    rows = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    xs = np.asarray(x[rows], dtype=np.float64)
    if routing is None:
        idx, w, _ = route(xs, conv(Wg), k)
    else:
        idx, w = routing
    n, d = xs.shape
    outs = np.zeros((n, k, d), dtype=np.float64)
    E = Wg.shape[0]
    for e in range(E):
        sel = np.nonzero(idx == e)  # (row, slot) pairs routed to expert e
        if sel[0].size == 0:
            continue
        o = swiglu_expert(xs[sel[0]], conv(W1[e]), conv(W3[e]), conv(W2[e]))
        outs[sel[0], sel[1]] = o
    y = np.zeros((n, d), dtype=np.float64)
    for j in range(k):
        y += w[:, j:j + 1] * outs[:, j]
    return y, idx, w


def permute(idx: np.ndarray, E: int):
    """Expert-contiguous order of the T*k assignments q = t*k + j.

    A counting sort written out: count each expert's assignments, take the
    exclusive prefix sum as the start of each expert's block, then walk the
    assignments in increasing q and place each at the next free row of its
    expert's block.  Within an expert the assignment ids therefore increase
    (stable).  Mixtral of Experts, Method: the batch is processed "grouped by
    expert"; Pitfalls: the reference layer scatters results back.

    Returns (offsets [E+1], perm [T*k], inv [T*k]), all int32, with
    perm[r] = the assignment at permuted row r and inv[q] = the row of q.
    """
    flat = np.asarray(idx, dtype=np.int64).ravel()
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    nxt = offsets[:E].copy()
    perm = np.empty(flat.size, dtype=np.int64)
    inv = np.empty(flat.size, dtype=np.int64)
    for q, e in enumerate(flat):
        r = nxt[e]
        perm[r] = q
        inv[q] = r
        nxt[e] = r + 1
    return offsets.astype(np.int32), perm.astype(np.int32), inv.astype(np.int32)


def routing_stats(idx: np.ndarray, E: int, seq_len: int = 0) -> np.ndarray:
    """Routing statistics of "Mixtral of Experts" §5 / tab. 5, by their
    definition, with plain loops.  Returns int64 [E + 3]:
    loads of the E experts (assignments per expert); then, over consecutive
    token pairs (t-1, t) inside a sequence (sequences of seq_len tokens;
    seq_len <= 0: one sequence), the number whose first choices agree, the
    number whose kept expert sets intersect (the card's "first or second
    choice" repetition for k = 2, whose uniform-routing rate 1 - C(6,2)/C(8,2)
    = 13/28 matches the quoted ~46%), and the number of pairs counted."""
    idx = np.asarray(idx)
    T, k = idx.shape
    load = [0] * E
    for t in range(T):
        for j in range(k):
            load[int(idx[t, j])] += 1
    first = overlap = pairs = 0
    for t in range(1, T):
        if seq_len > 0 and t % seq_len == 0:
            continue
        pairs += 1
        if idx[t, 0] == idx[t - 1, 0]:
            first += 1
        if set(idx[t].tolist()) & set(idx[t - 1].tolist()):
            overlap += 1
    return np.array(load + [first, overlap, pairs], dtype=np.int64)
