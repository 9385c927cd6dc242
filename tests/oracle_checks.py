"""Pins for the fp64 oracle: each check compares it with something other than
itself -- values printed on the pages, closed forms, special cases that reduce
to a textbook or library routine (torch fp64), brute force on tiny inputs and
invariants.  Every check takes an `oracle.Oracle` so the mutation tests can run
the same checks against deliberately broken copies of the oracle.

Pages cited:
  [P2] "Mixtral of Experts" flash cards (learn.ifs.name/d/jiang2024), section
       2.1 "Sparse Mixture of Experts": the layer equation, n and K.
  [P5] "Mixture of Experts: Why Mixtral Only Wakes Up Two Specialists"
       (neobadger.com), Part 3 Steps 1-4 and Part 4.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [float(v) for v in vals]
    return out


def rand_layer(seed, T, d, F, n, scale_x=1.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, d)) * scale_x
    Wg = g.standard_normal((d, n)) / math.sqrt(d)
    w1 = g.standard_normal((n, d, F)) / math.sqrt(d)
    w3 = g.standard_normal((n, d, F)) / math.sqrt(d)
    w2 = g.standard_normal((n, F, d)) / math.sqrt(F)
    return x, Wg, w1, w3, w2


def torch_swiglu(x, w1e, w3e, w2e):
    """Textbook SwiGLU FFN with torch's own silu and matmul, fp64."""
    X = torch.from_numpy(np.asarray(x, np.float64))
    a = X @ torch.from_numpy(np.asarray(w1e, np.float64))
    b = X @ torch.from_numpy(np.asarray(w3e, np.float64))
    h = torch.nn.functional.silu(a) * b
    return (h @ torch.from_numpy(np.asarray(w2e, np.float64))).numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# --------------------------------------------------------------------------
# Router, top-K, softmax
# --------------------------------------------------------------------------

def check_worked_example(O):
    """[P5] Part 3 Steps 1-3: logits (0.1, -0.4, 2.3, 0.0, -1.2, 0.6, 1.5, -0.3)
    -> experts 3 and 7 (1-based), weights about 0.69 and 0.31."""
    g = read_golden("worked_routing_example.txt")
    L = np.array(g["logits"])
    n = L.size
    # W_g = I: the logits are x itself.
    idx, gate, logits = O.router(L[None, :], np.eye(n), 2)
    assert list(idx[0] + 1) == [int(v) for v in g["top2_one_based"]]
    dec = int(g["gates_decimals"][0])
    assert [round(float(v), dec) for v in gate[0]] == g["gates_printed"]
    # The same logits produced by a non-square W_g (d=3 != n=8) whose first
    # row holds them: fails if the gate's operand is transposed.
    rng = np.random.default_rng(7)
    Wg = np.vstack([L[None, :], rng.standard_normal((2, n))])
    x = np.array([[1.0, 0.0, 0.0]])
    idx2, gate2, logits2 = O.router(x, Wg, 2)
    assert np.array_equal(idx2, idx) and np.allclose(gate2, gate, rtol=0, atol=1e-15)
    assert np.allclose(logits2[0], L, rtol=0, atol=0)


def check_two_way_softmax_closed_form(O):
    """K=2: the softmax over the two kept logits is the logistic function of
    their difference, g0 = 1/(1+e^-(L0-L1))."""
    rng = np.random.default_rng(3)
    for _ in range(20):
        L = rng.standard_normal(6) * 3
        idx, gate, _ = O.router(L[None, :], np.eye(6), 2)
        a, b = sorted(L)[-1], sorted(L)[-2]
        g0 = 1.0 / (1.0 + math.exp(-(a - b)))
        assert abs(gate[0, 0] - g0) < 1e-15 and abs(gate[0, 1] - (1 - g0)) < 1e-15


def check_logits_are_x_times_Wg(O):
    """Step 1: the logits are the bias-free linear map x . W_g (numpy matmul)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((17, 40))
    Wg = rng.standard_normal((40, 12))
    _, _, logits = O.router(x, Wg, 3)
    assert np.allclose(logits, x @ Wg, rtol=1e-13, atol=1e-13)


def check_topk_brute_force(O):
    """For tiny n the kept set maximises the sum of K logits over all K-subsets
    (brute force), ordered by descending logit."""
    rng = np.random.default_rng(5)
    for n, K in ((4, 2), (8, 2), (8, 3), (13, 2), (16, 4), (5, 5), (6, 1)):
        x = rng.standard_normal((40, 24))
        Wg = rng.standard_normal((24, n))
        idx, gate, _ = O.router(x, Wg, K)
        L = x @ Wg
        for t in range(x.shape[0]):
            best = max(itertools.combinations(range(n), K), key=lambda s: sum(L[t, list(s)]))
            assert sorted(idx[t].tolist()) == sorted(best)
            vals = L[t, idx[t]]
            assert all(vals[i] >= vals[i + 1] for i in range(K - 1))


def check_ties_go_to_lower_index(O):
    """Equal logits: the lower expert index is kept first (the reading taken
    where torch.topk leaves the order open)."""
    cases = [([1.0, 3.0, 3.0, 0.0], 2, [1, 2]),
             ([5.0, 5.0, 5.0, 5.0], 2, [0, 1]),
             ([0.0, 2.0, 1.0, 2.0, 2.0], 3, [1, 3, 4]),
             ([-1.0, -1.0, -2.0], 1, [0])]
    for L, K, want in cases:
        idx, gate, _ = O.router(np.array([L]), np.eye(len(L)), K)
        assert idx[0].tolist() == want, (L, idx)
        assert np.allclose(gate[0], np.full(K, 1.0 / K)) or len(set(np.array(L)[want])) > 1


def check_gate_invariants(O):
    """[P5] Step 3: positive weights that add up to 1, larger logit -> larger
    weight; K=1 gives weight exactly 1."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((64, 32))
    Wg = rng.standard_normal((32, 8)) * 2
    for K in (1, 2, 3, 8):
        _, gate, _ = O.router(x, Wg, K)
        assert np.all(gate > 0)
        assert np.allclose(gate.sum(1), 1.0, rtol=0, atol=1e-14)
        assert np.all(np.diff(gate, axis=1) <= 0)
        if K == 1:
            assert np.all(gate == 1.0)


def check_gates_to_bf16(O):
    """The routing code quoted in [P5] Part 3 computes the softmax in fp32 and
    casts the weights to the inputs' dtype.  Pins of that cast: the worked
    example's gates 0.689974 / 0.310026 (printed 0.69 / 0.31) become
    177/256 and 159/512 (nearest bf16); halfway cases go to the even mantissa;
    a double just above a bf16 halfway point that rounds onto it in fp32 then
    goes to the even neighbour (fp32 first, then bf16); values already in bf16
    are unchanged, and torch's fp32 -> bf16 cast agrees on random gates."""
    import torch
    g = O.gates_to_bf16(np.array([0.689974, 0.310026]))
    assert g[0] == 177 / 256 and g[1] == 159 / 512, g
    # ulp of bf16 is 2^-7 on [1, 2) and 2^-8 on [0.5, 1): these sit halfway
    ties = O.gates_to_bf16(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 0.5 + 2.0 ** -9, 0.5 + 3 * 2.0 ** -9]))
    assert list(ties) == [1.0, 1 + 2.0 ** -6, 0.5, 0.5 + 2.0 ** -7], ties
    # fp32 first: 1 + 2^-8 + 2^-30 is 1 + 2^-8 in fp32 (a tie in bf16 -> 1.0),
    # while rounding the double straight to bf16 would give 1 + 2^-7
    assert O.gates_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1.0
    exact = np.array([1.0, 0.5, 0.75, 2.0 ** -20, 0.0])
    assert np.array_equal(O.gates_to_bf16(exact), exact)
    rng = np.random.default_rng(21)
    r = rng.random(4096)
    ref = torch.from_numpy(r).float().to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.gates_to_bf16(r), ref)


# --------------------------------------------------------------------------
# Experts and the combine
# --------------------------------------------------------------------------

def check_silu(O):
    """silu(z) = z*sigmoid(z): special values and torch's silu."""
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    assert abs(O.silu(-40.0)) < 1e-15
    assert abs(O.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    z = np.linspace(-12, 12, 97)
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    got = np.array([O.silu(v) for v in z])
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-16)


def check_n1_is_plain_swiglu(O):
    """n=1, K=1: the layer is a plain SwiGLU FFN (torch fp64)."""
    x, Wg, w1, w3, w2 = rand_layer(21, 9, 48, 80, 1)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, 1)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    ref = torch_swiglu(x, w1[0], w3[0], w2[0])
    assert rel_l2(y, ref) < 1e-13


def check_expert_indexing(O):
    """One expert e of n on one token matches torch on w1[e], w3[e], w2[e]."""
    x, Wg, w1, w3, w2 = rand_layer(22, 3, 32, 48, 5)
    for e in range(5):
        got = O.expert(x[1], w1, w3, w2, e)
        ref = torch_swiglu(x[1:2], w1[e], w3[e], w2[e])[0]
        assert rel_l2(got, ref) < 1e-13


def check_K_equals_n_is_dense_mixture(O):
    """K=n: Top-K keeps everything, so y is the dense softmax-weighted sum of
    all experts (torch softmax and matmul, fp64)."""
    T, d, F, n = 11, 40, 56, 6
    x, Wg, w1, w3, w2 = rand_layer(23, T, d, F, n)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, n)
    p = torch.softmax(torch.from_numpy(x @ Wg), dim=1).numpy()
    ref = np.zeros((T, d))
    for e in range(n):
        ref += p[:, e:e + 1] * torch_swiglu(x, w1[e], w3[e], w2[e])
    assert rel_l2(y, ref) < 1e-13


def check_top2_layer_against_torch(O):
    """The Top-2 layer on random data against a torch restatement that
    builds the sparse gate vector (others -inf) and sums all experts."""
    T, d, F, n = 13, 32, 40, 8
    x, Wg, w1, w3, w2 = rand_layer(24, T, d, F, n)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, 2)
    L = torch.from_numpy(x @ Wg)
    top = torch.topk(L, 2, dim=1)
    masked = torch.full_like(L, float("-inf")).scatter(1, top.indices, top.values)
    p = torch.softmax(masked, dim=1).numpy()
    ref = np.zeros((T, d))
    for e in range(n):
        ref += p[:, e:e + 1] * torch_swiglu(x, w1[e], w3[e], w2[e])
    assert rel_l2(y, ref) < 1e-13


def check_relabel_invariance(O):
    """Relabelling experts together with their W_g columns leaves y unchanged
    and relabels the chosen indices."""
    T, d, F, n = 20, 24, 32, 7
    x, Wg, w1, w3, w2 = rand_layer(25, T, d, F, n)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, 2)
    perm = np.random.default_rng(1).permutation(n)  # new expert j is old perm[j]
    y2, idx2, gate2 = O.moe_forward(x, Wg[:, perm], w1[perm], w3[perm], w2[perm], 2)
    inv = np.argsort(perm)
    assert np.array_equal(inv[idx], idx2)
    assert np.allclose(gate, gate2, rtol=0, atol=1e-15)
    assert rel_l2(y2, y) < 1e-14


def check_unchosen_experts_do_not_matter(O):
    """[P5] Step 2: the experts not kept are not run: changing them leaves y
    bit-identical.  Also y is linear in w2 (scaling by 2 is exact)."""
    T, d, F, n = 3, 16, 24, 8
    x, Wg, w1, w3, w2 = rand_layer(26, T, d, F, n)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, 2)
    unused = sorted(set(range(n)) - set(idx.ravel().tolist()))
    assert unused, "seeded case should leave an expert unused"
    w1b, w3b, w2b = w1.copy(), w3.copy(), w2.copy()
    for e in unused:
        w1b[e] = 1e3
        w3b[e] = -7.0
        w2b[e] = 5.0
    yb, _, _ = O.moe_forward(x, Wg, w1b, w3b, w2b, 2)
    assert np.array_equal(y, yb)
    y2, _, _ = O.moe_forward(x, Wg, w1, w3, 2.0 * w2, 2)
    assert np.array_equal(y2, 2.0 * y)


def check_forward_with_routing_consistent(O):
    """Routing supplied from outside reproduces the full forward exactly, and
    a hand-made routing matches torch per token."""
    T, d, F, n = 10, 24, 32, 5
    x, Wg, w1, w3, w2 = rand_layer(27, T, d, F, n)
    y, idx, gate = O.moe_forward(x, Wg, w1, w3, w2, 2)
    y2 = O.forward_with_routing(x, idx, gate, w1, w3, w2)
    assert np.array_equal(y, y2)
    idx3 = np.array([[t % n, (t + 2) % n] for t in range(T)], np.int32)
    gate3 = np.array([[0.25, 0.75]] * T)
    y3 = O.forward_with_routing(x, idx3, gate3, w1, w3, w2)
    for t in range(T):
        ref = 0.25 * torch_swiglu(x[t:t + 1], w1[idx3[t, 0]], w3[idx3[t, 0]], w2[idx3[t, 0]]) + \
            0.75 * torch_swiglu(x[t:t + 1], w1[idx3[t, 1]], w3[idx3[t, 1]], w2[idx3[t, 1]])
        assert rel_l2(y3[t], ref[0]) < 1e-13


def check_bf16_inputs_widen_exactly(O):
    """bf16 bit patterns are read as the exact values they encode."""
    from moe_inputs import f32_to_bf16_bits, bf16_bits_to_f32
    x, Wg, w1, w3, w2 = rand_layer(28, 5, 32, 64, 4)
    xb, w1b, w3b, w2b = (f32_to_bf16_bits(a.astype(np.float32)) for a in (x, w1, w3, w2))
    y_b, idx_b, g_b = O.moe_forward(xb, Wg, w1b, w3b, w2b, 2)
    wide = [bf16_bits_to_f32(a).astype(np.float64) for a in (xb, w1b, w3b, w2b)]
    y_w, idx_w, g_w = O.moe_forward(wide[0], Wg, wide[1], wide[2], wide[3], 2)
    assert np.array_equal(idx_b, idx_w) and np.array_equal(g_b, g_w) and np.array_equal(y_b, y_w)


# --------------------------------------------------------------------------
# Dispatch (the per-expert segments)
# --------------------------------------------------------------------------

def check_dispatch(O):
    """Segments: counts add to T*K, each (token, slot) lands in exactly one
    row of its expert's segment, and the order equals a stable library sort
    of the flattened pairs by expert."""
    rng = np.random.default_rng(31)
    for T, n, K in ((1, 1, 1), (7, 4, 2), (50, 8, 2), (33, 16, 3), (64, 5, 5), (0, 3, 2)):
        idx = np.array([rng.permutation(n)[:K] for _ in range(T)], np.int32).reshape(T, K)
        counts, offsets, row_token, token_row = O.dispatch(idx, n)
        assert counts.sum() == T * K and offsets[0] == 0 and offsets[-1] == T * K
        assert np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=n))
        order = np.argsort(idx.ravel(), kind="stable")  # flattened pair ids, by expert
        assert np.array_equal(row_token, order // K)
        inv = np.empty(T * K, np.int64)
        inv[order] = np.arange(T * K)
        assert np.array_equal(token_row.ravel(), inv)
        for r in range(T * K):
            e = np.searchsorted(offsets, r, side="right") - 1
            t = row_token[r]
            k = list(idx[t]).index(e)
            assert token_row[t, k] == r


# --------------------------------------------------------------------------
# Load-balancing statistics and expert capacity ([P5] Part 5)
# --------------------------------------------------------------------------

def check_router_stats_closed_forms(O):
    """[P5] Part 5 Tool 2: f_i = share of the routed pairs sent to expert i,
    P_i = mean router probability (softmax over all n logits), aux =
    alpha * N * sum f_i P_i.  All-equal logits give P_i = 1/N exactly; the
    tie-break then sends every token to experts 0..K-1, so aux = alpha; a
    uniform routing with uniform probabilities also gives aux = alpha (the
    minimum of N * sum f_i P_i is 1)."""
    T, d, n, K = 24, 16, 8, 2
    x = np.random.default_rng(40).standard_normal((T, d))
    Wg = np.zeros((d, n))
    idx, _, _ = O.router(x, Wg, K)
    f, P, aux = O.router_stats(x, Wg, idx, 0.01)
    assert np.allclose(P, 1.0 / n, rtol=0, atol=1e-15)
    assert np.allclose(f, [0.5, 0.5] + [0.0] * 6, rtol=0, atol=0)
    assert abs(aux - 0.01) < 1e-15
    uni = np.array([[t % n, (t + 1) % n] for t in range(T)], np.int32)
    f2, P2, aux2 = O.router_stats(x, Wg, uni, 0.02)
    assert np.allclose(f2, 1.0 / n, rtol=0, atol=1e-15) and abs(aux2 - 0.02) < 1e-15


def check_router_stats_against_torch(O):
    """Random case against torch's softmax and a bincount."""
    T, d, n, K = 37, 24, 6, 2
    g = np.random.default_rng(41)
    x = g.standard_normal((T, d))
    Wg = g.standard_normal((d, n)) / math.sqrt(d)
    idx, _, _ = O.router(x, Wg, K)
    f, P, aux = O.router_stats(x, Wg, idx, 0.01)
    Pt = torch.softmax(torch.from_numpy(x @ Wg), dim=1).mean(0).numpy()
    ft = np.bincount(idx.ravel(), minlength=n) / (T * K)
    assert np.allclose(P, Pt, rtol=1e-13, atol=1e-15)
    assert np.allclose(f, ft, rtol=0, atol=1e-15)
    assert abs(aux - 0.01 * n * float((ft * Pt).sum())) < 1e-14
    assert abs(P.sum() - 1.0) < 1e-13 and abs(f.sum() - 1.0) < 1e-14


def check_dispatch_capacity(O):
    """[P5] Part 5 'What happens when an expert is full': at most C pairs per
    expert, the first ones in dispatch order kept, the overflow dropped."""
    rng = np.random.default_rng(42)
    for T, n, K, C in ((50, 4, 2, 10), (64, 8, 2, 0), (33, 5, 3, 7), (40, 3, 1, 100), (1, 2, 2, 1)):
        idx = np.array([rng.permutation(n)[:K] for _ in range(T)], np.int32).reshape(T, K)
        counts, offsets, row_token, token_row = O.dispatch_capacity(idx, n, C)
        full = np.bincount(idx.ravel(), minlength=n)
        assert np.array_equal(counts, np.minimum(full, C))
        assert np.array_equal(np.diff(offsets), counts) and offsets[0] == 0
        order = np.argsort(idx.ravel(), kind="stable")
        kept = []
        for e in range(n):
            pe = order[idx.ravel()[order] == e]
            kept.extend(pe[:C].tolist())
        kept = np.array(kept, np.int64)
        tr = token_row.ravel()
        assert np.array_equal(np.sort(np.nonzero(tr >= 0)[0]), np.sort(kept))
        assert np.array_equal(tr[kept], np.arange(kept.size))
        assert np.array_equal(row_token[:kept.size], kept // K)
        if C >= full.max():
            c0, o0, rt0, tr0 = O.dispatch(idx, n)
            assert np.array_equal(c0, counts) and np.array_equal(tr0, token_row)


# --------------------------------------------------------------------------
# Expert-choice routing ([P1] "How Experts Are Chosen", item 2)
# --------------------------------------------------------------------------

def check_expert_choice_full_capacity_is_dense(O):
    """C = T: every expert keeps every token, so y is the dense
    softmax-weighted sum of all experts -- the token-choice layer with K = n,
    and torch's dense restatement."""
    T, d, F, n = 9, 24, 40, 5
    x, Wg, w1, w3, w2 = rand_layer(43, T, d, F, n)
    y, sel, gate = O.expert_choice(x, Wg, w1, w3, w2, T)
    assert np.array_equal(sel, np.tile(np.arange(T), (n, 1)))
    y_tc, _, _ = O.moe_forward(x, Wg, w1, w3, w2, n)
    assert rel_l2(y, y_tc) < 1e-13
    p = torch.softmax(torch.from_numpy(x @ Wg), dim=1).numpy()
    ref = sum(p[:, e:e + 1] * torch_swiglu(x, w1[e], w3[e], w2[e]) for e in range(n))
    assert rel_l2(y, ref) < 1e-13
    assert np.allclose(gate, p.T, rtol=1e-13, atol=0)


def check_expert_choice_ties_and_unchosen_tokens(O):
    """All-equal scores (W_g = 0): every expert keeps tokens 0..C-1 with gate
    1/n; the other tokens get y = 0 exactly."""
    T, d, F, n, C = 10, 16, 24, 4, 3
    x, _, w1, w3, w2 = rand_layer(44, T, d, F, n)
    y, sel, gate = O.expert_choice(x, np.zeros((d, n)), w1, w3, w2, C)
    assert np.array_equal(sel, np.tile(np.arange(C), (n, 1)))
    assert np.all(gate == 0.25)
    assert np.all(y[C:] == 0.0)
    ref = sum(torch_swiglu(x[:C], w1[e], w3[e], w2[e]) for e in range(n)) / n
    assert rel_l2(y[:C], ref) < 1e-13


def check_expert_choice_selection_brute_force(O):
    """Each expert's kept set is its C best tokens by probability (lower index
    first on ties), cross-checked with a lexsort of torch's softmax."""
    rng = np.random.default_rng(45)
    for T, n, C in ((30, 4, 7), (17, 8, 17), (50, 3, 1)):
        d, F = 12, 16
        x, Wg, w1, w3, w2 = rand_layer(int(rng.integers(1000)), T, d, F, n)
        y, sel, gate = O.expert_choice(x, Wg, w1, w3, w2, C)
        p = torch.softmax(torch.from_numpy(x @ Wg), dim=1).numpy()
        for e in range(n):
            order = np.lexsort((np.arange(T), -p[:, e]))
            assert np.array_equal(sel[e], np.sort(order[:C]))
            assert np.allclose(gate[e], p[sel[e], e], rtol=1e-13, atol=0)
        # y restated per token from the selection
        yr = np.zeros_like(y)
        for e in range(n):
            for j in range(C):
                t = sel[e, j]
                yr[t] += gate[e, j] * torch_swiglu(x[t:t + 1], w1[e], w3[e], w2[e])[0]
        assert rel_l2(y, yr) < 1e-13


# --------------------------------------------------------------------------
# FP8 E4M3 experts
# --------------------------------------------------------------------------

def check_e4m3_codec(O):
    """E4M3 as the OCP 8-bit floating point specification defines it: largest
    finite 448 (S.1111.110), NaN S.1111.111, smallest normal 2^-6 (0x08),
    smallest subnormal 2^-9 (0x01); encode rounds to nearest, ties to even,
    saturating beyond 448; every non-NaN code round-trips."""
    assert O.e4m3_decode(0x7E) == 448.0 and O.e4m3_decode(0xFE) == -448.0
    assert math.isnan(O.e4m3_decode(0x7F)) and math.isnan(O.e4m3_decode(0xFF))
    assert O.e4m3_decode(0x08) == 2.0 ** -6 and O.e4m3_decode(0x01) == 2.0 ** -9
    assert O.e4m3_decode(0x38) == 1.0 and O.e4m3_decode(0x00) == 0.0
    vals = [O.e4m3_decode(c) for c in range(0x7F)]
    assert all(vals[i] < vals[i + 1] for i in range(len(vals) - 1))
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert O.e4m3_encode(O.e4m3_decode(c)) == c, c
    # ties to even, saturation, rounding
    assert O.e4m3_encode(1.0 + 1 / 16) == 0x38       # halfway 1 | 1.125 -> even (1)
    assert O.e4m3_encode(1.125 + 1 / 16) == 0x3A     # halfway 1.125 | 1.25 -> even (1.25)
    assert O.e4m3_encode(2.0 ** -10) == 0x00          # halfway 0 | 2^-9 -> even (0)
    assert O.e4m3_encode(3 * 2.0 ** -10) == 0x02      # halfway 2^-9 | 2^-8 -> even (2^-8)
    assert O.e4m3_encode(1e9) == 0x7E and O.e4m3_encode(-1e9) == 0xFE
    assert O.e4m3_encode(460.0) == 0x7E and O.e4m3_encode(-3.0) == 0xC4
    rng = np.random.default_rng(46)
    for v in rng.standard_normal(200) * 10:
        q = O.e4m3_decode(O.e4m3_encode(v))
        assert abs(q - v) <= max(abs(v) * 2.0 ** -4, 2.0 ** -10)


def check_e4m3_weight_quantization(O):
    """One scale per output column (max |w| / 448 over the reduction rows): the
    column maximum codes to +-448 and every value comes back within E4M3's
    relative step."""
    rng = np.random.default_rng(47)
    w = rng.standard_normal((3, 40, 24)).astype(np.float32)
    codes, scales = O.quantize_weights_e4m3(w)
    assert np.allclose(scales, np.abs(w).max(axis=1) / 448, rtol=1e-7, atol=0)
    deq = np.vectorize(O.e4m3_decode)(codes) * scales[:, None, :]
    assert np.all(np.abs(deq - w) <= np.abs(w) * 2.0 ** -4 + scales[:, None, :] * 2.0 ** -9)
    amax_rows = np.abs(w).argmax(axis=1)
    for e in range(3):
        for c in range(24):
            assert codes[e, amax_rows[e, c], c] in (0x7E, 0xFE)


def check_e4m3_forward_exact_case(O):
    """With every x row and weight column exactly representable after its
    scale (column and row maxima of 3.5 = 448 * 2^-7 make the scales powers
    of two), and ffn = 1 (the hidden row's single value codes to +-448), the
    E4M3 layer equals the exact layer up to the bf16 rounding of h."""
    T, d, F, n = 7, 16, 1, 3
    rng = np.random.default_rng(48)
    vals = [-3.5, -1.75, -0.875, 0.875, 1.75, 3.5]
    x = rng.choice([-3.5, -1.75, 0.0, 1.75, 3.5], size=(T, d))
    x[:, 0] = 3.5
    w1 = rng.choice(vals, size=(n, d, F)) / 8
    w3 = rng.choice(vals, size=(n, d, F)) / 8
    w2 = rng.choice(vals, size=(n, F, d)) / 8
    w1[:, 0, :] = w3[:, 0, :] = 3.5 / 8
    w2[:, :, 0] = 3.5 / 8
    idx = np.array([[t % n, (t + 1) % n] for t in range(T)], np.int32)
    gate = np.tile([[0.75, 0.25]], (T, 1))
    q1, s1 = O.quantize_weights_e4m3(w1)
    q3, s3 = O.quantize_weights_e4m3(w3)
    q2, s2 = O.quantize_weights_e4m3(w2)
    assert np.all(s1 == 2.0 ** -10) and np.all(s3 == 2.0 ** -10)
    assert np.all(np.log2(s2) == np.round(np.log2(s2)))   # every |value| is 448 * 2^k
    assert np.array_equal(np.vectorize(O.e4m3_decode)(q1) * s1[:, None, :], w1)
    assert np.array_equal(np.vectorize(O.e4m3_decode)(q2) * s2[:, None, :], w2)
    y8 = O.forward_e4m3(x, idx, gate, q1, s1, q3, s3, q2, s2)
    y = O.forward_with_routing(x, idx, gate, w1, w3, w2)
    assert rel_l2(y8, y) < 2.0 ** -8


def check_e4m3_forward_error_band(O):
    """On random data the E4M3 layer stays within the quantisation error band
    of the exact layer (and is not the exact layer)."""
    T, d, F, n = 12, 64, 96, 4
    x, Wg, w1, w3, w2 = rand_layer(49, T, d, F, n)
    idx, gate, _ = O.router(x, Wg, 2)
    q1, s1 = O.quantize_weights_e4m3(w1)
    q3, s3 = O.quantize_weights_e4m3(w3)
    q2, s2 = O.quantize_weights_e4m3(w2)
    y8 = O.forward_e4m3(x, idx, gate, q1, s1, q3, s3, q2, s2)
    y = O.forward_with_routing(x, idx, gate, w1, w3, w2)
    err = rel_l2(y8, y)
    assert 1e-3 < err < 0.08, err


# --------------------------------------------------------------------------
# 4-bit (E2M1, block-scaled) experts
# --------------------------------------------------------------------------

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def check_e2m1_codec(O):
    """E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit -- magnitudes
    0, 0.5, 1, 1.5, 2, 3, 4, 6; encode rounds to nearest with ties to the even
    mantissa, saturates at 6 and keeps the sign of zero."""
    for c in range(16):
        want = E2M1_VALUES[c & 7] * (-1.0 if c & 8 else 1.0)
        got = O.e2m1_decode(c)
        assert got == want and math.copysign(1.0, got) == (-1.0 if c & 8 else 1.0), c
        assert O.e2m1_encode(got) == c, c
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert O.e2m1_encode(v) == c and O.e2m1_encode(-v) == c | 8, v
    assert O.e2m1_encode(0.26) == 1 and O.e2m1_encode(0.74) == 1 and O.e2m1_encode(5.01) == 7
    assert O.e2m1_encode(6.5) == 7 and O.e2m1_encode(-1e30) == 15 and O.e2m1_encode(1e-30) == 0
    rng = np.random.default_rng(51)
    for v in rng.uniform(-8, 8, 500):
        q = O.e2m1_decode(O.e2m1_encode(v))
        nearest = min(E2M1_VALUES, key=lambda g: abs(abs(v) - g)) if abs(v) <= 6 else 6.0
        assert abs(q) == nearest or abs(abs(q) - abs(v)) == abs(nearest - abs(v))


def _fp4_exact_matrix(rng):
    """One expert matrix [32][6] whose blocks are E2M1 values x a power-of-two
    block scale (one block at 448) x the tensor scale 2^-8, each block
    reaching +-6 x its scale: quantisation must recover it exactly."""
    rows, cols = 32, 6
    st = 2.0 ** -8
    w = np.zeros((rows, cols))
    q_ref = np.zeros((rows, cols), int)
    sb_ref = np.zeros((rows // 16, cols))
    for b in range(rows // 16):
        for c in range(cols):
            sb = 448.0 if (b, c) == (0, 0) else 2.0 ** int(rng.integers(-3, 9))
            q = rng.integers(0, 16, 16)
            q[int(rng.integers(0, 16))] = 7 if rng.random() < 0.5 else 15     # the block maximum, +-6
            for r in range(16):
                w[16 * b + r, c] = E2M1_VALUES[q[r] & 7] * (-1 if q[r] & 8 else 1) * sb * st
            q_ref[16 * b:16 * b + 16, c] = q
            sb_ref[b, c] = sb
    return w, q_ref, sb_ref, st


def check_fp4_exact_case(O):
    """Exactly representable weights come back bit-exact: tensor scale =
    amax / 2688, block scales, codes, nibble order (column 2j low), and the
    dequantised matrix; negative zeros keep their sign code."""
    rng = np.random.default_rng(52)
    w, q_ref, sb_ref, st = _fp4_exact_matrix(rng)
    codes, bscale, tscale = O.quantize_weights_fp4(w[None].astype(np.float32))
    assert tscale[0] == np.float32(st)
    assert np.array_equal(np.vectorize(O.e4m3_decode)(bscale[0]), sb_ref)
    lo, hi = codes[0] & 0xF, codes[0] >> 4
    got = np.empty_like(q_ref)
    got[:, 0::2], got[:, 1::2] = lo, hi
    assert np.array_equal(got, q_ref)
    assert np.array_equal(O.dequantize_fp4(codes, bscale, tscale)[0], w)


def check_fp4_error_band(O):
    """Gaussian weights: every element within its block's E2M1 rounding bound
    (a quarter of the largest grid step, 2 x sb x st, plus the E4M3 rounding
    of sb), the whole matrix within the 4-bit error band, zero blocks exact."""
    rng = np.random.default_rng(53)
    w = rng.standard_normal((3, 64, 40)).astype(np.float32)
    w[1, 16:32, 5] = 0.0
    codes, bscale, tscale = O.quantize_weights_fp4(w)
    d = O.dequantize_fp4(codes, bscale, tscale)
    for e in range(3):
        assert tscale[e] == np.float32(np.abs(w[e]).max() / np.float32(2688.0))
        sb = np.vectorize(O.e4m3_decode)(bscale[e]).repeat(16, axis=0)
        bound = 1.0 * sb * tscale[e] + 1e-30
        assert np.all(np.abs(d[e] - w[e]) <= bound)
    assert np.all(d[1, 16:32, 5] == 0.0)
    err = np.linalg.norm(d - w) / np.linalg.norm(w)
    assert 0.03 < err < 0.15, err


def check_fp4_layer_uses_dequantised_weights(O):
    """The 4-bit layer is the layer of the dequantised weights: with exactly
    representable weights it equals the exact layer."""
    rng = np.random.default_rng(54)
    T, d, F, n, K = 9, 32, 32, 2, 2
    ws = []
    for _ in range(3):
        m = np.stack([_fp4_exact_matrix(rng)[0] for _ in range(n)])      # [n][32][6] each
        ws.append(m)
    # fit the exact matrices to the layer shapes: w1, w3 [n][d][F], w2 [n][F][d]
    w1 = np.concatenate([ws[0]] * 6, axis=2)[:, :, :F][:, :d]
    w3 = np.concatenate([ws[1]] * 6, axis=2)[:, :, :F][:, :d]
    w2 = np.concatenate([ws[2]] * 6, axis=2)[:, :, :d][:, :F]
    x = rng.standard_normal((T, d))
    idx = np.array([[0, 1]] * T, np.int32)
    gate = np.tile([[0.6, 0.4]], (T, 1))
    deq = [O.dequantize_fp4(*O.quantize_weights_fp4(w.astype(np.float32))) for w in (w1, w3, w2)]
    for a, b in zip(deq, (w1, w3, w2)):
        assert np.array_equal(a, b)
    y = O.forward_with_routing(x, idx, gate, *deq)
    y0 = O.forward_with_routing(x, idx, gate, w1, w3, w2)
    assert np.array_equal(y, y0)


def check_fp4_forward_is_layer_of_dequantised(O):
    """The 4-bit layer (weights dequantised where read) equals the layer of the
    dequantised matrices, up to summation order."""
    T, d, F, n = 7, 32, 48, 3
    x, Wg, w1, w3, w2 = rand_layer(55, T, d, F, n)
    idx, gate, _ = O.router(x, Wg, 2)
    q = [O.quantize_weights_fp4(w.astype(np.float32)) for w in (w1, w3, w2)]
    deq = [O.dequantize_fp4(*t) for t in q]
    y4 = O.forward_fp4(x, idx, gate, *q)
    y = O.forward_with_routing(x, idx, gate, *deq)
    assert rel_l2(y4, y) < 1e-12
    assert rel_l2(y, O.forward_with_routing(x, idx, gate, w1, w3, w2)) > 1e-3


def check_fp4_rows_match_the_weight_quantiser(O):
    """Per-row 4-bit quantisation of x equals the 4-bit weight quantiser run on
    each row as a one-column matrix (blocks of 16 along the row, the row's own
    tensor scale): two independent code paths of the same definition."""
    rng = np.random.default_rng(56)
    x = (rng.standard_normal((5, 64)) * rng.choice([1e-3, 1.0, 50.0], size=(5, 1))).astype(np.float32)
    x[2, 16:32] = 0.0
    x[4, :] = 0.0
    codes, bscale, rscale = O.quantize_rows_fp4(x)
    for t in range(5):
        m = np.stack([x[t], np.zeros_like(x[t])], axis=1)[None]          # [1][64][2]
        wc, wb, wt = O.quantize_weights_fp4(m)
        assert rscale[t] == wt[0]
        assert np.array_equal(bscale[t], wb[0, :, 0])
        assert np.array_equal(codes[t] & 0xF, wc[0, 0::2, 0] & 0xF)
        assert np.array_equal(codes[t] >> 4, wc[0, 1::2, 0] & 0xF)


def check_fp4_rows_exact_case(O):
    """A row made of E2M1 values x power-of-two block scales x 2^-8, every
    block reaching 6 x its scale and one block at scale 448, is recovered
    exactly (codes, block scales, row scale)."""
    rng = np.random.default_rng(57)
    w, q_ref, sb_ref, st = _fp4_exact_matrix(rng)        # [32][6]: 2 blocks per column
    x = w.T.astype(np.float32)                            # 6 rows of 32
    codes, bscale, rscale = O.quantize_rows_fp4(x)
    for t in range(6):
        # each row of the exact matrix is a column of it: its tensor scale is that column's
        col_amax = np.abs(w[:, t]).max()
        assert rscale[t] == np.float32(col_amax / np.float32(2688.0))
        got = np.empty(32, int)
        got[0::2], got[1::2] = codes[t] & 0xF, codes[t] >> 4
        if col_amax == 6 * 448 * st:                      # the row holding the 448 block
            assert np.array_equal(got, q_ref[:, t])
            assert np.array_equal(np.vectorize(O.e4m3_decode)(bscale[t]), sb_ref[:, t])


def check_w4a4_layer_band(O):
    """The layer with 4-bit weights and activations stays within the 4-bit
    band of the exact layer and moves further from it than weights-only
    quantisation does (the activations are really quantised)."""
    T, d, F, n = 10, 64, 64, 4
    x, Wg, w1, w3, w2 = rand_layer(58, T, d, F, n)
    idx, gate, _ = O.router(x, Wg, 2)
    q = [O.quantize_weights_fp4(w.astype(np.float32)) for w in (w1, w3, w2)]
    y_exact = O.forward_with_routing(x, idx, gate, w1, w3, w2)
    e_w4 = rel_l2(O.forward_fp4(x, idx, gate, *q), y_exact)
    e_w4a4 = rel_l2(O.forward_w4a4(x, idx, gate, *q), y_exact)
    assert e_w4 < e_w4a4 < 0.35, (e_w4, e_w4a4)


def check_w4a4_zero_rows_and_scaling(O):
    """Zero tokens give exact zeros; scaling a token by a power of two scales
    its output by the same power (every scale is a ratio of the row's own
    maximum, so the codes do not change)."""
    T, d, F, n = 6, 32, 32, 3
    x, Wg, w1, w3, w2 = rand_layer(59, T, d, F, n)
    x[1] = 0.0
    x[3] = 4.0 * x[2]
    idx = np.array([[0, 1], [1, 2], [2, 0], [2, 0], [0, 2], [1, 0]], np.int32)
    gate = np.tile([[0.5, 0.5]], (T, 1))
    q = [O.quantize_weights_fp4(w.astype(np.float32)) for w in (w1, w3, w2)]
    y = O.forward_w4a4(x.astype(np.float32), idx, gate, *q)
    assert np.all(y[1] == 0.0)
    xc, xb, xs = O.quantize_rows_fp4(x.astype(np.float32))
    assert np.array_equal(xc[3], xc[2]) and np.array_equal(xb[3], xb[2]) and xs[3] == 4 * xs[2]


ALL_CHECKS = [
    check_worked_example, check_two_way_softmax_closed_form, check_logits_are_x_times_Wg,
    check_topk_brute_force, check_ties_go_to_lower_index, check_gate_invariants, check_gates_to_bf16, check_silu,
    check_n1_is_plain_swiglu, check_expert_indexing, check_K_equals_n_is_dense_mixture,
    check_top2_layer_against_torch, check_relabel_invariance,
    check_unchosen_experts_do_not_matter, check_forward_with_routing_consistent,
    check_bf16_inputs_widen_exactly, check_dispatch,
    check_router_stats_closed_forms, check_router_stats_against_torch, check_dispatch_capacity,
    check_expert_choice_full_capacity_is_dense, check_expert_choice_ties_and_unchosen_tokens,
    check_expert_choice_selection_brute_force,
    check_e4m3_codec, check_e4m3_weight_quantization, check_e4m3_forward_exact_case,
    check_e4m3_forward_error_band,
    check_e2m1_codec, check_fp4_exact_case, check_fp4_error_band, check_fp4_layer_uses_dequantised_weights,
    check_fp4_forward_is_layer_of_dequantised,
    check_fp4_rows_match_the_weight_quantiser, check_fp4_rows_exact_case, check_w4a4_layer_band,
    check_w4a4_zero_rows_and_scaling,
]
