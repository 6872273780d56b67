"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something the pages print, a closed form,
an invariant, a library routine on a special case, or brute force on tiny
inputs.  None of them re-types the oracle's own formula.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- routing
def test_worked_router_example(golden_dir):
    """The printed router example selects experts 4 and 2 (best first)."""
    g = _golden(golden_dir, "router_worked_example.json")
    sel = oracle.select_topk(np.array(g["scores"]), g["top_k"])[0]
    assert sel.tolist() == g["selected_best_first"]


def test_two_way_gate_is_logistic_of_gap(golden_dir):
    """Closed form: with k = 2 the renormalised softmax is the logistic function of the score gap."""
    g = _golden(golden_dir, "router_worked_example.json")
    s = np.array(g["scores"])
    sel = oracle.select_topk(s, 2)
    w = oracle.gate_weights(s, sel)[0]
    gap = s[4] - s[2]
    assert w[0] == pytest.approx(1.0 / (1.0 + math.exp(-gap)), rel=1e-15)
    assert w[1] == pytest.approx(1.0 / (1.0 + math.exp(gap)), rel=1e-14)


def _lexsort_topk(row, K):
    # numpy's stable lexicographic sort: primary key descending score, secondary ascending index
    order = np.lexsort((np.arange(row.shape[0]), -row))
    return order[:K]


@pytest.mark.parametrize("N,K", [(8, 2), (6, 2), (32, 4), (256, 8), (5, 5), (7, 1)])
def test_topk_matches_library_sort_with_many_ties(N, K):
    """Selection equals a library stable sort (desc score, asc index) on tie-heavy scores."""
    rng = np.random.default_rng(N * 100 + K)
    scores = rng.integers(-3, 4, size=(200, N)).astype(np.float64)  # lots of exact ties
    scores[:5] = 0.0  # all-equal rows: selection must be 0..K-1
    sel = oracle.select_topk(scores, K)
    for t in range(scores.shape[0]):
        assert sel[t].tolist() == _lexsort_topk(scores[t], K).tolist()
    for t in range(5):
        assert sel[t].tolist() == list(range(K))


def test_topk_brute_force_over_subsets():
    """Brute force: the selected set is the K-subset with the largest score sum; among equal sums,
    the lexicographically smallest index tuple (integer scores, so sums are exact)."""
    rng = np.random.default_rng(7)
    for N, K in [(6, 2), (6, 3), (5, 1), (7, 4)]:
        for _ in range(60):
            s = rng.integers(-2, 3, size=N).astype(np.float64)
            best = None
            for sub in itertools.combinations(range(N), K):  # lexicographic order
                tot = sum(s[list(sub)])
                if best is None or tot > best[0]:
                    best = (tot, sub)
            sel = oracle.select_topk(s, K)[0]
            assert sorted(sel.tolist()) == list(best[1])
            # best-first order within the set: non-increasing scores, ties by index
            vals = s[sel]
            assert all(vals[i] >= vals[i + 1] for i in range(K - 1))


def test_tie_break_duplicate_router_columns():
    """Duplicate W_g columns give bit-equal scores; the lower expert index wins."""
    rng = np.random.default_rng(3)
    D, N = 16, 8
    Wg = rng.standard_normal((D, N)).astype(np.float32)
    Wg[:, 5] = Wg[:, 2]
    Wg[:, 6] = Wg[:, 2]
    x = rng.standard_normal((50, D)).astype(np.float32)
    s = oracle.router_scores(x.astype(np.float64), Wg, oracle.F32)
    sel = oracle.select_topk(s, 3)
    for t in range(50):
        picked = [e for e in sel[t].tolist() if e in (2, 5, 6)]
        assert picked == sorted(picked)
        if 5 in picked:
            assert 2 in picked
        if 6 in picked:
            assert 5 in picked and 2 in picked
    # signed zeros compare equal: a tie, lower index first
    assert oracle.select_topk(np.array([-0.0, 0.0, -1.0]), 1)[0].tolist() == [0]


def test_router_scores_match_library_matmul():
    """Router scores equal a library fp64 matmul (+ bias) on random inputs."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((20, 33)).astype(np.float32)
    Wg = rng.standard_normal((33, 7)).astype(np.float32)
    bg = rng.standard_normal(7).astype(np.float32)
    s = oracle.router_scores(x.astype(np.float64), Wg, oracle.F32, bg)
    ref = x.astype(np.float64) @ Wg.astype(np.float64) + bg.astype(np.float64)
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)


def test_bf16_widening_is_exact():
    """bf16 bit patterns widen to the same doubles torch produces."""
    t = torch.randn(40, dtype=torch.float32).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).reshape(1, -1)
    got = oracle.load_rows(bits, oracle.BF16, [0])[0]
    np.testing.assert_array_equal(got, t.to(torch.float64).numpy())


# --------------------------------------------------------------------------- gate weights
def test_gate_weights_sum_to_one_and_order():
    rng = np.random.default_rng(5)
    for N, K in [(8, 2), (32, 4), (256, 8), (6, 6)]:
        s = rng.standard_normal((100, N)) * 3
        sel = oracle.select_topk(s, K)
        w = oracle.gate_weights(s, sel)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
        assert np.all(w > 0)
        assert np.all(np.diff(w, axis=1) <= 1e-17)  # best slot carries the largest weight


def test_gate_weights_equal_masked_full_softmax():
    """softmax(KeepTopK(H, k)) with -inf masking (library softmax) equals the oracle's weights."""
    rng = np.random.default_rng(9)
    N, K = 16, 4
    s = rng.standard_normal((64, N)) * 2
    sel = oracle.select_topk(s, K)
    w = oracle.gate_weights(s, sel)
    masked = torch.full((64, N), -math.inf, dtype=torch.float64)
    st = torch.from_numpy(s)
    for t in range(64):
        masked[t, sel[t]] = st[t, sel[t]]
    G = torch.softmax(masked, dim=1).numpy()
    for t in range(64):
        np.testing.assert_allclose(w[t], G[t, sel[t]], rtol=1e-14)
        off = np.setdiff1d(np.arange(N), sel[t])
        assert np.all(G[t, off] == 0.0)


# --------------------------------------------------------------------------- activations
def test_activation_closed_forms():
    assert oracle.gelu(0.0) == 0.0
    assert oracle.silu(0.0) == 0.0
    assert oracle.gelu(1.0) == pytest.approx(0.8413447460685429, rel=1e-15)  # Phi(1)
    for v in [0.3, 1.7, 4.0, 9.0]:
        assert oracle.gelu(v) - oracle.gelu(-v) == pytest.approx(v, rel=1e-14)
        assert oracle.silu(v) - oracle.silu(-v) == pytest.approx(v, rel=1e-14)
    assert oracle.silu(2.0) == pytest.approx(2.0 / (1.0 + math.exp(-2.0)), rel=1e-15)


# --------------------------------------------------------------------------- experts / layer
def _rand_layer(rng, T, D, H, N, act, bias):
    x = rng.standard_normal((T, D)).astype(np.float32)
    Wg = (rng.standard_normal((D, N)) * 0.5).astype(np.float32)
    rows = H if act == oracle.ACT_GELU else 2 * H
    W1 = (rng.standard_normal((N, rows, D)) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((N, D, H)) * 0.2).astype(np.float32)
    b1 = (rng.standard_normal((N, H)) * 0.1).astype(np.float32) if bias else None
    b2 = (rng.standard_normal((N, D)) * 0.1).astype(np.float32) if bias else None
    return x, Wg, W1, W2, b1, b2


def _torch_expert(x64, act, W1e, W2e, b1e, b2e, H):
    W1t = torch.from_numpy(W1e.astype(np.float64))
    W2t = torch.from_numpy(W2e.astype(np.float64))
    if act == oracle.ACT_GELU:
        b1t = None if b1e is None else torch.from_numpy(b1e.astype(np.float64))
        b2t = None if b2e is None else torch.from_numpy(b2e.astype(np.float64))
        h = F.gelu(F.linear(x64, W1t, b1t), approximate="none")
        return F.linear(h, W2t, b2t)
    gu = F.linear(x64, W1t)
    return F.linear(F.silu(gu[:, :H]) * gu[:, H:], W2t)


@pytest.mark.parametrize("act,bias", [(oracle.ACT_GELU, True), (oracle.ACT_GELU, False), (oracle.ACT_SWIGLU, False)])
def test_one_expert_top1_is_dense_ffn(act, bias):
    """A 1-expert top-1 layer equals the dense FFN (library fp64 linear + activation)."""
    rng = np.random.default_rng(21 + act)
    T, D, H = 24, 16, 40
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, 1, act, bias)
    out = oracle.moe_layer(x, Wg, W1, W2, K=1, act=act, dtype_tag=oracle.F32, b1=b1, b2=b2, threads=2)
    assert np.all(out["w"] == 1.0)
    assert np.all(out["sel"] == 0)
    ref = _torch_expert(torch.from_numpy(x.astype(np.float64)), act, W1[0], W2[0],
                        None if b1 is None else b1[0], None if b2 is None else b2[0], H).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("act,N,K", [(oracle.ACT_GELU, 6, 2), (oracle.ACT_SWIGLU, 8, 3), (oracle.ACT_GELU, 4, 4)])
def test_sparse_layer_equals_dense_masked_gate(act, N, K):
    """Brute force: evaluate every expert, weight by the dense masked gate softmax(KeepTopK(H, k)),
    sum over all experts; equals the sparse oracle within 1e-12 relative."""
    rng = np.random.default_rng(31 + N + K)
    T, D, H = 40, 12, 20
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, act, act == oracle.ACT_GELU)
    bg = (rng.standard_normal(N) * 0.3).astype(np.float32)
    out = oracle.moe_layer(x, Wg, W1, W2, K=K, act=act, dtype_tag=oracle.F32, bg=bg, b1=b1, b2=b2, threads=3)
    x64 = torch.from_numpy(x.astype(np.float64))
    logits = x64 @ torch.from_numpy(Wg.astype(np.float64)) + torch.from_numpy(bg.astype(np.float64))
    np.testing.assert_allclose(out["scores"], logits.numpy(), rtol=1e-13, atol=1e-13)
    # KeepTopK by a library sort (torch.sort is stable when asked), then the masked softmax
    order = torch.sort(-logits, dim=1, stable=True).indices[:, :K]
    masked = torch.full_like(logits, -math.inf)
    masked.scatter_(1, order, logits.gather(1, order))
    G = torch.softmax(masked, dim=1)
    y = torch.zeros(T, D, dtype=torch.float64)
    for e in range(N):
        Ee = _torch_expert(x64, act, W1[e], W2[e], None if b1 is None else b1[e], None if b2 is None else b2[e], H)
        y += G[:, e:e + 1] * Ee
    np.testing.assert_allclose(out["y"], y.numpy(), rtol=1e-12, atol=1e-13)
    assert out["sel"].tolist() == order.numpy().tolist()


def test_selection_on_given_scores_keeps_fp64_weights():
    """With sel_scores the selection follows the given scores while weights use the fp64 scores."""
    rng = np.random.default_rng(41)
    T, D, H, N, K = 10, 8, 16, 6, 2
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_GELU, False)
    ref = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_GELU, dtype_tag=oracle.F32, threads=1)
    forced = np.zeros((T, N), dtype=np.float32)
    forced[:, 5] = 2.0
    forced[:, 3] = 1.0
    out = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_GELU, dtype_tag=oracle.F32, sel_scores=forced,
                           threads=1)
    assert np.all(out["sel"] == np.array([5, 3]))
    np.testing.assert_array_equal(out["scores"], ref["scores"])
    s = ref["scores"]
    np.testing.assert_allclose(out["w"][:, 0], 1 / (1 + np.exp(s[:, 3] - s[:, 5])), rtol=1e-14)


def test_layer_rows_threads_are_independent():
    rng = np.random.default_rng(43)
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, 37, 8, 16, 5, oracle.ACT_SWIGLU, False)
    a = oracle.moe_layer(x, Wg, W1, W2, K=2, act=oracle.ACT_SWIGLU, dtype_tag=oracle.F32, threads=1)
    b = oracle.moe_layer(x, Wg, W1, W2, K=2, act=oracle.ACT_SWIGLU, dtype_tag=oracle.F32, threads=5)
    for k in ("scores", "sel", "w", "y"):
        np.testing.assert_array_equal(a[k], b[k])


# --------------------------------------------------------------------------- shared expert, selection bias
@pytest.mark.parametrize("act,bias", [(oracle.ACT_GELU, True), (oracle.ACT_SWIGLU, False)])
def test_one_expert_with_shared_expert_is_two_dense_ffns(act, bias):
    """A 1-expert top-1 layer with a shared expert equals the sum of two dense FFNs
    (library fp64 linear + activation)."""
    rng = np.random.default_rng(51 + act)
    T, D, H = 20, 16, 24
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, 1, act, bias)
    _, _, S1, S2, sb1, sb2 = _rand_layer(rng, 1, D, H, 1, act, bias)
    out = oracle.moe_layer(x, Wg, W1, W2, K=1, act=act, dtype_tag=oracle.F32, b1=b1, b2=b2, threads=2,
                           S1=S1[0], S2=S2[0], sb1=None if sb1 is None else sb1[0],
                           sb2=None if sb2 is None else sb2[0])
    x64 = torch.from_numpy(x.astype(np.float64))
    ref = _torch_expert(x64, act, W1[0], W2[0], None if b1 is None else b1[0], None if b2 is None else b2[0], H)
    ref = ref + _torch_expert(x64, act, S1[0], S2[0], None if sb1 is None else sb1[0],
                              None if sb2 is None else sb2[0], H)
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_shared_expert_alone_when_routed_experts_are_zero():
    """Routed experts with all-zero weights contribute nothing: y is the shared FFN alone."""
    rng = np.random.default_rng(57)
    T, D, H, N = 12, 8, 16, 4
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_SWIGLU, False)
    _, _, S1, S2, _, _ = _rand_layer(rng, 1, D, H, 1, oracle.ACT_SWIGLU, False)
    out = oracle.moe_layer(x, Wg, np.zeros_like(W1), np.zeros_like(W2), K=2, act=oracle.ACT_SWIGLU,
                           dtype_tag=oracle.F32, S1=S1[0], S2=S2[0], threads=1)
    ref = _torch_expert(torch.from_numpy(x.astype(np.float64)), oracle.ACT_SWIGLU, S1[0], S2[0], None, None, H)
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_zero_selection_bias_is_the_plain_layer():
    rng = np.random.default_rng(61)
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, 30, 8, 16, 6, oracle.ACT_GELU, True)
    a = oracle.moe_layer(x, Wg, W1, W2, K=2, act=oracle.ACT_GELU, dtype_tag=oracle.F32, b1=b1, b2=b2, threads=1)
    b = oracle.moe_layer(x, Wg, W1, W2, K=2, act=oracle.ACT_GELU, dtype_tag=oracle.F32, b1=b1, b2=b2, threads=1,
                         bsel=np.zeros(6, np.float32))
    for k in ("scores", "sel", "w", "y"):
        np.testing.assert_array_equal(a[k], b[k])


def test_selection_bias_changes_the_kept_set_not_the_weights():
    """A selection bias picks the kept set by s + b; the weights are the masked softmax of the raw
    scores over that set (library masked softmax), and the scores themselves are unchanged."""
    rng = np.random.default_rng(63)
    T, D, H, N, K = 40, 8, 16, 6, 3
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_SWIGLU, False)
    bsel = np.array([0.0, 3.0, -1.0, 0.5, 9.0, -9.0], np.float32)
    out = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_SWIGLU, dtype_tag=oracle.F32, bsel=bsel, threads=2)
    logits = torch.from_numpy(x.astype(np.float64)) @ torch.from_numpy(Wg.astype(np.float64))
    np.testing.assert_allclose(out["scores"], logits.numpy(), rtol=1e-13, atol=1e-13)
    biased = logits + torch.from_numpy(bsel.astype(np.float64))
    order = torch.sort(-biased, dim=1, stable=True).indices[:, :K]
    assert out["sel"].tolist() == order.numpy().tolist()
    assert np.all(out["sel"][:, 0] == 4)             # the +9 bias always wins the first slot
    assert not np.any(out["sel"] == 5)               # the -9 bias never gets in
    masked = torch.full_like(logits, -math.inf)
    masked.scatter_(1, order, logits.gather(1, order))   # raw scores on the kept set
    G = torch.softmax(masked, dim=1)
    np.testing.assert_allclose(out["w"], G.gather(1, order).numpy(), rtol=1e-13, atol=1e-15)
    # the weight of the forced expert follows its raw score, not its bias
    assert np.any(out["w"][:, 0] < 0.5)


# --------------------------------------------------------------------------- capacity (drop)
def test_capacity_closed_forms():
    """C = ceil(cf T K / N): the expected assignments per expert times the capacity factor."""
    assert oracle.capacity(1.25, 16384, 8, 256) == 640        # 512 per expert x 1.25
    assert oracle.capacity(1.0, 8192, 2, 6) == 2731          # 2730.67 rounded up
    assert oracle.capacity(2.0, 10, 2, 8) == 5
    assert oracle.capacity(0.5, 7, 1, 7) == 1                # 0.5 rounded up
    assert oracle.capacity(0.0, 100, 2, 4) >= 2 ** 62        # no limit


def test_capacity_keeps_the_first_C_of_each_expert_in_row_order():
    """Brute force with a library routine: for each expert, the first C of its assignments in
    row-major (row, slot) order are kept (numpy flatnonzero), the others dropped."""
    rng = np.random.default_rng(71)
    T, N, K = 300, 8, 3
    sel = np.stack([rng.permutation(N)[:K] for _ in range(T)]).astype(np.int32)
    sel[:40, 0] = 2                                            # a burst on expert 2
    for C in (1, 7, 50, 113, 1000):
        keep = oracle.capacity_keep(sel, N, C)
        ref = np.zeros(T * K, dtype=np.uint8)
        flat = sel.ravel()
        for e in range(N):
            ref[np.flatnonzero(flat == e)[:C]] = 1
        np.testing.assert_array_equal(keep.ravel(), ref)
        counts = np.bincount(flat, minlength=N)
        np.testing.assert_array_equal(np.bincount(flat, weights=keep.ravel(), minlength=N), np.minimum(counts, C))


def test_capacity_layer_is_the_masked_dense_gate():
    """Brute force: every expert evaluated, weighted by the dense gate softmax(KeepTopK) times the
    keep mask of the capacity decision, summed; equals the capacity layer (library routines)."""
    rng = np.random.default_rng(73)
    T, D, H, N, K = 60, 10, 16, 5, 2
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_SWIGLU, False)
    bg = np.array([1.5, 0.5, 0.0, -0.5, -1.0], np.float32)   # skewed: expert 0 overflows
    out = oracle.moe_layer_capacity(x, Wg, W1, W2, K=K, act=oracle.ACT_SWIGLU, dtype_tag=oracle.F32, cf=0.8,
                                    bg=bg, threads=2)
    C = out["capacity"]
    assert C == math.ceil(0.8 * T * K / N)
    x64 = torch.from_numpy(x.astype(np.float64))
    logits = x64 @ torch.from_numpy(Wg.astype(np.float64)) + torch.from_numpy(bg.astype(np.float64))
    order = torch.sort(-logits, dim=1, stable=True).indices[:, :K]
    masked = torch.full_like(logits, -math.inf)
    masked.scatter_(1, order, logits.gather(1, order))
    G = torch.softmax(masked, dim=1)
    keep = np.zeros((T, N))
    flat = order.numpy().ravel()
    for e in range(N):
        idx = np.flatnonzero(flat == e)[:C]
        keep[idx // K, e] = 1.0
    assert keep.sum() < T * K                                  # something was dropped
    y = torch.zeros(T, D, dtype=torch.float64)
    for e in range(N):
        Ee = _torch_expert(x64, oracle.ACT_SWIGLU, W1[e], W2[e], None, None, H)
        y += (G[:, e:e + 1] * torch.from_numpy(keep[:, e:e + 1])) * Ee
    np.testing.assert_allclose(out["y"], y.numpy(), rtol=1e-12, atol=1e-13)
    # the kept gate weights are the unrenormalised ones of the plain layer
    plain = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_SWIGLU, dtype_tag=oracle.F32, bg=bg, threads=2)
    np.testing.assert_array_equal(out["w"], plain["w"])


def test_large_capacity_is_the_plain_layer():
    rng = np.random.default_rng(79)
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, 40, 8, 16, 4, oracle.ACT_GELU, True)
    a = oracle.moe_layer(x, Wg, W1, W2, K=2, act=oracle.ACT_GELU, dtype_tag=oracle.F32, b1=b1, b2=b2, threads=1)
    b = oracle.moe_layer_capacity(x, Wg, W1, W2, K=2, act=oracle.ACT_GELU, dtype_tag=oracle.F32, cf=4.0, b1=b1,
                                  b2=b2, threads=1)
    assert b["keep"].all()
    np.testing.assert_array_equal(a["y"], b["y"])


# --------------------------------------------------------------------------- reroute
def test_reroute_worked_examples():
    """Hand-worked cases of the next-candidate reroute (rows served in order, a refused slot
    goes to the best-ranked expert the row does not hold yet that still has room)."""
    # three rows prefer expert 0, then 1, then 2; one place each: 0, then 1, then 2
    v = np.array([[3.0, 2.0, 1.0]] * 4)
    sel = np.zeros((4, 1), np.int32)
    assert oracle.capacity_reroute(v, sel, 1)[:, 0].tolist() == [0, 1, 2, -1]
    assert oracle.capacity_reroute(v, sel, 2)[:, 0].tolist() == [0, 0, 1, 1]
    # two slots per row: row 1 loses both first choices; its first refused slot takes the
    # better of the two free experts (2), the second slot the next one (3)
    v = np.array([[4.0, 3.0, 2.0, 1.0]] * 2)
    sel = np.array([[0, 1], [0, 1]], np.int32)
    assert oracle.capacity_reroute(v, sel, 1).tolist() == [[0, 1], [2, 3]]
    # equal values: the lower index first, as in the selection
    v = np.ones((2, 4))
    assert oracle.capacity_reroute(v, sel, 1).tolist() == [[0, 1], [2, 3]]
    # an earlier row's reroute takes the place a later row selected first
    v = np.array([[3.0, 2.0, 1.0], [3.0, 2.0, 1.0], [1.0, 3.0, 2.0]])
    sel = np.array([[0], [0], [1]], np.int32)
    assert oracle.capacity_reroute(v, sel, 1)[:, 0].tolist() == [0, 1, 2]
    assert oracle.capacity_keep(sel, 3, 1)[:, 0].tolist() == [1, 0, 1]        # the drop, for contrast
    # a row never takes an expert twice: row 1 keeps expert 1 in slot 1, so its refused slot 0
    # cannot go to expert 1 although it has room; expert 2 is full, so slot 0 is dropped
    v = np.array([[3.0, 2.0, 1.0], [3.0, 2.0, 1.0]])
    sel = np.array([[0, 1], [0, 1]], np.int32)
    assert oracle.capacity_reroute(v, sel, np.int64(2)).tolist() == [[0, 1], [0, 1]]
    sel1 = np.array([[0, 2], [0, 1]], np.int32)
    assert oracle.capacity_reroute(v, sel1, 1).tolist() == [[0, 2], [-1, 1]]


def _deferred_acceptance(v, K, C):
    """Expert sets from deferred acceptance: every row proposes down its own ranking
    (larger value first, ties to the lower index) until it holds K experts or has asked
    them all; each expert keeps the C lowest-numbered rows proposing to it.  With one
    priority order shared by all experts this reaches the serial-dictatorship outcome,
    i.e. rows served in order each taking the K best experts still free."""
    T, N = v.shape
    pref = [sorted(range(N), key=lambda e: (-v[t, e], e)) for t in range(T)]
    nxt = [0] * T
    held = [set() for _ in range(T)]
    accepted = [set() for _ in range(N)]
    changed = True
    while changed:
        changed = False
        for t in range(T):
            while len(held[t]) < K and nxt[t] < N:
                e = pref[t][nxt[t]]
                nxt[t] += 1
                accepted[e].add(t)
                held[t].add(e)
                changed = True
                if len(accepted[e]) > C:
                    worst = max(accepted[e])
                    accepted[e].discard(worst)
                    held[worst].discard(e)
    return held


def test_reroute_equals_deferred_acceptance():
    """Against another algorithm: each row's set of serving experts equals the outcome of
    deferred acceptance with the row order as the experts' common priority; slots whose
    selected expert had room keep it, and refused slots take the new experts in rank order."""
    rng = np.random.default_rng(89)
    cases = 0
    for _ in range(200):
        T, N = int(rng.integers(1, 14)), int(rng.integers(2, 7))
        K, C = int(rng.integers(1, min(3, N) + 1)), int(rng.integers(1, 4))
        v = rng.integers(0, 4, size=(T, N)).astype(np.float64)       # many ties
        sel = oracle.select_topk(v, K)
        assign = oracle.capacity_reroute(v, sel, C)
        sets = _deferred_acceptance(v, K, C)
        for t in range(T):
            got = [e for e in assign[t].tolist() if e >= 0]
            assert len(set(got)) == len(got)
            assert set(got) == sets[t], (t, v, sel, assign)
            kept = [int(e) for e, a in zip(sel[t], assign[t]) if a == e]
            new = [int(a) for e, a in zip(sel[t], assign[t]) if a != e and a >= 0]
            order = sorted(range(N), key=lambda e: (-v[t, e], e))
            assert new == [e for e in order if e in set(new)]           # rank order across slots
            assert -1 not in assign[t] or len(got) == len(kept) + len(new)
        loads = np.bincount(assign[assign >= 0], minlength=N)
        assert (loads <= C).all()
        cases += int((assign != sel).any())
    assert cases > 50


def test_reroute_layer_against_single_expert_layers():
    """Two rows that both select expert 0 of two, one place each: the second row is served
    by expert 1 with its gate weight (1 at K = 1), i.e. exactly the one-expert layer of
    expert 1; the first row is the one-expert layer of expert 0.  With room for all the
    reroute layer is the plain layer."""
    rng = np.random.default_rng(97)
    T, D, H, N = 2, 6, 8, 2
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_GELU, True)
    bg = np.array([50.0, 0.0], np.float32)                       # both rows select expert 0
    out = oracle.moe_layer_capacity(x, Wg, W1, W2, K=1, act=oracle.ACT_GELU, dtype_tag=oracle.F32, cf=0.5,
                                    overflow="reroute", bg=bg, b1=b1, b2=b2, threads=1)
    assert out["capacity"] == 1 and out["assign"][:, 0].tolist() == [0, 1]
    for t, e in ((0, 0), (1, 1)):
        one = oracle.moe_layer(x[t:t + 1], Wg[:, e:e + 1], W1[e:e + 1], W2[e:e + 1], K=1, act=oracle.ACT_GELU,
                               dtype_tag=oracle.F32, b1=b1[e:e + 1], b2=b2[e:e + 1], threads=1)
        np.testing.assert_allclose(out["y"][t], one["y"][0], rtol=1e-14, atol=1e-15)
    drop = oracle.moe_layer_capacity(x, Wg, W1, W2, K=1, act=oracle.ACT_GELU, dtype_tag=oracle.F32, cf=0.5,
                                     bg=bg, b1=b1, b2=b2, threads=1)
    assert (drop["y"][1] == 0).all()
    plain = oracle.moe_layer(x, Wg, W1, W2, K=1, act=oracle.ACT_GELU, dtype_tag=oracle.F32, bg=bg, b1=b1, b2=b2,
                             threads=1)
    big = oracle.moe_layer_capacity(x, Wg, W1, W2, K=1, act=oracle.ACT_GELU, dtype_tag=oracle.F32, cf=4.0,
                                    overflow="reroute", bg=bg, b1=b1, b2=b2, threads=1)
    np.testing.assert_array_equal(big["y"], plain["y"])
    np.testing.assert_array_equal(big["assign"], plain["sel"])


# --------------------------------------------------------------------------- backward
def _objective(x, Wg, W1, W2, bg, b1, b2, bsel, dy, K, act, a_s, a_i):
    """sum(y * dy) + a_s * switch + a_i * cv2_importance, from the pinned forward and statistics."""
    out = oracle.moe_layer(x, Wg, W1, W2, K=K, act=act, dtype_tag=oracle.F32, bg=bg, b1=b1, b2=b2, bsel=bsel,
                           threads=1)
    st = oracle.aux_stats(out["scores"], out["sel"], out["w"], Wg.shape[1])
    return float((out["y"] * dy).sum() + a_s * st["switch"] + a_i * st["cv2_importance"]), out["sel"]


@pytest.mark.parametrize("act", [oracle.ACT_GELU, oracle.ACT_SWIGLU])
def test_backward_matches_central_differences(act):
    """Every gradient of the backward against central differences of the pinned forward (and
    statistics) on a tiny layer with router and selection biases and both trainable auxiliary
    losses.  The step is the difference of the two fp32-rounded perturbed values, so rounding of
    the stored parameter does not enter; entries whose perturbation changes the kept set are
    skipped."""
    rng = np.random.default_rng(91 + act)
    T, D, H, N, K = 7, 6, 5, 4, 2
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, act, act == oracle.ACT_GELU)
    bg = (rng.standard_normal(N) * 0.3).astype(np.float32)
    bsel = (rng.standard_normal(N) * 0.2).astype(np.float32)
    dy = rng.standard_normal((T, D))
    a_s, a_i = 0.7, 1.3
    g = oracle.moe_layer_backward(x, Wg, W1, W2, dy, K=K, act=act, dtype_tag=oracle.F32, bg=bg, b1=b1, b2=b2,
                                  bsel=bsel, alpha_switch=a_s, alpha_importance=a_i)
    params = dict(x=x, Wg=Wg, bg=bg, W1=W1, W2=W2)
    if act == oracle.ACT_GELU:
        params.update(b1=b1, b2=b2)
    names = dict(x="dx", Wg="dWg", bg="dbg", W1="dW1", W2="dW2", b1="db1", b2="db2")
    _, sel0 = _objective(x, Wg, W1, W2, bg, b1, b2, bsel, dy, K, act, a_s, a_i)
    checked = 0
    for name, arr in params.items():
        for flat in rng.choice(arr.size, size=min(8, arr.size), replace=False):
            idx = np.unravel_index(flat, arr.shape)
            base = arr[idx]
            vals = {}
            for sgn in (1, -1):
                arr[idx] = np.float32(base + sgn * 1e-3)
                kw = dict(params)
                Jv, sel = _objective(kw["x"], kw["Wg"], kw["W1"], kw["W2"], kw["bg"], kw.get("b1", b1),
                                     kw.get("b2", b2), bsel, dy, K, act, a_s, a_i)
                vals[sgn] = (Jv, float(arr[idx]), np.array_equal(sel, sel0))
            arr[idx] = base
            if not (vals[1][2] and vals[-1][2]):
                continue
            fd = (vals[1][0] - vals[-1][0]) / (vals[1][1] - vals[-1][1])
            an = g[names[name]][idx]
            assert an == pytest.approx(fd, rel=2e-5, abs=2e-7), (name, idx)
            checked += 1
    assert checked >= 30


@pytest.mark.parametrize("act,bias", [(oracle.ACT_GELU, True), (oracle.ACT_SWIGLU, False)])
def test_backward_one_expert_top1_is_dense_ffn_autograd(act, bias):
    """A 1-expert top-1 layer's backward is the dense FFN's (library autograd in fp64); the router
    gets no gradient (its only gate weight is the constant 1)."""
    rng = np.random.default_rng(95 + act)
    T, D, H = 9, 8, 12
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, 1, act, bias)
    dy = rng.standard_normal((T, D))
    g = oracle.moe_layer_backward(x, Wg, W1, W2, dy, K=1, act=act, dtype_tag=oracle.F32, b1=b1, b2=b2)
    xt = torch.from_numpy(x.astype(np.float64)).requires_grad_()
    W1t = torch.from_numpy(W1[0].astype(np.float64)).requires_grad_()
    W2t = torch.from_numpy(W2[0].astype(np.float64)).requires_grad_()
    b1t = torch.from_numpy(b1[0].astype(np.float64)).requires_grad_() if bias else None
    b2t = torch.from_numpy(b2[0].astype(np.float64)).requires_grad_() if bias else None
    if act == oracle.ACT_GELU:
        y = F.linear(F.gelu(F.linear(xt, W1t, b1t), approximate="none"), W2t, b2t)
    else:
        gu = F.linear(xt, W1t)
        y = F.linear(F.silu(gu[:, :H]) * gu[:, H:], W2t)
    (y * torch.from_numpy(dy)).sum().backward()
    np.testing.assert_allclose(g["dx"], xt.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["dW1"][0], W1t.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["dW2"][0], W2t.grad.numpy(), rtol=1e-12, atol=1e-13)
    if bias:
        np.testing.assert_allclose(g["db1"][0], b1t.grad.numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(g["db2"][0], b2t.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.all(g["dWg"] == 0) and np.all(g["dbg"] == 0)


def test_activation_derivatives_closed_forms():
    """GELU'(0) = 1/2, GELU'(v) + GELU'(-v) = 1 (odd part of GELU is v/2); SiLU'(0) = 1/2."""
    assert oracle.lib().orc_gelu_grad(0.0) == pytest.approx(0.5, rel=1e-15)
    assert oracle.lib().orc_silu_grad(0.0) == pytest.approx(0.5, rel=1e-15)
    for v in (0.3, 1.1, 2.7):
        assert oracle.lib().orc_gelu_grad(v) + oracle.lib().orc_gelu_grad(-v) == pytest.approx(1.0, rel=1e-14)
        assert oracle.lib().orc_silu_grad(v) + oracle.lib().orc_silu_grad(-v) == pytest.approx(1.0, rel=1e-14)


# --------------------------------------------------------------------------- statistics
def test_balance_loss_extremes(golden_dir):
    g = _golden(golden_dir, "balance_loss_extremes.json")
    N = 8
    assert oracle.simple_balance_loss(np.full(N, 5.0)) == pytest.approx(g["uniform_value"], rel=1e-15)
    onehot = np.zeros(N)
    onehot[3] = 10
    assert oracle.simple_balance_loss(onehot) == pytest.approx(N, rel=1e-15)  # top-1, all on one
    two = np.zeros(N)
    two[[0, 1]] = 10
    # top-2 with distinct experts per token cannot put everything on one expert: the maximum is N/K
    assert oracle.simple_balance_loss(two) == pytest.approx(N / 2, rel=1e-15)
    assert oracle.simple_balance_loss(np.zeros(N)) == 0.0


def test_cv_squared_closed_forms():
    N = 8
    assert oracle.cv_squared(np.full(N, 3.0)) == 0.0
    onehot = np.zeros(N)
    onehot[0] = 7.0
    assert oracle.cv_squared(onehot) == pytest.approx(N - 1, rel=1e-14)
    assert oracle.cv_squared(np.array([1.0, 2.0, 3.0, 4.0])) == pytest.approx(1.25 / 6.25, rel=1e-15)
    assert oracle.cv_squared(np.zeros(N)) == 0.0


def test_aux_stats_invariants_and_library_checks():
    rng = np.random.default_rng(51)
    T, N, K = 300, 16, 4
    s = rng.standard_normal((T, N)) * 2
    sel = oracle.select_topk(s, K)
    w = oracle.gate_weights(s, sel)
    st = oracle.aux_stats(s, sel, w, N)
    np.testing.assert_array_equal(st["counts"], np.bincount(sel.ravel(), minlength=N).astype(np.float64))
    assert st["importance"].sum() == pytest.approx(T, rel=1e-13)
    assert st["p_mean"].sum() == pytest.approx(1.0, rel=1e-13)
    np.testing.assert_allclose(st["p_mean"], torch.softmax(torch.from_numpy(s), 1).mean(0).numpy(), rtol=1e-13)
    f = st["counts"] / (T * K)
    assert st["switch"] == pytest.approx(N * float(np.dot(f, st["p_mean"])), rel=1e-13)
    assert st["simple"] == pytest.approx(N * float(np.sum(f * f)), rel=1e-13)
    assert st["cv2_importance"] == pytest.approx(float(np.var(st["importance"]) / np.mean(st["importance"]) ** 2),
                                                 rel=1e-12)
    assert st["cv2_load"] == pytest.approx(float(np.var(st["counts"]) / np.mean(st["counts"]) ** 2), rel=1e-12)


def test_aux_stats_uniform_and_empty():
    N, K = 8, 2
    T = 4 * N
    s = np.zeros((T, N))  # all-equal scores: P = 1/N exactly
    sel = np.array([[(2 * t) % N, (2 * t + 1) % N] for t in range(T)], dtype=np.int32)  # uniform load
    w = np.full((T, K), 0.5)
    st = oracle.aux_stats(s, sel, w, N)
    assert st["switch"] == pytest.approx(1.0, rel=1e-15)
    assert st["simple"] == pytest.approx(1.0, rel=1e-15)
    assert st["cv2_importance"] == 0.0 and st["cv2_load"] == 0.0
    empty = oracle.aux_stats(np.zeros((0, N)), np.zeros((0, K), np.int32), np.zeros((0, K)), N)
    assert empty["switch"] == 0.0 and empty["simple"] == 0.0
    assert np.all(empty["counts"] == 0)


def test_demo_scenario_balanced_vs_biased():
    """The chapter's demo: 10 tokens, 8 experts, top-2; a router biased towards a few experts
    concentrates the load and raises N * sum f^2."""
    rng = np.random.default_rng(61)
    T, D, H, N, K = 10, 16, 32, 8, 2
    x, Wg, W1, W2, b1, b2 = _rand_layer(rng, T, D, H, N, oracle.ACT_GELU, False)
    Wg = (rng.standard_normal((D, N)) * 0.02).astype(np.float32)
    bal = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_GELU, dtype_tag=oracle.F32, threads=1)
    bias = np.zeros(N, dtype=np.float32)
    bias[[1, 6]] = 5.0
    biased = oracle.moe_layer(x, Wg, W1, W2, K=K, act=oracle.ACT_GELU, dtype_tag=oracle.F32, bg=bias, threads=1)
    sb = oracle.aux_stats(bal["scores"], bal["sel"], bal["w"], N)
    sz = oracle.aux_stats(biased["scores"], biased["sel"], biased["w"], N)
    assert sb["counts"].sum() == T * K and sz["counts"].sum() == T * K
    assert sorted(np.nonzero(sz["counts"])[0].tolist()) == [1, 6]
    assert sz["simple"] == pytest.approx(N / K)
    assert sz["simple"] > sb["simple"] >= 1.0


# --------------------------------------------------------------------------- accounting
def test_expert_total_is_four_times_active(golden_dir):
    g = _golden(golden_dir, "param_accounting.json")["ratio_case"]
    D, H, N, K = 64, 256, g["n_experts"], g["top_k"]
    router = D * N
    tot = oracle.total_params(D, H, N, K)
    act = oracle.active_params(D, H, N, K)
    assert (tot - router) == g["expert_total_over_active"] * (act - router)
    assert oracle.expert_params(D, H) == 2 * D * H


def test_gpt2_moe_parameter_totals(golden_dir):
    """GPT-2-small dims + 6 experts/top-2 reproduce the printed 446M total / 220M active."""
    gg = _golden(golden_dir, "param_accounting.json")
    d = gg["gpt2_small_dims"]
    c = gg["gpt2_case"]
    D, H, L, V, C = d["d_model"], d["d_hidden"], d["layers"], d["vocab"], d["context"]
    ln = 2 * D
    attn = D * 3 * D + 3 * D + D * D + D
    non_moe_block = 2 * ln + attn
    embed_and_head = V * D + C * D + ln + V * D
    total = embed_and_head + L * (non_moe_block + oracle.total_params(D, H, c["n_experts"], c["top_k"], has_bias=True))
    active = embed_and_head + L * (non_moe_block + oracle.active_params(D, H, c["n_experts"], c["top_k"],
                                                                        has_bias=True))
    assert round(total / 1e6) == c["total_millions_printed"]
    assert round(active / 1e6) == c["active_millions_printed"]
