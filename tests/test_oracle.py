"""Pins of the CPU oracle against facts other than itself.

Each test checks one oracle function against brute force, a closed form, a
textbook routine or an invariant of the mathematics, chosen so that a dropped
term, a wrong sign or index, or a transposed operand fails at least one of
them. No test here needs a GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle

U32 = 2.0 ** -24


def bf16_values(rng, shape, std=1.0):
    """Random values that are exactly representable in bf16."""
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * std)
    return v.to(torch.bfloat16).to(torch.float32).numpy()


def tiny_layer(rng, T=8, d=8, E=4, k=2, f=16, wscale=0.4):
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((E, d)) * 0.7
    b = rng.standard_normal(E) * 0.3
    Wg = rng.standard_normal((E, f, d)) * wscale
    Wu = rng.standard_normal((E, f, d)) * wscale
    Wd = rng.standard_normal((E, d, f)) * wscale
    return x, Wr, b, Wg, Wu, Wd


# ------------------------------------------------------------ router logits

def test_logits_f32_within_summation_error_bound(rng):
    T, d, E = 64, 512, 16
    x = bf16_values(rng, (T, d))
    Wr = bf16_values(rng, (E, d), 0.05)
    b = rng.standard_normal(E).astype(np.float32)
    z32 = oracle.router_logits_f32(x, Wr, b).astype(np.float64)
    z64 = oracle.router_logits_f64(x, Wr, b)
    # recursive summation of d exact products, then one rounded add of b:
    # |err| <= gamma_d * sum|x_i w_i| + u * |z|  (Higham, Accuracy and Stability, ch. 3)
    gamma = d * U32 / (1 - d * U32)
    bound = gamma * (np.abs(x.astype(np.float64)) @ np.abs(Wr.astype(np.float64)).T) + U32 * np.abs(z64) + 1e-30
    assert np.all(np.abs(z32 - z64) <= bound)


def test_logits_one_hot_rows_pick_router_columns(rng):
    d, E = 32, 8
    Wr = rng.standard_normal((E, d)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    x = np.eye(d, dtype=np.float32)
    z = oracle.router_logits_f32(x, Wr, b)
    expect = (Wr.T + b[None, :]).astype(np.float32)  # one fp32 add per entry
    assert np.array_equal(z, expect)


def test_logits_bf16_fma_equals_rounded_add_of_exact_products(rng):
    # for bf16 operands every product is exact in fp32, so fma == one rounded add
    T, d, E = 16, 96, 8
    x = bf16_values(rng, (T, d))
    Wr = bf16_values(rng, (E, d), 0.1)
    b = bf16_values(rng, (E,))
    z = oracle.router_logits_f32(x, Wr, b)
    acc = np.zeros((T, E), np.float32)
    for i in range(d):
        acc = (acc + np.outer(x[:, i], Wr[:, i]).astype(np.float32)).astype(np.float32)
    assert np.array_equal(z, (acc + b[None, :]).astype(np.float32))


# ----------------------------------------------------------------- routing

def brute_topk(z, k):
    """Top-k by sorting (-z, index) lexicographically; NaN after every number."""
    T, E = z.shape
    out = np.empty((T, k), np.int32)
    for t in range(T):
        keys = [((1, 0.0) if math.isnan(z[t, e]) else (0, -z[t, e]), e) for e in range(E)]
        keys.sort()
        out[t] = [e for _, e in keys[:k]]
    return out


@pytest.mark.parametrize("E,k", [(4, 2), (8, 2), (64, 8), (16, 16), (5, 1), (33, 7)])
def test_route_selection_matches_brute_force_with_ties(rng, E, k):
    T = 200
    z = np.round(rng.standard_normal((T, E)) * 2) / 2  # coarse grid: many exact ties
    z[::7, : E // 2] = 0.5
    idx, w, flags = oracle.route(z, k)
    assert flags == 0
    assert np.array_equal(idx, brute_topk(z, k))


def test_route_nan_ranks_last_and_nonfinite_flags():
    z = np.array([[np.nan, 1.0, -np.inf, 2.0],
                  [0.0, np.nan, np.nan, -1.0],
                  [-np.inf, -np.inf, 3.0, 1.0]])
    idx, w, flags = oracle.route(z, 2)
    assert idx.tolist() == [[3, 1], [0, 3], [2, 3]]
    assert flags == 0 and np.allclose(w.sum(1), 1)
    idx, w, flags = oracle.route(z, 3)
    assert idx.tolist() == [[3, 1, 2], [0, 3, 1], [2, 3, 0]]
    assert flags & oracle.FLAG_NONFINITE
    # selected (2, 1, -inf): the softmax is defined; by hand e^0 / (1 + e^-1)
    # = 0.7310586, e^-1 / (1 + e^-1) = 0.2689414, and exactly 0 for -inf
    np.testing.assert_allclose(w[0], [0.7310585786300049, 0.2689414213699951, 0.0], rtol=1e-15)
    assert w[0, 2] == 0.0
    # selected (0, -1, NaN): undefined, 1/k each
    assert np.all(w[1] == 1.0 / 3)
    # selected (3, 1, -inf): e^0 / (1 + e^-2) = 0.8807971, e^-2 / (1 + e^-2) = 0.1192029
    np.testing.assert_allclose(w[2], [0.8807970779778823, 0.11920292202211755, 0.0], rtol=1e-15)


def test_route_undefined_softmax_falls_back_to_uniform_weights():
    inf = np.inf
    # all selected -inf (0/0), +inf selected (inf - inf), NaN selected
    for row, k in (([-inf, -inf, -inf, -inf], 2), ([inf, 1.0, 0.0, 2.0], 2),
                   ([inf, inf, 0.0, 2.0], 3), ([1.0, np.nan, np.nan, np.nan], 2)):
        idx, w, flags = oracle.route(np.array([row]), k)
        assert flags & oracle.FLAG_NONFINITE, row
        assert np.all(w == 1.0 / k), row
    # one finite logit with -inf after it: the whole weight on the finite one
    idx, w, flags = oracle.route(np.array([[-inf, 0.25, -inf, -inf]]), 3)
    assert flags == 0
    assert idx.tolist() == [[1, 0, 2]] and w.tolist() == [[1.0, 0.0, 0.0]]
    # a NaN outside the selection does not matter
    idx, w, flags = oracle.route(np.array([[np.nan, 1.0, 1.0, 0.0]]), 2)
    assert flags == 0 and idx.tolist() == [[1, 2]] and w.tolist() == [[0.5, 0.5]]


def test_route_weights_properties(rng):
    z = rng.standard_normal((300, 12)) * 3
    for k in (1, 2, 5, 12):
        idx, w, _ = oracle.route(z, k)
        assert np.all(np.abs(w.sum(1) - 1) <= 1e-12)
        assert np.all(w >= 0)
        assert np.all(np.diff(w, axis=1) <= 0)
        if k == 1:
            assert np.all(w == 1.0)


def test_route_k_equals_E_is_plain_softmax(rng):
    import scipy.special
    z = rng.standard_normal((50, 9)) * 2
    idx, w, _ = oracle.route(z, 9)
    full = scipy.special.softmax(z, axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, idx, axis=1), rtol=1e-13, atol=1e-15)


def test_route_topk_weights_equal_renormalised_full_softmax(rng):
    import scipy.special
    z = rng.standard_normal((80, 16))
    idx, w, _ = oracle.route(z, 4)
    p = np.take_along_axis(scipy.special.softmax(z, axis=1), idx, axis=1)
    np.testing.assert_allclose(w, p / p.sum(1, keepdims=True), rtol=1e-12)


# ------------------------------------------------------------------ layout

def check_layout(idx, lay, E, G):
    T, k = idx.shape
    P = T * k
    counts = np.bincount(idx.ravel(), minlength=E)
    assert np.array_equal(lay["counts"], counts)
    assert lay["counts"].sum() == P
    assert np.array_equal(lay["offsets"], np.concatenate([[0], np.cumsum(counts)]))
    rop, por = lay["row_of_pair"], lay["pair_of_row"]
    assert np.array_equal(np.sort(rop), np.arange(P))
    assert np.array_equal(por[rop], np.arange(P))
    # rows sorted by (expert, token), strictly increasing
    e_of_row = idx.ravel()[por]
    t_of_row = por // k
    key = e_of_row.astype(np.int64) * (T + 1) + t_of_row
    assert np.all(np.diff(key) > 0)
    # independent construction: stable argsort of the expert id of each pair
    assert np.array_equal(por, np.argsort(idx.ravel(), kind="stable"))
    per = E // G
    assert np.array_equal(lay["group_counts"], counts.reshape(G, per).sum(1))
    assert np.array_equal(lay["group_offsets"], lay["offsets"][::per])


@pytest.mark.parametrize("T,E,k,G", [(1, 4, 2, 2), (257, 8, 2, 1), (1000, 64, 8, 4), (33, 16, 16, 16)])
def test_layout_invariants(rng, T, E, k, G):
    z = rng.standard_normal((T, E))
    z[:, E - 1] -= 1e4 if k < E else 0  # one starved expert
    idx, _, _ = oracle.route(z, k)
    lay = oracle.dispatch_layout(idx, E, G)
    check_layout(idx, lay, E, G)
    if k < E:
        assert lay["counts"][E - 1] == 0


def test_layout_rejects_indivisible_groups():
    with pytest.raises(ValueError):
        oracle.dispatch_layout(np.zeros((2, 1), np.int32), 6, 4)


def test_layout_empty_batch():
    lay = oracle.dispatch_layout(np.zeros((0, 2), np.int32), 4, 2)
    assert lay["counts"].tolist() == [0, 0, 0, 0]
    assert lay["offsets"].tolist() == [0] * 5
    assert lay["group_offsets"].tolist() == [0, 0, 0]


# ----------------------------------------------------------------- forward

def test_permute_then_combine_of_identity_returns_x(rng):
    T, d, E, k = 40, 12, 6, 3
    x = rng.standard_normal((T, d))
    idx, w, _ = oracle.route(rng.standard_normal((T, E)), k)
    lay = oracle.dispatch_layout(idx, E, 1)
    xp = oracle.permute(x, lay["pair_of_row"], k)
    for r in range(T * k):
        assert np.array_equal(xp[r], x[lay["pair_of_row"][r] // k])
    Y = oracle.combine(xp, w, lay["row_of_pair"])
    np.testing.assert_allclose(Y, x, rtol=1e-13, atol=1e-14)


def test_closed_form_single_token():
    # x = (1, 0); gate row (1, 0), up row (2, 0): h1 = 1, h2 = 2,
    # a = 2 * silu(1) = 2 / (1 + e^-1); down column (1, -1): Y = (a, -a)
    x = np.array([[1.0, 0.0]])
    Wr = np.zeros((1, 2)); b = np.zeros(1)
    Wg = np.array([[[1.0, 0.0]]]); Wu = np.array([[[2.0, 0.0]]]); Wd = np.array([[[1.0], [-1.0]]])
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k=1)
    a = 2.0 / (1.0 + math.exp(-1.0))
    assert fw["h1"][0, 0] == 1.0 and fw["h2"][0, 0] == 2.0
    assert abs(fw["a"][0, 0] - a) < 1e-15
    np.testing.assert_allclose(fw["Y"], [[a, -a]], rtol=1e-15)


def test_one_expert_top1_is_plain_swiglu_mlp(rng):
    T, d, f = 20, 10, 14  # d != f so a transposed weight cannot pass
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=T, d=d, E=1, k=1, f=f)
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k=1)
    X = torch.from_numpy(x)
    ref = (torch.nn.functional.silu(X @ torch.from_numpy(Wg[0]).T) * (X @ torch.from_numpy(Wu[0]).T)) \
        @ torch.from_numpy(Wd[0]).T
    np.testing.assert_allclose(fw["Y"], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_two_experts_mix_by_gate_weights(rng):
    # k = E = 2: Y = g0 FFN_{S0}(x) + g1 FFN_{S1}(x) with g the 2-way softmax
    T, d, f = 6, 5, 7
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=T, d=d, E=2, k=2, f=f)
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k=2, logits="f64")
    X = torch.from_numpy(x)
    outs = [(torch.nn.functional.silu(X @ torch.from_numpy(Wg[e]).T) * (X @ torch.from_numpy(Wu[e]).T))
            @ torch.from_numpy(Wd[e]).T for e in range(2)]
    p = torch.softmax(torch.from_numpy(x @ Wr.T + b), dim=1)
    ref = p[:, :1] * outs[0] + p[:, 1:] * outs[1]
    np.testing.assert_allclose(fw["Y"], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_permuted_path_equals_per_token_brute_force(rng):
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=37, d=9, E=5, k=3, f=11)
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k=3)
    Y, ys = oracle.tokens_fwd(x, fw["idx"], fw["w"], Wg, Wu, Wd)
    np.testing.assert_allclose(fw["Y"], Y, rtol=1e-13, atol=1e-14)
    for t in range(x.shape[0]):
        for j in range(3):
            r = fw["row_of_pair"][t * 3 + j]
            np.testing.assert_allclose(fw["yp"][r], ys[t, j], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- backward

def loss(x, Wr, b, Wg, Wu, Wd, k, dY):
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k, logits="f64")
    return float((fw["Y"] * dY).sum()), fw["idx"]


@pytest.mark.parametrize("k", [1, 2])
def test_backward_matches_central_finite_differences(rng, k):
    T, d, E, f = 8, 8, 4, 16
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=T, d=d, E=E, k=k, f=f)
    dY = rng.standard_normal((T, d))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k, logits="f64")
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, k)
    params = dict(x=x, Wr=Wr, b=b, Wg=Wg, Wu=Wu, Wd=Wd)
    grads = dict(x=bw["dX"], Wr=bw["dWr"], b=bw["db"], Wg=bw["dWg"], Wu=bw["dWu"], Wd=bw["dWd"])
    h = 1e-6
    skipped = 0
    checked = 0
    for name, P in params.items():
        flat = P.reshape(-1)
        G = grads[name].reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp, ip = loss(**params, k=k, dY=dY)
            flat[i] = old - h
            lm, im = loss(**params, k=k, dY=dY)
            flat[i] = old
            if not (np.array_equal(ip, fw["idx"]) and np.array_equal(im, fw["idx"])):
                skipped += 1  # the perturbation crossed a top-k boundary
                continue
            fd = (lp - lm) / (2 * h)
            assert abs(fd - G[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, G[i])
            checked += 1
    assert checked > 0.95 * (checked + skipped)


def test_route_gradient_sums_to_zero_per_token(rng):
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=30, d=6, E=7, k=3, f=5)
    dY = rng.standard_normal((30, 6))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 3)
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 3)
    assert np.all(np.abs(bw["dz"].sum(1)) <= 1e-12 * (1 + np.abs(bw["dz"]).sum(1)))
    assert abs(bw["db"].sum()) <= 1e-11
    # dz is zero off the selected experts
    mask = np.ones_like(bw["dz"], bool)
    np.put_along_axis(mask, fw["idx"], False, axis=1)
    assert np.all(bw["dz"][mask] == 0)


def test_empty_expert_gradients_untouched(rng):
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=12, d=6, E=4, k=2, f=5)
    b[3] = -1e4
    dY = rng.standard_normal((12, 6))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 2)
    assert fw["counts"][3] == 0
    acc = dict(dWg=rng.standard_normal(Wg.shape), dWu=rng.standard_normal(Wu.shape),
               dWd=rng.standard_normal(Wd.shape))
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 2, acc=acc)
    for n in ("dWg", "dWu", "dWd"):
        assert np.array_equal(bw[n][3], acc[n][3])
    bw0 = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 2)
    assert not bw0["dWg"][3].any() and not bw0["dWd"][3].any()


def test_empty_batch_leaves_accumulators_unchanged(rng):
    _, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=1, d=6, E=4, k=2, f=5)
    x = np.zeros((0, 6)); dY = np.zeros((0, 6))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 2)
    assert fw["Y"].shape == (0, 6) and fw["counts"].sum() == 0
    acc = dict(dWg=rng.standard_normal(Wg.shape), dWu=rng.standard_normal(Wu.shape),
               dWd=rng.standard_normal(Wd.shape), dWr=rng.standard_normal(Wr.shape),
               db=rng.standard_normal(4))
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 2, acc=acc)
    for n in acc:
        assert np.array_equal(bw[n], acc[n])
    assert bw["dX"].shape == (0, 6)


def test_microbatch_accumulation_equals_one_concatenated_pass(rng):
    d, E, k, f = 6, 4, 2, 5
    _, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=1, d=d, E=E, k=k, f=f)
    sizes = [9, 4, 1, 0]
    xs = [rng.standard_normal((n, d)) for n in sizes]
    dYs = [rng.standard_normal((n, d)) for n in sizes]
    acc = None
    for x, dY in zip(xs, dYs):
        fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, k)
        bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, k, acc=acc)
        acc = {n: bw[n] for n in ("dWg", "dWu", "dWd", "dWr", "db")}
    X = np.concatenate(xs); DY = np.concatenate(dYs)
    fw = oracle.layer_forward(X, Wr, b, Wg, Wu, Wd, k)
    bw = oracle.layer_backward(fw, X, DY, Wr, Wg, Wu, Wd, k)
    for n in acc:
        np.testing.assert_allclose(acc[n], bw[n], rtol=1e-12, atol=1e-13)


def test_per_token_backward_equals_permuted_backward(rng):
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=23, d=7, E=5, k=2, f=9)
    dY = rng.standard_normal((23, 7))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 2)
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 2)
    Y, ys = oracle.tokens_fwd(x, fw["idx"], fw["w"], Wg, Wu, Wd)
    dz, dX = oracle.tokens_bwd(x, dY, fw["idx"], fw["w"], ys, Wr, Wg, Wu, Wd)
    np.testing.assert_allclose(dz, bw["dz"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dX, bw["dX"], rtol=1e-12, atol=1e-13)


def test_wgrad_columns_equal_full_weight_gradients(rng):
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=31, d=7, E=4, k=2, f=9)
    dY = rng.standard_normal((31, 7))
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 2)
    bw = oracle.layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, 2)
    for e in range(4):
        rows = np.arange(fw["offsets"][e], fw["offsets"][e + 1])
        pairs = fw["pair_of_row"][rows]
        toks = pairs // 2
        gs = fw["w"].ravel()[pairs]
        cols = np.array([0, 3, 8], np.int32)
        og, ou, od = oracle.wgrad_columns(x[toks], dY[toks], gs, Wg[e], Wu[e], Wd[e], cols)
        np.testing.assert_allclose(og, bw["dWg"][e][cols], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ou, bw["dWu"][e][cols], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(od, bw["dWd"][e][:, cols].T, rtol=1e-12, atol=1e-13)


def test_planted_mistakes_are_caught(rng):
    """A mistake planted in the oracle's results (on the CPU) fails a pin."""
    x, Wr, b, Wg, Wu, Wd = tiny_layer(rng, T=10, d=6, E=4, k=2, f=7)
    fw = oracle.layer_forward(x, Wr, b, Wg, Wu, Wd, 2)
    Y, _ = oracle.tokens_fwd(x, fw["idx"], fw["w"], Wg, Wu, Wd)
    # combine with swapped slot weights
    bad = oracle.combine(fw["yp"], fw["w"][:, ::-1], fw["row_of_pair"])
    assert not np.allclose(bad, Y)
    # an up projection used in place of the gate
    _, _, _, yp_bad = oracle.expert_ffn_fwd(fw["xp"], Wu, Wg, Wd, fw["offsets"])
    assert not np.allclose(oracle.combine(yp_bad, fw["w"], fw["row_of_pair"]), Y)
    # a permutation off by one row
    bad_rop = np.roll(fw["row_of_pair"], 1)
    assert not np.allclose(oracle.combine(fw["yp"], fw["w"], bad_rop), Y)


# ------------------------------------------- auxiliary load-balancing loss

@pytest.mark.parametrize("E,k", [(4, 2), (8, 1), (64, 8)])
def test_aux_loss_uniform_routing_closed_form(E, k):
    """Equal logits and equal counts: importance 1/E, loss alpha, entropy ln E."""
    T = 6 * E
    z = np.zeros((T, E))
    counts = np.full(E, T * k // E, np.int32)
    out = oracle.aux_loss(z, counts, k, 0.02)
    assert np.allclose(out["importance"], 1.0 / E, rtol=0, atol=1e-15)
    assert abs(out["loss"] - 0.02) < 1e-15
    assert abs(out["entropy"] - math.log(E)) < 1e-12


def test_aux_loss_collapsed_routing_closed_form():
    """Every token sends its only pair to expert 0 and its softmax is (almost)
    one-hot there: the loss reaches its maximum alpha * E and the entropy 0."""
    T, E = 9, 5
    z = np.zeros((T, E))
    z[:, 0] = 60.0
    counts = np.array([T, 0, 0, 0, 0], np.int32)
    out = oracle.aux_loss(z, counts, 1, 0.5)
    p0 = 1.0 / (1.0 + (E - 1) * math.exp(-60.0))
    assert abs(out["loss"] - 0.5 * E * p0) < 1e-14
    assert out["entropy"] < 1e-20


def test_aux_loss_matches_scipy_softmax_and_entropy(rng):
    from scipy.special import softmax
    from scipy.stats import entropy
    T, E, k = 37, 12, 3
    z = rng.standard_normal((T, E)) * 2.0
    counts = rng.integers(0, 20, E).astype(np.int32)
    out = oracle.aux_loss(z, counts, k, 0.01)
    p = softmax(z, axis=1)
    P = p.mean(axis=0)
    f = counts / (T * k)
    assert np.allclose(out["importance"], P, rtol=1e-13, atol=0)
    assert abs(out["loss"] - 0.01 * E * float(np.dot(f, P))) < 1e-15
    assert abs(out["entropy"] - float(np.mean(entropy(p, axis=1)))) < 1e-12


def test_aux_loss_gradient_matches_central_finite_differences(rng):
    T, E, k, alpha, dL = 5, 6, 2, 0.3, 1.7
    z = rng.standard_normal((T, E))
    counts = rng.integers(1, 9, E).astype(np.int32)
    dz = oracle.aux_loss_bwd(z, counts, k, alpha, dL)
    h = 1e-6
    num = np.zeros_like(z)
    for t in range(T):
        for e in range(E):
            zp = z.copy(); zp[t, e] += h
            zm = z.copy(); zm[t, e] -= h
            num[t, e] = dL * (oracle.aux_loss(zp, counts, k, alpha)["loss"] -
                              oracle.aux_loss(zm, counts, k, alpha)["loss"]) / (2 * h)
    assert np.abs(dz - num).max() <= 1e-7 * np.abs(num).max()
    # a softmax gradient: every token's row sums to zero
    assert np.abs(dz.sum(axis=1)).max() < 1e-15


def test_aux_loss_router_gradient_matches_finite_differences(rng):
    """The balance loss composed with z = x Wr^T + b: its gradient through the
    dense router backward matches central differences in x, Wr and b."""
    T, d, E, k, alpha = 4, 5, 6, 2, 0.7
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((E, d)) * 0.5
    b = rng.standard_normal(E) * 0.3
    counts = rng.integers(1, 5, E).astype(np.int32)

    def loss(x_, Wr_, b_):
        return oracle.aux_loss(oracle.router_logits_f64(x_, Wr_, b_), counts, k, alpha)["loss"]

    dz = oracle.aux_loss_bwd(oracle.router_logits_f64(x, Wr, b), counts, k, alpha)
    dX, dWr, db = oracle.router_bwd(x, Wr, dz, np.zeros((T, d)))
    h = 1e-6
    for arr, grad in ((x, dX), (Wr, dWr), (b, db)):
        num = np.zeros_like(arr)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h; lp = loss(x, Wr, b)
            flat[i] = old - h; lm = loss(x, Wr, b)
            flat[i] = old
            num.reshape(-1)[i] = (lp - lm) / (2 * h)
        assert np.abs(grad - num).max() <= 1e-6 * max(np.abs(num).max(), 1e-12)


def test_aux_loss_planted_mistake_is_caught():
    """Counting the fraction per token instead of per routed pair (dropping k)
    breaks the uniform closed form."""
    T, E, k = 24, 4, 2
    z = np.zeros((T, E))
    counts = np.full(E, T * k // E, np.int32)
    good = oracle.aux_loss(z, counts, k, 1.0)["loss"]
    bad = oracle.aux_loss(z, counts, 1, 1.0)["loss"]  # k dropped from f's denominator
    assert abs(good - 1.0) < 1e-15 and abs(bad - 1.0) > 0.5
