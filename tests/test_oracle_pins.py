"""Pins of the CPU oracle to what the pages and the mathematics fix (no GPU).

Each test ties one oracle function to something other than itself: a library
routine (torch.softmax in float64), a closed form, an invariant the pages
state, or a hand-worked example from tests/golden/.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import skvgen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bf16_bits(x):
    """float array -> bf16 bit patterns (round to nearest even, via torch)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_vals(bits):
    return skvgen.bf16_to_f64(bits)


def rand_bf16(*shape, scale=1.0):
    return bf16_bits(RNG.standard_normal(shape) * scale)


def torch_attention(q, K, V, scale, mask=None):
    """Library reference: softmax(scale * q K^T) V in float64 (torch CPU)."""
    qt = torch.tensor(bf16_vals(q), dtype=torch.float64)
    Kt = torch.tensor(bf16_vals(K), dtype=torch.float64)
    Vt = torch.tensor(bf16_vals(V), dtype=torch.float64)
    z = scale * (qt @ Kt.T)
    if mask is not None:
        z = z.masked_fill(~torch.tensor(mask), float("-inf"))
    p = torch.softmax(z, dim=-1)
    return (p @ Vt).numpy(), torch.logsumexp(z, dim=-1).numpy()


# ----------------------------------------------------------------------------- plain attention

@pytest.mark.parametrize("L", [1, 5, 63, 64, 65, 130])
def test_attend_matches_torch_softmax(L):
    d, nq = 16, 3
    q = rand_bf16(1, nq, d)
    K = rand_bf16(1, L, d)
    V = rand_bf16(1, L, d)
    s = 1 / math.sqrt(d)
    O, lse = oracle.attend(q, K, V, [[np.arange(L)] * nq], s)
    Ot, lt = torch_attention(q[0], K[0], V[0], s)
    np.testing.assert_allclose(O[0], Ot, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], lt, rtol=1e-13)


def test_attend_subset_matches_masked_softmax():
    d, L = 8, 40
    q = rand_bf16(1, 1, d)
    K = rand_bf16(1, L, d)
    V = rand_bf16(1, L, d)
    sub = np.array(sorted(RNG.choice(L, 11, replace=False)))
    O, lse = oracle.attend(q, K, V, [[sub]], 0.3)
    mask = np.zeros((1, L), dtype=bool)
    mask[0, sub] = True
    Ot, lt = torch_attention(q[0], K[0], V[0], 0.3, mask)
    np.testing.assert_allclose(O[0], Ot, atol=1e-12)
    np.testing.assert_allclose(lse[0], lt, rtol=1e-13)


def test_attend_identical_keys_closed_form():
    # all keys equal -> uniform weights: O = mean(V), lse = z + ln n
    d, L = 8, 37
    q = rand_bf16(1, 1, d)
    k = rand_bf16(1, d)
    K = np.repeat(k[None], L, axis=1)
    V = rand_bf16(1, L, d)
    s = 0.25
    O, lse = oracle.attend(q, K, V, [[np.arange(L)]], s)
    z = s * float(bf16_vals(q[0, 0]) @ bf16_vals(k[0]))
    np.testing.assert_allclose(O[0, 0], bf16_vals(V[0]).mean(axis=0), atol=1e-13)
    assert abs(lse[0, 0] - (z + math.log(L))) < 1e-12


def test_attend_dominant_key_and_empty_set():
    d, L = 8, 20
    q = bf16_bits(np.eye(d)[0][None, None] * 8)
    K = np.zeros((1, L, d), dtype=np.uint16)
    K[0, 7] = bf16_bits(np.eye(d)[0] * 64)  # logit 8*64*0.5 = 256 above the rest
    V = rand_bf16(1, L, d)
    O, lse = oracle.attend(q, K, V, [[np.arange(L)]], 0.5)
    np.testing.assert_allclose(O[0, 0], bf16_vals(V[0, 7]), atol=1e-12)
    O, lse = oracle.attend(q, K, V, [[np.array([], dtype=np.int64)]], 0.5)
    assert np.all(O == 0) and lse[0, 0] == -np.inf


def test_attend_causal_chunk_matches_masked_softmax():
    # query-chunk token t sees the context and chunk keys 0..t
    d, Lc, T = 8, 23, 5
    q = rand_bf16(1, T, d)
    K = rand_bf16(1, Lc + T, d)
    V = rand_bf16(1, Lc + T, d)
    idx = [[oracle.keys_chunk(Lc, t) for t in range(T)]]
    O, lse = oracle.attend(q, K, V, idx, 0.4)
    mask = np.zeros((T, Lc + T), dtype=bool)
    for t in range(T):
        mask[t, :Lc + t + 1] = True
    Ot, lt = torch_attention(q[0], K[0], V[0], 0.4, mask)
    np.testing.assert_allclose(O[0], Ot, atol=1e-12)
    np.testing.assert_allclose(lse[0], lt, rtol=1e-13)


# ----------------------------------------------------------------------------- key sets

def test_window_key_set():
    # Flux sparse layers: sink + recent window; overlapping ranges counted once
    assert list(oracle.keys_window(10, 3, 4)) == [0, 1, 2, 6, 7, 8, 9]
    assert list(oracle.keys_window(6, 3, 4)) == [0, 1, 2, 3, 4, 5]
    assert list(oracle.keys_window(5, 64, 4096)) == [0, 1, 2, 3, 4]


def test_window_covering_everything_is_full_attention():
    d, L = 8, 100
    q = rand_bf16(1, 1, d)
    K = rand_bf16(1, L, d)
    V = rand_bf16(1, L, d)
    a = oracle.attend(q, K, V, [[oracle.keys_window(L, 64, 4096)]], 0.3)
    b = oracle.attend(q, K, V, [[oracle.keys_full(L)]], 0.3)
    np.testing.assert_array_equal(a[0], b[0])


def test_art_traversal_puts_block0_first():
    assert list(oracle.art_traversal(5)) == [0, 4, 3, 2, 1]
    assert list(oracle.art_traversal(5, [3, 1, 4, 2])) == [0, 3, 1, 4, 2]  # order omits 0
    assert list(oracle.art_traversal(4, [2, 0, 3, 1])) == [0, 2, 3, 1]


# ----------------------------------------------------------------------------- ART metrics and rule

def test_art_metric_closed_forms():
    e0, e1 = np.eye(8)[0], np.eye(8)[1]
    assert oracle.art_metrics(e0, 2 * e0) == (1.0, 0.0)
    ds, dc = oracle.art_metrics(e0, e1)
    assert ds == 0.0 and abs(dc - 1.0) < 1e-15
    ds, dc = oracle.art_metrics(e0, e0 + e1)
    assert abs(ds - (math.sqrt(2) - 1)) < 1e-15 and abs(dc - (1 - 1 / math.sqrt(2))) < 1e-15
    ds, dc = oracle.art_metrics(2 * e0, -e0)
    assert abs(ds - 0.5) < 1e-15 and abs(dc - 2.0) < 1e-15
    # zero-norm conventions
    z = np.zeros(8)
    assert oracle.art_metrics(z, z) == (0.0, 0.0)
    assert oracle.art_metrics(z, e0) == (math.inf, 1.0)
    assert oracle.art_metrics(e0, z) == (1.0, 1.0)


def _read_trajectory():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "art_trajectory.txt")) if l.strip() and not l.startswith("#")]
    tau, phi = map(float, rows[0])
    traj, passes, stops = [], None, {}
    for r in rows[1:]:
        if r[0] == "pass":
            passes = [int(v) for v in r[1:]]
        elif r[0] == "stop":
            stops[int(r[1])] = int(r[2])
        else:
            traj.append([float(v) for v in r])
    return tau, phi, np.array(traj), passes, stops


def test_art_rule_on_hand_trajectory():
    tau, phi, x, passes, stops = _read_trajectory()
    got = []
    for t in range(1, len(x)):
        ds, dc = oracle.art_metrics(x[t - 1], x[t])
        got.append(int(ds < tau and dc < phi))
    assert got == passes
    for p, want in stops.items():
        c, _ = oracle.art_stop(x, tau, phi, p)
        assert c == want, (p, c, want)


def test_art_rule_strict_thresholds():
    # identical probes: metrics are 0 up to rounding; with tau = phi = 0 the strict
    # test never passes, so traversal never stops ("ART" 2.2: below)
    x = np.ones((6, 8))
    assert oracle.art_stop(x, 0.0, 0.0, 1)[0] == 6
    assert oracle.art_stop(x, 1e-9, 1e-9, 1)[0] == 2
    assert oracle.art_stop(x, 1e-9, 1e-9, 5)[0] == 6
    assert oracle.art_stop(x, 1e-9, 1e-9, 6)[0] == 6


def _art_inputs(L, d=128, G=4, seed=7):
    rng = np.random.default_rng(seed)
    q = bf16_bits(rng.standard_normal((1, G, d)))
    K = bf16_bits(rng.standard_normal((1, L, d)))
    V = bf16_bits(rng.standard_normal((1, L, d)))
    return q, K, V


@pytest.mark.parametrize("L", [64 * 9, 64 * 9 + 17])
def test_art_never_stopping_equals_full_attention(L):
    # tau = phi = 0: ART consumes every block and equals full attention
    q, K, V = _art_inputs(L)
    nb = (L + 63) // 64
    s = 1 / math.sqrt(128)
    O, lse, cons, _ = oracle.art(q, K, V, [L], 64, [oracle.art_traversal(nb)], s, 0.0, 0.0, 4)
    Of, lf = oracle.attend(q, K, V, [[np.arange(L)] * 4], s)
    assert np.all(cons == nb)
    np.testing.assert_allclose(O, Of, atol=1e-12)
    np.testing.assert_allclose(lse, lf, rtol=1e-13)


def test_full_traversal_is_block_permutation_invariant():
    # "ART" 2.4: reordering KV blocks introduces no approximation error
    L = 64 * 12 + 5
    q, K, V = _art_inputs(L, seed=3)
    nb = 13
    s = 1 / math.sqrt(128)
    ref = oracle.art(q, K, V, [L], 64, [oracle.art_traversal(nb, list(range(nb)))], s, 0.0, 0.0, 4)
    for trial in range(4):
        order = list(RNG.permutation(nb))
        got = oracle.art(q, K, V, [L], 64, [oracle.art_traversal(nb, order)], s, 0.0, 0.0, 4)
        np.testing.assert_allclose(got[0], ref[0], atol=1e-12)
        np.testing.assert_allclose(got[1], ref[1], rtol=1e-12)


def test_art_block0_consumed_and_dominant_sink_stops_at_one_plus_p():
    # a sink key whose logit dominates makes the probe constant (= v_0[0:8])
    # from block 0 on, so every test passes and the walk stops after exactly
    # 1 + p blocks -- even though the order given never lists block 0.
    L, d, G, p = 64 * 20, 128, 4, 4
    rng = np.random.default_rng(11)
    q = bf16_bits(rng.standard_normal((1, G, d)))
    qs = bf16_vals(q[0]).sum(axis=0)
    K = bf16_bits(rng.standard_normal((1, L, d)) * 0.1)
    K[0, 0] = bf16_bits(qs / np.linalg.norm(qs) * 60.0)
    V = bf16_bits(rng.standard_normal((1, L, d)))
    s = 1 / math.sqrt(128)
    order = list(range(19, 0, -1))  # recency-first, no block 0
    O, lse, cons, mg = oracle.art(q, K, V, [L], 64, [oracle.art_traversal(20, order)], s, 1e-3, 1e-4, p)
    assert np.all(cons == 1 + p)
    # result = attention over the consumed blocks: block 0 and the p most recent
    keys = np.concatenate([np.arange(64), np.arange(L - 64 * p, L)])
    Oc, lc = oracle.attend(q, K, V, [[keys] * G], s)
    np.testing.assert_allclose(O, Oc, atol=1e-12)
    np.testing.assert_allclose(lse, lc, rtol=1e-13)


def test_art_forced_stop_equals_prefix_attention():
    L = 64 * 10
    q, K, V = _art_inputs(L, seed=5)
    s = 1 / math.sqrt(128)
    trav = oracle.art_traversal(10)
    forced = np.array([[3, 1, 10, 6]], dtype=np.int32)
    O, lse, cons, _ = oracle.art(q, K, V, [L], 64, [trav], s, 1e-3, 1e-4, 4, forced=forced)
    assert list(cons[0]) == [3, 1, 10, 6]
    for g in range(4):
        keys = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in trav[:forced[0, g]]])
        Oc, lc = oracle.attend(q[:, g:g + 1], K, V, [[keys]], s)
        np.testing.assert_allclose(O[0, g], Oc[0, 0], atol=1e-12)


def test_art_probe_trajectory_matches_rule():
    # the stop point of a real decode equals the rule applied to the probe
    # trajectory, x_t = normalised partial output after t+1 blocks, dims 0..7
    L, G = 64 * 16, 4
    q, K, V = _art_inputs(L, seed=9)
    s = 1 / math.sqrt(128)
    trav = oracle.art_traversal(16)
    tau, phi, p = 0.05, 0.02, 2
    O, lse, cons, _ = oracle.art(q, K, V, [L], 64, [trav], s, tau, phi, p)
    for g in range(G):
        xs = []
        for t in range(16):
            keys = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in trav[:t + 1]])
            Ot, _ = oracle.attend(q[:, g:g + 1], K, V, [[keys]], s)
            xs.append(Ot[0, 0, :8])
        c, _ = oracle.art_stop(np.array(xs), tau, phi, p)
        assert cons[0, g] == c


# ----------------------------------------------------------------------------- merge

@pytest.mark.parametrize("S", [1, 2, 3, 8])
def test_merge_of_shards_equals_unsharded(S):
    # "Pulsar Attention" Phase 2: per-shard partials merged exactly
    d, L, nq = 16, 300, 3
    q = rand_bf16(1, nq, d)
    K = rand_bf16(1, L, d)
    V = rand_bf16(1, L, d)
    cuts = np.sort(RNG.choice(np.arange(1, L), S - 1, replace=False)) if S > 1 else []
    bounds = [0, *cuts, L]
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        O, l = oracle.attend(q, K, V, [[np.arange(a, b)] * nq], 0.25)
        parts_o.append(O[0])
        parts_l.append(l[0])
    # plus an empty shard, which must carry zero weight
    parts_o.append(np.zeros((nq, d)))
    parts_l.append(np.full(nq, -np.inf))
    Om, lm = oracle.merge(np.array(parts_o), np.array(parts_l))
    Of, lf = oracle.attend(q, K, V, [[np.arange(L)] * nq], 0.25)
    np.testing.assert_allclose(Om, Of[0], atol=1e-12)
    np.testing.assert_allclose(lm, lf[0], rtol=1e-13)


def test_merge_all_empty_and_single():
    o = np.zeros((3, 2, 4))
    l = np.full((3, 2), -np.inf)
    Om, lm = oracle.merge(o, l)
    assert np.all(Om == 0) and np.all(lm == -np.inf)
    o1 = RNG.standard_normal((1, 2, 4))
    l1 = RNG.standard_normal((1, 2))
    Om, lm = oracle.merge(o1, l1)
    np.testing.assert_array_equal(Om, o1[0])
    np.testing.assert_array_equal(lm, l1[0])


# ----------------------------------------------------------------------------- centroid selection

def test_select_known_ranking_and_ties():
    d, C, G = 8, 16, 4
    q = np.zeros((1, G, d), dtype=np.uint16)
    q[0, 0] = bf16_bits(np.eye(d)[0])          # sum over heads = e0
    cent = np.zeros((1, C, d), dtype=np.uint16)
    score = [5, 9, 1, 9, 3, 7, 7, 0, 2, 8, 4, 6, 6, 9, 1, 5]
    for c, s in enumerate(score):
        cent[0, c] = bf16_bits(np.eye(d)[0] * s)
    ids, sc = oracle.select(q, cent, 5)
    # best: 9 (ids 1, 3, 13), 8 (id 9), then 7 (ids 5, 6): tie -> lower id 5
    assert list(ids[0]) == [1, 3, 5, 9, 13]
    np.testing.assert_array_equal(sc[0], score)
    ids, _ = oracle.select(q, cent, C)
    assert list(ids[0]) == list(range(C))


def test_select_uses_sum_over_group_heads():
    # the group's score is (sum_g q_g) . c, so heads cancelling out matter
    d, C = 4, 3
    q = np.zeros((1, 2, d), dtype=np.uint16)
    q[0, 0] = bf16_bits([1, 0, 0, 0])
    q[0, 1] = bf16_bits([-1, 1, 0, 0])
    cent = bf16_bits(np.array([[[9, 0, 0, 0], [0, 1, 0, 0], [0, 0, 5, 0]]]))
    ids, sc = oracle.select(q, cent, 1)
    assert list(ids[0]) == [1]
    np.testing.assert_array_equal(sc[0], [0, 1, 0])


def test_select_shared_is_each_requests_own_selection_brute_force():
    """Shared fixed context ("Squeezed Attention" Q1): every request ranks the
    same centroids with its own summed query.  Checked against scores written
    out as explicit sums and a ranking by (score desc, id asc), per request."""
    rng = np.random.default_rng(7)
    U, G, d, C, k = 5, 2, 8, 20, 6
    q = bf16_bits(rng.integers(-3, 4, size=(U, G, d)).astype(np.float64))
    cent = bf16_bits(rng.integers(-2, 3, size=(C, d)).astype(np.float64))  # many exact ties
    ids, sc = oracle.select_shared(q, cent, k)
    qv = skvgen.bf16_to_f64(q)
    cv = skvgen.bf16_to_f64(cent)
    for u in range(U):
        score = [sum(sum(qv[u, g, j] for g in range(G)) * cv[c, j] for j in range(d)) for c in range(C)]
        np.testing.assert_array_equal(sc[u], score)
        best = sorted(range(C), key=lambda c: (-score[c], c))[:k]
        assert list(ids[u]) == sorted(best)


def test_select_shared_identical_and_permuted_requests():
    rng = np.random.default_rng(8)
    U, G, d, C, k = 4, 4, 16, 64, 9
    q = bf16_bits(rng.standard_normal((U, G, d)))
    cent = bf16_bits(rng.standard_normal((C, d)))
    ids, _ = oracle.select_shared(q, cent, k)
    q2 = q.copy()
    q2[2] = q2[0]                         # two identical requests choose identically
    ids2, _ = oracle.select_shared(q2, cent, k)
    np.testing.assert_array_equal(ids2[2], ids2[0])
    perm = [3, 1, 0, 2]                   # the requests' order does not matter
    ids3, _ = oracle.select_shared(q[perm], cent, k)
    np.testing.assert_array_equal(ids3, ids[perm])


def test_select_all_clusters_is_full_attention():
    wl = skvgen.Workload("tiny-mix", B=1, Hq=4, Hkv=1, L=700, c_log2=4, mixture=True, seed=99)
    K, off, cent = skvgen.host_mixture_group(wl, 0, 0)
    _, V = skvgen.host_kv_group(wl, 0, 0)
    q = skvgen.host_q(wl)[:, 0]
    ids, _ = oracle.select(q, cent[None], 16)
    keys = oracle.keys_segments(off[ids[0]], off[ids[0] + 1])
    assert list(keys) == list(range(700))
    a = oracle.attend(q, K[None], V[None], [[keys] * 4], wl.scale)
    b = oracle.attend(q, K[None], V[None], [[np.arange(700)] * 4], wl.scale)
    np.testing.assert_array_equal(a[0], b[0])


def test_squeezed_six_key_example():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "squeezed_six_keys.txt")) if l.strip() and not l.startswith("#")]
    d = int(rows[0][0])
    keys = np.array([[float(v) for v in r] for r in rows[1:7]])
    vals = np.array([[float(v) for v in r] for r in rows[7:13]])
    off = [int(v) for v in rows[13]]
    qv = np.array([float(v) for v in rows[14]])
    want = int(rows[15][1])
    cent = np.array([keys[off[c]:off[c + 1]].mean(axis=0) for c in range(2)])
    ids, _ = oracle.select(bf16_bits(qv[None, None]), bf16_bits(cent[None]), 1)
    assert ids[0, 0] == want
    sel = oracle.keys_segments([off[want]], [off[want + 1]])
    s = 1 / math.sqrt(d)
    O, lse = oracle.attend(bf16_bits(qv[None, None]), bf16_bits(keys[None]), bf16_bits(vals[None]), [[sel]], s)
    # closed form: logits 2, 2, 1.5 over D, E, F with one-hot values
    e2, e15 = math.exp(2.0), math.exp(1.5)
    Z = 2 * e2 + e15
    np.testing.assert_allclose(O[0, 0], [e2 / Z, e2 / Z, e15 / Z, 0.0], atol=1e-15)
    assert abs(lse[0, 0] - math.log(Z)) < 1e-14


def test_topk_boundary_gap():
    g = oracle.topk_boundary_gap(np.array([[3.0, 1.0, 2.0, 2.0]]), 2)
    assert g[0] == 0.0
    g = oracle.topk_boundary_gap(np.array([[4.0, 1.0, 2.0]]), 1)
    assert abs(g[0] - 0.5) < 1e-15


# ----------------------------------------------------------------------------- layer routing

def test_route_constant_tokens_closed_form():
    # every token of every layer equals c: both pooled vectors are c, so the
    # logit is c * (sum of the layer's weights) + bias
    L, B, T, F = 3, 2, 7, 16
    c = 0.375
    q = np.full((L, B, T, F), bf16_bits([c])[0], dtype=np.uint16)
    w = RNG.standard_normal((L, 2 * F))
    bias = RNG.standard_normal(L)
    z, r = oracle.route(q, w, bias, 3, 2)
    want = c * w.sum(axis=1) + bias
    np.testing.assert_allclose(z, np.repeat(want[:, None], B, axis=1), rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(r, (z > 0).astype(np.uint8))


def test_route_one_hot_weights_pick_one_pooled_feature():
    # a weight vector with a single 1 reads one feature of one pooled vector:
    # the mean of that feature over the prefix (or suffix) tokens, by a loop
    L, B, T, F = 2, 3, 9, 8
    q = bf16_bits(RNG.standard_normal((L, B, T, F)))
    vals = bf16_vals(q)
    n_p, n_s = 4, 3
    for j, suffix in ((5, False), (2, True)):
        w = np.zeros((L, 2 * F))
        w[:, F * suffix + j] = 1.0
        z, _ = oracle.route(q, w, np.zeros(L), n_p, n_s)
        for l in range(L):
            for b in range(B):
                toks = range(T - n_s, T) if suffix else range(n_p)
                s = 0.0
                for t in toks:
                    s += vals[l, b, t, j]
                assert z[l, b] == pytest.approx(s / len(toks), rel=1e-15, abs=1e-15)


def test_route_brute_force_tiny():
    L, B, T, F = 2, 2, 5, 4
    q = bf16_bits(RNG.standard_normal((L, B, T, F)))
    vals = bf16_vals(q)
    w = RNG.standard_normal((L, 2 * F))
    bias = RNG.standard_normal(L)
    n_p, n_s = 2, 4  # prefix and suffix overlap: each is pooled on its own
    z, r = oracle.route(q, w, bias, n_p, n_s)
    for l in range(L):
        for b in range(B):
            acc = bias[l]
            for j in range(F):
                pre = sum(vals[l, b, t, j] for t in range(n_p)) / n_p
                suf = sum(vals[l, b, t, j] for t in range(T - n_s, T)) / n_s
                acc += w[l, j] * pre + w[l, F + j] * suf
            assert z[l, b] == pytest.approx(acc, rel=1e-12, abs=1e-12)
            assert r[l, b] == (1 if acc > 0 else 0)


def test_route_hard_decision_is_strict():
    # zero queries and zero bias give a zero logit: not above zero, so sparse
    L, B, T, F = 1, 2, 3, 8
    q = np.zeros((L, B, T, F), dtype=np.uint16)
    z, r = oracle.route(q, RNG.standard_normal((L, 2 * F)), np.zeros(L), 1, 1)
    assert np.all(z == 0.0) and np.all(r == 0)
    z, r = oracle.route(q, RNG.standard_normal((L, 2 * F)), np.full(L, 1e-30), 1, 1)
    assert np.all(r == 1)


# ----------------------------------------------------------------------------- two-level selection

def _hier(U, G, d, C1, per, seed):
    rng = np.random.default_rng(seed)
    C = C1 * per
    q = bf16_bits(rng.standard_normal((U, G, d)))
    fine = bf16_bits(rng.standard_normal((U, C, d)))
    coarse = bf16_bits(bf16_vals(fine).reshape(U, C1, per, d).mean(axis=2))
    off = np.tile(np.arange(0, C + 1, per), (U, 1))
    return q, coarse, off, fine


def test_select2_all_coarse_is_flat_selection():
    # keeping every coarse cluster leaves every fine cluster a candidate: the
    # second level is then exactly the one-level top-k
    q, coarse, off, fine = _hier(3, 4, 16, 8, 5, 11)
    for k2 in (1, 7, 40):
        got = oracle.select2(q, coarse, off, fine, 8, k2)
        want, _ = oracle.select(q, fine, k2)
        np.testing.assert_array_equal(got, want)


def test_select2_picks_the_best_candidates_only():
    # fine clusters outside the chosen coarse clusters never appear, and the
    # chosen ones are the k2 best candidates by a plain sort (score desc, index asc)
    q, coarse, off, fine = _hier(4, 2, 8, 10, 6, 12)
    k1, k2 = 3, 5
    got = oracle.select2(q, coarse, off, fine, k1, k2)
    qs = bf16_vals(q).sum(axis=1)
    for u in range(4):
        sc1 = bf16_vals(coarse[u]) @ qs[u]
        top1 = sorted(range(10), key=lambda i: (-sc1[i], i))[:k1]
        cand = [c for i in sorted(top1) for c in range(off[u][i], off[u][i + 1])]
        sc2 = bf16_vals(fine[u]) @ qs[u]
        want = sorted(sorted(cand, key=lambda c: (-sc2[c], c))[:k2])
        assert list(got[u]) == want


def test_select2_fewer_candidates_than_k2():
    # 2 coarse clusters of 3 fine ones each can offer only 6 candidates
    q, coarse, off, fine = _hier(1, 1, 8, 4, 3, 13)
    got = oracle.select2(q, coarse, off, fine, 2, 9)
    assert (got[0, :6] >= 0).all() and (got[0, 6:] == -1).all()
    assert list(got[0, :6]) == sorted(got[0, :6])


def test_select2_squeezed_hierarchy_example():
    rows, expect = {}, {}
    for line in open(os.path.join(GOLDEN, "squeezed_hierarchy.txt")):
        s = line.split()
        if not s or s[0].startswith("#"):
            continue
        if s[0].startswith("expect_"):
            expect[s[0]] = s[1:]
        else:
            rows[s[0]] = [float(x) for x in s[1:]]
    names = ["apple", "banana", "carrot", "dog", "elephant", "fish"]
    keys = np.array([rows[n] for n in names])
    fine_members = [[0, 1], [2], [3, 4], [5]]           # A1, A2, B1, B2
    coarse_members = [[0, 1, 2], [3, 4, 5]]             # A, B
    fine = bf16_bits(np.array([keys[m].mean(axis=0) for m in fine_members]))[None]
    coarse = bf16_bits(np.array([keys[m].mean(axis=0) for m in coarse_members]))[None]
    off = np.array([[0, 2, 4]])
    q = bf16_bits(np.array(rows["query"]))[None, None]
    got = oracle.select2(q, coarse, off, fine, 1, 1)
    fine_names = ["A1", "A2", "B1", "B2"]
    assert [fine_names[i] for i in got[0]] == expect["expect_fine"]
    assert [names[i] for i in fine_members[got[0][0]]] == expect["expect_keys"]


def test_oracle_threads_do_not_change_results():
    # the OpenMP loops run over independent units: one thread or many, the
    # results are the same bits (the CPU baseline times both)
    n0 = oracle.threads()
    q = bf16_bits(RNG.standard_normal((6, 4, 16)))
    K = bf16_bits(RNG.standard_normal((6, 70, 16)))
    V = bf16_bits(RNG.standard_normal((6, 70, 16)))
    keys = [[np.arange(70)] * 4 for _ in range(6)]  # per unit, per query row
    a = oracle.attend(q, K, V, keys, 0.25)
    oracle.set_threads(1)
    try:
        assert oracle.threads() == 1
        b = oracle.attend(q, K, V, keys, 0.25)
    finally:
        oracle.set_threads(n0)
    assert oracle.threads() == n0
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ----------------------------------------------------------------------------- lookahead (Forecast)

def test_forecast_one_hot_weights_read_one_input():
    rng = np.random.default_rng(11)
    d = 128
    x = bf16_bits(rng.standard_normal((3, d)))
    perm = rng.permutation(d)
    w = np.zeros((3, d, d))
    w[:, perm, np.arange(d)] = 1.0             # output j reads input perm[j]
    f = oracle.forecast(x, bf16_bits(w))
    np.testing.assert_array_equal(f, x[:, perm])


def test_forecast_small_integers_are_exact():
    rng = np.random.default_rng(12)
    d = 128
    x = rng.integers(-2, 3, size=(4, d))
    w = rng.integers(-1, 2, size=(4, d, d))
    f = oracle.forecast(bf16_bits(x.astype(float)), bf16_bits(w.astype(float)))
    exact = np.einsum("uij,ui->uj", w, x)      # |sum| <= 256: exact in bf16
    np.testing.assert_array_equal(skvgen.bf16_to_f64(f), exact)


def test_forecast_sums_in_fp32_in_input_order_and_rounds_to_nearest_even():
    d = 128
    x = np.zeros((3, d))
    w = np.zeros((3, d, d))
    # 2^24 + 1 rounds to 2^24 in fp32, then - 2^24 gives 0 (another order gives 1)
    x[0, :3] = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    w[0, :3, 0] = 1.0
    # 1 + 2^-8 is halfway between two bf16 values: to the even one, 1.0;
    # 1 + 3 * 2^-8 is halfway too: to the even one, 1 + 2^-6
    x[1, :2] = [1.0, 2.0 ** -8]
    w[1, :2, 0] = 1.0
    x[2, :2] = [1.0, 3 * 2.0 ** -8]
    w[2, :2, 0] = 1.0
    f = skvgen.bf16_to_f64(oracle.forecast(bf16_bits(x), bf16_bits(w)))
    assert f[0, 0] == 0.0
    assert f[1, 0] == 1.0
    assert f[2, 0] == 1.0 + 2.0 ** -6


def test_forecast_close_to_the_exact_projection():
    rng = np.random.default_rng(13)
    d = 128
    x = bf16_bits(rng.standard_normal((5, d)))
    w = bf16_bits(rng.standard_normal((5, d, d)) / 16)
    f = skvgen.bf16_to_f64(oracle.forecast(x, w))
    ref = np.einsum("uij,ui->uj", skvgen.bf16_to_f64(w), skvgen.bf16_to_f64(x))
    # one bf16 rounding (relative 2^-8) plus fp32 accumulation error
    bound = np.abs(ref) * 2.0 ** -8 + d * 2.0 ** -23 * np.einsum(
        "uij,ui->uj", np.abs(skvgen.bf16_to_f64(w)), np.abs(skvgen.bf16_to_f64(x)))
    assert np.all(np.abs(f - ref) <= bound)


def test_keys_blocks_short_last_block():
    np.testing.assert_array_equal(oracle.keys_blocks([2, 0, -1], 150),
                                  np.r_[np.arange(0, 64), np.arange(128, 150)])
