"""Pins of the CPU oracle against what the pages and the mathematics fix.

The pages ("PIVOT", picx.dev summary of the paper, Methodology, Eq. 1-9)
print no numeric example, so the oracle is pinned by:
  * a hand-worked example (tests/golden/hand_example.json) with one-hot keys,
  * closed forms (one-hot keys reduce q.k to one coordinate),
  * reductions the equations imply (g=1 Reuse == dense, c >= L Refine == dense,
    g=1 Refine == dense, identical members Reuse == dense),
  * a library routine for TopK order (numpy lexsort) and brute-force selection,
  * invariants (causal mask, row counts, -1 padding, lower-index ties).
Each pin is chosen so that a plausible slip (a dropped ReLU, ReLU after the
head sum, a transposed operand, a wrong mean divisor, the proxy scanning
s <= group start, the wrong tie order) fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

from top_token_selection_proxy_b200 import inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")))


def _hand():
    q = np.array(GOLD["q"], np.float32)
    w = np.array(GOLD["w"], np.float32)
    k = np.array(GOLD["keys"], np.float32)
    return q, w, k


def _rand(L, H, d, seed, dtype=np.float32, scale=1.0):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((L, H, d)) * scale).astype(np.float32)
    w = rng.standard_normal((L, H)).astype(np.float32)
    k = (rng.standard_normal((L, d)) / np.sqrt(d)).astype(np.float32)
    if dtype == np.uint16:
        return inputs.to_bf16_bits(q), w, inputs.to_bf16_bits(k)
    return q, w, k


def _onehot(L, H, seed):
    """q, w random; k_s = e_s so that q_{t,j} . k_s = q_{t,j,s} (closed form)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, H, L)).astype(np.float32)
    w = rng.standard_normal((L, H)).astype(np.float32)
    k = np.eye(L, dtype=np.float32)
    return q, w, k


# ----------------------------------------------------------------- golden


def test_golden_dense(orc):
    q, w, k = _hand()
    idx, val = orc.dense(q, w, k, GOLD["k"])
    assert idx.tolist() == GOLD["dense_idx"]
    for t, row in enumerate(GOLD["dense_scores"]):
        for r, s in enumerate(idx[t]):
            if s >= 0:
                assert val[t, r] == row[s]


def test_golden_proxy(orc):
    q, w, k = _hand()
    for i, rows in enumerate(([0, 1], [2, 3])):
        qb, wb = orc.proxy(q, w, rows)
        assert qb.reshape(2, 4).tolist() == GOLD["proxy_g2"]["qbar"][i]
        assert wb.tolist() == GOLD["proxy_g2"]["wbar"][i]
        assert orc.proxy_scores(q, w, k, 2, i).tolist() == GOLD["proxy_g2"]["scores"][i]


def test_golden_reuse(orc):
    q, w, k = _hand()
    idx, _ = orc.reuse(q, w, k, GOLD["k"], 2)
    assert idx.tolist() == GOLD["reuse_g2_idx"]


@pytest.mark.parametrize("c", [3, 2])
def test_golden_refine(orc, c):
    q, w, k = _hand()
    idx, _, cand, _ = orc.refine(q, w, k, GOLD["k"], c, 2)
    assert cand.tolist() == GOLD[f"refine_g2_c{c}_cand"]
    assert idx.tolist() == GOLD[f"refine_g2_c{c}_idx"]


# ----------------------------------------------------------------- TopK order


def test_topn_matches_lexsort(orc):
    rng = np.random.default_rng(1)
    for trial in range(20):
        m = int(rng.integers(1, 300))
        f = np.round(rng.standard_normal(m) * 3) / 4  # many exact ties
        f[rng.random(m) < 0.1] = -0.0
        idx = rng.permutation(10 * m)[:m].astype(np.int64)
        n = int(rng.integers(1, m + 5))
        got, gv = orc.topn(f, n, idx)
        order = np.lexsort((idx, -f))  # library: key -f ascending, then idx ascending
        want = idx[order][: min(n, m)]
        assert got.tolist() == want.tolist()
        assert np.array_equal(gv, f[order][: min(n, m)])


def test_topn_brute_force_selection(orc):
    """Top-n by repeated 'best remaining' selection (no sort) on tiny arrays."""
    rng = np.random.default_rng(2)
    for _ in range(50):
        m = int(rng.integers(1, 12))
        f = rng.integers(-3, 4, size=m).astype(np.float64)
        n = int(rng.integers(1, m + 2))
        left = list(range(m))
        want = []
        for _ in range(min(n, m)):
            best = left[0]
            for i in left[1:]:
                if f[i] > f[best] or (f[i] == f[best] and i < best):
                    best = i
            want.append(best)
            left.remove(best)
        got, _ = orc.topn(f, n)
        assert got.tolist() == want


# ----------------------------------------------------------------- Eq. 1 closed forms


def test_onehot_scores_closed_form(orc):
    L, H = 9, 3
    q, w, k = _onehot(L, H, 3)
    idx, val = orc.dense(q, w, k, L)
    for t in range(L):
        # q_{t,j} . e_s = q[t,j,s]  =>  I_{t,s} = sum_j w_{t,j} max(0, q[t,j,s])
        closed = np.array([sum(float(w[t, j]) * max(0.0, float(q[t, j, s])) for j in range(H))
                           for s in range(t + 1)])
        got = {int(s): v for s, v in zip(idx[t], val[t]) if s >= 0}
        assert sorted(got) == list(range(t + 1))
        for s, v in got.items():
            assert abs(v - closed[s]) <= 1e-12 * (1 + abs(closed[s]))


def test_relu_inside_head_sum(orc):
    """ReLU acts per head before the w-weighted sum: one head negative, one positive."""
    L, H, d = 2, 2, 2
    k = np.eye(2, dtype=np.float32)
    q = np.zeros((L, H, d), np.float32)
    q[1, 0] = [-4.0, 1.0]  # head 0: dot with k0 = -4, with k1 = 1
    q[1, 1] = [2.0, 3.0]   # head 1: dot with k0 = 2, with k1 = 3
    w = np.array([[1, 1], [1.0, 1.0]], np.float32)
    _, val = orc.dense(q, w, k, 2, 1, 2)
    # I_{1,0} = max(0,-4) + max(0,2) = 2 ; I_{1,1} = 1 + 3 = 4.  ReLU after the sum would give
    # max(0,-2) = 0 and 4; no ReLU gives -2 and 4.
    assert sorted(val[0].tolist()) == [2.0, 4.0]


def test_negative_w_and_zero_ties(orc):
    """All-zero queries with w < 0: every score is -0.0 -> lowest indices win."""
    L, H, d, topk = 20, 4, 8, 5
    q = np.zeros((L, H, d), np.float32)
    w = -np.ones((L, H), np.float32)
    k = np.random.default_rng(4).standard_normal((L, d)).astype(np.float32)
    idx, val = orc.dense(q, w, k, topk)
    for t in range(L):
        n = min(topk, t + 1)
        assert idx[t, :n].tolist() == list(range(n))
        assert (idx[t, n:] == -1).all()
        assert np.all(val[t, :n] == 0.0)


def test_duplicate_keys_lower_index(orc):
    """Equal keys give equal scores; the lower index must win."""
    L, H, d = 12, 2, 4
    q, w, k = _rand(L, H, d, 5)
    k[7] = k[2]
    k[9] = k[2]
    idx, val = orc.dense(q, w, k, 12)
    row = idx[11].tolist()
    assert row.index(2) < row.index(7) < row.index(9)


def test_scale_and_sign(orc):
    """Positive homogeneity: scaling every key by a>0 scales each score by a;
    flipping w's sign negates scores (and reverses the order of nonzero ones)."""
    L, H, d = 16, 3, 8
    q, w, k = _rand(L, H, d, 6)
    _, v1 = orc.dense(q, w, k, L, L - 1, L)
    _, v2 = orc.dense(q, w, (2.0 * k).astype(np.float32), L, L - 1, L)
    assert np.allclose(np.sort(v2[0]), np.sort(2.0 * v1[0]), rtol=1e-12, atol=0)
    _, v3 = orc.dense(q, (-w).astype(np.float32), k, L, L - 1, L)
    assert np.allclose(np.sort(v3[0]), np.sort(-v1[0]), rtol=1e-12, atol=0)


# ----------------------------------------------------------------- masks and counts


@pytest.mark.parametrize("dt", [np.float32, np.uint16])
def test_causal_and_counts(orc, dt):
    L, H, d, topk, c, g = 37, 3, 16, 6, 12, 4
    q, w, k = _rand(L, H, d, 7, dt)
    for name, res in (("dense", orc.dense(q, w, k, topk)[0]),
                      ("reuse", orc.reuse(q, w, k, topk, g)[0]),
                      ("refine", orc.refine(q, w, k, topk, c, g)[0])):
        for t in range(L):
            n = min(topk, t + 1)  # c >= k + g - 1 here, so Refine rows are full too
            v = res[t][res[t] >= 0]
            assert v.size == n, (name, t)
            assert (v <= t).all(), (name, t)
            assert len(set(v.tolist())) == n
            assert (res[t, n:] == -1).all()


def test_refine_candidates_within_group_prefix(orc):
    """Eq. 7 candidates come from s <= group end; members then mask s <= t."""
    L, H, d, topk, c, g = 40, 2, 8, 3, 6, 8
    q, w, k = _rand(L, H, d, 8)
    _, _, cand, _ = orc.refine(q, w, k, topk, c, g)
    for i in range(cand.shape[0]):
        e = min(i * g + g, L) - 1
        v = cand[i][cand[i] >= 0]
        assert v.size == min(c, e + 1)
        assert (v <= e).all()
    # The last member of a group sees the in-group keys: with c >= L, row e equals dense row e.
    idx_r, _, _, _ = orc.refine(q, w, k, topk, L, g)
    idx_d, _ = orc.dense(q, w, k, topk)
    assert np.array_equal(idx_r, idx_d)


# ----------------------------------------------------------------- reductions


@pytest.mark.parametrize("dt", [np.float32, np.uint16])
def test_reuse_g1_is_dense(orc, dt):
    L, H, d, topk = 45, 4, 16, 7
    q, w, k = _rand(L, H, d, 9, dt)
    a, av = orc.reuse(q, w, k, topk, 1)
    b, bv = orc.dense(q, w, k, topk)
    assert np.array_equal(a, b)
    assert np.array_equal(np.nan_to_num(av, nan=7.0), np.nan_to_num(bv, nan=7.0))


@pytest.mark.parametrize("dt", [np.float32, np.uint16])
@pytest.mark.parametrize("g", [1, 3, 4])
def test_refine_c_ge_L_is_dense(orc, dt, g):
    L, H, d, topk = 33, 3, 8, 5
    q, w, k = _rand(L, H, d, 10, dt)
    a, av, _, _ = orc.refine(q, w, k, topk, L, g)
    b, bv = orc.dense(q, w, k, topk)
    assert np.array_equal(a, b)
    assert np.array_equal(np.nan_to_num(av, nan=7.0), np.nan_to_num(bv, nan=7.0))


def test_refine_g1_is_dense(orc):
    L, H, d, topk, c = 50, 3, 8, 4, 8
    q, w, k = _rand(L, H, d, 11, np.uint16)
    a, _, _, _ = orc.refine(q, w, k, topk, c, 1)
    b, _ = orc.dense(q, w, k, topk)
    assert np.array_equal(a, b)


def test_identical_members_reuse_is_dense(orc):
    """If every member of a group has the same q and w, the proxy equals them exactly."""
    L, H, d, topk, g = 32, 3, 8, 5, 4
    q, w, k = _rand(L, H, d, 12, np.uint16)
    for i in range(L // g):
        q[i * g:(i + 1) * g] = q[i * g]
        w[i * g:(i + 1) * g] = w[i * g]
    a, _ = orc.reuse(q, w, k, topk, g)
    b, _ = orc.dense(q, w, k, topk)
    assert np.array_equal(a, b)


def test_reuse_topk_plus_g_minus_1_shortcut(orc):
    """Eq. 6 per-member sort equals: proxy top-(k+g-1) over s <= e, drop s > t, keep k."""
    L, H, d, topk, g = 53, 3, 8, 6, 5
    q, w, k = _rand(L, H, d, 13, np.uint16)
    idx, _ = orc.reuse(q, w, k, topk, g)
    for i in range((L + g - 1) // g):
        f = orc.proxy_scores(q, w, k, g, i)
        top, _ = orc.topn(f, topk + g - 1)
        for t in range(i * g, min(i * g + g, L)):
            want = [s for s in top.tolist() if s <= t][:topk]
            got = idx[t][idx[t] >= 0].tolist()
            assert got == want, (i, t)


def test_partial_last_group(orc):
    """L % g != 0: the last group pools only its real members (here one -> equals dense)."""
    L, H, d, topk, g = 21, 2, 8, 4, 4
    q, w, k = _rand(L, H, d, 14, np.uint16)
    a, _ = orc.reuse(q, w, k, topk, g)
    b, _ = orc.dense(q, w, k, topk)
    assert np.array_equal(a[20], b[20])


# ----------------------------------------------------------------- pooling (Eq. 4)


def test_mean_divisor(orc):
    """Members 2x and 0 pool to x exactly, w likewise (a sum would give 2x)."""
    L, H, d = 2, 2, 4
    k = np.eye(d, dtype=np.float32)
    x = np.array([[0.5, -1.25, 3.0, 0.0], [2.0, 0.75, -0.5, 1.0]], np.float32)
    q = np.zeros((L, H, d), np.float32)
    q[0] = 2 * x
    w = np.array([[1.5, -0.5], [0.0, 0.0]], np.float32)
    qb, wb = orc.proxy(q, w, [0, 1])
    assert qb.reshape(H, d).tolist() == x.tolist()
    assert wb.tolist() == [0.75, -0.25]
    f = orc.proxy_scores(q, w, k[:L], 2, 0)
    closed = [0.75 * max(0.0, x[0, s]) - 0.25 * max(0.0, x[1, s]) for s in range(L)]
    assert f.tolist() == closed


def test_bf16_rounding_of_mean(orc):
    """bf16 inputs: the mean is rounded to nearest even bf16 (the scan's operand)."""
    one = 1.0
    ulp = 2.0 ** -7
    cases = [
        ((one, one + ulp), one),                    # halfway, 1.0 is even -> down
        ((one + ulp, one + 2 * ulp), one + 2 * ulp),  # halfway, odd below -> up
        ((one, one + 2 * ulp), one + ulp),          # exact
        ((-one, -(one + ulp)), -one),               # sign symmetric
    ]
    for (a, b), want in cases:
        q = inputs.to_bf16_bits(np.array([a, b], np.float32).reshape(2, 1, 1))
        w = np.ones((2, 1), np.float32)
        qb, _ = orc.proxy(q, w, [0, 1])
        assert qb[0] == want, (a, b, qb[0], want)
    # a mean of three needs true rounding: (1 + 1 + (1+ulp)) / 3 = 1 + ulp/3 -> 1.0
    q = inputs.to_bf16_bits(np.array([one, one, one + ulp], np.float32).reshape(3, 1, 1))
    qb, _ = orc.proxy(q, np.ones((3, 1), np.float32), [0, 1, 2])
    assert qb[0] == one


# ----------------------------------------------------------------- decode (Eq. 3)


@pytest.mark.parametrize("variant", [0, 1])
def test_decode_mirrors_prefill_last_group(orc, variant):
    """A decode sequence whose keys are a prefill prefix and whose g rows are that
    prefix's last g queries gives the prefill result of the last group."""
    L, H, d, topk, c, g = 24, 3, 8, 4, 8, 4
    q, w, k = _rand(L, H, d, 15, np.uint16)
    P = [24, 16]
    kc = np.concatenate([k[:P[0]], k[:P[1]]])
    off = np.array([0, P[0], P[0] + P[1]], np.int64)
    qd = np.concatenate([q[P[0] - g:P[0]], q[P[1] - g:P[1]]])
    wd = np.concatenate([w[P[0] - g:P[0]], w[P[1] - g:P[1]]])
    got, _, _, _ = orc.decode(qd, wd, kc, off, topk, c, g, variant)
    for b, p in enumerate(P):
        qq, ww, kk = q[:p], w[:p], k[:p]
        if variant == 0:
            want, _ = orc.reuse(qq, ww, kk, topk, g)
        else:
            want, _, _, _ = orc.refine(qq, ww, kk, topk, c, g)
        assert np.array_equal(got[b * g:(b + 1) * g], want[p - g:p])


# ----------------------------------------------------------------- generators


def test_generator_shapes_and_determinism():
    spec = inputs.PrefillSpec("t", L=64, H=4, d=32, k=4, c=8, g=4, seed=3)
    a = inputs.make_prefill(spec, chunk=16)
    b = inputs.make_prefill(spec, chunk=16)  # same seed, same draw (threads do not matter)
    assert a["q"].shape == (64, 4, 32) and a["q"].dtype == np.uint16
    assert a["k"].shape == (64, 32) and a["w"].shape == (64, 4)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["k"], b["k"])
    assert np.array_equal(a["w"], b["w"])
    # the chunk carry makes the rows one AR(1) chain: q_t - rho q_{t-1} is the innovation,
    # whose variance is 1/d, also across a chunk boundary (rows 15 -> 16)
    qf = inputs.make_prefill(
        inputs.PrefillSpec("t", L=64, H=64, d=32, k=4, c=8, g=4, dtype=inputs.F32, seed=3), chunk=16)["q"]
    innov = qf[1:] - np.float32(0.95) * qf[:-1]
    assert abs(innov[15].var() * 32 - 1) < 0.3
    assert abs(innov[20].var() * 32 - 1) < 0.3
    ds = inputs.DecodeSpec("d", B=3, p_lo=10, p_hi=20, H=2, d=16, k=2, c=4, g=4, seed=5)
    x = inputs.make_decode(ds)
    assert x["q"].shape == (12, 2, 16) and x["k"].shape[0] == x["offsets"][-1]
    assert np.array_equal(x["w"][0], x["w"][3])


def test_bf16_bits_rne():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], np.float32)
    back = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(v))
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 * 2 ** -7, -2.5]


def test_sample_groups_edges():
    s = inputs.sample_groups(16384, 8, 2048, 4096, 256, 7)
    assert s.size == 256 and s[0] == 0 and s[-1] == 16383
    assert 511 in s and 256 in s  # P_i straddles c=4096 and k+g-1=2055


# ---------------------------------------------------------------- proxy aggregation (Table 2 variants)


@pytest.mark.parametrize("dt", [inputs.F32, inputs.BF16])
@pytest.mark.parametrize("mode,member", [("first", 0), ("last", -1)])
def test_single_query_proxy_member_row_is_dense(orc, dt, mode, member):
    """With a first- (last-) query proxy, that member's Reuse row ranks its own
    query's scores over s <= t: exactly its dense row, bit for bit."""
    L, g, topk = 61, 4, 9
    x = inputs.random_prefill(L, 3, 16, dt, seed=83)
    di, dv = orc.dense(x["q"], x["w"], x["k"], topk)
    try:
        orc.set_aggregation(mode)
        ui, uv = orc.reuse(x["q"], x["w"], x["k"], topk, g)
    finally:
        orc.set_aggregation("mean")
    G = (L + g - 1) // g
    rows = [min(i * g + g, L) - 1 if member == -1 else i * g for i in range(G)]
    assert np.array_equal(ui[rows], di[rows])
    assert np.array_equal(np.nan_to_num(uv[rows], nan=7.0), np.nan_to_num(dv[rows], nan=7.0))
    # the other members rank the proxy's scores, not their own
    other = [i * g + 1 for i in range(G) if i * g + 1 < L and i * g + 1 not in rows]
    assert any(not np.array_equal(ui[t], di[t]) for t in other)


@pytest.mark.parametrize("mode", ["first", "last"])
def test_aggregation_reductions(orc, mode):
    """g = 1: every aggregation is the query itself (Reuse = dense).  c >= L: the
    candidate set is the whole prefix whatever the proxy (Refine = dense)."""
    L, topk = 40, 7
    x = inputs.random_prefill(L, 4, 16, inputs.F32, seed=84)
    di, dv = orc.dense(x["q"], x["w"], x["k"], topk)
    try:
        orc.set_aggregation(mode)
        ui, uv = orc.reuse(x["q"], x["w"], x["k"], topk, 1)
        ri, rv, _, _ = orc.refine(x["q"], x["w"], x["k"], topk, L, 4)
    finally:
        orc.set_aggregation("mean")
    nz = lambda v: np.nan_to_num(v, nan=7.0)  # short rows are NaN padded
    assert np.array_equal(ui, di) and np.array_equal(nz(uv), nz(dv))
    assert np.array_equal(ri, di) and np.array_equal(nz(rv), nz(dv))


# ----------------------------------------------------------------- the batch scorer used by the GPU checks


def test_scores_batch_prefix_form_hand_example(orc):
    """Prefix form (plen): row t of the hand-worked example holds I_{t,s} for s <= t, as
    derived by hand in the golden file, and NaN past its prefix."""
    q, w, k = _hand()
    L = q.shape[0]
    qv, wv = orc.query_rows(q, w, range(L))
    F = orc.scores_batch(qv, wv, k, plen=np.arange(L) + 1)
    assert F.shape == (L, L)
    for t in range(L):
        assert F[t, :t + 1].tolist() == GOLD["dense_scores"][t][:t + 1]
        assert np.isnan(F[t, t + 1:]).all()


def test_scores_batch_key_rows_form_closed_form(orc):
    """key_rows form: entry i scores key key_rows[r, i] (NaN where it is -1).  With one-hot
    keys k_s = e_s the score has the closed form sum_j w_j max(0, q_{j,s})."""
    L, H = 11, 3
    q, w, k = _onehot(L, H, 21)
    rows = [2, 7, 10]
    qv, wv = orc.query_rows(q, w, rows)
    rng = np.random.default_rng(22)
    kr = rng.integers(0, L, size=(len(rows), 6))
    kr[0, 1] = -1
    kr[2, 4] = -1
    kr[1, 5] = -1
    F = orc.scores_batch(qv, wv, k, key_rows=kr)
    for r, t in enumerate(rows):
        for i, s in enumerate(kr[r]):
            if s < 0:
                assert np.isnan(F[r, i])
                continue
            closed = sum(float(w[t, j]) * max(0.0, float(q[t, j, s])) for j in range(H))
            assert abs(F[r, i] - closed) <= 1e-12 * (1 + abs(closed)), (r, i)


def test_scores_batch_key_base_offsets_each_vector(orc):
    """key_base: vector r reads its keys from row key_base[r] on, in both forms.  The keys
    are a block of filler rows followed by one-hot rows, so only the right offset lands on
    the closed form; a vector with base 0 must see the filler instead."""
    H, n1 = 2, 7
    rng = np.random.default_rng(23)
    filler = (rng.standard_normal((5, n1)) + 3.0).astype(np.float32)
    k = np.concatenate([filler, np.eye(n1, dtype=np.float32)])
    qv = rng.standard_normal((3, H * n1))
    wv = rng.standard_normal((3, H))
    base = np.array([5, 5, 0])
    Fp = orc.scores_batch(qv, wv, k, plen=np.array([n1, 4, n1]), key_base=base)
    kr = np.array([[0, 3, 6], [6, -1, 1], [0, 1, 2]])
    Fk = orc.scores_batch(qv, wv, k, key_rows=kr, key_base=base, m=3)
    for r in range(2):  # one-hot block at rows 5..11
        qq = qv[r].reshape(H, n1)
        closed = [sum(wv[r, j] * max(0.0, qq[j, s]) for j in range(H)) for s in range(n1)]
        plen = (n1, 4)[r]
        assert np.allclose(Fp[r, :plen], closed[:plen], rtol=1e-12, atol=1e-12)
        assert np.isnan(Fp[r, plen:]).all()
        for i, s in enumerate(kr[r]):
            assert np.isnan(Fk[r, i]) if s < 0 else abs(Fk[r, i] - closed[s]) <= 1e-12
    # base 0: filler rows, whose scores are the plain double dot products
    qq = qv[2].reshape(H, n1)
    want = [sum(wv[2, j] * max(0.0, float(np.dot(qq[j].astype(np.float64), filler[s].astype(np.float64))))
                for j in range(H)) for s in range(3)]
    assert np.allclose(Fk[2], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dt", [np.float32, np.uint16])
def test_scores_batch_agrees_with_the_pinned_entry_points(orc, dt):
    """The batch scorer reproduces what the pinned calls return: the dense indexer's row
    scores, the proxy scores of a group (prefix form) and a Refine member row's scores
    over its candidate set (key_rows form), value for value."""
    L, H, d, topk, c, g = 45, 3, 16, 7, 14, 4
    q, w, k = _rand(L, H, d, 24, dt)
    didx, dval = orc.dense(q, w, k, topk)
    rows = [0, 13, 44]
    qv, wv = orc.query_rows(q, w, rows)
    F = orc.scores_batch(qv, wv, k, plen=np.array(rows) + 1)
    for r, t in enumerate(rows):
        for s, v in zip(didx[t], dval[t]):
            if s >= 0:
                assert F[r, s] == v
    groups = [0, 5, (L + g - 1) // g - 1]
    mem = [list(range(i * g, min(i * g + g, L))) for i in groups]
    pq, pw = orc.proxies(q, w, mem)
    Fp = orc.scores_batch(pq, pw, k, plen=np.array([m[-1] + 1 for m in mem]))
    for r, i in enumerate(groups):
        ps = orc.proxy_scores(q, w, k, g, i)
        assert np.array_equal(Fp[r, :ps.size], ps)
    ridx, rval, cand, _ = orc.refine(q, w, k, topk, c, g)
    t = 22
    grp = t // g
    qv, wv = orc.query_rows(q, w, [t])
    C = cand[grp:grp + 1].astype(np.int64)
    M = orc.scores_batch(qv, wv, k, key_rows=C)
    for s, v in zip(ridx[t], rval[t]):
        if s >= 0:
            assert M[0, list(C[0]).index(s)] == v
