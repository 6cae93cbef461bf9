"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, a library routine,
brute force on tiny inputs, a published known-answer vector, or a statistical
law -- chosen so that a dropped term, a wrong sign, a swapped operand or a
miswired counter in the oracle fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x):
    """Round-to-nearest-even float32 -> bf16 bit patterns (uint16)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- Philox

def test_philox_known_answers(oracle_lib):
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(t, 16) for t in line.split()])
    assert len(rows) == 3
    for r in rows:
        out = O.philox4x32_10(r[0:4], r[4:6])
        assert [int(x) for x in out] == r[6:10]


def test_draw_word_is_keyed_by_seed_halves(oracle_lib):
    seed = 0x0123456789ABCDEF
    direct = O.philox4x32_10([5, 6, 7, 8], [seed & 0xFFFFFFFF, seed >> 32])
    for w in range(4):
        assert O.draw_word(seed, 5, 6, 7, 8, w) == int(direct[w])


# ----------------------------------------------------------------------------- uniform / Gumbel

def test_uniform_range_and_grid(oracle_lib):
    assert O.uniform(0) == 2.0 ** -24
    assert O.uniform(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    # (2k + 1) 2^-24 with k the top 23 bits
    for x in (0x200, 0x12345678, 0x80000000):
        assert O.uniform(x) == (2 * (x >> 9) + 1) * 2.0 ** -24


def test_gumbel_inverts_its_cdf(oracle_lib):
    for x in (0, 1 << 9, 0x40000000, 0x80000000, 0xFFFFFFFF):
        g = O.gumbel(x)
        assert math.exp(-math.exp(-g)) == pytest.approx(O.uniform(x), rel=1e-12)


def test_uniform_token_exact_mapping(oracle_lib):
    rng = np.random.default_rng(0)
    for x in rng.integers(0, 2 ** 32, 200, dtype=np.uint64):
        x = int(x)
        assert O.uniform_token(x, 1024) == x >> 22          # V = 2^10: top 10 bits
        assert O.uniform_token(x, 262144) == x >> 14
        assert O.uniform_token(x, 262000) == (x * 262000) >> 32
    assert O.uniform_token(0xFFFFFFFF, 7) == 6


def test_renoise_tokens_uniform_chi_square(oracle_lib):
    V = 1024
    cfg = O.Config(B=1, L=V * 64, V=V, seed=11)
    st = O.State(cfg).init()  # initial canvas uses the same token mapping
    counts = np.bincount(st.canvas[0], minlength=V)
    assert st.canvas.min() >= 0 and st.canvas.max() < V
    chi = scipy.stats.chisquare(counts)
    assert chi.pvalue > 1e-3


# ----------------------------------------------------------------------------- temperature

def test_temperature_schedule(oracle_lib):
    cfg = O.Config(num_steps=48)
    T = [O.temperature(cfg, s) for s in range(48)]
    assert T[0] == pytest.approx(0.8, abs=1e-15)
    assert T[47] == pytest.approx(0.4, abs=1e-15)
    d = np.diff(T)
    assert np.allclose(d, -0.4 / 47, atol=1e-15)
    assert O.temperature(O.Config(num_steps=1), 0) == 0.8
    assert O.temperature(O.Config(greedy=1), 5) == 1.0


# ----------------------------------------------------------------------------- entropy

@pytest.mark.parametrize("V", [7, 1024, 262144])
@pytest.mark.parametrize("T", [0.4, 0.8, 1.0])
def test_entropy_uniform_logits_is_log_V(oracle_lib, V, T):
    row = np.full(V, 1.25, np.float32)
    H, pmax, amax, Hd = O.row_stats(row, 1.0 / T)
    assert H == pytest.approx(math.log(V), abs=1e-9)
    assert Hd == pytest.approx(math.log(V), abs=1e-9)
    assert pmax == pytest.approx(1.0 / V, rel=1e-12)
    assert amax == 0  # lowest index among equal maxima


def test_entropy_one_hot_is_zero(oracle_lib):
    row = np.full(1000, -1e4, np.float32)
    row[417] = 0.0
    H, pmax, amax, _ = O.row_stats(row, 1.0 / 0.8)
    assert abs(H) < 1e-12 and pmax == pytest.approx(1.0, abs=1e-12) and amax == 417


@pytest.mark.parametrize("a,b,T", [(0.0, 0.0, 0.8), (1.5, -0.5, 0.8), (3.0, 2.0, 0.4), (-2, 5, 1.0)])
def test_entropy_two_tokens_is_binary_entropy(oracle_lib, a, b, T):
    row = np.full(64, -1e4, np.float32)
    row[10], row[20] = a, b
    p = 1.0 / (1.0 + math.exp(-(a - b) / T))
    hb = -(p * math.log(p) + (1 - p) * math.log(1 - p))
    H, pmax, amax, _ = O.row_stats(row, 1.0 / T)
    assert H == pytest.approx(hb, abs=1e-12)
    assert pmax == pytest.approx(max(p, 1 - p), abs=1e-12)
    assert amax == (10 if a >= b else 20)


def test_entropy_matches_scipy_on_random_rows(oracle_lib):
    rng = np.random.default_rng(1)
    for V, scale in [(50, 1.0), (1000, 3.0), (4096, 0.3), (20000, 5.0)]:
        z = (rng.standard_normal(V) * scale).astype(np.float32)
        for T in (0.4, 0.63, 0.8):
            H, pmax, amax, Hd = O.row_stats(z, 1.0 / T)
            p = scipy.special.softmax(z.astype(np.float64) / T)
            assert H == pytest.approx(scipy.stats.entropy(p), abs=1e-10)
            assert Hd == pytest.approx(H, abs=1e-10)
            assert pmax == pytest.approx(p.max(), rel=1e-10)
            assert amax == int(np.argmax(z))


def test_entropy_temperature_scaling_identity(oracle_lib):
    rng = np.random.default_rng(2)
    z = (rng.standard_normal(3000) * 2).astype(np.float64)
    for T in (0.4, 0.55, 0.8):
        zs = (z / T).astype(np.float32)
        H1, *_ = O.row_stats(z.astype(np.float32), 1.0 / T)
        H2, *_ = O.row_stats(zs, 1.0)
        assert H1 == pytest.approx(H2, abs=1e-5)  # float32 rounding of z/T only


def test_bf16_rows_decode_exactly(oracle_lib):
    rng = np.random.default_rng(3)
    z = (rng.standard_normal(5000) * 4).astype(np.float32)
    bits = bf16_bits(z)
    zf = bf16_to_f32(bits)
    a = O.row_stats(bits, 1.0 / 0.7)
    b = O.row_stats(zf, 1.0 / 0.7)
    assert a == b


def test_entropy_bounds_on_random_rows(oracle_lib):
    rng = np.random.default_rng(4)
    for _ in range(20):
        V = int(rng.integers(2, 3000))
        z = (rng.standard_normal(V) * rng.uniform(0.1, 10)).astype(np.float32)
        H, pmax, _, _ = O.row_stats(z, 1.0 / rng.uniform(0.3, 1.0))
        assert -1e-12 <= H <= math.log(V) + 1e-9
        assert 1.0 / V - 1e-15 <= pmax <= 1.0


# ----------------------------------------------------------------------------- Gumbel-max draw

def _chi_square_draws(cfg, z, T, n):
    counts = np.zeros(cfg.V, np.int64)
    for k in range(n):
        x, _, _ = O.sample(cfg, z, 1.0 / T, 0, k % 50000, k // 50000)
        counts[x] += 1
    p = scipy.special.softmax(z.astype(np.float64) / T)
    keep = p * n >= 5
    exp_ = p * n
    obs = np.append(counts[keep], counts[~keep].sum())
    ex = np.append(exp_[keep], exp_[~keep].sum())
    if ex[-1] == 0:
        obs, ex = obs[:-1], ex[:-1]
    return scipy.stats.chisquare(obs, ex)


@pytest.mark.parametrize("G", [1, 8, 64])
def test_two_level_gumbel_draw_follows_softmax(oracle_lib, G):
    rng = np.random.default_rng(5)
    V = 64
    z = (rng.standard_normal(V) * 1.5).astype(np.float32)
    cfg = O.Config(B=1, L=1, V=V, group_size=G, seed=99)
    res = _chi_square_draws(cfg, z, 0.7, 100000)
    assert res.pvalue > 1e-3, res


def test_two_level_equals_flat_when_one_group(oracle_lib):
    rng = np.random.default_rng(6)
    V = 300
    z = (rng.standard_normal(V) * 2).astype(np.float32)
    one = O.Config(B=1, L=1, V=V, group_size=512, seed=7)
    for k in range(300):
        a, ma, g = O.sample(one, z, 1 / 0.6, 0, k, 3)
        b, mb = O.sample_flat(one, z, 1 / 0.6, 0, k, 3)
        assert a == b and g == 0


def test_flat_draw_matches_counter_layout(oracle_lib):
    """Recompute a flat draw from raw Philox words with the documented counters."""
    V, l, s, b, seed, T = 40, 3, 9, 2, 0xABCDEF12345, 0.8
    rng = np.random.default_rng(7)
    z = rng.standard_normal(V).astype(np.float32)
    cfg = O.Config(B=4, L=8, V=V, seed=seed, group_size=64)
    best, arg = -np.inf, -1
    for v in range(V):
        w = O.philox4x32_10([v >> 2, l, s, b | (0 << 24)], [seed & 0xFFFFFFFF, seed >> 32])[v & 3]
        u = (2 * (int(w) >> 9) + 1) * 2.0 ** -24
        sc = float(z[v]) / T - math.log(-math.log(u))
        if sc > best:
            best, arg = sc, v
    assert O.sample_flat(cfg, z, 1 / T, b, l, s)[0] == arg


def test_group_draw_uses_group_stream(oracle_lib):
    """With group_size 1 the group level alone decides, from the group stream."""
    V, l, s, b, seed, T = 33, 1, 4, 0, 77, 0.5
    z = np.random.default_rng(8).standard_normal(V).astype(np.float32)
    cfg = O.Config(B=1, L=4, V=V, seed=seed, group_size=1)
    best, arg = -np.inf, -1
    for j in range(V):
        w = O.philox4x32_10([j >> 2, l, s, b | (3 << 24)], [seed, 0])[j & 3]
        sc = float(z[j]) / T + O.gumbel(int(w))
        if sc > best:
            best, arg = sc, j
    tok, _, grp = O.sample(cfg, z, 1 / T, b, l, s)
    assert tok == arg and grp == arg


def test_element_draw_in_a_later_group_uses_global_ids(oracle_lib):
    """The element level of the two-level draw, when the winning group is not
    group 0: recomputed from raw Philox words whose counters carry the GLOBAL
    vocabulary id v (ctr = (v >> 2, l, s, b), word v & 3).  One group holds
    logits 40 above every other, so the group level always picks it; a
    local-id counter (v - 64 j*) would draw other tokens, which the second
    half of the test checks."""
    V, G, seed, T = 640, 64, 0x5EED0BADC0FFEE, 0.7
    rng = np.random.default_rng(17)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    n_local_differs = 0
    for trial in range(24):
        jstar = 1 + trial % 9  # groups 1 .. 9
        z = (rng.standard_normal(V) - 40.0).astype(np.float32)
        z[jstar * G:(jstar + 1) * G] += 40.0
        l, s, b = trial % 7, 3 + trial, 2 + trial % 5
        cfg = O.Config(B=8, L=8, V=V, seed=seed, group_size=G)
        tok, _, grp = O.sample(cfg, z, 1 / T, b, l, s)
        assert grp == jstar

        def draw(local):
            best, arg = -np.inf, -1
            for v in range(jstar * G, (jstar + 1) * G):
                vc = v - jstar * G if local else v
                w = int(O.philox4x32_10([vc >> 2, l, s, b], key)[vc & 3])
                u = (2 * (w >> 9) + 1) * 2.0 ** -24
                sc = float(z[v]) / T - math.log(-math.log(u))
                if sc > best:
                    best, arg = sc, v
            return arg

        assert tok == draw(local=False)
        n_local_differs += draw(local=True) != tok
    assert n_local_differs >= 12  # the pin tells the two counter layouts apart


def test_initial_canvas_matches_raw_philox_words(oracle_lib):
    """Initial canvas token of (b, l): word l & 3 of Philox4x32-10 at
    ctr = (l >> 2, 0, 0, b | 2 << 24) with b the GLOBAL canvas index
    (canvas_offset + local index), mapped to (x * V) >> 32; nothing
    committed, stop flag clear."""
    for V, seed, off in ((1024, 11, 0), (262144, 0xFEEDFACE12345678, 7), (1000, 3, 1 << 20)):
        L, B = 37, 3
        cfg = O.Config(B=B, L=L, V=V, seed=seed, canvas_offset=off)
        st = O.State(cfg).init()
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for bl in range(B):
            bg = off + bl
            for l in range(L):
                w = int(O.philox4x32_10([l >> 2, 0, 0, bg | (2 << 24)], key)[l & 3])
                assert st.canvas[bl, l] == (w * V) >> 32, (V, bl, l)
        assert not st.committed.any() and not st.stop.any() and not st.stable.any()


def test_argmax_ties_take_the_lowest_index(oracle_lib):
    """Equal maxima: the argmax is the first of them (within one group, across
    groups, and across a group boundary)."""
    V = 300
    for where in ([5, 6], [5, 200], [63, 64], [0, 299], [130, 131, 140]):
        row = np.zeros(V, np.float32)
        row[where] = 3.5
        _, pmax, amax, _ = O.row_stats(row, 1.0 / 0.8)
        assert amax == min(where)
        # k equal maxima of e^(3.5/T) among V - k ones
        e = math.exp(3.5 / 0.8)
        assert pmax == pytest.approx(e / (len(where) * e + V - len(where)), rel=1e-12)


@pytest.mark.parametrize("k", [1, 3, 64, 100])
def test_masked_row_is_the_softmax_of_the_finite_logits(oracle_lib, k):
    """-inf logits drop out: k equal finite logits among -inf ones give
    H = ln k and pmax = 1/k, the argmax is the first finite one, and no draw
    lands on a masked token."""
    V = 500
    rng = np.random.default_rng(k)
    finite = np.sort(rng.choice(V, size=k, replace=False))
    row = np.full(V, -np.inf, np.float32)
    row[finite] = 1.25
    for T in (0.4, 1.0):
        H, pmax, amax, _ = O.row_stats(row, 1.0 / T)
        assert H == pytest.approx(math.log(k), abs=1e-12)
        assert pmax == pytest.approx(1.0 / k, rel=1e-12)
        assert amax == finite[0]
    cfg = O.Config(B=1, L=4, V=V)
    drawn = {O.sample(cfg, row, 1.0 / 0.8, 0, l, s)[0] for l in range(4) for s in range(60)}
    assert drawn <= set(finite.tolist())
    if k > 1:
        assert len(drawn) > 1  # equal logits: the draw is not stuck on one token


def test_single_token_vocabulary(oracle_lib):
    """V = 1: entropy 0, pmax 1, argmax 0, and every draw is token 0."""
    cfg = O.Config(B=1, L=2, V=1)
    for z in (-3.0, 0.0, 7.5):
        row = np.array([z], np.float32)
        H, pmax, amax, _ = O.row_stats(row, 1.0 / 0.4)
        assert H == 0.0 and pmax == 1.0 and amax == 0
        assert all(O.sample(cfg, row, 1.0 / 0.4, 0, l, s)[0] == 0 for l in range(2)
                   for s in range(5))


def test_single_finite_logit_is_always_drawn(oracle_lib):
    V = 1000
    cfg = O.Config(B=1, L=8, V=V)
    for j in (0, 63, 64, 999):
        row = np.full(V, -np.inf, np.float32)
        row[j] = -40.0
        assert O.row_stats(row, 1.0)[2] == j
        assert all(O.sample(cfg, row, 1.0 / 0.8, 0, l, s)[0] == j for l in range(8)
                   for s in range(4))


def test_draw_concentrates_on_dominant_token(oracle_lib):
    z = np.zeros(4096, np.float32)
    z[1234] = 60.0
    cfg = O.Config(B=1, L=1, V=4096, seed=1)
    for k in range(50):
        assert O.sample(cfg, z, 1 / 0.8, 0, k, 0)[0] == 1234


# ----------------------------------------------------------------------------- commit rules

def _decide_all_open(rule, H, pmax=None, gamma=0.1, theta=0.9, quota=2, s=0, N=48):
    L = len(H)
    cfg = O.Config(B=1, L=L, V=1000, num_steps=N, rule=rule, entropy_bound=gamma,
                   stop_entropy=-1.0, threshold=theta, quota=quota)
    st = O.State(cfg).init()
    amax = np.arange(L, dtype=np.int32) + 100
    smp = np.arange(L, dtype=np.int32) + 500
    pm = np.zeros(L) if pmax is None else np.asarray(pmax, np.float64)
    before = st.canvas[0].copy()
    mg = O.canvas_decide(st, 0, s, np.asarray(H, np.float64), amax, pm, smp)
    return st, mg, before, smp


def test_eb_commit_matches_brute_force(oracle_lib):
    rng = np.random.default_rng(9)
    for trial in range(400):
        L = int(rng.integers(1, 9))
        H = np.round(rng.exponential(rng.choice([0.01, 0.05, 0.3]), L), 6)
        st, mg, _, smp = _decide_all_open(O.RULE_EB, H)
        got = set(np.nonzero(st.committed[0])[0].tolist())
        # brute force: the largest subset with sum <= gamma; among those the smallest sum
        best = None
        for k in range(L, -1, -1):
            cands = [c for c in itertools.combinations(range(L), k) if H[list(c)].sum() <= 0.1]
            if cands:
                best = min(cands, key=lambda c: (H[list(c)].sum(), sorted(H[list(c)]), c))
                break
        if len(best) == 0:  # nothing fits: the single lowest-entropy position
            best = (int(np.lexsort((np.arange(L), H))[0]),)
        exp_set = set(best)
        sums = [H[list(c)].sum() for c in itertools.combinations(range(L), len(best))]
        unique = sorted(sums).count(min(sums)) == 1
        if unique:
            assert got == exp_set, (H, got, exp_set)
        else:
            assert len(got) == len(exp_set)
        assert len(got) >= 1
        for l in got:
            assert st.canvas[0, l] == smp[l]


def test_eb_mi_commit_matches_brute_force(oracle_lib):
    rng = np.random.default_rng(10)
    for trial in range(300):
        L = int(rng.integers(1, 9))
        H = np.round(rng.exponential(rng.choice([0.02, 0.08, 0.3]), L), 6)
        st, mg, _, _ = _decide_all_open(O.RULE_EB_MI, H)
        got = np.nonzero(st.committed[0])[0].tolist()
        k_best = 0
        for k in range(1, L + 1):
            for c in itertools.combinations(range(L), k):
                h = H[list(c)]
                if h.sum() - h.max() <= 0.1:
                    k_best = max(k_best, k)
        assert len(got) == k_best
        h = H[got]
        assert h.sum() - h.max() <= 0.1 + 1e-15
        # the committed set is a lowest-entropy prefix
        if len(got) < L:
            rest = np.delete(H, got)
            assert h.max() <= rest.min()


def test_br_commit_threshold_plus_quota(oracle_lib):
    rng = np.random.default_rng(11)
    for trial in range(200):
        L = int(rng.integers(1, 9))
        p = np.round(rng.uniform(0, 1, L), 4)
        q = int(rng.integers(0, 4))
        st, mg, _, smp = _decide_all_open(O.RULE_BR, np.ones(L), pmax=p, quota=q)
        got = set(np.nonzero(st.committed[0])[0].tolist())
        over = {i for i in range(L) if p[i] >= 0.9}
        rest = sorted((i for i in range(L) if p[i] < 0.9), key=lambda i: (-p[i], i))
        assert got == over | set(rest[:q])


def test_br_editing_threshold_reedits_confident_committed_positions(oracle_lib):
    """BlockRefinement with editing (diffusers "DiffusionGemma", Schedulers:
    editing_threshold lets the scheduler re-edit committed tokens), as read
    here: a position committed before the step whose argmax differs from its
    token takes the argmax iff its pmax >= editing_threshold; it stays
    committed; open positions follow the ordinary rule."""
    L = 6
    cfg = O.Config(B=1, L=L, V=1000, rule=O.RULE_BR, stop_entropy=-1.0, threshold=0.9,
                   quota=1, greedy=1, editing_threshold=0.6)
    st = O.State(cfg).init()
    st.committed[0, :4] = 1
    st.canvas[0, :4] = [10, 11, 12, 13]
    amax = np.array([20, 21, 12, 23, 24, 25], np.int32)
    pmax = np.array([0.61, 0.59, 0.99, 0.6, 0.2, 0.1])
    H = np.full(L, 0.5)
    mg = O.canvas_decide(st, 0, 3, H, amax, pmax, np.zeros(L, np.int32))
    # 0: differs, confident -> edited; 1: below the threshold -> kept;
    # 2: argmax equals the token -> untouched; 3: pmax == threshold -> edited
    assert st.canvas[0, :4].tolist() == [20, 11, 12, 23]
    assert st.committed[0, :4].all()
    assert mg["n_edit"] == 2
    assert abs(mg["edit_margin"] - 0.0) < 1e-12  # position 3 sits on the threshold
    # the open positions: quota 1 commits the higher pmax (position 4)
    assert st.committed[0, 4] == 1 and st.canvas[0, 4] == 24 and st.committed[0, 5] == 0
    # disabled (negative) or under another rule: no edits
    for rule, eps in ((O.RULE_BR, -1.0), (O.RULE_EB, 0.6)):
        cfg2 = O.Config(B=1, L=L, V=1000, rule=rule, stop_entropy=-1.0, greedy=1,
                        editing_threshold=eps)
        st2 = O.State(cfg2).init()
        st2.committed[0, :4] = 1
        st2.canvas[0, :4] = [10, 11, 12, 13]
        mg2 = O.canvas_decide(st2, 0, 3, H, amax, pmax, np.zeros(L, np.int32))
        assert st2.canvas[0, :4].tolist() == [10, 11, 12, 13] and mg2["n_edit"] == 0


def test_br_editing_is_not_applied_when_the_stop_fires(oracle_lib):
    L = 3
    cfg = O.Config(B=1, L=L, V=1000, rule=O.RULE_BR, stop_entropy=0.5, stability_steps=1,
                   greedy=1, editing_threshold=0.1)
    st = O.State(cfg).init()
    st.committed[0, 0] = 1
    st.canvas[0, 0] = 10
    st.prev[0] = [20, 21, 22]
    st.stable[0] = 0
    H = np.full(L, 0.01)  # mean below the stop entropy, argmax unchanged
    mg = O.canvas_decide(st, 0, 4, H, np.array([20, 21, 22], np.int32), np.full(L, 0.99),
                         np.zeros(L, np.int32))
    assert mg["fired"] == 1 and mg["n_edit"] == 0
    assert st.canvas[0].tolist() == [10, 21, 22]  # frozen token kept, open ones take the argmax


def test_commit_takes_sample_or_argmax_when_greedy(oracle_lib):
    H = np.array([0.01, 0.5, 0.02, 0.9])
    st, mg, before, smp = _decide_all_open(O.RULE_EB, H)
    assert set(np.nonzero(st.committed[0])[0]) == {0, 2}
    assert st.canvas[0, 0] == smp[0] and st.canvas[0, 2] == smp[2]
    cfg = O.Config(B=1, L=4, V=1000, rule=O.RULE_EB, stop_entropy=-1.0, greedy=1)
    st2 = O.State(cfg).init()
    O.canvas_decide(st2, 0, 0, H, np.array([7, 8, 9, 10], np.int32), np.zeros(4),
                    np.array([1, 2, 3, 4], np.int32))
    assert st2.canvas[0, 0] == 7 and st2.canvas[0, 2] == 9


def test_last_step_commits_everything(oracle_lib):
    H = np.array([0.5, 0.6, 0.7])
    st, mg, _, smp = _decide_all_open(O.RULE_EB, H, s=47, N=48)
    assert st.committed[0].all() and st.stop[0] == O.STOP_LAST_STEP
    assert (st.canvas[0] == smp).all()


def test_renoise_changes_only_open_positions(oracle_lib):
    H = np.array([0.01, 0.5, 0.6, 0.7, 0.8])
    cfg = O.Config(B=1, L=5, V=1 << 20, rule=O.RULE_EB, stop_entropy=-1.0, seed=3)
    st = O.State(cfg).init()
    st.committed[0, 4] = 1
    st.canvas[0, 4] = 42
    O.canvas_decide(st, 0, 5, H, np.zeros(5, np.int32), np.zeros(5), np.full(5, 9, np.int32))
    assert st.canvas[0, 4] == 42 and st.committed[0, 0] == 1 and st.canvas[0, 0] == 9
    for l in (1, 2, 3):  # renoised from stream 1 at step 5
        w = O.draw_word(3, l >> 2, 0, 5, 0 | (1 << 24), l & 3)
        assert st.canvas[0, l] == O.uniform_token(w, 1 << 20)


# ----------------------------------------------------------------------------- adaptive stop

def _conf_logits(L, V, targets, gap):
    z = np.zeros((L, V), np.float32)
    z[np.arange(L), targets] = gap
    return z


def test_stop_fires_at_predicted_step(oracle_lib):
    # bound 0: exactly one commit per step, so the canvas stays open long enough
    L, V = 16, 512
    cfg = O.Config(B=1, L=L, V=V, num_steps=30, seed=5, entropy_bound=0.0)
    st = O.State(cfg).init()
    tgt = (np.arange(L) * 31) % V
    fired_at = None
    for s in range(30):
        # uncertain, moving targets for s < 6, then near-deterministic fixed targets
        z = _conf_logits(L, V, tgt if s >= 6 else (tgt + s) % V, 40.0 if s >= 6 else 0.5)
        out = O.step_canvas(st, 0, z, s)
        if out is None:
            break
        assert out["margins"]["n_commit"] >= 1
        if out["margins"]["fired"]:
            fired_at = s
            break
    # s = 6 is the first confident step; its argmax differs from s = 5, so the
    # stability condition first holds at s = 7.
    assert fired_at == 7
    assert st.stop[0] == O.STOP_ADAPTIVE and st.committed[0].all()
    # positions still open when it fired took the argmax
    assert (st.canvas[0][8:] == tgt[8:]).sum() >= L - 8


def test_stop_blocked_by_one_flipping_position(oracle_lib):
    L, V = 4, 512
    cfg = O.Config(B=1, L=L, V=V, num_steps=12, seed=5, entropy_bound=0.0)
    st = O.State(cfg).init()
    tgt = np.array([3, 100, 200, 511])
    for s in range(12):
        t = tgt.copy()
        t[2] = 7 if s % 2 else 8  # flips every step
        out = O.step_canvas(st, 0, _conf_logits(L, V, t, 40.0), s)
        if out is None:
            break
        assert not out["margins"]["fired"]
    assert st.stop[0] != O.STOP_ADAPTIVE


def test_stop_disabled_with_negative_threshold(oracle_lib):
    L, V = 4, 64
    cfg = O.Config(B=1, L=L, V=V, num_steps=6, stop_entropy=-1.0, entropy_bound=0.0)
    st = O.State(cfg).init()
    z = _conf_logits(L, V, np.arange(L), 40.0)
    for s in range(6):
        out = O.step_canvas(st, 0, z, s)
        if out is None:
            break
        assert not out["margins"]["fired"]


# ----------------------------------------------------------------------------- invariants

def test_trajectory_invariants(oracle_lib):
    rng = np.random.default_rng(12)
    B, L, V, N = 3, 16, 300, 12
    for rule in (O.RULE_EB, O.RULE_EB_MI, O.RULE_BR):
        cfg = O.Config(B=B, L=L, V=V, num_steps=N, rule=rule, seed=21, quota=2,
                       greedy=int(rule == O.RULE_BR))
        st = O.State(cfg).init()
        assert ((st.canvas >= 0) & (st.canvas < V)).all() and not st.committed.any()
        for s in range(N):
            z = (rng.standard_normal((B, L, V)) * 2).astype(np.float32)
            z[:, np.arange(L), (np.arange(L) * 7) % V] += rng.uniform(0, 20, (B, L)).astype(np.float32)
            for i in range(B):
                before = st.copy()
                out = O.step_canvas(st, i, z[i], s)
                if before.stop[i]:
                    assert out is None
                    assert (st.canvas[i] == before.canvas[i]).all()
                    continue
                assert (st.committed[i] >= before.committed[i]).all()       # never reverts
                keep = before.committed[i] == 1
                assert (st.canvas[i][keep] == before.canvas[i][keep]).all()  # never changes
                assert ((st.canvas[i] >= 0) & (st.canvas[i] < V)).all()
                assert (out["H"] >= -1e-12).all() and (out["H"] <= math.log(V) + 1e-9).all()
                n_new = int(st.committed[i].sum() - before.committed[i].sum())
                if rule != O.RULE_BR and (before.committed[i] == 0).any():
                    assert n_new >= 1
                if st.stop[i]:
                    assert st.committed[i].all()
        assert st.stop.all()  # everything stops by the last step


# ----------------------------------------------------------------------------- vocabulary slices

def test_slices_combine_to_the_full_row(oracle_lib):
    """Vocabulary-sharded logits: the slices' records, combined, give the
    full row's entropy, max probability, argmax and two-level draw.  Checked
    against the full-row functions for random partitions on group boundaries,
    including -inf logits and a slice of -inf only."""
    rng = np.random.default_rng(31)
    G = 64
    for trial in range(60):
        ng = int(rng.integers(2, 12))
        V = ng * G - int(rng.integers(0, G))
        z = rng.normal(0.0, rng.choice([0.5, 3.0]), V)
        if trial % 3 == 0:
            z[rng.integers(0, V)] += 15.0
        if trial % 4 == 1:
            z[rng.random(V) < 0.2] = -np.inf
        cuts = sorted(set(rng.choice(np.arange(1, ng), size=int(rng.integers(1, min(4, ng))),
                                     replace=False).tolist()))
        bounds = [0] + [c * G for c in cuts] + [V]
        if trial % 5 == 2:  # one slice of -inf only
            z[bounds[0]:bounds[1]] = -np.inf
            z[bounds[-2]] = 1.0  # keep the row finite somewhere
        cfg = O.Config(B=1, L=4, V=V, group_size=G, seed=int(rng.integers(1 << 30)))
        inv_T = float(rng.choice([1.0, 1.25, 2.5]))
        row = z.astype(np.float32)
        slices = [O.slice_record(cfg, np.ascontiguousarray(row[lo:hi]), lo, inv_T, 0, 2, 7)
                  for lo, hi in zip(bounds[:-1], bounds[1:])]
        H, pm, am, x = O.combine_slices(slices, inv_T)
        H0, pm0, am0, _ = O.row_stats(row, inv_T)
        x0, margin, _ = O.sample(cfg, row, inv_T, 0, 2, 7)
        assert am == am0
        assert abs(H - H0) <= 1e-12 * max(1.0, abs(H0)) and abs(pm - pm0) <= 1e-12
        if margin > 1e-9:  # not an exact tie between two draws
            assert x == x0, (trial, x, x0)
