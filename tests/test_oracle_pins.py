"""Pins of the oracle against what the pages and the mathematics fix.

No pin here re-runs the oracle against itself: each checks a value the pages
state (the multi-item equivalence s^MIS = s, the pair count
(K-1) L (L+1) / 2, the tree mask and position rule, the interface's RMS), a
closed form of the mathematics (softmax, RoPE rotation, RMSNorm, a constructed
two-token attention), or a special case in which the model reduces to a
computation that can be written down by hand.
"""
import math

import numpy as np
import pytest

from oracle import ranker as R
from synth import workloads as W
from synth.rng import Stream, mix

TINY = W.TINY


def _tiny_model():
    return R.OracleModel(TINY, W.model_weights(TINY))


def _tiny_table(model, n_items=64, gamma=0.0):
    a = W.item_vectors(n_items, TINY.d)
    return R.table_f32(R.interface(a, gamma, R.embedding_rho(model.embed)))


def _blank_weights(shape: W.ModelShape, fill=0.0):
    """Weights with every matrix set to `fill` and every norm gain to 1."""
    out = []
    for _, shp, init in W.weight_names(shape):
        out.append(np.ones(shp, np.float32) if init == "ones" else np.full(shp, fill, np.float32))
    return out


def _idx(shape, name):
    return [n for n, _, _ in W.weight_names(shape)].index(name)


# --------------------------------------------------------------------------
# generator
# --------------------------------------------------------------------------

def test_splitmix64_reference_sequence():
    # SplitMix64 from state 1234567: the first outputs of the reference
    # implementation (Vigna, splitmix64.c), used as test vectors by many ports.
    st = np.uint64(1234567)
    idx = np.arange(1, 6, dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = mix(st + idx * np.uint64(0x9E3779B97F4A7C15))
    assert [int(v) for v in got] == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                                     4593380528125082431, 16408922859458223821]


def test_normals_moments_and_chunk_independence():
    s = Stream(5, 1).normal(400_001)
    assert abs(s.mean()) < 0.01 and abs(s.std() - 1.0) < 0.01
    # chunked generation on the thread pool gives the same values as one chunk
    a = Stream(5, 1)
    b = Stream(5, 1)
    x = a.normal(100_000, chunk_pairs=1 << 10)
    y = b.normal(100_000, chunk_pairs=1 << 20)
    assert np.array_equal(x, y)


# --------------------------------------------------------------------------
# continuous interface (DuoLM summary page, 前置知识 / 核心方法)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("gamma", [0.0, 0.3, -1.2])
def test_interface_rms_closed_form(gamma):
    a = W.item_vectors(64, 128).astype(np.float64) * 3.7
    rho = 0.0280669
    zf = (np.exp(gamma) * rho) * a / R.rms(a)[:, None]   # before FP16 storage
    assert np.allclose(R.rms(zf), math.exp(gamma) * rho, rtol=1e-13, atol=0)
    z16 = R.interface(a, gamma, rho).astype(np.float64)
    # FP16 storage: each element moves by at most half an ulp (2^-11 relative
    # in the normal range), so the row RMS moves by at most that much.
    assert np.all(np.abs(R.rms(z16) / (math.exp(gamma) * rho) - 1.0) <= 2.0 ** -11)
    # round to nearest: the stored value is the closest FP16 value
    up = np.nextafter(z16.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(z16.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    assert np.all(np.abs(zf - z16) <= np.abs(zf - up) + 0.0)
    assert np.all(np.abs(zf - z16) <= np.abs(zf - dn) + 0.0)


def test_embedding_rho_is_the_mean_of_row_rms():
    """rho of the synthetic configurations: the mean over embedding rows of
    each row's RMS (DuoLM summary page, 前置知识 / 核心方法: z = e^gamma *
    rho * a / RMS(a), with rho the reference scale of the native embeddings).
    Rows are chosen with integer RMS, so each reduction someone might write
    by mistake gives a different number: the RMS of the whole table, the
    mean of squares, the mean absolute value, an epsilon under the root."""
    rows = np.array([[4.0, 4.0, 2.0, 0.0],     # RMS 3, mean |x| 2.5
                     [8.0, -6.0, 0.0, 0.0],    # RMS 5, mean |x| 3.5
                     [0.5, -0.5, 0.5, 0.5]])   # RMS 0.5
    for scale in (1.0, 2.0 ** -6):             # 2^-6: the N(0, 0.02) range, still exact
        e = rows * scale
        want = (3.0 + 5.0 + 0.5) / 3.0 * scale
        got = R.embedding_rho(e.astype(np.float32))
        assert got == pytest.approx(want, rel=1e-15, abs=0)
        assert abs(float(np.sqrt(np.mean(e * e))) - want) > 0.1 * want     # RMS of the whole table
        assert abs(float(np.mean(e * e)) - want) > 0.1 * want              # mean of squares
        assert abs(float(np.mean(np.abs(e))) - want) > 0.1 * want          # mean |x|
    # an epsilon under the root would move the result: no epsilon here
    tiny = np.full((2, 4), 2.0 ** -20, np.float32)
    assert R.embedding_rho(tiny) == 2.0 ** -20
    # rows are independent of their order; scaling one row by s moves rho by
    # (s - 1) RMS(row) / n_rows
    assert R.embedding_rho(rows[::-1].astype(np.float32)) == pytest.approx(8.5 / 3.0, rel=1e-15)
    r2 = rows.copy()
    r2[1] *= 4.0
    assert R.embedding_rho(r2.astype(np.float32)) == pytest.approx((3.0 + 20.0 + 0.5) / 3.0, rel=1e-15)


def test_interface_scale_invariance():
    # RMS normalisation makes z independent of the scale of a.
    a = W.item_vectors(16, 128).astype(np.float64)
    assert np.array_equal(R.interface(a, 0.1, 0.02), R.interface(a * 8.0, 0.1, 0.02))


# --------------------------------------------------------------------------
# single steps against closed forms
# --------------------------------------------------------------------------

def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    for n in [1, 2, 7, 300]:
        q = rng.normal(size=32) * 5
        K = rng.normal(size=(n, 32)) * 5
        V = rng.normal(size=(n, 32))
        p, _ = R.attend(q, K, V, 1 / math.sqrt(32))
        assert abs(p.sum() - 1.0) < 1e-12 and np.all(p >= 0)


def test_attention_two_keys_closed_form():
    q = np.array([1.0, 0.0, 0.0, 0.0])
    K = np.array([[2.0, 0, 0, 0], [0.0, 0, 0, 0]])
    V = np.array([[1.0, 2.0, 3.0, 4.0], [-1.0, 0.0, 5.0, 0.0]])
    p, o = R.attend(q, K, V, 0.5)  # logits 1 and 0
    e = math.e
    assert p[0] == pytest.approx(e / (1 + e), abs=1e-15)
    assert np.allclose(o, (e * V[0] + V[1]) / (1 + e), atol=1e-15)


def test_attention_zero_query_is_mean():
    rng = np.random.default_rng(1)
    V = rng.normal(size=(9, 16))
    p, o = R.attend(np.zeros(16), rng.normal(size=(9, 16)), V, 0.25)
    assert np.allclose(p, 1 / 9, atol=1e-15) and np.allclose(o, V.mean(0), atol=1e-14)


def test_rope_closed_form_pairs_and_frequencies():
    # head_dim 4, theta 100: pair (0, 2) turns by pos rad, pair (1, 3) by pos/10.
    for pos in [0, 1, 5, 37]:
        e0 = R.rope(np.array([1.0, 0, 0, 0]), pos, 100.0)
        assert np.allclose(e0, [math.cos(pos), 0, math.sin(pos), 0], atol=1e-15)
        e1 = R.rope(np.array([0, 1.0, 0, 0]), pos, 100.0)
        assert np.allclose(e1, [0, math.cos(pos / 10), 0, math.sin(pos / 10)], atol=1e-15)
        e2 = R.rope(np.array([0, 0, 1.0, 0]), pos, 100.0)
        assert np.allclose(e2, [-math.sin(pos), 0, math.cos(pos), 0], atol=1e-15)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(2)
    q, k = rng.normal(size=128), rng.normal(size=128)
    dots = [R.rope(q, p + 9, 1e6) @ R.rope(k, p, 1e6) for p in [0, 11, 500, 2000]]
    assert np.allclose(dots, dots[0], rtol=1e-10)
    assert np.linalg.norm(R.rope(q, 1234, 1e4)) == pytest.approx(np.linalg.norm(q), rel=1e-14)


def test_rmsnorm_closed_form():
    x = np.full(64, -3.0)
    g = np.linspace(0.5, 2.0, 64).astype(np.float32)
    y = R.rmsnorm(x, g, 1e-6)
    assert np.allclose(y, -3.0 / math.sqrt(9.0 + 1e-6) * g.astype(np.float64), rtol=1e-15)
    z = R.rmsnorm(np.arange(1.0, 9.0), np.ones(8, np.float32), 0.0)
    assert math.sqrt(np.mean(z * z)) == pytest.approx(1.0, abs=1e-15)


# --------------------------------------------------------------------------
# tree mask, positions and pair count (DuoLM summary page, 研究动机 and
# 方法步骤详情 step 4)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("L,K,b", [(48, 8, 1), (1, 1, 1), (5, 3, 4), (17, 6, 2), (3, 1, 5)])
def test_tree_mask_brute_force_and_positions(L, K, b):
    lay = R.mis_layout(np.zeros(L, np.int32), np.zeros((K, b), np.int32))
    m = R.tree_mask(L, K, b)
    got = np.zeros_like(m)
    for r in range(lay.n_rows):
        got[r, lay.key_idx[lay.key_ptr[r]:lay.key_ptr[r + 1]]] = True
    assert np.array_equal(got, m)
    # every candidate sees the prefix and only its own branch
    for j in range(K):
        for i in range(b):
            row = L + j * b + i
            assert m[row, :L].all()
            others = [L + jj * b + ii for jj in range(K) for ii in range(b) if jj != j]
            assert not m[row, others].any()
    # unified logical position: branch token i of every candidate sits at L + i
    assert np.array_equal(lay.pos[:L], np.arange(L))
    assert np.array_equal(lay.pos[L:].reshape(K, b), np.broadcast_to(L + np.arange(b), (K, b)))


@pytest.mark.parametrize("L,K,b", [(48, 8, 1), (296, 100, 1), (1, 1, 1), (5, 3, 4), (2132, 256, 4)])
def test_pair_elimination_count(L, K, b):
    mis = L * (L + 1) // 2 + K * sum(L + i + 1 for i in range(b))
    small = L < 400
    if small:
        lay = R.mis_layout(np.zeros(L, np.int32), np.zeros((K, b), np.int32))
        assert lay.n_pairs() == mis
        ind = R.independent_layout(np.zeros(L, np.int32), np.zeros(b, np.int32)).n_pairs() * K
    else:
        ind = K * (L + b) * (L + b + 1) // 2
    assert ind - mis == (K - 1) * L * (L + 1) // 2


# --------------------------------------------------------------------------
# the multi-item equivalence s^MIS = s, bit for bit
# --------------------------------------------------------------------------

def test_mis_equals_independent_tiny():
    m = _tiny_model()
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    assert np.array_equal(R.score_mis(m, tab, req), R.score_independent(m, tab, req))


@pytest.mark.parametrize("seed,n_hist,fb,K,b", [(11, 0, 0, 1, 1), (12, 2, (1, 9), 5, 4), (13, 3, (3, 12), 7, 2)])
def test_mis_equals_independent_ragged(seed, n_hist, fb, K, b):
    m = _tiny_model()
    tab = _tiny_table(m)
    wl = W.custom(TINY, 64, seed, 2, n_hist, fb if n_hist else 1, K, b, n_instr=1 + seed % 3)
    for req in wl.requests:
        assert np.array_equal(R.score_mis(m, tab, req), R.score_independent(m, tab, req))


def test_candidates_do_not_see_each_other():
    m = _tiny_model()
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    base = R.score_mis(m, tab, req)
    # replacing one candidate leaves every other score unchanged, bit for bit
    br = req.branch_ids.copy()
    br[3, 0] = TINY.vocab + 63
    alt = R.forward(m, tab, R.mis_layout(req.prefix_ids, br))
    keep = [j for j in range(req.K) if j != 3]
    assert np.array_equal(alt[keep], base[keep]) and alt[3] != base[3]
    # scores come back in input order: permuting candidates permutes scores
    perm = np.array([5, 0, 7, 2, 1, 6, 4, 3])
    assert np.array_equal(R.forward(m, tab, R.mis_layout(req.prefix_ids, req.branch_ids[perm])), base[perm])


def test_causal_prefix():
    m = _tiny_model()
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    lay = R.independent_layout(req.prefix_ids, req.branch_ids[0])
    _, layers = R.forward(m, tab, lay, want_layers=True)
    ids2 = lay.ids.copy()
    ids2[30] = (ids2[30] + 1) % TINY.vocab
    lay2 = R.Layout(ids2, lay.pos, lay.key_ptr, lay.key_idx, lay.out_rows)
    _, layers2 = R.forward(m, tab, lay2, want_layers=True)
    assert np.array_equal(layers[:, :30], layers2[:, :30])
    assert not np.array_equal(layers[-1, 30:], layers2[-1, 30:])


def test_prefix_rows_of_a_shorter_call_equal_those_of_the_whole_sequence():
    """The reading behind prefix KV reuse: in the packed multi-item layout a
    prefix row's residual at every layer (hence its K/V) is the same whether
    the call held the prefix up to some cut with its own candidates, or the
    whole prefix with other candidates."""
    m = _tiny_model()
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    c = 29
    short = R.mis_layout(req.prefix_ids[:c], req.branch_ids[:3])
    full = R.mis_layout(req.prefix_ids, req.branch_ids[3:])
    _, ls = R.forward(m, tab, short, want_layers=True)
    _, lf = R.forward(m, tab, full, want_layers=True)
    assert np.array_equal(ls[:, :c], lf[:, :c])
    # the branches of the short call sit at position c, those of the whole one at L
    assert short.pos[c] == c and full.pos[req.L] == req.L


# --------------------------------------------------------------------------
# whole-model special cases with hand-computable results
# --------------------------------------------------------------------------

def _one_layer(shape):
    import dataclasses
    return dataclasses.replace(shape, n_layers=1)


def test_embedding_lookup_and_head_when_layers_are_silent():
    # With W_o = 0 and W_down = 0 every layer adds zero, so the scored hidden
    # state is the looked-up row of the last branch token.
    shp = TINY
    w = [a.copy() for a in W.model_weights(shp)]
    for l in range(shp.n_layers):
        w[_idx(shp, f"l{l}.wo")][:] = 0
        w[_idx(shp, f"l{l}.w_down")][:] = 0
    m = R.OracleModel(shp, w)
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    s = R.score_mis(m, tab, req)
    head = w[-1].astype(np.float64)
    for j in range(req.K):
        row = tab[req.branch_ids[j, -1] - shp.vocab].astype(np.float64)
        h = row / math.sqrt(np.mean(row * row) + shp.rms_eps)
        assert s[j] == pytest.approx(float(head @ h), rel=1e-12)
    # a vocabulary id as last token reads the embedding instead
    br = req.branch_ids.copy()
    br[0, 0] = 17
    s2 = R.forward(m, tab, R.mis_layout(req.prefix_ids, br))
    e = m.embed[17].astype(np.float64)
    assert s2[0] == pytest.approx(float(head @ (e / math.sqrt(np.mean(e * e) + shp.rms_eps))), rel=1e-12)


def test_uniform_attention_follows_mask_and_kv_groups():
    # q = 0 (W_q = 0) makes every softmax uniform over the visible keys, so a
    # row's attention output is the mean of the visible values of its kv head.
    # W_v copies normed coordinates [0, 64) (kv head g <- coords 32g..32g+31),
    # W_o = identity puts query head h in coords 32h..32h+31, the MLP is off.
    shp = _one_layer(TINY)
    w = _blank_weights(shp)
    w[0] = W.model_weights(TINY)[0].copy()
    wv = w[_idx(shp, "l0.wv")]
    wv[np.arange(64), np.arange(64)] = 1.0
    w[_idx(shp, "l0.wo")][np.arange(128), np.arange(128)] = 1.0
    m = R.OracleModel(shp, w)
    tab = _tiny_table(m)
    wl = W.custom(TINY, 64, 21, 1, 2, (2, 4), 4, 3)
    req = wl.requests[0]
    lay = R.mis_layout(req.prefix_ids, req.branch_ids)
    _, layers = R.forward(m, tab, lay, want_layers=True)
    x0 = layers[0]
    n0 = x0 / np.sqrt(np.mean(x0 * x0, axis=1, keepdims=True) + shp.rms_eps)
    mask = R.tree_mask(req.L, req.K, wl.branch_len)
    for r in range(lay.n_rows):
        vis = np.nonzero(mask[r])[0]
        exp = x0[r].copy()
        for h in range(4):
            g = h // 2
            exp[32 * h:32 * h + 32] += n0[vis, 32 * g:32 * g + 32].mean(axis=0)
        assert np.allclose(layers[1][r], exp, rtol=1e-13, atol=1e-15)


def test_attention_scale_and_qk_norm_two_tokens():
    # Tokens A and B = -A at position 0 (RoPE is the identity there).  W_q and
    # W_k copy coords [0, 32) into head 0, W_v likewise, W_o = identity, MLP off.
    # After QK-norm q1 = -u, k0 = u, k1 = -u with |u|^2 = 32, so row 1 gives
    # logits -sqrt(32) (key 0) and +sqrt(32) (key 1) under the 1/sqrt(32) scale.
    # eps = 1e-30 keeps the all-zero heads at zero and is below fp64 resolution
    # for the others, so the closed form holds to rounding.
    import dataclasses
    shp = dataclasses.replace(_one_layer(TINY), rms_eps=1e-30)
    w = _blank_weights(shp)
    rng = np.random.default_rng(3)
    emb = np.zeros((shp.vocab, shp.d), np.float32)
    emb[1] = rng.normal(size=shp.d).astype(np.float32)
    emb[2] = -emb[1]
    w[0] = emb
    for nm in ["l0.wq", "l0.wk", "l0.wv"]:
        w[_idx(shp, nm)][np.arange(32), np.arange(32)] = 1.0
    w[_idx(shp, "l0.wo")][np.arange(128), np.arange(128)] = 1.0
    m = R.OracleModel(shp, w)
    lay = R.Layout(np.array([1, 2], np.int32), np.array([0, 0], np.int32),
                   np.array([0, 1, 3], np.int64), np.array([0, 0, 1], np.int32), np.array([1], np.int32))
    _, layers = R.forward(m, np.zeros((1, shp.d), np.float32), lay, want_layers=True)
    a = emb[1].astype(np.float64)
    nA = a / math.sqrt(np.mean(a * a) + shp.rms_eps)
    p_self = 1.0 / (1.0 + math.exp(-2.0 * math.sqrt(32.0)))
    exp = -a.copy()
    exp[:32] += (1 - p_self) * nA[:32] + p_self * (-nA[:32])
    assert np.allclose(layers[1][1, :32], exp[:32], rtol=1e-12, atol=1e-14)
    # row 0 sees only itself: its output is its own value
    exp0 = a.copy()
    exp0[:32] += nA[:32]
    assert np.allclose(layers[1][0, :32], exp0[:32], rtol=1e-12, atol=1e-14)


def test_swiglu_mlp_orientation():
    # Attention silent (W_o = 0).  W_gate row i reads coord pi(i) scaled by 3,
    # W_up row i reads coord sigma(i), W_down row c reads hidden unit tau(c):
    # x_c += silu(3 n_pi(tau c)) * n_sigma(tau c).
    shp = _one_layer(TINY)
    w = _blank_weights(shp)
    w[0] = W.model_weights(TINY)[0].copy()
    rng = np.random.default_rng(4)
    pi, sigma = rng.integers(0, 128, 256), rng.integers(0, 128, 256)
    tau = rng.permutation(256)[:128]
    w[_idx(shp, "l0.w_gate")][np.arange(256), pi] = 3.0
    w[_idx(shp, "l0.w_up")][np.arange(256), sigma] = 1.0
    w[_idx(shp, "l0.w_down")][np.arange(128), tau] = 1.0
    m = R.OracleModel(shp, w)
    ids = np.array([5, 77, 300], np.int32)
    lay = R.Layout(ids, np.arange(3, dtype=np.int32), np.array([0, 1, 3, 6], np.int64),
                   np.array([0, 0, 1, 0, 1, 2], np.int32), np.array([2], np.int32))
    _, layers = R.forward(m, np.zeros((1, shp.d), np.float32), lay, want_layers=True)
    x0 = layers[0]
    n = x0 / np.sqrt(np.mean(x0 * x0, axis=1, keepdims=True) + shp.rms_eps)
    for r in range(3):
        for c in range(128):
            hdn = tau[c]
            g = 3.0 * n[r, pi[hdn]]
            exp = x0[r, c] + g / (1 + math.exp(-g)) * n[r, sigma[hdn]]
            assert layers[1][r, c] == pytest.approx(exp, rel=1e-13, abs=1e-16)


def test_qk_norm_makes_scores_invariant_to_qk_scale():
    w = [a.copy() for a in W.model_weights(TINY)]
    m = R.OracleModel(TINY, w)
    tab = _tiny_table(m)
    req = W.tiny().requests[0]
    base = R.score_mis(m, tab, req)
    for l in range(TINY.n_layers):
        w[_idx(TINY, f"l{l}.wq")] *= 4.0
        w[_idx(TINY, f"l{l}.wk")] *= 2.0
    s = R.score_mis(R.OracleModel(TINY, w), tab, req)
    assert np.allclose(s, base, rtol=0, atol=1e-5)
    # scaling the values is not normalised away
    w2 = [a.copy() for a in W.model_weights(TINY)]
    w2[_idx(TINY, "l0.wv")] *= 4.0
    assert not np.allclose(R.score_mis(R.OracleModel(TINY, w2), tab, req), base, atol=1e-3)


def _fp16_rne(x) -> float:
    """Nearest FP16 value of an exact rational (ties to even mantissa)."""
    from fractions import Fraction
    x = Fraction(x)
    if x == 0:
        return 0.0
    s, x = (-1 if x < 0 else 1), abs(x)
    e = max(x.numerator.bit_length() - x.denominator.bit_length() - 1, -14)
    while Fraction(2) ** e > x and e > -14:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    step = Fraction(2) ** (e - 10)  # 10 fraction bits; subnormal spacing below 2^-14
    q, r = divmod(x, step)
    q = int(q)
    if r * 2 > step or (r * 2 == step and q % 2 == 1):
        q += 1
    return s * float(q * step)


def test_interface_golden_at_the_pages_rho():
    """tests/golden/interface_rho.txt: the pages' rho, vectors with rational
    RMS; the oracle's FP16 table rows equal the exact rational z rounded to
    nearest even, and RMS(z) = rho before rounding."""
    import os
    from fractions import Fraction
    path = os.path.join(os.path.dirname(__file__), "golden", "interface_rho.txt")
    rho_s, rows = None, []
    for line in open(path, encoding="utf-8"):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "rho":
            rho_s = f[1]
        elif f[0] == "gamma":
            assert float(f[1]) == 0.0
        elif f[0] == "a":
            rows.append([Fraction(v) for v in f[1:]])
    rho = Fraction(rho_s)
    assert rho == Fraction(280669, 10 ** 7)
    got = R.interface(np.array([[float(v) for v in a] for a in rows]), 0.0, float(rho))
    for a, z16 in zip(rows, got):
        ms = sum(v * v for v in a) / len(a)
        rms = Fraction(int(round(float(ms) ** 0.5 * 2)), 2)  # the vectors' RMS are halves
        assert rms * rms == ms
        z = [rho * v / rms for v in a]
        assert sum(v * v for v in z) / len(z) == rho * rho  # RMS(z) = rho, exactly
        assert [float(v) for v in z16] == [_fp16_rne(v) for v in z]


def test_fp16_rounding_helper():
    from fractions import Fraction as F
    assert _fp16_rne(F(1, 3)) == float(np.float16(1 / 3))
    assert _fp16_rne(F(-1000, 7)) == float(np.float16(-1000 / 7))
    assert _fp16_rne(F(1, 2 ** 20)) == 2.0 ** -20              # subnormal, exact
    assert _fp16_rne(1 + F(1, 2 ** 11)) == 1.0                 # tie to the even mantissa
    assert _fp16_rne(1 + F(3, 2 ** 11)) == 1 + 2.0 ** -9       # tie to the even mantissa
    assert _fp16_rne(F(3, 2 ** 25)) == 2.0 ** -23              # subnormal tie: 1.5 ulp -> 2 ulp
