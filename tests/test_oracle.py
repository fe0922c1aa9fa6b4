"""Pins for the fp64 CPU oracle, against facts fixed by the pages and by
mathematics rather than by the oracle itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one causal mask, a wrong
log base) fails at least one of them; ``test_planted_mistakes_are_caught``
checks that claim on mutated copies of the oracle.
"""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
from exact_attention_127_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(None, 1)
            vals[key] = val
    return vals


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# ---------------------------------------------------------------------------
# Worked values printed on the pages
# ---------------------------------------------------------------------------
def test_golden_rescale_factor_exp_minus_2():
    """Page 3, follow-up 2: block maxima 10 then 12 give factor exp(-2)."""
    g = _golden("online_softmax_rescale.txt")
    m1, m2, factor = float(g["block1_max"]), float(g["block2_max"]), float(g["factor"])
    x = np.array([3.0, m1, -1.0, 0.5, m2, 7.0, 11.0, -4.0])
    p, m, l, factors = oracle.online_softmax(x, block=4)
    assert factors[1] == pytest.approx(factor, rel=1e-15, abs=0)
    assert factor == pytest.approx(math.exp(m1 - m2), rel=1e-15)
    assert m == m2
    # the statistics after both blocks are the full-vector ones
    assert l == pytest.approx(np.exp(x - m2).sum(), rel=1e-15)


def test_golden_exercise_online_matches_two_pass():
    """Page 2, practice exercise 2: online softmax (block 4) == two-pass to 1e-6."""
    g = _golden("online_softmax_exercise.txt")
    n, std, block, tol = int(g["length"]), float(g["std"]), int(g["block"]), float(g["tolerance"])
    x = _rand(n, 21, std)
    p_online, _, _, _ = oracle.online_softmax(x, block)
    p_two = oracle.softmax_two_pass(x)
    assert np.max(np.abs(p_online - p_two)) < tol
    # in fp64 the agreement is far tighter than the page's bound
    assert np.max(np.abs(p_online - p_two)) < 1e-15


def test_softmax_two_pass_special_cases():
    # constant vector -> uniform
    p = oracle.softmax_two_pass(np.full(7, 3.25))
    assert np.allclose(p, 1 / 7, rtol=0, atol=1e-16)
    # two entries: logistic function
    p = oracle.softmax_two_pass(np.array([0.0, 2.0]))
    assert p[1] == pytest.approx(1 / (1 + math.exp(-2.0)), rel=1e-15)
    # shift by a huge constant (needs the max subtraction): still finite
    p = oracle.softmax_two_pass(np.array([1000.0, 1001.0]))
    assert p[1] == pytest.approx(1 / (1 + math.exp(-1.0)), rel=1e-15)


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d", [1, 4, 64])
def test_single_key_returns_its_value_row(d):
    q, k, v = (_rand((1, 1, 1, d), s) for s in (1, 2, 3))
    scale = 0.37
    O, L = oracle.attention(q, k, v, causal=False, scale=scale)
    assert np.array_equal(O[0, 0, 0], v[0, 0, 0])
    assert L[0, 0, 0] == pytest.approx(scale * float(np.dot(q[0, 0, 0], k[0, 0, 0])),
                                       rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("N", [1, 2, 5, 130])
def test_causal_row0_is_v0(N):
    q, k, v = (_rand((2, 1, N, 8), s) for s in (4, 5, 6))
    O, L = oracle.attention_rows(q, k, v, causal=True, scale=0.5, rows=[0])
    for h in range(2):
        assert np.array_equal(O[h, 0], v[h, 0, 0])
        assert L[h, 0] == pytest.approx(0.5 * float(np.dot(q[h, 0, 0], k[h, 0, 0])),
                                        rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_values(causal):
    N, d = 37, 6
    q = np.zeros((1, 2, N, d))
    k, v = _rand((1, 2, N, d), 7), _rand((1, 2, N, d), 8)
    O, L = oracle.attention(q, k, v, causal=causal, scale=0.125)
    for h in range(2):
        for i in range(N):
            n = i + 1 if causal else N
            assert np.allclose(O[0, h, i], v[0, h, :n].mean(axis=0), rtol=0, atol=1e-14)
            assert L[0, h, i] == pytest.approx(math.log(n), rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_keys_average_values_and_shift_lse(causal):
    N, d = 19, 5
    q = _rand((1, 1, N, d), 9)
    krow = _rand(d, 10)
    k = np.broadcast_to(krow, (1, 1, N, d)).copy()
    v = _rand((1, 1, N, d), 11)
    scale = 0.8
    O, L = oracle.attention(q, k, v, causal=causal, scale=scale)
    for i in range(N):
        n = i + 1 if causal else N
        s = scale * float(np.dot(q[0, 0, i], krow))
        assert np.allclose(O[0, 0, i], v[0, 0, :n].mean(axis=0), rtol=0, atol=1e-13)
        assert L[0, 0, i] == pytest.approx(s + math.log(n), rel=1e-13, abs=1e-13)


def test_scale_multiplies_scores():
    """scale=2 on (q, k) equals scale=1 on (2q, k): the scale enters the scores."""
    q, k, v = (_rand((1, 2, 23, 8), s) for s in (12, 13, 14))
    O1, L1 = oracle.attention(q, k, v, causal=True, scale=2.0)
    O2, L2 = oracle.attention(2.0 * q, k, v, causal=True, scale=1.0)
    assert np.allclose(O1, O2, rtol=0, atol=1e-14)
    assert np.allclose(L1, L2, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Invariances of the definition
# ---------------------------------------------------------------------------
def test_key_value_permutation_invariance_noncausal():
    q, k, v = (_rand((2, 2, 41, 16), s) for s in (15, 16, 17))
    perm = np.random.default_rng(18).permutation(41)
    O1, L1 = oracle.attention(q, k, v, causal=False, scale=0.25)
    O2, L2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], causal=False, scale=0.25)
    assert np.allclose(O1, O2, rtol=0, atol=1e-13)
    assert np.allclose(L1, L2, rtol=0, atol=1e-13)
    # ... and a permutation that is not joint changes the result
    O3, _ = oracle.attention(q, k[:, :, perm], v, causal=False, scale=0.25)
    assert not np.allclose(O1, O3, atol=1e-3)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_moves_lse_not_output(causal):
    """Adding c to every key row shifts row i's scores by scale*q_i.c: O is
    unchanged, LSE_i moves by exactly that amount (the invariance the online
    recurrence rests on, "GPU 学习日报 Day 21" section 5.2)."""
    q, k, v = (_rand((1, 2, 33, 8), s) for s in (19, 20, 21))
    c = _rand(8, 22)
    scale = 0.3
    O1, L1 = oracle.attention(q, k, v, causal=causal, scale=scale)
    O2, L2 = oracle.attention(q, k + c, v, causal=causal, scale=scale)
    shift = scale * np.einsum("bhnd,d->bhn", q, c)
    assert np.allclose(O1, O2, rtol=0, atol=1e-12)
    assert np.allclose(L2 - L1, shift, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k, v = (_rand((1, 1, 50, 8), s, 3.0) for s in (23, 24, 25))
    for i in (0, 1, 17, 49):
        p = oracle.prob_row(q, k, v, causal, 0.35, head=0, row=i)
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p >= 0)
        if causal:
            assert np.all(p[i + 1:] == 0)
            assert np.all(p[:i + 1] > 0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 4, 7, 128, 1000])
def test_online_recurrence_equals_two_pass(causal, block):
    """Page 2 section 5.3 (one pass, rescaled accumulator, normalise at the
    end) agrees with the three-step definition in fp64."""
    q, k, v = (_rand((1, 2, 300, 16), s, 2.0) for s in (26, 27, 28))
    rows = [0, 1, 127, 128, 129, 200, 299]
    O1, L1 = oracle.attention_rows(q, k, v, causal, 0.25, rows=rows)
    O2, L2 = oracle.attention_rows_online(q, k, v, causal, 0.25, block, rows=rows)
    assert np.max(np.abs(O1 - O2)) < 1e-12
    assert np.max(np.abs(L1 - L2)) < 1e-12


# ---------------------------------------------------------------------------
# Brute force, no max subtraction, in 40-digit decimal arithmetic
# ---------------------------------------------------------------------------
def _brute(q, k, v, causal, scale):
    getcontext().prec = 40
    N, d = q.shape
    O = np.zeros((N, d))
    L = np.zeros(N)
    sc = Decimal(repr(scale))
    for i in range(N):
        keys = range(i + 1) if causal else range(N)
        e = []
        for j in keys:
            s = sum(Decimal(repr(float(q[i, c]))) * Decimal(repr(float(k[j, c])))
                    for c in range(d))
            e.append((j, (sc * s).exp()))
        z = sum(x for _, x in e)
        for c in range(d):
            O[i, c] = float(sum(x * Decimal(repr(float(v[j, c]))) for j, x in e) / z)
        L[i] = float(z.ln())
    return O, L


@pytest.mark.parametrize("N,d", [(1, 1), (2, 3), (5, 4), (8, 2), (7, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(N, d, causal):
    q, k, v = (_rand((1, 1, N, d), 30 + s) for s in range(3))
    scale = 0.7
    O, L = oracle.attention(q, k, v, causal=causal, scale=scale)
    Ob, Lb = _brute(q[0, 0], k[0, 0], v[0, 0], causal, scale)
    assert np.max(np.abs(O[0, 0] - Ob)) < 1e-12
    assert np.max(np.abs(L[0, 0] - Lb)) < 1e-12


# ---------------------------------------------------------------------------
# Large logits (the peaked long-context workload's distribution)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_large_logits_stay_bounded(causal):
    q, k = _rand((1, 1, 256, 128), 40, 4.0), _rand((1, 1, 256, 128), 41, 4.0)
    v = np.random.default_rng(42).uniform(-1, 1, (1, 1, 256, 128))
    scale = 1 / math.sqrt(128)
    rows = [0, 1, 100, 255]
    O, L = oracle.attention_rows(q, k, v, causal, scale, rows=rows)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    for n, i in enumerate(rows):
        keys = slice(0, i + 1) if causal else slice(0, 256)
        s = scale * (k[0, 0, keys] @ q[0, 0, i])
        assert L[0, n] >= s.max() - 1e-9                  # LSE >= max score
        assert L[0, n] <= s.max() + math.log(s.size) + 1e-9
        lo, hi = v[0, 0, keys].min(axis=0), v[0, 0, keys].max(axis=0)
        assert np.all(O[0, n] >= lo - 1e-12) and np.all(O[0, n] <= hi + 1e-12)


# ---------------------------------------------------------------------------
# Inputs: bf16 values reach the oracle exactly
# ---------------------------------------------------------------------------
def test_bf16_inputs_widen_exactly():
    q, k, v = inputs.make_qkv(1, 2, 40, 8, seed=7)
    O1, L1 = oracle.attention(q, k, v, causal=True, scale=0.5)
    O2, L2 = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                              causal=True, scale=0.5)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_rows_and_heads_selection():
    q, k, v = (_rand((2, 3, 20, 4), s) for s in (50, 51, 52))
    Oall, Lall = oracle.attention(q, k, v, causal=True, scale=0.9)
    O, L = oracle.attention_rows(q, k, v, True, 0.9, rows=[3, 19], heads=[4, 1])
    assert np.array_equal(O[0], Oall.reshape(6, 20, 4)[4, [3, 19]])
    assert np.array_equal(L[1], Lall.reshape(6, 20)[1, [3, 19]])


def test_bad_arguments_rejected():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_rows(q, q, q, False, 1.0, rows=[4])
    with pytest.raises(ValueError):
        oracle.attention_rows(q, q, np.zeros((1, 1, 5, 2)), False, 1.0)
    with pytest.raises(ValueError):
        oracle.attention_rows_online(q, q, q, False, 1.0, block=0)


# ---------------------------------------------------------------------------
# The pins above are sensitive: plant one mistake at a time in a copy of the
# oracle source (CPU only), rebuild it, and check that some pin fails.
# ---------------------------------------------------------------------------
MUTANTS = {
    "dropped_term": ("for (int64_t c = 0; c < d; ++c) acc += qi[c] * K[j * d + c];\n        s[j] = scale * acc;",
                     "for (int64_t c = 0; c + 1 < d; ++c) acc += qi[c] * K[j * d + c];\n        s[j] = scale * acc;"),
    "wrong_sign": ("s[j] = exp(s[j] - m); l += s[j];", "s[j] = exp(m - s[j]); l += s[j];"),
    "transposed_v": ("o_i[c] += s[j] * V[j * d + c];", "o_i[c] += s[j] * V[c * N + j];"),
    "causal_off_by_one": ("causal ? (i + 1 < N ? i + 1 : N) : N", "causal ? (i + 2 < N ? i + 2 : N) : N"),
    "lse_base2": ("*lse_i = m + log(l);\n    if (p_out)", "*lse_i = m + log2(l);\n    if (p_out)"),
    "scale_dropped": ("s[j] = scale * acc;\n    }\n    /* step 2", "s[j] = acc;\n    }\n    /* step 2"),
}


def _pins_pass():
    """A compact run of the pins above; True when all hold."""
    try:
        for causal in (False, True):
            for (N, d) in [(5, 4), (7, 3)]:
                test_brute_force_tiny(N, d, causal)
            test_zero_queries_average_values(causal)
            test_key_shift_moves_lse_not_output(causal)
        test_causal_row0_is_v0(5)
        test_single_key_returns_its_value_row(4)
        test_decode_brute_force(1, 7, 4)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutant, tmp_path, monkeypatch):
    import ctypes
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation site for {mutant} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", str(path), "-o", str(lib),
                    "-lm", "-lpthread"], check=True)
    # build the real library first so that its argtypes can be copied over
    real = oracle._lib()
    mut = ctypes.CDLL(str(lib))
    for name in ("oracle_softmax_two_pass", "oracle_online_softmax", "oracle_attention_rows",
                 "oracle_attention_rows_online", "oracle_attention_prob_row",
                 "oracle_attention_rows_qk"):
        getattr(mut, name).argtypes = getattr(real, name).argtypes
        getattr(mut, name).restype = getattr(real, name).restype
    assert _pins_pass()
    monkeypatch.setattr(oracle, "_LIB", mut)
    assert not _pins_pass(), f"planted mistake {mutant!r} went unnoticed"


# ---------------------------------------------------------------------------
# Decode (one query against many keys): attention_qk
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("Nq,Nk,d", [(1, 1, 3), (1, 7, 4), (3, 5, 2), (1, 8, 1)])
def test_decode_brute_force(Nq, Nk, d):
    q = _rand((1, 1, Nq, d), 60)
    k, v = _rand((1, 1, Nk, d), 61), _rand((1, 1, Nk, d), 62)
    O, L = oracle.attention_qk(q, k, v, 0.6)
    getcontext().prec = 40
    for i in range(Nq):
        e = []
        for j in range(Nk):
            s = sum(Decimal(repr(float(q[0, 0, i, c]))) * Decimal(repr(float(k[0, 0, j, c])))
                    for c in range(d))
            e.append((Decimal(repr(0.6)) * s).exp())
        z = sum(e)
        for c in range(d):
            ref = float(sum(x * Decimal(repr(float(v[0, 0, j, c]))) for j, x in enumerate(e)) / z)
            assert abs(O[0, i, c] - ref) < 1e-12
        assert abs(L[0, i] - float(z.ln())) < 1e-12


def test_decode_single_key_and_zero_query():
    q, k, v = _rand((2, 1, 1, 8), 63), _rand((2, 1, 1, 8), 64), _rand((2, 1, 1, 8), 65)
    O, L = oracle.attention_qk(q, k, v, 0.4)
    for h in range(2):
        assert np.array_equal(O[h, 0], v[h, 0, 0])
        assert L[h, 0] == pytest.approx(0.4 * float(q[h, 0, 0] @ k[h, 0, 0]), rel=1e-14, abs=1e-14)
    k2, v2 = _rand((1, 1, 50, 8), 66), _rand((1, 1, 50, 8), 67)
    O, L = oracle.attention_qk(np.zeros((1, 1, 1, 8)), k2, v2, 0.4)
    assert np.allclose(O[0, 0], v2[0, 0].mean(axis=0), rtol=0, atol=1e-14)
    assert L[0, 0] == pytest.approx(math.log(50), rel=1e-14)


@pytest.mark.parametrize("split", [1, 17, 64, 99])
def test_split_and_merge_matches_whole(split):
    """Q31, follow-up 3 (split K/V, compute the parts, merge) with the merge
    rule of the online recurrence ("GPU 学习日报 Day 21", section 5.2): weights e^{LSE_part}."""
    N = 100
    q = _rand((1, 2, 1, 16), 68, 2.0)
    k, v = _rand((1, 2, N, 16), 69, 2.0), _rand((1, 2, N, 16), 70)
    O, L = oracle.attention_qk(q, k, v, 0.25)
    O1, L1 = oracle.attention_qk(q, k[:, :, :split], v[:, :, :split], 0.25)
    O2, L2 = oracle.attention_qk(q, k[:, :, split:], v[:, :, split:], 0.25)
    M = np.maximum(L1, L2)
    w1, w2 = np.exp(L1 - M), np.exp(L2 - M)
    Lm = M + np.log(w1 + w2)
    Om = (w1[..., None] * O1 + w2[..., None] * O2) / (w1 + w2)[..., None]
    assert np.max(np.abs(Om - O)) < 1e-13
    assert np.max(np.abs(Lm - L)) < 1e-13


def test_decode_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.attention_qk(np.zeros((1, 1, 1, 4)), np.zeros((1, 1, 5, 4)), np.zeros((1, 1, 6, 4)), 1.0)
    with pytest.raises(ValueError):
        oracle.attention_qk(np.zeros((1, 1, 1, 4)), np.zeros((1, 2, 5, 4)), np.zeros((1, 2, 5, 4)), 1.0)
