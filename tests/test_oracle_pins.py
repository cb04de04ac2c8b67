"""Pins of the CPU oracle against facts that do not come from the oracle.

Each check ties a piece of the oracle to a published test vector, a library
routine, a closed form, an invariant of the method, or brute force on tiny
inputs, so that a plausible slip (a dropped term, a wrong sign or index, a
transposed operand) fails at least one of them.  Method: "ResidualQuant: KV
Cache Quantization for Looped Transformers with 2-Bit Residuals" (Abstract).
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle


def _bf16_bits(a):
    """Round float values to bf16 (torch's RN conversion) and return the bits."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _parse_ints(s):
    return [int(v, 0) for v in s.split()]


# ---------------------------------------------------------------------------
# generator and scalar formats
# ---------------------------------------------------------------------------

def test_splitmix64_published_vector(golden):
    g = golden("splitmix64_seed0.txt")
    seed = int(g["seed"])
    for i in range(5):
        assert oracle.splitmix64(seed, i) == int(g[str(i)], 16)


def test_signs_follow_top_bit():
    # sign i is -1 exactly when output i has its top bit set
    for seed in (0, 1, 7, 2**63 + 5):
        D = oracle.signs(seed, 128)
        for i in range(128):
            top = oracle.splitmix64(seed, i) >> 63
            assert D[i] == (-1 if top else 1)
    # balanced-ish and seed dependent
    assert abs(int(oracle.signs(0, 4096).sum())) < 300
    assert not np.array_equal(oracle.signs(0, 128), oracle.signs(1, 128))


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        [0.0, -0.0, 65504.0, 65519.99, 6.1e-5, 5.96e-8, 2.98e-8, 1 / 3, 0.1, 1 + 2**-11,
         1 + 3 * 2**-11, 2048 + 1, 2048 + 3],
    ])
    for v in vals:
        assert oracle.f64_to_f16(v) == int(np.float16(v).view(np.uint16)), v
    for h in range(0, 65536, 7):
        f = np.array([h], dtype=np.uint16).view(np.float16)[0]
        if np.isfinite(f):
            assert oracle.f16_to_f64(h) == float(f)


def test_bf16_widening_is_bit_shift():
    bits = np.array([0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x4049], dtype=np.uint16)
    f = oracle.bf16_to_f32(bits)
    assert f[0] == 1.0 and f[1] == -1.0 and f[4] == np.float32(3.140625)
    lib = oracle.lib()
    for b in bits:
        assert lib.orq_bf16_to_f32(int(b)) == float(oracle.bf16_to_f32(np.array([b]))[0])


# ---------------------------------------------------------------------------
# rotation
# ---------------------------------------------------------------------------

def test_cd_constant():
    # RN_f32(2^-3.5): the binary32 pattern of sqrt(2) with exponent -4
    assert np.float32(oracle.cd_f32(128)).view(np.uint32) == 0x3DB504F3
    assert oracle.cd_f32(64) == 0.125
    for d in (2, 4, 8, 16, 32, 256):
        assert oracle.cd_f32(d) == np.float32(1.0 / math.sqrt(d))


@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128])
def test_hadamard_matches_scipy(d):
    H = scipy.linalg.hadamard(d)
    for i in range(d):
        for j in range(d):
            assert oracle.hadamard_entry(i, j) == H[i, j]


@pytest.mark.parametrize("d", [4, 64, 128])
@pytest.mark.parametrize("seed", [0, 3])
def test_rotation_matrix_orthogonal_and_closed_form(d, seed):
    R = oracle.rotation_matrix_f64(d, seed)
    assert np.abs(R @ R.T - np.eye(d)).max() < 1e-12
    H = scipy.linalg.hadamard(d).astype(np.float64)
    D = oracle.signs(seed, d).astype(np.float64)
    assert np.abs(R - H @ np.diag(D) / math.sqrt(d)).max() < 1e-15
    # Rot e_j = c_d D_jj H[:, j]
    for j in (0, 1, d - 1):
        e = np.zeros(d)
        e[j] = 1
        assert np.abs(R @ e - D[j] * H[:, j] / math.sqrt(d)).max() < 1e-15


@pytest.mark.parametrize("d", [4, 64, 128])
def test_fwht_f64_equals_matrix(d):
    rng = np.random.default_rng(d)
    v = rng.standard_normal(d)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    assert np.abs(oracle.fwht_f64(v) - H @ v).max() < 1e-12 * np.abs(v).sum()


@pytest.mark.parametrize("d", [4, 64, 128])
def test_rotate_f32_within_rounding_of_definition(d):
    rng = np.random.default_rng(100 + d)
    R = oracle.rotation_matrix_f64(d, 5)
    for _ in range(50):
        r = (rng.standard_normal(d) * np.exp(rng.standard_normal(d))).astype(np.float32)
        y32 = oracle.rotate_f32(r, 5).astype(np.float64)
        y64 = R @ r.astype(np.float64)
        bound = (math.log2(d) + 2) * 2.0 ** -23 * np.abs(r).sum() / math.sqrt(d)
        assert np.abs(y32 - y64).max() <= bound
    # exact on a power-of-two basis vector (no rounding anywhere)
    e = np.zeros(d, dtype=np.float32)
    e[3] = 1.0
    y = oracle.rotate_f32(e, 5).astype(np.float64)
    assert np.array_equal(y, (R @ e.astype(np.float64)).astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

def _levels(codes, bits):
    return 2 * codes.astype(np.int64) - (2 ** bits - 1)


@pytest.mark.parametrize("bits", [2, 4])
def test_code_rule_is_nearest_level_brute_force(bits):
    # For u off the decision boundaries, floor(u) + 2^(b-1) is the code whose
    # level (in u units, l/2) is nearest; at a boundary the upper one wins.
    rng = np.random.default_rng(bits)
    half = 2 ** (bits - 1)
    for g in (1, 2, 3, 5, 8):
        for _ in range(300):
            y = (rng.standard_normal(g) * rng.choice([1e-3, 1.0, 50.0])).astype(np.float32)
            c, _, _, _ = oracle.quantize_group_f32(y, bits)
            amax = np.float32(np.abs(y).max())
            inv = np.float32(np.float32(half - 0.5) / amax)
            u = (y * inv).astype(np.float32)
            cand = np.arange(2 ** bits)
            for i in range(g):
                dist = np.abs(u[i].astype(np.float64) - (cand - half + 0.5))
                best = cand[dist == dist.min()]
                assert c[i] == best.max()


def test_tie_goes_up_and_is_counted():
    c, _, _, ties = oracle.quantize_group_f32(np.array([1.5, 1.0, -1.0, 0.0], np.float32), 2)
    # inv = 1.5 / 1.5 = 1; u = (1.5, 1, -1, 0): 1, -1 and 0 are boundaries
    assert list(c) == [3, 3, 1, 2]
    assert ties == 3


@pytest.mark.parametrize("bits", [2, 4])
def test_ls_scale_beats_brute_force_scan(bits):
    rng = np.random.default_rng(10 + bits)
    for trial in range(40):
        g = int(rng.integers(1, 9))
        y = rng.standard_normal(g).astype(np.float32)
        if trial % 5 == 0:      # adversarial: one outlier
            y[0] *= 40
        c, s_star, _, _ = oracle.quantize_group_f32(y, bits)
        lv = _levels(c, bits).astype(np.float64)
        yd = y.astype(np.float64)
        f = lambda s: np.sum((yd[:, None] - s[None, :] * lv[:, None]) ** 2, axis=0)
        grid = np.linspace(0.0, 2.0 * abs(s_star) + 1e-12, 100001)
        assert f(np.array([s_star]))[0] <= f(grid).min() + 1e-12
        # normal equation of the least-squares fit
        assert abs(np.dot(yd - s_star * lv, lv)) < 1e-9 * (1 + np.abs(yd).sum())


@pytest.mark.parametrize("bits", [2, 4])
def test_zero_group(bits):
    c, s, h, ties = oracle.quantize_group_f32(np.zeros(32, np.float32), bits)
    assert (c == 2 ** (bits - 1)).all() and s == 0.0 and h == 0 and ties == 0
    # subnormal-only groups are treated as zero (inv = 0)
    tiny = np.full(8, 1e-40, dtype=np.float32)
    c, s, h, _ = oracle.quantize_group_f32(tiny, bits)
    assert (c == 2 ** (bits - 1)).all()


@pytest.mark.parametrize("bits", [2, 4])
def test_on_grid_group_reconstructs_exactly(bits):
    rng = np.random.default_rng(20 + bits)
    top = 2 ** bits - 1
    for _ in range(100):
        g = 32
        lv = rng.choice(np.arange(-top, top + 1, 2), size=g)
        lv[0] = top * rng.choice([-1, 1])        # the group spans the grid
        s = 2.0 ** int(rng.integers(-8, 3))
        y = (s * lv).astype(np.float32)
        c, s_star, h, _ = oracle.quantize_group_f32(y, bits)
        assert np.array_equal(_levels(c, bits), lv)
        assert s_star == s
        assert oracle.f16_to_f64(h) == s


def test_golden_encode_examples(golden):
    g = golden("tiny_encode_d4.txt")
    seed = int(g["seed"])
    assert list(oracle.signs(seed, 4)) == _parse_ints(g["signs"])
    for ex in "ABC":
        bits = int(g[f"{ex} bits"])
        x = _bf16_bits([float(v) for v in g[f"{ex} x"].split()])
        ref = _bf16_bits([float(v) for v in g[f"{ex} ref"].split()])
        y = oracle.rotate_f32(oracle.bf16_to_f32(x) - oracle.bf16_to_f32(ref), seed)
        assert list(y) == [float(v) for v in g[f"{ex} y"].split()]
        words, scales, ties = oracle.encode_rows_f32(x[None], ref[None], bits, 4, seed)
        codes = oracle.unpack_codes(words, bits, 4)[0]
        assert list(codes) == _parse_ints(g[f"{ex} codes"])
        assert int(words[0, 0]) == int(g[f"{ex} word"], 16)
        assert int(scales[0, 0]) == int(g[f"{ex} scale_f16"], 16)
        assert ties == int(g[f"{ex} ties"])


def test_golden_packing(golden):
    g = golden("packing.txt")
    for key, bits in (("int2", 2), ("int2b", 2), ("int4", 4)):
        codes = np.array(_parse_ints(g[f"{key} codes"]), dtype=np.uint8)
        want = np.array(_parse_ints(g[f"{key} words"]), dtype=np.uint32)
        assert np.array_equal(oracle.pack_codes(codes, bits), want)
        assert np.array_equal(oracle.unpack_codes(want, bits, codes.size), codes)


# ---------------------------------------------------------------------------
# encoder: fp32 spec vs fp64 definition, reconstruction invariants
# ---------------------------------------------------------------------------

def _rows(rng, n, d, sigma):
    ref = rng.standard_normal((n, d)) * np.exp(0.5 * rng.standard_normal(d))
    x = ref + sigma * rng.standard_normal((n, d))
    return _bf16_bits(x), _bf16_bits(ref)


@pytest.mark.parametrize("d,g,bits", [(64, 32, 2), (128, 32, 2), (128, 64, 2), (128, 32, 4)])
def test_f32_spec_agrees_with_f64_definition(d, g, bits):
    rng = np.random.default_rng(d + g + bits)
    x, ref = _rows(rng, 60, d, 0.1)
    words, scales, _ = oracle.encode_rows_f32(x, ref, bits, g, 9)
    codes32 = oracle.unpack_codes(words, bits, d)
    mism = near = 0
    for i in range(x.shape[0]):
        c64, s64, bd = oracle.encode_row_f64(x[i], ref[i], bits, g, 9)
        diff = codes32[i] != c64
        near += int((bd < 1e-4).sum())
        # every disagreement is an element sitting on a decision boundary
        assert (bd[diff] < 1e-4).all()
        mism += int(diff.sum())
        s32 = np.array([oracle.f16_to_f64(h) for h in scales[i]])
        groups_ok = np.array([not diff[k * g:(k + 1) * g].any() for k in range(d // g)])
        # where the codes agree the stored scale is the fp16 of the f64 scale
        # to within one fp16 ulp
        assert np.all(np.abs(s32 - s64)[groups_ok] <= 2.0 ** -10 * np.abs(s64)[groups_ok] + 2.0 ** -24)
    assert mism <= near


@pytest.mark.parametrize("bits", [2, 4])
def test_zero_residual_reconstructs_reference_exactly(bits):
    rng = np.random.default_rng(3)
    _, ref = _rows(rng, 8, 128, 0.0)
    words, scales, _ = oracle.encode_rows_f32(ref, ref, bits, 32, 11)
    assert (oracle.unpack_codes(words, bits, 128) == 2 ** (bits - 1)).all()
    assert (scales == 0).all()
    rec = oracle.reconstruct_rows_f64(ref, words, scales, bits, 32, 11)
    assert np.array_equal(rec, oracle.bf16_to_f32(ref).astype(np.float64))


@pytest.mark.parametrize("d,g,bits", [(64, 32, 2), (128, 64, 2), (128, 32, 4)])
def test_reconstruction_matches_independent_hadamard_route(d, g, bits):
    # ref + Rot^T (s16 * l), with Rot built from scipy's Hadamard matrix and
    # the oracle's pinned signs; plus the isometry ||r - r_hat|| = ||y - y_hat||.
    rng = np.random.default_rng(d * bits)
    x, ref = _rows(rng, 10, d, 0.2)
    seed = 77
    words, scales, _ = oracle.encode_rows_f32(x, ref, bits, g, seed)
    rec = oracle.reconstruct_rows_f64(ref, words, scales, bits, g, seed)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    Rot = H @ np.diag(oracle.signs(seed, d).astype(np.float64)) / math.sqrt(d)
    codes = oracle.unpack_codes(words, bits, d)
    for i in range(x.shape[0]):
        s = np.repeat([oracle.f16_to_f64(h) for h in scales[i]], g)
        yhat = s * _levels(codes[i], bits)
        want = oracle.bf16_to_f32(ref[i]).astype(np.float64) + Rot.T @ yhat
        assert np.abs(rec[i] - want).max() < 1e-12
        r = oracle.bf16_to_f32(x[i]).astype(np.float64) - oracle.bf16_to_f32(ref[i])
        y = Rot @ r
        rhat = rec[i] - oracle.bf16_to_f32(ref[i])
        assert abs(np.linalg.norm(r - rhat) - np.linalg.norm(y - yhat)) < 1e-12
        # the residual code actually helps: error well below the residual
        assert np.linalg.norm(r - rhat) < 0.75 * np.linalg.norm(r)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _sdpa64(q, K, V, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :].transpose(1, 2),
        torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None], scale=scale)
    return out[0, 0].numpy()


@pytest.mark.parametrize("T,G,d", [(1, 1, 64), (37, 4, 64), (300, 1, 128)])
def test_attention_matches_sdpa(T, G, d):
    rng = np.random.default_rng(T)
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((T, d)) * 2
    V = rng.standard_normal((T, d))
    out = oracle.attention_f64(q, K, V, 1 / math.sqrt(d))
    assert np.abs(out - _sdpa64(q, K, V, 1 / math.sqrt(d))).max() < 1e-12
    # scores far beyond exp's range: only a max-subtracted softmax survives
    out = oracle.attention_f64(q, K * 400, V, 1 / math.sqrt(d))
    assert np.isfinite(out).all()
    assert np.abs(out - _sdpa64(q, K * 400, V, 1 / math.sqrt(d))).max() < 1e-9


@pytest.mark.parametrize("T,G,d,g", [(1, 4, 64, 32), (100, 1, 128, 32), (77, 4, 128, 64)])
def test_reference_loop_decode_is_plain_attention(T, G, d, g):
    rng = np.random.default_rng(T + G)
    _, rk = _rows(rng, T, d, 0)
    _, rv = _rows(rng, T, d, 0)
    q = _bf16_bits(rng.standard_normal((G, d)))
    out = oracle.decode_attention_f64(q, rk, rv, None, None, None, None, 16, g, 5)
    want = _sdpa64(oracle.bf16_to_f32(q).astype(np.float64), oracle.bf16_to_f32(rk).astype(np.float64),
                   oracle.bf16_to_f32(rv).astype(np.float64), 1 / math.sqrt(d))
    assert np.abs(out - want).max() < 1e-12
    # zero scales reduce a residual loop to the reference loop
    for bits in (2, 4):
        wpr = d * bits // 32
        codes = rng.integers(0, 2 ** 32, size=(T, wpr), dtype=np.uint32)
        zs = np.zeros((T, d // g), dtype=np.uint16)
        out2 = oracle.decode_attention_f64(q, rk, rv, codes, codes, zs, zs, bits, g, 5)
        assert np.abs(out2 - want).max() < 1e-12


@pytest.mark.parametrize("bits", [2, 4])
def test_residual_loop_decode_is_attention_over_reconstruction(bits):
    rng = np.random.default_rng(50 + bits)
    T, G, d, g, seed = 64, 4, 64, 32, 123
    xk, rk = _rows(rng, T, d, 0.3)
    xv, rv = _rows(rng, T, d, 0.3)
    q = _bf16_bits(rng.standard_normal((G, d)))
    wk, sk, _ = oracle.encode_rows_f32(xk, rk, bits, g, seed)
    wv, sv, _ = oracle.encode_rows_f32(xv, rv, bits, g, seed)
    out = oracle.decode_attention_f64(q, rk, rv, wk, wv, sk, sv, bits, g, seed)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    Rot = H @ np.diag(oracle.signs(seed, d).astype(np.float64)) / math.sqrt(d)

    def rebuild(ref, w, s):
        lv = _levels(oracle.unpack_codes(w, bits, d), bits)
        sc = np.repeat(np.vectorize(oracle.f16_to_f64)(s), g, axis=1)
        return oracle.bf16_to_f32(ref).astype(np.float64) + (sc * lv) @ Rot

    want = _sdpa64(oracle.bf16_to_f32(q).astype(np.float64), rebuild(rk, wk, sk),
                   rebuild(rv, wv, sv), 1 / math.sqrt(d))
    assert np.abs(out - want).max() < 1e-10
    # and the quantised loop is close to, but not identical with, the BF16 loop
    exact = _sdpa64(oracle.bf16_to_f32(q).astype(np.float64), oracle.bf16_to_f32(xk).astype(np.float64),
                    oracle.bf16_to_f32(xv).astype(np.float64), 1 / math.sqrt(d))
    err = np.abs(out - exact).max()
    assert 0 < err < 0.5


# ---------------------------------------------------------------------------
# least-squares refinement (alternating code / scale refits)
# ---------------------------------------------------------------------------

def _levels(codes, bits):
    return 2 * codes.astype(np.int64) - ((1 << bits) - 1)


def test_refinement_worked_example(golden):
    # hand-derived in tests/golden/ls_refinement_g8.txt
    g = golden("ls_refinement_g8.txt")
    y = np.array([float(v) for v in g["y"].split()], dtype=np.float32)
    for it, ck, sk in ((0, "codes0", "s0"), (1, "codes1", "s1"), (2, "codes2", "s2")):
        codes, s32, _ = oracle.quantize_group_refined_f32(y, 2, it)
        assert codes.tolist() == [int(v) for v in g[ck].split()]
        assert abs(s32 - float(g[sk])) <= 1e-6
        c64, s64, err, done = oracle.quantize_group_refined_f64(y.astype(np.float64), 2, it)
        assert c64.tolist() == codes.tolist()
    _, _, err, _ = oracle.quantize_group_refined_f64(y.astype(np.float64), 2, 1)
    assert abs(err[0] - float(g["err0"])) < 1e-3 and abs(err[1] - float(g["err1"])) < 1e-3


@pytest.mark.parametrize("bits,group", [(2, 32), (2, 64), (4, 32), (4, 64)])
def test_refinement_error_never_increases(bits, group):
    # nearest-level codes minimise the error for a fixed scale, and the
    # least-squares scale minimises it for fixed codes: the error of the
    # alternation can only go down
    rng = np.random.default_rng(100 + bits + group)
    for trial in range(300):
        kind = trial % 3
        if kind == 0:
            y = rng.standard_normal(group)
        elif kind == 1:
            y = rng.laplace(size=group)
        else:
            y = rng.standard_normal(group) * 0.1
            y[rng.integers(group)] = 5.0          # one outlier sets the absmax
        _, _, err, done = oracle.quantize_group_refined_f64(y, bits, 8)
        assert np.all(np.diff(err) <= 1e-12 * err[0]), (trial, err)


@pytest.mark.parametrize("bits", [2, 4])
def test_refit_codes_are_the_nearest_levels(bits):
    # brute force over every level, independent of the floor rule
    rng = np.random.default_rng(7 + bits)
    top = (1 << bits) - 1
    all_levels = np.arange(-top, top + 1, 2)
    for _ in range(200):
        y = rng.standard_normal(32)
        _, s0, _, _ = oracle.quantize_group_refined_f64(y, bits, 0)
        c1, _, _, _ = oracle.quantize_group_refined_f64(y, bits, 1)
        best = all_levels[np.argmin(np.abs(y[:, None] - s0 * all_levels[None, :]), axis=1)]
        assert np.array_equal(_levels(c1, bits), best)


@pytest.mark.parametrize("bits", [2, 4])
def test_refinement_fixed_point_on_an_exact_grid(bits):
    # y = s l with s a power of two and levels that include the outermost:
    # every quantity is exact, the first step already lands on the grid and
    # no refit moves it
    rng = np.random.default_rng(3)
    top = (1 << bits) - 1
    lv = rng.choice(np.arange(-top, top + 1, 2), size=32)
    lv[5] = top
    y = (0.25 * lv).astype(np.float32)
    for it in (0, 1, 4):
        codes, s32, h = oracle.quantize_group_refined_f32(y, bits, it)
        assert np.array_equal(_levels(codes, bits), lv)
        assert s32 == 0.25 and oracle.f16_to_f64(h) == 0.25


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 64)])
def test_zero_refits_keep_the_unrefined_codes(bits, group):
    rng = np.random.default_rng(11)
    for _ in range(100):
        y = rng.standard_normal(group).astype(np.float32)
        c_ref, _, s_ref, _ = oracle.quantize_group_f32(y, bits)
        codes, _, h = oracle.quantize_group_refined_f32(y, bits, 0)
        assert np.array_equal(codes, c_ref)
        a, b = oracle.f16_to_f64(h), oracle.f16_to_f64(s_ref)
        assert abs(a - b) <= 1e-3 * abs(b) + 2.0 ** -24


def test_fixed_order_dot_within_its_rounding_bound():
    rng = np.random.default_rng(5)
    for g in (8, 32, 64):
        for _ in range(100):
            y = rng.standard_normal(g).astype(np.float32)
            lv = rng.choice([-3, -1, 1, 3], size=g)
            exact = float(np.sum(y.astype(np.float64) * lv))
            got = oracle.ls_dot_f32(y, lv)
            bound = g * 2.0 ** -23 * float(np.sum(np.abs(y.astype(np.float64) * lv)))
            assert abs(got - exact) <= bound
        yi = rng.integers(-50, 50, size=g).astype(np.float32)     # all sums exact
        lv = rng.choice([-3, -1, 1, 3], size=g)
        assert oracle.ls_dot_f32(yi, lv) == float(np.sum(yi.astype(np.int64) * lv))


# ---------------------------------------------------------------------------
# compressed reference (the final loop stored as rotated codes)
# ---------------------------------------------------------------------------

def _bf16(v):
    a = np.asarray(v, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _rand_bf16(rng, shape, scale=1.0):
    return _bf16((rng.standard_normal(shape) * scale).astype(np.float32))


def test_cr_reference_codes_are_the_zero_reference_encoder():
    # quantising Rot(ref) is what the plain encoder does to ref against a
    # zero reference: same codes (scales differ only in their sum order)
    rng = np.random.default_rng(41)
    ref = _rand_bf16(rng, (50, 128))
    rw, rs, _, _ = oracle.encode_rows_cr_f32(None, ref, 4, 2, 32, 9)
    w4, s4, _ = oracle.encode_rows_f32(ref, np.zeros_like(ref), 4, 32, 9)
    assert np.array_equal(rw, w4)
    a = np.vectorize(oracle.f16_to_f64)(rs)
    b = np.vectorize(oracle.f16_to_f64)(s4)
    assert np.all(np.abs(a - b) <= 1e-3 * np.abs(b) + 2.0 ** -24)


def test_cr_exact_grid_reference_round_trips_exactly():
    # d = 4, Rot = (1/2) H D: choose the rotated reference on the INT4 grid
    # s l with s = 1/4 (levels include +-15), so that ref = D H y / 2 is a
    # short dyadic vector, exact in bf16; then the reference reconstructs
    # exactly, and a non-final loop equal to it gets a zero residual
    d, seed = 4, 20                      # seed 20: all signs +1 for d = 4
    assert list(oracle.signs(seed, d)) == [1, 1, 1, 1]
    lv = np.array([15, -1, 3, -5])
    y = 0.25 * lv
    H = np.array([[oracle.hadamard_entry(i, j) for j in range(d)] for i in range(d)])
    ref = H.T @ y / 2.0
    rb = _bf16(ref)
    assert np.array_equal(oracle.bf16_to_f32(rb).astype(np.float64), ref)
    rw, rs, w, s = oracle.encode_rows_cr_f32(rb[None], rb[None], 4, 2, 4, seed)
    codes = oracle.unpack_codes(rw[0], 4, d)
    assert np.array_equal(2 * codes.astype(int) - 15, lv)
    assert oracle.f16_to_f64(int(rs[0, 0])) == 0.25
    K_ref = oracle.reconstruct_rows_cr_f64(rw, rs, None, None, 4, 2, 4, seed, d)
    K_l = oracle.reconstruct_rows_cr_f64(rw, rs, w, s, 4, 2, 4, seed, d)
    assert np.array_equal(K_ref[0], ref) and np.array_equal(K_l[0], ref)
    assert oracle.f16_to_f64(int(s[0, 0])) == 0.0


def test_cr_reconstruction_is_orthogonal():
    # ||K^_l - x|| equals the rotated-domain error ||z + s l - R x||, with R
    # the explicit rotation matrix: checks that reconstruction applies R^T
    rng = np.random.default_rng(43)
    d, g, seed = 64, 32, 12
    ref = _rand_bf16(rng, (6, d))
    x = _bf16(oracle.bf16_to_f32(ref) + 0.2 * rng.standard_normal((6, d)).astype(np.float32))
    rw, rs, w, s = oracle.encode_rows_cr_f32(x, ref, 8, 4, g, seed)
    K = oracle.reconstruct_rows_cr_f64(rw, rs, w, s, 8, 4, g, seed, d)
    R = oracle.rotation_matrix_f64(d, seed)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    for i in range(6):
        cr = oracle.unpack_codes(rw[i], 8, d).astype(int)
        c = oracle.unpack_codes(w[i], 4, d).astype(int)
        sr = np.repeat([oracle.f16_to_f64(int(h)) for h in rs[i]], g)
        sl = np.repeat([oracle.f16_to_f64(int(h)) for h in s[i]], g)
        z = sr * (2 * cr - 255) + sl * (2 * c - 15)
        assert abs(np.linalg.norm(K[i] - xf[i]) - np.linalg.norm(z - R @ xf[i])) < 1e-9


@pytest.mark.parametrize("ref_bits", [4, 8])
def test_cr_residual_moves_the_loop_closer(ref_bits):
    rng = np.random.default_rng(44 + ref_bits)
    d, g, seed = 128, 32, 3
    ref = _rand_bf16(rng, (40, d))
    x = _bf16(oracle.bf16_to_f32(ref) + 0.1 * rng.standard_normal((40, d)).astype(np.float32))
    rw, rs, w, s = oracle.encode_rows_cr_f32(x, ref, ref_bits, 2, g, seed)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    K_ref = oracle.reconstruct_rows_cr_f64(rw, rs, None, None, ref_bits, 2, g, seed, d)
    K_l = oracle.reconstruct_rows_cr_f64(rw, rs, w, s, ref_bits, 2, g, seed, d)
    assert np.linalg.norm(K_l - xf) < np.linalg.norm(K_ref - xf)


def _nearest_levels_on_absmax_grid(e, bits):
    """Brute force over the 2^b points amax*l/(2^b - 1), l odd: the level of
    the nearest point per coordinate, and the gap to the runner-up (how far
    the coordinate sits from a decision boundary)."""
    top = (1 << bits) - 1
    levels = np.arange(-top, top + 1, 2)
    grid = np.abs(e).max() * levels / top
    dist = np.abs(e[:, None] - grid[None, :])
    order = np.argsort(dist, axis=1, kind="stable")
    near = np.take_along_axis(dist, order[:, :2], axis=1)
    return levels[order[:, 0]], near[:, 1] - near[:, 0]


def _check_cr_residual_base(x, ref, ref_bits, bits, g, seed):
    """The residual of a non-final loop is quantised against the
    reconstructed reference in the rotated domain, e = R x - z with
    z = s_ref l_ref (ResidualQuant Abstract: the final loop is the reference;
    this format stores that reference itself as rotated codes).  e is formed
    here in fp64 from the explicit rotation matrix and the reference's own
    codes and scales; the loop's codes must be the nearest levels of e on its
    absmax grid (away from decision boundaries) and its scales the
    least-squares optimum for those codes, to one fp16 step."""
    d = x.shape[-1]
    rw, rs, w, s = oracle.encode_rows_cr_f32(x, ref, ref_bits, bits, g, seed)
    R = oracle.rotation_matrix_f64(d, seed)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    rtop, top = (1 << ref_bits) - 1, (1 << bits) - 1
    checked = 0
    for i in range(x.shape[0]):
        cr = oracle.unpack_codes(rw[i], ref_bits, d).astype(int)
        sr = np.repeat([oracle.f16_to_f64(int(h)) for h in rs[i]], g)
        e = R @ xf[i] - sr * (2 * cr - rtop)
        lv = 2 * oracle.unpack_codes(w[i], bits, d).astype(int) - top
        for k in range(d // g):
            eg, lg = e[k * g:(k + 1) * g], lv[k * g:(k + 1) * g]
            want, gap = _nearest_levels_on_absmax_grid(eg, bits)
            clear = gap > 1e-4 * np.abs(eg).max()
            assert clear.sum() >= g // 2
            assert np.array_equal(lg[clear], want[clear]), (i, k)
            s_opt = float(eg @ lg) / float(lg @ lg)
            s16 = oracle.f16_to_f64(int(s[i, k]))
            step = 2.0 ** (math.floor(math.log2(abs(s_opt))) - 10)
            assert abs(s16 - s_opt) <= step + 1e-6 * abs(s_opt), (i, k, s16, s_opt)
            checked += 1
    return checked


@pytest.mark.parametrize("ref_bits", [4, 8])
def test_cr_loop_equal_to_reference_encodes_the_reference_error(ref_bits):
    # a non-final loop identical to the final loop: its residual is the
    # reference's own quantisation error R ref - z, which is not zero, so the
    # loop must end up strictly closer to ref than the reference codes alone
    rng = np.random.default_rng(60 + ref_bits)
    d, g, seed = 128, 32, 5
    ref = _rand_bf16(rng, (12, d), scale=2.0)
    assert _check_cr_residual_base(ref, ref, ref_bits, 2, g, seed) == 12 * d // g
    rw, rs, w, s = oracle.encode_rows_cr_f32(ref, ref, ref_bits, 2, g, seed)
    assert np.all(s != 0)
    rf = oracle.bf16_to_f32(ref).astype(np.float64)
    K_ref = oracle.reconstruct_rows_cr_f64(rw, rs, None, None, ref_bits, 2, g, seed, d)
    K_l = oracle.reconstruct_rows_cr_f64(rw, rs, w, s, ref_bits, 2, g, seed, d)
    for i in range(ref.shape[0]):
        assert np.linalg.norm(K_l[i] - rf[i]) < np.linalg.norm(K_ref[i] - rf[i])


@pytest.mark.parametrize("ref_bits,bits,g", [(4, 2, 32), (4, 4, 64), (8, 2, 64)])
def test_cr_residual_is_taken_against_the_reconstructed_reference(ref_bits, bits, g):
    rng = np.random.default_rng(70 + ref_bits + bits + g)
    d, seed = 128, 8
    ref = _rand_bf16(rng, (10, d))
    x = _bf16(oracle.bf16_to_f32(ref) + 0.1 * rng.standard_normal((10, d)).astype(np.float32))
    assert _check_cr_residual_base(x, ref, ref_bits, bits, g, seed) == 10 * d // g
