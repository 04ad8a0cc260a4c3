"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here:
  * library routines: scipy.linalg.hadamard, NumPy's legacy MT19937 / RandomState.randn,
    NumPy's float16 conversion, np.searchsorted, np.argmin, np.unpackbits, matmul;
  * closed forms: Gaussian Lloyd-Max levels from exact integrals, the expected relative
    distortion of a group-normalised Gaussian source, the Hadamard image of a constant
    or one-hot vector;
  * values printed on the pages (tests/golden/pages_constants.json);
  * brute force on tiny inputs (exhaustive 1-D k-means).
A plausible slip anywhere in the oracle (a dropped term, wrong sign or index, transposed
operand, wrong packing bit order) fails at least one of these.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.integrate as si
import scipy.linalg as sl
import scipy.special as sp
import scipy.stats as st

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))
G128 = GOLD["group_size"]["value"]


# ----------------------------------------------------------------------------------------
# independent closed forms
# ----------------------------------------------------------------------------------------

def gauss_lloyd_closed(L, iters=100000, tol=1e-15):
    """Gaussian Lloyd-Max levels from exact truncated-normal centroids."""
    c = st.norm.ppf((np.arange(L) + 0.5) / L)
    for _ in range(iters):
        b = np.concatenate([[-np.inf], (c[:-1] + c[1:]) / 2, [np.inf]])
        p = st.norm.cdf(b[1:]) - st.norm.cdf(b[:-1])
        new = (st.norm.pdf(b[:-1]) - st.norm.pdf(b[1:])) / p
        if np.max(np.abs(new - c)) < tol:
            c = new
            break
        c = new
    b = np.concatenate([[-np.inf], (c[:-1] + c[1:]) / 2, [np.inf]])
    p = st.norm.cdf(b[1:]) - st.norm.cdf(b[:-1])
    mse = 1.0 - float(np.sum(p * c * c))
    return c, mse


def sphere_coord_density(g):
    """Density of t = sqrt(g) * u_i, u uniform on the unit sphere in R^g."""
    lognorm = sp.gammaln(g / 2) - sp.gammaln((g - 1) / 2) - 0.5 * math.log(g * math.pi)
    return lambda t: math.exp(lognorm) * max(0.0, 1.0 - t * t / g) ** ((g - 3) / 2)


def expected_rel_mse(levels_unscaled, g):
    """E[(t - Q(t))^2] with Q = nearest level, t ~ sqrt(g) * sphere coordinate."""
    f = sphere_coord_density(g)
    c = np.asarray(levels_unscaled, np.float64)
    mids = (c[:-1] + c[1:]) / 2
    edges = np.concatenate([[-math.sqrt(g)], mids, [math.sqrt(g)]])
    tot = 0.0
    for k in range(len(c)):
        val, _ = si.quad(lambda t: (t - c[k]) ** 2 * f(t), edges[k], edges[k + 1], limit=200)
        tot += val
    return tot


def unpack_fields(packed, field_bits, g):
    """Independent LSB-first unpack with numpy.unpackbits."""
    bits = np.unpackbits(packed.reshape(-1, packed.shape[-1]), axis=-1, bitorder="little")
    bits = bits.reshape(-1, g, field_bits).astype(np.int64)
    return (bits * (1 << np.arange(field_bits))).sum(-1).reshape(packed.shape[:-1] + (g,))


def scipy_H(g):
    return sl.hadamard(g).astype(np.float64) / math.sqrt(g)


# ----------------------------------------------------------------------------------------
# Hadamard
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("g", [8, 16, 128, 256])
def test_hadamard_matches_scipy_and_is_orthonormal(g):
    H = oracle.hadamard(g)
    Hint = np.rint(H * math.sqrt(g)).astype(np.int64)
    assert np.array_equal(Hint, sl.hadamard(g))
    assert np.array_equal(Hint @ Hint.T, g * np.eye(g, dtype=np.int64))
    assert np.allclose(H @ H, np.eye(g), atol=1e-14)  # symmetric, self-inverse


def test_hadamard_sylvester_recursion():
    H64 = np.rint(oracle.hadamard(64) * 8).astype(np.int64)
    H128 = np.rint(oracle.hadamard(128) * math.sqrt(128)).astype(np.int64)
    assert np.array_equal(H128, np.block([[H64, H64], [H64, -H64]]))


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.hadamard(96)


# ----------------------------------------------------------------------------------------
# MT19937 / randn: bit-exact against NumPy's legacy RandomState
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 5489, 2**32 - 1])
def test_mt19937_raw_matches_numpy(seed):
    rs = np.random.RandomState(seed)
    assert np.array_equal(oracle.mt_uint32(seed, 2000),
                          rs._bit_generator.random_raw(2000).astype(np.uint32))


@pytest.mark.parametrize("seed", [0, 3, 12345])
def test_randn_matches_numpy_legacy(seed):
    n = GOLD["lloyd_samples"]["value"]
    assert np.array_equal(oracle.randn(seed, n), np.random.RandomState(seed).randn(n))


# ----------------------------------------------------------------------------------------
# Lloyd-Max
# ----------------------------------------------------------------------------------------

def test_closed_form_helper_reproduces_page_ternary_constant():
    c, mse = gauss_lloyd_closed(3)
    assert abs(c[2] - GOLD["ternary_level"]["value"]) < 5e-8
    assert abs(c[1]) < 1e-12


@pytest.mark.parametrize("L,iters,tol", [(3, 300, 1.5e-5), (4, 400, 5e-5), (8, 3000, 3e-4)])
def test_lloyd_on_quantile_sample_converges_to_closed_form(L, iters, tol):
    n = 200000
    x = sp.ndtri((np.arange(n) + 0.5) / n)
    c = oracle.lloyd_on_sorted(x, L, iters)
    ref, _ = gauss_lloyd_closed(L)
    assert np.max(np.abs(c - ref)) < tol


@pytest.mark.parametrize("L,tol_level,tol_mse", [(4, 5e-3, 0.01), (8, 1.5e-2, 0.01),
                                                 (16, 3e-2, 0.01)])
def test_lloyd_max_with_page_parameters_near_closed_form(L, tol_level, tol_mse):
    c = oracle.lloyd_max(L, GOLD["lloyd_samples"]["value"], GOLD["lloyd_iters"]["value"], 0)
    ref, ref_mse = gauss_lloyd_closed(L)
    assert np.all(np.diff(c) > 0)
    assert np.max(np.abs(c - ref)) < tol_level
    # sample MSE of the codebook on the same samples, nearest-level assignment
    x = np.sort(np.random.RandomState(0).randn(GOLD["lloyd_samples"]["value"]))
    k = np.searchsorted((c[:-1] + c[1:]) / 2, x, side="left")
    mse = float(np.mean((x - c[k]) ** 2))
    assert abs(mse - ref_mse) / ref_mse < tol_mse


def test_lloyd_max_two_bit_matches_textbook_levels():
    # The classical optimum 4-level quantiser of a unit Gaussian (J. Max, "Quantizing for
    # minimum distortion", IRE Trans. Inf. Theory, 1960) has levels +-0.4528 / +-1.510 and
    # mean squared error 0.1175.
    c = oracle.lloyd_max(4)
    assert np.allclose(np.abs(c), [1.5104, 0.4528, 0.4528, 1.5104], atol=5e-3)
    _, mse = gauss_lloyd_closed(4)
    assert abs(mse - 0.1175) < 1e-4


def test_lloyd_three_levels_near_page_ternary_constant():
    c = oracle.lloyd_max(3)
    assert abs((c[2] - c[0]) / 2 - GOLD["ternary_level"]["value"]) < 2e-3


def _brute_kmeans_1d(x, L):
    """Exhaustive optimum over contiguous partitions of sorted x into L non-empty cells."""
    n = len(x)
    best = np.inf
    import itertools
    for cuts in itertools.combinations(range(1, n), L - 1):
        parts = np.split(x, cuts)
        best = min(best, sum(float(np.sum((p - p.mean()) ** 2)) for p in parts))
    return best


@pytest.mark.parametrize("seed", range(12))
def test_lloyd_fixed_point_against_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(6, 12))
    L = int(rng.integers(2, 5))
    x = np.sort(rng.standard_normal(n) * rng.uniform(0.5, 3))
    c = oracle.lloyd_on_sorted(x, L, 500)
    b = (c[:-1] + c[1:]) / 2
    k = np.searchsorted(b, x, side="left")
    # centroid condition holds for every non-empty cell
    for j in range(L):
        if np.any(k == j):
            assert abs(c[j] - x[k == j].mean()) < 1e-12
    sse = float(np.sum((x - c[k]) ** 2))
    assert sse >= _brute_kmeans_1d(x, L) - 1e-12


def test_lloyd_reaches_brute_force_optimum_on_separated_clusters():
    x = np.sort(np.array([-5.1, -5.0, -4.8, 0.1, 0.2, 0.25, 6.0, 6.3]))
    c = oracle.lloyd_on_sorted(x, 3, 200)
    k = np.searchsorted((c[:-1] + c[1:]) / 2, x)
    assert abs(float(np.sum((x - c[k]) ** 2)) - _brute_kmeans_1d(x, 3)) < 1e-12


def test_lloyd_zero_iterations_is_quantile_init():
    x = np.sort(np.random.default_rng(1).standard_normal(101))
    c = oracle.lloyd_on_sorted(x, 4, 0)
    assert np.array_equal(c, x[((np.arange(4) + 0.5) / 4 * 101).astype(int)])


# ----------------------------------------------------------------------------------------
# Codebooks
# ----------------------------------------------------------------------------------------

def test_ternary_codebook_is_page_constant_scaled():
    cb = oracle.codebook(0, G128)
    t = GOLD["ternary_level"]["value"]
    assert cb.dtype == np.float32 and cb.size == 3
    assert np.array_equal(cb, (np.array([-t, 0.0, t]) / math.sqrt(G128)).astype(np.float32))


@pytest.mark.parametrize("bits", GOLD["cb_bits"]["value"])
def test_codebook_sizes_scale_and_order(bits):
    cb = oracle.codebook(bits, G128)
    assert cb.size == 2 ** bits
    assert np.all(np.diff(cb) > 0)
    ref, _ = gauss_lloyd_closed(2 ** bits)
    assert np.max(np.abs(cb.astype(np.float64) * math.sqrt(G128) - ref)) < 3e-2
    # a different group size only rescales
    cb64 = oracle.codebook(bits, 64)
    assert np.allclose(cb64 * 8.0, cb * math.sqrt(128), rtol=1e-6)


def test_levels_and_fields():
    assert [oracle.levels(b) for b in (0, 2, 3, 4)] == [3, 4, 8, 16]
    assert [oracle.field_bits(b) for b in (0, 2, 3, 4)] == [2, 2, 3, 4]
    assert oracle.levels(2) == GOLD["levels_2bit"]["value"]
    assert oracle.levels(1) == -1 and oracle.levels(5) == -1


# ----------------------------------------------------------------------------------------
# Rounding helpers
# ----------------------------------------------------------------------------------------

def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]),
        # exact halfway cases between neighbouring fp16 values
        (np.arange(1, 2000) + 0.5) * 2.0 ** -10 + 1.0,
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16_bits(x) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    back = np.array([oracle.f16_bits_to_f64(h) for h in ref[:2000]])
    assert np.array_equal(back, ref[:2000].view(np.float16).astype(np.float64))


def test_bf16_rounding_halfway_cases():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    assert oracle.f64_to_bf16_bits(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.f64_to_bf16_bits(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.f64_to_bf16_bits(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.f64_to_bf16_bits(-2.0) == 0xC000
    assert oracle.f64_to_bf16_bits(3.0e38 * 1.2) == 0x7F80


def test_bf16_rounding_matches_torch_on_fp32_values():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    xs = (rng.standard_normal(5000) * 10.0 ** rng.uniform(-20, 20, 5000)).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f64_to_bf16_bits(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------------------
# Quantise
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_quantize_on_hadamard_domain_construction(bits):
    """Choose the rotated vector r, feed w = H r, and predict every output independently."""
    g = G128
    rng = np.random.default_rng(100 + bits)
    rows, G = 16, 4
    r = rng.standard_normal((rows, G, g)) * rng.uniform(0.01, 3, (rows, G, 1))
    H = scipy_H(g)
    w = (r @ H).reshape(rows, G * g)  # per group w = H r (H symmetric)
    packed, norms = oracle.quantize(w, bits, g)
    cb = oracle.codebook(bits, g).astype(np.float64)
    n = np.linalg.norm(r, axis=-1, keepdims=True)
    u = r / n
    mids = (cb[:-1] + cb[1:]) / 2
    want = np.searchsorted(mids, u, side="left")
    got = unpack_fields(packed, oracle.field_bits(bits), g)
    near = np.min(np.abs(u[..., None] - mids), axis=-1) < 1e-12
    assert np.array_equal(got[~near], want[~near])
    assert np.array_equal(norms, n[..., 0].astype(np.float16).view(np.uint16))


def test_quantize_spike_group_follows_hadamard_row_signs():
    g = G128
    for bits in (2, 4):
        for p in (0, 1, 77, 127):
            w = np.zeros((1, g))
            w[0, p] = 0.37
            packed, norms = oracle.quantize(w, bits, g)
            got = unpack_fields(packed, oracle.field_bits(bits), g)[0, 0]
            cb = oracle.codebook(bits, g).astype(np.float64)
            signs = sl.hadamard(g)[:, p]
            want = np.array([np.argmin(np.abs(s / math.sqrt(g) - cb)) for s in signs])
            assert np.array_equal(got, want)
            if bits == 2:  # both sides pick the outer level
                assert set(got.tolist()) <= {0, 3}
            assert norms[0, 0] == np.float16(0.37).view(np.uint16)


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_quantize_zero_group(bits):
    g = G128
    packed, norms = oracle.quantize(np.zeros((2, 3 * g), np.float32), bits, g)
    cb = oracle.codebook(bits, g)
    want = int(np.argmin(np.abs(cb.astype(np.float64))))  # first index on ties
    assert np.all(norms == 0)
    assert np.all(unpack_fields(packed, oracle.field_bits(bits), g) == want)


def test_quantize_padding_equals_explicit_zero_columns():
    rng = np.random.default_rng(7)
    w = rng.standard_normal((5, 300)).astype(np.float32)
    wp = np.zeros((5, 384), np.float32)
    wp[:, :300] = w
    for bits in (2, 3):
        a = oracle.quantize(w, bits)
        b = oracle.quantize(wp, bits)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_quantize_bf16_input_reads_top_half_of_fp32():
    rng = np.random.default_rng(8)
    w32 = rng.standard_normal((4, 256)).astype(np.float32)
    bf = (w32.view(np.uint32) >> 16).astype(np.uint16)
    exact = (bf.astype(np.uint32) << 16).view(np.float32)
    assert all(np.array_equal(x, y) for x, y in zip(oracle.quantize(bf, 2), oracle.quantize(exact, 2)))


def test_fake_quantize_bf16_input_reads_top_half_of_fp32():
    rng = np.random.default_rng(9)
    w32 = (rng.standard_normal((3, 300)) * 0.02).astype(np.float32)
    bf = (w32.view(np.uint32) >> 16).astype(np.uint16)
    exact = (bf.astype(np.uint32) << 16).view(np.float32)
    for bits in (0, 3):
        assert np.array_equal(oracle.fake_quantize(bf, bits), oracle.fake_quantize(exact, bits))


def test_norm_is_rotation_invariant():
    rng = np.random.default_rng(9)
    w = rng.standard_normal((64, 512)) * 0.02
    _, norms = oracle.quantize(w, 2)
    want = np.linalg.norm(w.reshape(64, 4, 128), axis=-1).astype(np.float16).view(np.uint16)
    assert np.array_equal(norms, want)


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_relative_mse_matches_sphere_closed_form(bits):
    rng = np.random.default_rng(11)
    w = rng.standard_normal((2048, 1024)) * 0.02
    packed, norms = oracle.quantize(w, bits)
    w_hat = oracle.dequantize(packed, norms, 2048, 1024, bits)
    got = oracle.rel_mse(w, w_hat)
    levels = oracle.codebook(bits).astype(np.float64) * math.sqrt(128)
    want = expected_rel_mse(levels, 128)
    assert abs(got - want) / want < 0.01


def test_page_distortion_figures_are_relative_rmse():
    rng = np.random.default_rng(13)
    w = rng.standard_normal((2048, 512))
    out = {}
    for bits in (2, 4):
        p, n = oracle.quantize(w, bits)
        out[bits] = math.sqrt(oracle.rel_mse(w, oracle.dequantize(p, n, 2048, 512, bits)))
    assert abs(out[2] - GOLD["distortion_2bit"]["value"]) < 0.05
    assert abs(out[4] - GOLD["distortion_4bit"]["value"]) < 0.01


# ----------------------------------------------------------------------------------------
# Dequantise
# ----------------------------------------------------------------------------------------

def _pack_fields(idx, field_bits):
    """Independent LSB-first pack with numpy.packbits."""
    bits = ((idx[..., None] >> np.arange(field_bits)) & 1).astype(np.uint8)
    flat = bits.reshape(idx.shape[:-1] + (-1,))
    return np.packbits(flat, axis=-1, bitorder="little")


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_dequantize_constant_index_group_is_scaled_first_basis_vector(bits):
    g = G128
    L = oracle.levels(bits)
    cb = oracle.codebook(bits, g).astype(np.float64)
    idx = np.repeat(np.arange(L)[:, None], g, axis=1)  # row k: every index = k
    packed = _pack_fields(idx, oracle.field_bits(bits))[:, None, :]
    norms = np.full((L, 1), np.float16(1.75).view(np.uint16), np.uint16)
    out = oracle.dequantize(packed, norms, L, g, bits)
    want = np.zeros((L, g))
    want[:, 0] = 1.75 * cb * math.sqrt(g)
    assert np.allclose(out, want, atol=1e-15, rtol=1e-14)


def test_dequantize_one_hot_index_group_is_hadamard_column():
    # indices all pointing at the zero ternary level except one: w_hat = n * c * H[:, p]
    g = G128
    cb = oracle.codebook(0, g).astype(np.float64)
    idx = np.ones((1, g), np.int64)
    idx[0, 5] = 2
    packed = _pack_fields(idx, 2)[:, None, :]
    norms = np.array([[np.float16(3.0).view(np.uint16)]], np.uint16)
    out = oracle.dequantize(packed, norms, 1, g, 0)
    assert np.allclose(out[0], 3.0 * cb[2] * scipy_H(g)[:, 5], atol=1e-15)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequantize_preserves_group_norm(bits):
    rng = np.random.default_rng(20 + bits)
    g, L = G128, oracle.levels(bits)
    idx = rng.integers(0, L, (8, 3, g))
    packed = _pack_fields(idx, bits)
    normv = rng.uniform(0.1, 4, (8, 3)).astype(np.float16)
    out = oracle.dequantize(packed, normv.view(np.uint16), 8, 3 * g, bits).reshape(8, 3, g)
    cb = oracle.codebook(bits, g).astype(np.float64)
    want = normv.astype(np.float64) * np.linalg.norm(cb[idx], axis=-1)
    assert np.allclose(np.linalg.norm(out, axis=-1), want, rtol=1e-13)


def test_dequantize_clamps_unused_ternary_code():
    g = G128
    idx = np.full((1, g), 3)
    packed = _pack_fields(idx, 2)[:, None, :]
    norms = np.array([[np.float16(1.0).view(np.uint16)]], np.uint16)
    idx2 = np.full((1, g), 2)
    packed2 = _pack_fields(idx2, 2)[:, None, :]
    assert np.array_equal(oracle.dequantize(packed, norms, 1, g, 0),
                          oracle.dequantize(packed2, norms, 1, g, 0))


def test_quantize_dequantize_indices_idempotent_and_norm_closed_form():
    rng = np.random.default_rng(21)
    w = rng.standard_normal((256, 512)) * 0.02
    p1, n1 = oracle.quantize(w, 2)
    w1 = oracle.dequantize(p1, n1, 256, 512, 2)
    p2, n2 = oracle.quantize(w1, 2)
    assert np.array_equal(p1, p2)
    cb = oracle.codebook(2).astype(np.float64)
    idx = unpack_fields(p1, 2, 128)
    want = (n1.view(np.float16).astype(np.float64) * np.linalg.norm(cb[idx], axis=-1))
    assert np.array_equal(n2, want.astype(np.float16).view(np.uint16))


# ----------------------------------------------------------------------------------------
# fake quantisation (the pages' cq_quantize output)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_fake_quantize_spike_closed_form(bits):
    """A group holding one value a at position p rotates to s_i |a| / sqrt(g) with
    s_i = sign(a) (-1)^popcount(i & p), so every component picks C+ (the level nearest
    +1/sqrt(g)) or C- (nearest -1/sqrt(g)).  Writing C_i = (C+ + C-)/2 + s_i (C+ - C-)/2 and
    using the orthogonality of the Walsh rows, the inverse rotation is
        w_hat = n16 sqrt(g) [ sign(a) (C+ - C-)/2 e_p + (C+ + C-)/2 e_0 ],
    n16 = fp16(|a|).  A dropped term, a wrong sign, index or scale fails it."""
    g = G128
    cb = oracle.codebook(bits, g).astype(np.float64)
    cp = cb[np.argmin(np.abs(cb - 1 / math.sqrt(g)))]
    cm = cb[np.argmin(np.abs(cb + 1 / math.sqrt(g)))]
    for p in (0, 1, 77, 127):
        for a in (0.37, -2.5):
            w = np.zeros((1, 2 * g))
            w[0, g + p] = a  # second group; the first stays zero
            got = oracle.fake_quantize(w, bits, g)
            n16 = float(np.float16(abs(a)))
            want = np.zeros(2 * g)
            want[g + p] += n16 * math.sqrt(g) * math.copysign(1.0, a) * (cp - cm) / 2
            want[g] += n16 * math.sqrt(g) * (cp + cm) / 2
            assert np.allclose(got[0], want, rtol=1e-12, atol=1e-15), (bits, p, a)


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_fake_quantize_relative_mse_matches_sphere_closed_form(bits):
    rng = np.random.default_rng(31)
    w = rng.standard_normal((1024, 1024)) * 0.02
    got = oracle.rel_mse(w, oracle.fake_quantize(w, bits))
    want = expected_rel_mse(oracle.codebook(bits).astype(np.float64) * math.sqrt(128), 128)
    assert abs(got - want) / want < 0.015


def test_fake_quantize_zero_and_ragged_groups():
    """Zero groups stay zero, and a ragged last group equals the zero-padded computation
    with the padding columns dropped."""
    rng = np.random.default_rng(32)
    w = rng.standard_normal((5, 300)) * 0.02
    w[2, :] = 0.0
    pad = np.zeros((5, 384))
    pad[:, :300] = w
    for bits in (0, 2, 4):
        got = oracle.fake_quantize(w, bits)
        assert np.all(got[2] == 0.0)
        assert np.array_equal(got, oracle.fake_quantize(pad, bits)[:, :300])


def test_unpack_index_matches_numpy_fields():
    rng = np.random.default_rng(22)
    for bits in (2, 3, 4):
        idx = rng.integers(0, 2 ** bits, (1, 128))
        blk = _pack_fields(idx, bits)[0]
        assert [oracle.unpack_index(blk, bits, i) for i in range(128)] == idx[0].tolist()


# ----------------------------------------------------------------------------------------
# GEMV
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols,batch", [(37, 300, 1), (16, 512, 8), (9, 260, 20)])
def test_gemv_matches_hadamard_domain_identity(rows, cols, batch):
    rng = np.random.default_rng(rows + cols)
    w = rng.standard_normal((rows, cols)) * 0.02
    x = rng.standard_normal((batch, cols))
    packed, norms = oracle.quantize(w, 2)
    y = oracle.dequant_gemv(packed, norms, rows, cols, 2, x)
    # y = sum_j n_j <c[idx_j], H x_j>, with x zero padded
    G = packed.shape[1]
    xp = np.zeros((batch, G * 128))
    xp[:, :cols] = x
    xt = xp.reshape(batch, G, 128) @ scipy_H(128)
    cb = oracle.codebook(2).astype(np.float64)
    q = cb[unpack_fields(packed, 2, 128)] * norms.view(np.float16).astype(np.float64)[..., None]
    want = np.einsum("rjk,bjk->br", q, xt)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-14)
    w_hat = oracle.dequantize(packed, norms, rows, cols, 2)
    assert np.allclose(y, x @ w_hat.T, rtol=1e-12, atol=1e-14)


def test_gemv_bf16_activations():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((8, 256))
    x = rng.standard_normal((2, 256)).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    p, n = oracle.quantize(w, 3)
    assert np.array_equal(oracle.dequant_gemv(p, n, 8, 256, 3, xb),
                          oracle.dequant_gemv(p, n, 8, 256, 3, xf))


# ----------------------------------------------------------------------------------------
# Sizes (page 2 "Per-Group Storage Breakdown")
# ----------------------------------------------------------------------------------------

def test_packed_bytes_formula_and_config_totals():
    extra = GOLD["bytes_per_group_extra"]["value"]
    assert oracle.packed_bytes(256, 512, 2) == 256 * 4 * 32
    assert oracle.norm_bytes(256, 512) == 256 * 4 * extra
    assert oracle.packed_bytes(768, 1000, 3) == 768 * 8 * 48
    assert oracle.packed_bytes(1, 1, 0) == 32
    # 45M-parameter stand-in weight set: indices + norms at 2-bit
    shapes = [(8192, 768)] + [(768, 768), (768, 768), (768, 256), (768, 256), (768, 2048),
                              (2048, 768)] * 8 + [(768, 1000)]
    idx = sum(oracle.packed_bytes(r, c, 2) for r, c in shapes)
    nb = sum(oracle.norm_bytes(r, c) for r, c in shapes)
    assert (idx, nb, idx + nb) == (11206656, 700416, 11907072)
    assert sum(r * c for r, c in shapes) == 44808192


def test_oracle_results_do_not_depend_on_its_thread_count():
    """The oracle spreads independent groups over threads; every output is computed by one
    thread in a fixed order, so 1 thread and many give identical bits."""
    rng = np.random.default_rng(40)
    w = rng.standard_normal((67, 1000)) * 0.02
    x = rng.standard_normal((3, 1000))
    for bits in (0, 2, 3, 4):
        p1, n1 = oracle.quantize(w, bits, nthreads=1)
        p8, n8 = oracle.quantize(w, bits, nthreads=8)
        assert np.array_equal(p1, p8) and np.array_equal(n1, n8)
        d1 = oracle.dequantize(p1, n1, 67, 1000, bits, nthreads=1)
        d8 = oracle.dequantize(p1, n1, 67, 1000, bits, nthreads=8)
        assert np.array_equal(d1, d8)
        y1 = oracle.dequant_gemv(p1, n1, 67, 1000, bits, x, nthreads=1)
        y8 = oracle.dequant_gemv(p1, n1, 67, 1000, bits, x, nthreads=8)
        assert np.array_equal(y1, y8)
