"""Pins of the CPU oracle against things other than itself.

Library routines (scipy's Hadamard), closed forms, invariants that the
definitions force, brute force on tiny inputs and hand-derived fixtures under
tests/golden/.  Each test names the plausible oracle mistake it would catch.
"""

import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg

from oracle import kvq_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def outlier_tile(rng, t, d=128, n_out=4, mult=20.0):
    x = rng.standard_normal((t, d))
    ch = rng.choice(d, size=n_out, replace=False)
    x[:, ch] *= mult
    return x.astype(np.float16)


# --------------------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_equals_scipy(d):
    # wrong recursion / order / sign -> differs from the library matrix
    h = o.sylvester_hadamard(d)
    np.testing.assert_array_equal(np.rint(h * math.sqrt(d)), scipy.linalg.hadamard(d))


def test_hadamard_popcount_closed_form():
    h = o.sylvester_hadamard(128) * math.sqrt(128)
    for j, k in itertools.product(range(0, 128, 7), range(128)):
        assert h[j, k] == (-1) ** bin(j & k).count("1")


def test_hadamard_orthonormal_symmetric():
    h = o.sylvester_hadamard(128)
    np.testing.assert_allclose(h @ h, np.eye(128), atol=1e-13)
    np.testing.assert_array_equal(h, h.T)


def test_rotation_side_and_norm():
    # X' = X H acts on token rows: row e_k maps to row k of H; e_0 maps to
    # the constant vector 1/sqrt(d); norms are preserved.
    h = o.sylvester_hadamard(128)
    for k in (0, 1, 37, 127):
        e = np.zeros((1, 128))
        e[0, k] = 1.0
        np.testing.assert_allclose(o.rotate(e)[0], h[k], atol=0)
    np.testing.assert_allclose(o.rotate(np.eye(1, 128))[0], np.full(128, 1 / math.sqrt(128)), atol=1e-15)
    x = np.random.default_rng(1).standard_normal((64, 128))
    np.testing.assert_allclose(np.linalg.norm(o.rotate(x), axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


# --------------------------------------------------------------------------- normalization

def pop_std(a, axis):
    m = a.mean(axis=axis, keepdims=True)
    return np.sqrt(((a - m) ** 2).mean(axis=axis))


@pytest.mark.parametrize("iters", [1, 2, 3, 8])
def test_rows_unit_std_after_token_step(iters):
    # channel step first, token step last; ddof 0.  A swapped order, ddof 1
    # or a dropped division leaves some row std away from 1.
    rng = np.random.default_rng(10 + iters)
    xr = o.rotate(outlier_tile(rng, 64))
    y, c, r = o.sinkhorn_normalize(xr, iters)
    np.testing.assert_allclose(pop_std(y, 1), 1.0, rtol=1e-12)


def test_reconstruction_identity():
    # Y_ij R_i C_j == X'_ij: catches C / R accumulated by division or on the wrong axis
    rng = np.random.default_rng(3)
    xr = o.rotate(outlier_tile(rng, 64))
    y, c, r = o.sinkhorn_normalize(xr, 5)
    np.testing.assert_allclose(y * r[:, None] * c[None, :], xr, rtol=1e-12, atol=1e-12)


def test_energy_identity_of_channel_stds():
    # After a token step every row has unit std, so summing squares by rows
    # and by columns gives mean_j sigma_j^2 = 1 + mean_i mu_i^2 - mean_j nu_j^2
    # (mu = row means, nu = column means).  A wrong axis or ddof breaks it.
    rng = np.random.default_rng(4)
    for t in (32, 64, 128):
        y, _, _ = o.sinkhorn_normalize(o.rotate(outlier_tile(rng, t)), 3)
        mu = y.mean(axis=1)
        nu = y.mean(axis=0)
        lhs = (pop_std(y, 0) ** 2).mean()
        rhs = 1.0 + (mu ** 2).mean() - (nu ** 2).mean()
        assert abs(lhs - rhs) < 1e-12


@pytest.mark.parametrize("t", [32, 64, 128])
def test_channel_variances_equalized_at_large_n(t):
    # The method equalizes the channels' variances.  With the centred std the
    # fixed point has one common channel std (not necessarily 1, see the
    # energy identity); at n = 32 they agree to 1e-3.
    rng = np.random.default_rng(20 + t)
    y, _, _ = o.sinkhorn_normalize(o.rotate(outlier_tile(rng, t)), 32)
    s = pop_std(y, 0)
    assert s.max() / s.min() - 1.0 < 1e-3
    # For plain N(0,1) tiles the common value sits next to 1.
    x = rng.standard_normal((t, 128)).astype(np.float16)
    y, _, _ = o.sinkhorn_normalize(o.rotate(x), 32)
    s = pop_std(y, 0)
    assert s.max() / s.min() - 1.0 < 1e-3
    assert abs(s.mean() - 1.0) < 0.02


def test_clamp_on_zero_variance_channel():
    # Tile whose rotated image is k_i * sqrt(d)/2 * (e0 + e1), k_i = 1..64:
    # channels 2..127 are exactly zero, so the first channel step clamps them
    # to sigma = eps while channels 0, 1 get the closed-form std
    # std(1..64) * sqrt(d)/2 = sqrt((64^2 - 1)/12) * sqrt(128)/2.
    d = 128
    h = o.sylvester_hadamard(d)
    v = (h[:, 0] + h[:, 1]) * math.sqrt(d) / 2   # entries in {0, 1}
    k = np.arange(1, 65, dtype=np.float64)
    x = (k[:, None] * v[None, :])                  # exact integers in fp16
    xr = o.rotate(x)
    assert not xr[:, 2:].any()
    y, c, r = o.sinkhorn_normalize(xr, 1)
    sigma0 = math.sqrt((64 ** 2 - 1) / 12) * math.sqrt(d) / 2
    np.testing.assert_allclose(c[2:] / c[0], 1e-6 / sigma0, rtol=1e-12)
    np.testing.assert_allclose(c[1], c[0], rtol=0)


def test_renormalization_keeps_metadata_finite():
    # degenerate tiles: all zero, and 64 identical tokens (every rotated
    # channel is constant over the tile, so the clamp fires on every channel in
    # every iteration).  max C stays in [1, 2), the metadata stays finite, the
    # zero tile comes back exactly and the constant tile as well as 4-bit RTN
    # of its one row allows.
    rng = np.random.default_rng(14)
    row = rng.standard_normal(128).astype(np.float16)
    for x in (np.zeros((64, 128), np.float16), np.tile(row, (64, 1))):
        for n in (1, 2, 8):
            for dt in (np.float64, np.float32):
                q = o.quantize_tile(x, 4, n, dtype=dt, return_parts=True)
                assert 1.0 <= q["c"].max() < 2.0
                for key in ("s_t", "z_t", "c_t"):
                    assert np.all(np.isfinite(q[key]))
                _, xh = o.dequantize_tile(q["codes"], q["s_t"], q["z_t"], q["c_t"])
                ref = x.astype(np.float64)
                if not ref.any():
                    assert not xh.any()
                else:
                    assert np.linalg.norm(xh - ref) / np.linalg.norm(ref) < 0.15
                    np.testing.assert_allclose(xh, xh[:1].repeat(64, 0), rtol=0, atol=0)


@pytest.mark.parametrize("dt", [np.float64, np.float32])
def test_identical_tokens_clamp_every_channel(dt):
    # 64 identical tokens: every rotated channel is exactly constant over the
    # tile, so every channel std is 0 and every sigma is the clamp eps; all C
    # come out equal and every token row is the same.
    row = np.random.default_rng(15).standard_normal(128).astype(np.float16)
    q = o.quantize_tile(np.tile(row, (64, 1)), 4, 3, dtype=dt, return_parts=True)
    assert np.all(q["c"] == q["c"][0])
    assert np.all(q["codes"] == q["codes"][:1])


def test_scale_equivariance():
    # X -> 2^k X (exact in fp16): codes and C~ unchanged (C is renormalized to
    # max in [1, 2)), s~ and z~ scaled by 2^k
    rng = np.random.default_rng(5)
    x = outlier_tile(rng, 64, mult=5.0)
    a = o.quantize_tile(x, 4, 4)
    b = o.quantize_tile((x.astype(np.float32) * 4).astype(np.float16), 4, 4)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["c_t"], b["c_t"])
    np.testing.assert_array_equal(a["s_t"].astype(np.float32) * 4, b["s_t"].astype(np.float32))
    np.testing.assert_array_equal(a["z_t"].astype(np.float32) * 4, b["z_t"].astype(np.float32))


def test_token_permutation_equivariance():
    rng = np.random.default_rng(6)
    x = outlier_tile(rng, 64)
    perm = rng.permutation(64)
    a = o.quantize_tile(x, 4, 4)
    b = o.quantize_tile(x[perm], 4, 4)
    np.testing.assert_array_equal(a["codes"][perm], b["codes"])
    np.testing.assert_array_equal(a["s_t"][perm], b["s_t"])
    np.testing.assert_array_equal(a["c_t"], b["c_t"])


# --------------------------------------------------------------------------- RTN

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_rtn_brute_force_and_bounds(bits):
    # brute force: each code is the nearest grid point c*s + z (fp64, no ties);
    # min row entry -> 0, max -> 2^b - 1, error <= s/2, codes in range.
    rng = np.random.default_rng(30 + bits)
    y = rng.standard_normal((16, 128)) * rng.uniform(0.1, 3, size=(16, 1))
    codes, s, z = o.asymmetric_rtn(y, bits)
    qmax = (1 << bits) - 1
    grid = np.arange(qmax + 1)[None, None, :] * s[:, None, None] + z[:, None, None]
    brute = np.abs(y[:, :, None] - grid).argmin(axis=2)
    np.testing.assert_array_equal(codes, brute)
    assert codes.max() <= qmax
    np.testing.assert_array_equal(codes[np.arange(16), y.argmin(1)], 0)
    np.testing.assert_array_equal(codes[np.arange(16), y.argmax(1)], qmax)
    err = np.abs(y - (codes * s[:, None] + z[:, None]))
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-12))


def test_rtn_golden_rows():
    # hand-derived rows, tests/golden/rtn_worked_examples.txt
    path = os.path.join(GOLDEN, "rtn_worked_examples.txt")
    cases = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, codes = line.split("|")
            cases.append((int(bits), [float(v) for v in vals.split()], [int(c) for c in codes.split()]))
    assert cases
    for bits, vals, want in cases:
        codes, s, z = o.asymmetric_rtn(np.array([vals]), bits)
        assert codes[0].tolist() == want, (bits, vals)


def test_plain_rtn_baseline_golden_rows():
    # hand-derived rows, tests/golden/plain_rtn_worked_examples.txt: the
    # fp16 rounding of the scale moves the reconstruction (a baseline that
    # skipped it, used 2^(b+1) - 1 levels or scaled its input would not match)
    path = os.path.join(GOLDEN, "plain_rtn_worked_examples.txt")
    rows = 0
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, codes, s16, z16, recon = line.split("|")
            x = np.array([[float(v) for v in vals.split()]], dtype=np.float16)
            want = np.array([float(v) for v in recon.split()])
            got = o.plain_rtn_baseline(x, int(bits))
            np.testing.assert_array_equal(got[0], want)
            c, s, z = o.asymmetric_rtn(x.astype(np.float64), int(bits))
            assert c[0].tolist() == [int(v) for v in codes.split()]
            assert float(np.float16(s[0])) == float(s16) and float(np.float16(z[0])) == float(z16)
            rows += 1
    assert rows == 3


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_plain_rtn_baseline_brute_force(bits):
    # every code is the nearest point of the exact grid z + c s (brute force
    # over c), the reconstruction uses the fp16-rounded s and z, the row min
    # comes back exactly, and the error stays within s/2 plus the fp16
    # rounding of s times the code
    rng = np.random.default_rng(60 + bits)
    x = (rng.standard_normal((32, 128)) * rng.uniform(0.05, 40, size=(32, 1))
         + rng.uniform(-5, 5, size=(32, 1))).astype(np.float16)
    xd = x.astype(np.float64)
    qmax = (1 << bits) - 1
    z = xd.min(axis=1)
    s = (xd.max(axis=1) - z) / qmax
    grid = np.arange(qmax + 1)[None, None, :] * s[:, None, None] + z[:, None, None]
    dist = np.abs(xd[:, :, None] - grid)
    near = dist <= dist.min(axis=2, keepdims=True) * (1 + 1e-12) + 1e-300
    # an exact tie between two grid points goes to the even code (half to even)
    code = np.where(near.sum(axis=2) > 1, np.argmax(near & (np.arange(qmax + 1) % 2 == 0), axis=2),
                    dist.argmin(axis=2))
    s16 = s.astype(np.float16).astype(np.float64)
    z16 = z.astype(np.float16).astype(np.float64)
    got = o.plain_rtn_baseline(x, bits)
    np.testing.assert_array_equal(got, code * s16[:, None] + z16[:, None])
    np.testing.assert_array_equal(got[np.arange(32), xd.argmin(axis=1)], z)
    bound = s[:, None] / 2 + code * np.abs(s16 - s)[:, None]
    assert np.all(np.abs(got - xd) <= bound * (1 + 1e-12))
    assert not np.array_equal(s16, s)  # the fp16 rounding of s is exercised


def test_constant_row_gives_zero_scale():
    y = np.full((2, 128), 0.75)
    codes, s, z = o.asymmetric_rtn(y, 4)
    assert np.all(codes == 0) and np.all(s == 0) and np.all(z == 0.75)


# --------------------------------------------------------------------------- tile quantizer

@pytest.mark.parametrize("t,bits,iters", [(32, 2, 1), (64, 4, 4), (128, 3, 8), (64, 2, 0), (64, 8, 4)])
def test_dequantized_tile_within_half_step(t, bits, iters):
    # X^' - X' is bounded by (s/2) R_i C_j plus the fp16 rounding of the
    # metadata; a missing R or C factor in s~, z~ or C~ breaks it by orders of magnitude.
    rng = np.random.default_rng(40 + t + bits)
    x = outlier_tile(rng, t)
    q = o.quantize_tile(x, bits, iters, return_parts=True)
    xr_hat, x_hat = o.dequantize_tile(q["codes"], q["s_t"], q["z_t"], q["c_t"])
    half = (q["s"] * q["r"])[:, None] * q["c"][None, :] / 2
    fp16_slack = 2.0 ** -10 * (np.abs(q["xr"]) + (q["s"] * q["r"])[:, None] * q["c"][None, :] * ((1 << bits) - 1))
    assert np.all(np.abs(xr_hat - q["xr"]) <= half + 3 * fp16_slack)
    # original domain: the inverse rotation is exact up to rounding
    np.testing.assert_allclose(x_hat, xr_hat @ o.sylvester_hadamard(128), rtol=0, atol=1e-12)
    err = np.linalg.norm(x_hat - x.astype(np.float64)) / np.linalg.norm(x.astype(np.float64))
    assert err < {2: 0.7, 3: 0.3, 4: 0.15, 8: 0.02}[bits]


@pytest.mark.parametrize("t,bits,iters", [(t, b, n) for t in (32, 64, 128) for b in (2, 3, 4) for n in (1, 4, 8)])
def test_method_beats_plain_rtn_on_outliers(t, bits, iters):
    # the method's point: lower reconstruction MSE than plain per-token RTN
    rng = np.random.default_rng(1000 + 7 * t + 3 * bits + iters)
    d = 128
    x = rng.standard_normal((t, d))
    k = max(1, round(rng.uniform(0.01, 0.05) * d))
    ch = rng.choice(d, size=k, replace=False)
    x[:, ch] *= np.exp(rng.uniform(np.log(5), np.log(50), size=k))
    x = x.astype(np.float16)
    q = o.quantize_tile(x, bits, iters)
    _, x_hat = o.dequantize_tile(q["codes"], q["s_t"], q["z_t"], q["c_t"])
    ref = x.astype(np.float64)
    mse_method = ((x_hat - ref) ** 2).mean()
    mse_plain = ((o.plain_rtn_baseline(x, bits) - ref) ** 2).mean()
    assert mse_method < mse_plain


def test_float32_mode_agrees_with_fp64():
    # the parity tests run the quantizer in float32 (the GPU's precision for
    # the code decision); it must agree with fp64 except at rare near-ties
    rng = np.random.default_rng(8)
    x = outlier_tile(rng, 64)
    a = o.quantize_tile(x, 4, 4)
    b = o.quantize_tile(x, 4, 4, dtype=np.float32)
    diff = a["codes"].astype(int) - b["codes"].astype(int)
    assert np.abs(diff).max() <= 1 and (diff != 0).mean() < 1e-3


# --------------------------------------------------------------------------- format

@pytest.mark.parametrize("bits,is_v", [(2, False), (3, False), (4, False), (8, False), (2, True), (3, True),
                                       (4, True), (8, True)])
def test_code_positions_are_a_bijection(bits, is_v):
    pos = sorted(o.code_bit_position(c, p, bits, is_v) for p in range(16) for c in range(128))
    assert pos == list(range(0, 16 * 128 * bits, bits))


def test_layout_sizes_hand_computed():
    # K, T=64, b=4: 16*128*4/8 = 1024 codes + 64 meta + 32 channels*2 B = 1152
    assert o.page_layout(4, 64)["page_bytes"] == 1152
    # V, T=128, b=2: 512 + 64 + 16*2 = 608;  T=32, b=3: 768 + 64 + 64*2 = 960
    assert o.page_layout(2, 128)["page_bytes"] == 608
    assert o.page_layout(3, 32)["page_bytes"] == 960
    assert o.page_layout(4, 64)["cslice_channels"] == 32
    # b=8, T=64: 2048 + 64 + 32*2 = 2176
    assert o.page_layout(8, 64)["page_bytes"] == 2176


def test_code_positions_golden():
    # hand-derived positions from the written layout, tests/golden/format_positions.txt
    path = os.path.join(GOLDEN, "format_positions.txt")
    n = 0
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            kind, bits, ch, tok, want = line.split()
            got = o.code_bit_position(int(ch), int(tok), int(bits), kind == "V")
            assert got == int(want), line
            n += 1
    assert n >= 8


@pytest.mark.parametrize("bits,is_v", [(2, True), (4, True), (8, True), (3, False), (4, False), (8, False)])
def test_pack_unpack_roundtrip(bits, is_v):
    rng = np.random.default_rng(bits + 10 * is_v)
    codes = rng.integers(0, 1 << bits, size=(16, 128)).astype(np.uint8)
    region = o.pack_page_codes(codes, bits, is_v)
    assert region.size == 16 * 128 * bits // 8
    np.testing.assert_array_equal(o.unpack_page_codes(region, bits, is_v), codes)


def test_tile_pages_roundtrip():
    rng = np.random.default_rng(9)
    x = outlier_tile(rng, 64)
    q = o.quantize_tile(x, 4, 2)
    lay = o.page_layout(4, 64)
    pool = np.zeros((10, 2, lay["page_bytes"]), dtype=np.uint8)
    blocks = [7, 2, 9, 0]
    o.write_tile_pages(pool, blocks, 1, q, 4, 64, True)
    back = o.read_tile_pages(pool, blocks, 1, 4, 64, True)
    for key in ("codes", "s_t", "z_t", "c_t"):
        np.testing.assert_array_equal(back[key], q[key])
    assert not pool[:, 0].any()


# --------------------------------------------------------------------------- decode

def brute_attention(q, k, v, scale):
    # pure-Python loops, tiny sizes only
    logits = [scale * sum(q[j] * k[i][j] for j in range(len(q))) for i in range(len(k))]
    m = max(logits)
    w = [math.exp(a - m) for a in logits]
    tot = sum(w)
    return [sum(w[i] * v[i][j] for i in range(len(k))) / tot for j in range(len(q))]


def test_attention_brute_force():
    rng = np.random.default_rng(11)
    q = rng.standard_normal(128)
    k = rng.standard_normal((9, 128))
    v = rng.standard_normal((9, 128))
    want = brute_attention(q.tolist(), k.tolist(), v.tolist(), 1 / math.sqrt(128))
    np.testing.assert_allclose(o.attention_fp64(q, k, v), want, rtol=1e-12, atol=1e-14)


def test_attention_special_cases():
    rng = np.random.default_rng(12)
    k = rng.standard_normal((5, 128))
    v = rng.standard_normal((5, 128))
    np.testing.assert_allclose(o.attention_fp64(rng.standard_normal(128), k[:1], v[:1]), v[0], rtol=1e-15)
    np.testing.assert_allclose(o.attention_fp64(np.zeros(128), k, v), v.mean(axis=0), rtol=1e-13)


def test_decode_gqa_mapping_and_tail():
    # query head h reads KV head h // g; the raw tail follows the tiles
    rng = np.random.default_rng(13)
    g, hkv, t = 4, 2, 32
    rows_k = [rng.standard_normal((t + 3, 128)).astype(np.float16) for _ in range(hkv)]
    rows_v = [(float(4 * h) + rng.standard_normal((t + 3, 128))).astype(np.float16) for h in range(hkv)]
    k_hat, v_hat = [], []
    for h in range(hkv):
        tk, tail_k = o.quantize_sequence(rows_k[h], t, 4, 2)
        tv, tail_v = o.quantize_sequence(rows_v[h], t, 4, 2)
        assert tail_k.shape[0] == 3
        k_hat.append(o.sequence_kv_hat(tk, tail_k))
        v_hat.append(o.sequence_kv_hat(tv, tail_v))
        assert k_hat[-1].shape == (t + 3, 128)
        np.testing.assert_array_equal(k_hat[-1][t:], rows_k[h][t:].astype(np.float64))
    qh = rng.standard_normal((g * hkv, 128))
    out = o.decode_sequence(qh, k_hat, v_hat, g)
    for h in range(g * hkv):
        # KV head 1's values sit near 4, KV head 0's near 0
        assert abs(out[h].mean() - 4.0 * (h // g)) < 0.6
        np.testing.assert_array_equal(out[h], o.attention_fp64(qh[h], k_hat[h // g], v_hat[h // g]))


# --------------------------------------------------------------------------- randomized rotation (variant)

def test_splitmix64_matches_published_first_output():
    # a wrong constant, shift or update order in the generator changes it
    lines = [ln for ln in open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) if not ln.startswith("#")]
    want = int(lines[0].strip(), 16)
    assert o.splitmix64_outputs(0, 1)[0] == want


def test_rotation_signs_seed0_plain_and_seeded_balanced():
    np.testing.assert_array_equal(o.rotation_signs(128, 0), np.ones(128))
    for seed in (1, 12345, 0xDEADBEEF):
        s = o.rotation_signs(128, seed)
        assert set(np.unique(s)) == {-1.0, 1.0}
        assert 0.3 < np.mean(s < 0) < 0.7  # a stuck sign bit would give 0 or 1
    assert not np.array_equal(o.rotation_signs(128, 1), o.rotation_signs(128, 2))


def test_randomized_rotation_is_orthogonal_and_inverted():
    # X' = X D_s H keeps inner products between rows (Gram matrix), and the
    # dequantization's inverse X' H D_s recovers X: a sign applied on the
    # wrong side (H D_s instead of D_s H) breaks the inversion
    rng = np.random.default_rng(21)
    x = rng.standard_normal((16, 128))
    seed = 777
    xr = o.rotate(x, seed=seed)
    np.testing.assert_allclose(xr @ xr.T, x @ x.T, rtol=1e-12, atol=1e-10)
    back = (xr @ o.sylvester_hadamard(128)) * o.rotation_signs(128, seed)[None, :]
    np.testing.assert_allclose(back, x, atol=1e-12)
    wrong = (xr * o.rotation_signs(128, seed)[None, :]) @ o.sylvester_hadamard(128)
    assert not np.allclose(wrong, x, atol=1e-3)
    # a unit row e_k maps to s_k times row k of H
    h = o.sylvester_hadamard(128)
    s = o.rotation_signs(128, seed)
    for k in (0, 5, 127):
        e = np.zeros((1, 128))
        e[0, k] = 1.0
        np.testing.assert_allclose(o.rotate(e, seed=seed)[0], s[k] * h[k], atol=0)


def test_randomized_rotation_dequantizes_and_decodes():
    # dequantized tile within one step per element; decode over the seeded
    # quantization equals brute-force attention on its original-domain rows
    rng = np.random.default_rng(22)
    seed, t = 4242, 32
    x = outlier_tile(rng, t)
    q = o.quantize_tile(x, 4, 4, return_parts=True, seed=seed)
    xr_hat, x_hat = o.dequantize_tile(q["codes"], q["s_t"], q["z_t"], q["c_t"], seed)
    step = (q["s"] * q["r"])[:, None] * q["c"][None, :]
    fp16_slack = 2.0 ** -10 * (np.abs(q["xr"]) + step * 15)
    assert np.all(np.abs(xr_hat - q["xr"]) <= step / 2 + 3 * fp16_slack)
    err = np.linalg.norm(x_hat - x.astype(np.float64)) / np.linalg.norm(x.astype(np.float64))
    assert err < 0.15
    rows_k = rng.standard_normal((t + 5, 128)).astype(np.float16)
    rows_v = rng.standard_normal((t + 5, 128)).astype(np.float16)
    tk, tail_k = o.quantize_sequence(rows_k, t, 4, 2, seed=seed)
    tv, tail_v = o.quantize_sequence(rows_v, t, 4, 2, seed=seed)
    k_hat, v_hat = o.sequence_kv_hat(tk, tail_k, seed), o.sequence_kv_hat(tv, tail_v, seed)
    qv = rng.standard_normal(128)
    want = brute_attention(qv.tolist(), k_hat.tolist(), v_hat.tolist(), 1 / math.sqrt(128))
    np.testing.assert_allclose(o.decode_sequence(qv[None], [k_hat], [v_hat], 1)[0], want, rtol=1e-11, atol=1e-13)
    # the keys really are the seeded reconstruction: closer to the raw rows
    # than the unseeded decoder's reading of the same codes
    k_plain = o.sequence_kv_hat(tk, tail_k, 0)
    assert np.linalg.norm(k_hat - rows_k) < 0.5 * np.linalg.norm(k_plain - rows_k)


# --------------------------------------------------------------------------- chunked prefill

def _ctx(rng, hkv, length, t=32):
    """Context of ``length`` tokens per KV head as the cache holds it."""
    k_hat, v_hat = [], []
    for _ in range(hkv):
        rk = rng.standard_normal((length, 128)).astype(np.float16)
        rv = rng.standard_normal((length, 128)).astype(np.float16)
        tk, tail_k = o.quantize_sequence(rk, t, 4, 2)
        tv, tail_v = o.quantize_sequence(rv, t, 4, 2)
        k_hat.append(o.sequence_kv_hat(tk, tail_k))
        v_hat.append(o.sequence_kv_hat(tv, tail_v))
    return k_hat, v_hat


def test_prefill_causal_count_closed_form():
    # all keys equal -> uniform weights over exactly the visible keys.  With
    # context values 0 and new value j+1 at chunk position j, token i's
    # output is (1 + ... + (i+1)) / (L + i + 1): an off-by-one in the mask or
    # a dropped context shifts it
    L, n, g = 7, 5, 2
    u = np.full(128, 0.25)
    k_hat = [np.tile(u, (L, 1))]
    v_hat = [np.zeros((L, 128))]
    k_new = np.tile(u, (n, 1, 1)).astype(np.float16)
    v_new = np.zeros((n, 1, 128), dtype=np.float16)
    v_new[:, 0, 0] = np.arange(1, n + 1)
    q = np.random.default_rng(31).standard_normal((n, g, 128))
    out = o.prefill_chunk_sequence(q, k_hat, v_hat, k_new, v_new, g)
    for i in range(n):
        want = (i + 1) * (i + 2) / 2 / (L + i + 1)
        for h in range(g):
            assert out[i, h, 0] == pytest.approx(want, rel=1e-13)
            assert np.all(out[i, h, 1:] == 0)


def test_prefill_two_key_softmax_closed_form():
    # one context key, chunk of one token: weight of the new key is the
    # logistic of the score difference times the scale
    rng = np.random.default_rng(32)
    q = rng.standard_normal((1, 1, 128))
    k1, k2 = rng.standard_normal((1, 128)), rng.standard_normal((1, 1, 128)).astype(np.float16)
    v1 = np.zeros((1, 128))
    v2 = np.ones((1, 1, 128), dtype=np.float16)
    for scale in (None, 0.05):
        sc = 1 / math.sqrt(128) if scale is None else scale
        a = float(q[0, 0] @ k1[0]) * sc
        b = float(q[0, 0] @ k2[0, 0].astype(np.float64)) * sc
        w2 = 1.0 / (1.0 + math.exp(a - b))
        out = o.prefill_chunk_sequence(q, [k1], [v1], k2, v2, 1, scale)
        np.testing.assert_allclose(out[0, 0], np.full(128, w2), rtol=1e-12)


def test_prefill_gqa_mapping():
    # query head h reads KV head h // g: values constant per KV head
    rng = np.random.default_rng(33)
    hkv, g, L, n = 3, 4, 40, 6
    k_hat = [rng.standard_normal((L, 128)) for _ in range(hkv)]
    v_hat = [np.full((L, 128), float(kv + 1)) for kv in range(hkv)]
    k_new = rng.standard_normal((n, hkv, 128)).astype(np.float16)
    v_new = np.broadcast_to(np.arange(1, hkv + 1, dtype=np.float16)[None, :, None], (n, hkv, 128)).copy()
    out = o.prefill_chunk_sequence(rng.standard_normal((n, hkv * g, 128)), k_hat, v_hat, k_new, v_new, g)
    for h in range(hkv * g):
        np.testing.assert_allclose(out[:, h], float(h // g + 1), rtol=1e-13)


def test_prefill_one_token_is_decode_over_appended_cache():
    # a chunk of one token is a decode step over the context plus that row
    rng = np.random.default_rng(34)
    hkv, g = 2, 3
    k_hat, v_hat = _ctx(rng, hkv, 75)
    k_new = rng.standard_normal((1, hkv, 128)).astype(np.float16)
    v_new = rng.standard_normal((1, hkv, 128)).astype(np.float16)
    q = rng.standard_normal((1, hkv * g, 128))
    out = o.prefill_chunk_sequence(q, k_hat, v_hat, k_new, v_new, g)
    k_app = [np.concatenate([k_hat[h], k_new[:, h].astype(np.float64)]) for h in range(hkv)]
    v_app = [np.concatenate([v_hat[h], v_new[:, h].astype(np.float64)]) for h in range(hkv)]
    np.testing.assert_array_equal(out[0], o.decode_sequence(q[0], k_app, v_app, g))


def test_prefill_later_rows_do_not_leak():
    # changing chunk rows after position i leaves token i's output alone;
    # changing row i itself moves it
    rng = np.random.default_rng(35)
    hkv, g, n = 1, 2, 6
    k_hat, v_hat = _ctx(rng, hkv, 33)
    k_new = rng.standard_normal((n, hkv, 128)).astype(np.float16)
    v_new = rng.standard_normal((n, hkv, 128)).astype(np.float16)
    q = rng.standard_normal((n, hkv * g, 128))
    base = o.prefill_chunk_sequence(q, k_hat, v_hat, k_new, v_new, g)
    for i in range(n - 1):
        k2, v2 = k_new.copy(), v_new.copy()
        k2[i + 1:] = rng.standard_normal(k2[i + 1:].shape)
        v2[i + 1:] = rng.standard_normal(v2[i + 1:].shape)
        out = o.prefill_chunk_sequence(q, k_hat, v_hat, k2, v2, g)
        np.testing.assert_array_equal(out[:i + 1], base[:i + 1])
        assert np.abs(out[i + 1] - base[i + 1]).max() > 1e-3
        v3 = v_new.copy()
        v3[i] += np.float16(1.0)
        assert np.abs(o.prefill_chunk_sequence(q, k_hat, v_hat, k_new, v3, g)[i] - base[i]).max() > 1e-4


def test_prefill_empty_context_is_causal_attention():
    # no cached tokens: plain causal attention over the chunk (brute force)
    rng = np.random.default_rng(36)
    n = 4
    k_new = rng.standard_normal((n, 1, 128)).astype(np.float16)
    v_new = rng.standard_normal((n, 1, 128)).astype(np.float16)
    q = rng.standard_normal((n, 1, 128))
    out = o.prefill_chunk_sequence(q, [np.zeros((0, 128))], [np.zeros((0, 128))], k_new, v_new, 1)
    for i in range(n):
        want = brute_attention(q[i, 0].tolist(), k_new[:i + 1, 0].astype(np.float64).tolist(),
                               v_new[:i + 1, 0].astype(np.float64).tolist(), 1 / math.sqrt(128))
        np.testing.assert_allclose(out[i, 0], want, rtol=1e-12, atol=1e-14)


def test_lse_merge_of_parts_is_attention_over_all_keys():
    # the merge both split paths rely on: per part (max m, sum l, unnormalized
    # accumulator a) in the log2 domain, merged with weights 2^(m_s - max m),
    # reproduces attention over all keys; empty parts contribute nothing
    rng = np.random.default_rng(37)
    L = 300
    q = rng.standard_normal(128)
    k = rng.standard_normal((L, 128)) * 3
    v = rng.standard_normal((L, 128))
    want = o.attention_fp64(q, k, v)
    scale = math.log2(math.e) / math.sqrt(128)
    for cuts in ([0, 100, 100, 217, 300], [0, 1, 299, 300], [0, 300]):
        parts = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            if a == b:
                parts.append((-math.inf, 0.0, np.zeros(128)))
                continue
            s = (k[a:b] @ q) * scale
            m = s.max()
            p = np.exp2(s - m)
            parts.append((m, p.sum(), p @ v[a:b]))
        mm = max(m for m, l, _ in parts if l > 0)
        l_tot = sum(l * 2.0 ** (m - mm) for m, l, _ in parts if l > 0)
        acc = sum(a * 2.0 ** (m - mm) for m, l, a in parts if l > 0)
        np.testing.assert_allclose(acc / l_tot, want, rtol=1e-11, atol=1e-13)



# --------------------------------------------------------------------------- head sizes 64 and 256 (format)

@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits,is_v", [(2, False), (3, False), (4, False), (8, False), (2, True), (3, True),
                                       (4, True), (8, True)])
def test_code_positions_are_a_bijection_at_other_head_sizes(d, bits, is_v):
    # every (channel, token) of a page gets its own field inside p*d*b bits
    pos = [o.code_bit_position(ch, tok, bits, is_v, d) for tok in range(16) for ch in range(d)]
    assert len(set(pos)) == len(pos)
    assert min(pos) >= 0 and max(pos) + bits <= 16 * d * bits
    assert all(p % bits == 0 for p in pos)


def test_grouped_v_positions_golden_other_head_sizes():
    # hand-derived from the layout rule (n = c // 8, g = c % 8, t = (tok % 8) // 2,
    # u = tok // 8, s = tok % 2, h = 16 / b, k = 2 (n // h) + u, e = n % h,
    # lane 4 g + t, rows of min(4, d b / 64) words):
    # d = 64, b = 2, channel 9, token 3: n 1, g 1, t 1, u 0, s 1; h 8, k 0, e 1,
    #   lane 5, row width 2 -> byte 5 * 8 = 40, bit 320 + 2 (1 + 8) = 338
    assert o.code_bit_position(9, 3, 2, True, 64) == 338
    # d = 64, b = 2, channel 63, token 15: n 7, g 7, t 3, u 1, s 1; k 1, e 7, lane 31
    #   -> byte 31 * 8 + 4 = 252, bit 2016 + 2 (7 + 8) = 2046 (the page's last field)
    assert o.code_bit_position(63, 15, 2, True, 64) == 2046
    # d = 256, b = 4, channel 200, token 9: n 25, g 0, t 0, u 1, s 1; h 4, k 13, e 1,
    #   lane 0, rows of 4 -> byte (3 * 32) * 16 + 4 = 1540, bit 12320 + 4 (1 + 4) = 12340
    assert o.code_bit_position(200, 9, 4, True, 256) == 12340
    # d = 128 keeps its layout: rows of 4 words for every b
    assert o.code_bit_position(9, 3, 2, True, 128) == (5 * 16) * 8 + 2 * (1 + 8)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits,is_v", [(2, True), (4, True), (8, True), (3, False), (4, False)])
def test_pack_unpack_roundtrip_other_head_sizes(d, bits, is_v):
    rng = np.random.default_rng(50 + d + bits)
    codes = rng.integers(0, 1 << bits, size=(16, d)).astype(np.uint8)
    region = o.pack_page_codes(codes, bits, is_v)
    assert region.size == 16 * d * bits // 8
    np.testing.assert_array_equal(o.unpack_page_codes(region, bits, is_v, d=d), codes)


@pytest.mark.parametrize("d,t,bits", [(64, 64, 4), (256, 64, 2), (256, 128, 4), (64, 32, 8)])
def test_layout_and_tile_pages_roundtrip_other_head_sizes(d, t, bits):
    lay = o.page_layout(bits, t, d)
    # codes p d b / 8 | 64 B of metadata | d p / T channels of C, each padded to 16 B
    assert lay["codes"] == -(-16 * d * bits // 8 // 16) * 16
    assert lay["cslice_channels"] == d * 16 // t
    assert lay["page_bytes"] == lay["codes"] + 64 + -(-2 * (d * 16 // t) // 16) * 16
    rng = np.random.default_rng(60 + d + t + bits)
    for is_v in (False, True):
        tile = o.quantize_tile(outlier_tile(rng, t, d=d), bits, 2)
        pool = np.zeros((t // 16 + 3, 1, lay["page_bytes"]), dtype=np.uint8)
        blocks = list(rng.permutation(pool.shape[0])[: t // 16])
        o.write_tile_pages(pool, blocks, 0, tile, bits, t, is_v)
        back = o.read_tile_pages(pool, blocks, 0, bits, t, is_v, d=d)
        for k in ("codes", "s_t", "z_t", "c_t"):
            np.testing.assert_array_equal(np.asarray(back[k]).view(np.uint8), np.asarray(tile[k]).view(np.uint8))


@pytest.mark.parametrize("d", [64, 256])
def test_dequantized_tile_within_half_step_other_head_sizes(d):
    rng = np.random.default_rng(70 + d)
    x = outlier_tile(rng, 64, d=d)
    q = o.quantize_tile(x, 4, 4, return_parts=True)
    xr_hat, x_hat = o.dequantize_tile(q["codes"], q["s_t"], q["z_t"], q["c_t"])
    half = (q["s"] * q["r"])[:, None] * q["c"][None, :] / 2
    fp16_slack = 2.0 ** -10 * (np.abs(q["xr"]) + (q["s"] * q["r"])[:, None] * q["c"][None, :] * 15)
    assert np.all(np.abs(xr_hat - q["xr"]) <= half + 3 * fp16_slack)
    np.testing.assert_allclose(x_hat, xr_hat @ o.sylvester_hadamard(d), rtol=0, atol=1e-12)
    err = np.linalg.norm(x_hat - x.astype(np.float64)) / np.linalg.norm(x.astype(np.float64))
    assert err < 0.15


def test_prefill_causal_closed_form_at_d64():
    # the attention functions take d from the rows (scale 1/sqrt(64)): same
    # uniform-weight closed form as at d = 128
    L, n = 5, 3
    u = np.full(64, 0.5)
    v_new = np.zeros((n, 1, 64), dtype=np.float16)
    v_new[:, 0, 0] = np.arange(1, n + 1)
    out = o.prefill_chunk_sequence(np.ones((n, 1, 64)), [np.tile(u, (L, 1))], [np.zeros((L, 64))],
                                   np.tile(u, (n, 1, 1)).astype(np.float16), v_new, 1)
    for i in range(n):
        assert out[i, 0, 0] == pytest.approx((i + 1) * (i + 2) / 2 / (L + i + 1), rel=1e-13)
    # and the one-key logistic weight uses 1/sqrt(64)
    q = np.random.default_rng(38).standard_normal((1, 1, 64))
    k1, k2 = np.random.default_rng(39).standard_normal((1, 64)), np.zeros((1, 1, 64), dtype=np.float16)
    w2 = 1.0 / (1.0 + math.exp(float(q[0, 0] @ k1[0]) / 8.0))
    got = o.prefill_chunk_sequence(q, [k1], [np.zeros((1, 64))], k2, np.ones((1, 1, 64), dtype=np.float16), 1)
    np.testing.assert_allclose(got[0, 0], np.full(64, w2), rtol=1e-12)
