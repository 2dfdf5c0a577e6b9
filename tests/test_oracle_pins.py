"""Pins for the CPU oracle: checks against facts the pages and mathematics fix.

Nothing here re-types the oracle's own formulas.  Each check comes from an
independent source: the Sylvester recursion for Hadamard matrices,
orthogonality, the quantizer's half-step error bound, exact recovery of values
already on the int4 grid, hand-derived round-half-even ties and byte layouts
(tests/golden), closed-form attention cases, the page's 40 GB -> 12.5 GB
footprint, and a brute-force numpy softmax on tiny inputs.
"""
import os

import numpy as np
import pytest

import oracle
from conftest import GOLDEN


def sylvester(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def rand_signs(rng, d):
    return (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_sylvester_recursion(d):
    R = oracle.rotation_matrix(d, np.ones(d, np.int8))
    np.testing.assert_array_equal(np.rint(R * np.sqrt(d)), sylvester(d))


@pytest.mark.parametrize("d", [4, 32, 128, 256])
def test_hadamard_integer_identity(d):
    H = np.array([[oracle.hadamard_entry(i, j) for j in range(d)] for i in range(d)], np.int64)
    np.testing.assert_array_equal(H @ H, d * np.eye(d, dtype=np.int64))


def test_rotation_hand_values():
    with open(os.path.join(GOLDEN, "rotation_d2_d4.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    i, cases = 0, 0
    while i < len(lines):
        head = dict(kv.split("=") for kv in lines[i].split())
        d = int(head["d"])
        signs = np.array([int(s) for s in head["signs"].split(",")], np.int8)
        want = np.array([[float(x) for x in lines[i + 1 + r].split()] for r in range(d)])
        R = oracle.rotation_matrix(d, signs)
        np.testing.assert_allclose(R * np.sqrt(d), want, rtol=0, atol=1e-15)
        i += 1 + d
        cases += 1
    assert cases == 3


@pytest.mark.parametrize("d", [32, 64, 128, 256])
def test_rotation_orthogonal(d):
    rng = np.random.default_rng(d)
    R = oracle.rotation_matrix(d, rand_signs(rng, d))
    assert np.max(np.abs(R.T @ R - np.eye(d))) <= 1e-15


def test_rotation_off_is_identity():
    np.testing.assert_array_equal(oracle.rotation_matrix(64, None), np.eye(64))


@pytest.mark.parametrize("d", [128, 256])
def test_rotation_preserves_norm_and_dot(d):
    rng = np.random.default_rng(7)
    s = rand_signs(rng, d)
    R = oracle.rotation_matrix(d, s)
    x = rng.standard_normal((16, d))
    y = x @ R.T
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    assert abs((R @ q) @ (R @ k) - q @ k) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(k)


def test_rotate_rounds_once_to_fp32():
    rng = np.random.default_rng(3)
    d = 128
    s = rand_signs(rng, d)
    x = rng.standard_normal((8, d)).astype(np.float32)
    y = oracle.rotate(x, s)
    exact = x.astype(np.float64) @ oracle.rotation_matrix(d, s).T
    # one rounding of the fp64 product: within half an fp32 ulp (plus fp64 noise)
    ulp = np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(y.astype(np.float64) - exact) <= 0.5 * ulp + 1e-15)


def test_wht_inverse_is_transpose():
    rng = np.random.default_rng(11)
    d = 128
    R = oracle.rotation_matrix(d, rand_signs(rng, d))
    x = rng.standard_normal(d)
    np.testing.assert_allclose(R.T @ (R @ x), x, atol=1e-13)


# ------------------------------------------------------------ quantization

def _read_ties():
    with open(os.path.join(GOLDEN, "quant_ties.txt")) as f:
        lines = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    groups = []
    for i in range(0, len(lines), 3):
        assert lines[i][0] == "scale" and lines[i + 1][0] == "values" and lines[i + 2][0] == "codes"
        groups.append((float(lines[i][1]), np.array(lines[i + 1][1:], np.float32),
                       np.array(lines[i + 2][1:], np.int64)))
    return groups


def test_quantizer_hand_ties_round_half_even():
    groups = _read_ties()
    assert len(groups) == 4
    y = np.concatenate([g[1] for g in groups])[None, :]    # d = 128, four groups
    codes, scales = oracle.quantize_vectors(y)
    np.testing.assert_array_equal(scales[0], np.array([g[0] for g in groups], np.float32))
    np.testing.assert_array_equal(codes[0].astype(np.int64), np.concatenate([g[2] for g in groups]))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_quantizer_half_step_bound_and_absmax_code(d):
    rng = np.random.default_rng(d + 1)
    y = (rng.standard_normal((64, d)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    y[0, :32] = 0.0                                   # an all-zero group
    codes, scales = oracle.quantize_vectors(y)
    assert codes.min() >= -7 and codes.max() <= 7
    s = np.repeat(scales.astype(np.float64), 32, axis=1)
    err = np.abs(y.astype(np.float64) - s * codes)
    assert np.all(err <= s / 2 * (1 + 2.0 ** -20))
    grp = np.abs(codes.reshape(64, d // 32, 32)).max(axis=2)
    nonzero = np.abs(y.reshape(64, d // 32, 32)).max(axis=2) > 0
    assert np.all(grp[nonzero] == 7)
    assert np.all(scales[~nonzero] == 0) and np.all(grp[~nonzero] == 0)


@pytest.mark.parametrize("d", [32, 128, 256])
def test_quantizer_exact_recovery_on_grid(d):
    rng = np.random.default_rng(d + 2)
    n = 32
    c = rng.integers(-7, 8, (n, d)).astype(np.int8)
    c.reshape(n, d // 32, 32)[:, :, 5] = rng.choice([-7, 7], (n, d // 32))
    e = rng.integers(-20, 20, (n, d // 32)).astype(np.float64)
    s0 = np.exp2(e)
    y = (np.repeat(s0, 32, axis=1) * c).astype(np.float32)
    codes, scales = oracle.quantize_vectors(y)
    np.testing.assert_array_equal(codes, c)
    np.testing.assert_array_equal(scales, s0.astype(np.float32))


def test_quantizer_scale_is_fp32_division_by_seven():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((40, 32)).astype(np.float32)
    _, scales = oracle.quantize_vectors(y)
    amax = np.abs(y).max(axis=1)
    np.testing.assert_array_equal(scales[:, 0], (amax / np.float32(7)).astype(np.float32))


# ----------------------------------------------------------------- packing

def test_pack_hand_layout():
    with open(os.path.join(GOLDEN, "pack_layout.txt")) as f:
        lines = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for i in range(0, len(lines), 3):
        d = int(lines[i][0].split("=")[1])
        codes = np.zeros((1, d), np.int8)
        for tok in lines[i + 1][1:]:
            k, c = tok.split(":")
            codes[0, int(k)] = int(c)
        want = np.zeros(d // 2, np.uint8)
        for tok in lines[i + 2][1:]:
            k, b = tok.split(":")
            want[int(k)] = int(b, 16)
        packed = oracle.pack(codes)
        np.testing.assert_array_equal(packed[0], want)
        np.testing.assert_array_equal(oracle.unpack(packed, d), codes)


@pytest.mark.parametrize("d", [32, 64, 128, 256])
def test_pack_is_a_bijection(d):
    idx = sorted(oracle.packed_byte_index(d, i) * 2 + (i % 32) % 2 for i in range(d))
    assert idx == list(range(d))                     # every nibble used exactly once
    rng = np.random.default_rng(d)
    c = rng.integers(-8, 8, (50, d)).astype(np.int8)
    np.testing.assert_array_equal(oracle.unpack(oracle.pack(c), d), c)


def test_compression_closed_form():
    with open(os.path.join(GOLDEN, "compression.txt")) as f:
        vals = dict(ln.split() for ln in f if ln.strip() and not ln.startswith("#"))
    d = int(vals["head_dim"])
    cache = oracle.empty_cache(1, 1, 1, d)
    int4_bytes = cache[0].nbytes + cache[1].nbytes
    assert int4_bytes == int(vals["int4_bytes_per_vector"])
    assert 2 * d == int(vals["bf16_bytes_per_vector"])
    assert (2 * d) / int4_bytes == float(vals["ratio"])
    n = 80 * 8 * 2 * 131072
    assert n * 2 * d == int(vals["llama70b_128k_bf16_bytes"]) == 40 * 2 ** 30
    assert n * int4_bytes == int(vals["llama70b_128k_int4_bytes"]) == int(12.5 * 2 ** 30)


# ---------------------------------------------------------- quantize-append

def test_quantize_append_positions_and_untouched_rows():
    rng = np.random.default_rng(9)
    B, H, n, d, cap = 2, 3, 5, 64, 16
    k = rng.standard_normal((B, H, n, d)).astype(np.float32)
    v = rng.standard_normal((B, H, n, d)).astype(np.float32)
    cache = oracle.empty_cache(B, H, cap, d)
    for a in cache:
        a[...] = 0xAB if a.dtype == np.uint8 else -1.0
    pos = np.array([0, 9], np.int32)
    oracle.quantize_append(k, v, pos, None, cache)
    kp, ks, vp, vs = cache
    for b in range(B):
        rows = np.arange(pos[b], pos[b] + n)
        codes, scales = oracle.quantize_vectors(k[b].reshape(-1, d))
        np.testing.assert_array_equal(kp[b][:, rows].reshape(-1, d // 2), oracle.pack(codes))
        np.testing.assert_array_equal(ks[b][:, rows].reshape(-1, d // 32), scales)
        codes, scales = oracle.quantize_vectors(v[b].reshape(-1, d))
        np.testing.assert_array_equal(vp[b][:, rows].reshape(-1, d // 2), oracle.pack(codes))
        other = np.setdiff1d(np.arange(cap), rows)
        assert np.all(kp[b][:, other] == 0xAB) and np.all(vs[b][:, other] == -1.0)


def test_quantize_append_bf16_input_is_exact_conversion():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((1, 1, 4, 128)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)      # truncate to bf16
    xb = (bits.astype(np.uint32) << 16).view(np.float32)
    c1 = oracle.empty_cache(1, 1, 4, 128)
    c2 = oracle.empty_cache(1, 1, 4, 128)
    s = rand_signs(rng, 128)
    oracle.quantize_append(bits, bits, [0], s, c1)
    oracle.quantize_append(xb, xb, [0], s, c2)
    for a, b in zip(c1, c2):
        np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------- decode

def _random_cache(rng, B, H, T, d):
    codes_k = rng.integers(-7, 8, (B, H, T, d)).astype(np.int8)
    codes_v = rng.integers(-7, 8, (B, H, T, d)).astype(np.int8)
    sk = rng.uniform(0.05, 0.5, (B, H, T, d // 32)).astype(np.float32)
    sv = rng.uniform(0.05, 0.5, (B, H, T, d // 32)).astype(np.float32)
    kp = oracle.pack(codes_k.reshape(-1, d)).reshape(B, H, T, d // 2)
    vp = oracle.pack(codes_v.reshape(-1, d)).reshape(B, H, T, d // 2)
    khat = np.repeat(sk.astype(np.float64), 32, axis=-1) * codes_k
    vhat = np.repeat(sv.astype(np.float64), 32, axis=-1) * codes_v
    return (kp, sk, vp, sv), khat, vhat


def _numpy_attention(q, k, v, scale):
    """Independent brute force: softmax(scale * q k^T) v with a plain exp/sum."""
    s = scale * (k @ q)
    w = np.exp(s - s.max())
    return (w / w.sum()) @ v


@pytest.mark.parametrize("T", [1, 2, 3, 7, 40])
@pytest.mark.parametrize("d", [32, 64])
def test_decode_brute_force_rotation_off(T, d):
    rng = np.random.default_rng(T * 100 + d)
    B, Hkv, G = 2, 2, 3
    cache, khat, vhat = _random_cache(rng, B, Hkv, T, d)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    scale = 1 / np.sqrt(d)
    out = oracle.sdpa_int4_decode(q, cache, [T] * B, None, scale, Hkv)
    for b in range(B):
        for h in range(Hkv * G):
            want = _numpy_attention(q[b, h].astype(np.float64), khat[b, h // G], vhat[b, h // G], scale)
            np.testing.assert_allclose(out[b, h], want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T", [1, 5, 33])
def test_decode_rotation_on_is_attention_in_unrotated_basis(T):
    """With rotation, the cache holds R k; attention must equal plain attention
    over the dequantized vectors mapped back by R^T (catches a missing or
    transposed rotation of q or of the output)."""
    rng = np.random.default_rng(T)
    d, Hkv, G = 64, 1, 2
    s = rand_signs(rng, d)
    R = oracle.rotation_matrix(d, s)
    cache, khat_r, vhat_r = _random_cache(rng, 1, Hkv, T, d)
    q = rng.standard_normal((1, G, d)).astype(np.float32)
    out = oracle.sdpa_int4_decode(q, cache, [T], s, 0.3, Hkv)
    k_unrot = khat_r[0, 0] @ R          # rows: R^T k_r
    v_unrot = vhat_r[0, 0] @ R
    for h in range(G):
        want = _numpy_attention(q[0, h].astype(np.float64), k_unrot, v_unrot, 0.3)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-11, atol=1e-12)


def test_decode_single_token_returns_value():
    rng = np.random.default_rng(1)
    d = 128
    cache, _, vhat = _random_cache(rng, 1, 1, 1, d)
    q = rng.standard_normal((1, 4, d)).astype(np.float32)
    out = oracle.sdpa_int4_decode(q, cache, [1], None, 1.0, 1)
    for h in range(4):
        np.testing.assert_array_equal(out[0, h], vhat[0, 0, 0])


def test_decode_constant_scores_give_mean():
    rng = np.random.default_rng(2)
    d, T = 128, 37
    cache, _, vhat = _random_cache(rng, 1, 1, T, d)
    q = np.zeros((1, 2, d), np.float32)
    s = rand_signs(rng, d)
    out = oracle.sdpa_int4_decode(q, cache, [T], s, 1.0, 1)
    R = oracle.rotation_matrix(d, s)
    np.testing.assert_allclose(out[0, 0], vhat[0, 0].mean(axis=0) @ R, rtol=0, atol=1e-13)


def test_decode_gqa_head_mapping_and_ctx_lens():
    rng = np.random.default_rng(4)
    B, Hkv, G, d, cap = 2, 4, 2, 32, 9
    cache, khat, vhat = _random_cache(rng, B, Hkv, cap, d)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    ctx = [9, 4]
    out = oracle.sdpa_int4_decode(q, cache, ctx, None, 0.5, Hkv)
    for b in range(B):
        for h in range(Hkv * G):
            T = ctx[b]
            want = _numpy_attention(q[b, h].astype(np.float64), khat[b, h // G, :T], vhat[b, h // G, :T], 0.5)
            np.testing.assert_allclose(out[b, h], want, rtol=1e-12, atol=1e-13)


def test_decode_large_scores_are_stable():
    rng = np.random.default_rng(6)
    d, T = 128, 64
    cache, khat, vhat = _random_cache(rng, 1, 1, T, d)
    q = (rng.standard_normal((1, 1, d)) * 300).astype(np.float32)
    out = oracle.sdpa_int4_decode(q, cache, [T], None, 1.0, 1)
    assert np.all(np.isfinite(out))
    want = _numpy_attention(q[0, 0].astype(np.float64), khat[0, 0], vhat[0, 0], 1.0)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-10, atol=1e-12)


def test_decode_bf16_query_equals_fp32_of_same_values():
    rng = np.random.default_rng(8)
    d, T = 128, 10
    cache, _, _ = _random_cache(rng, 1, 1, T, d)
    x = rng.standard_normal((1, 2, d)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xb = (bits.astype(np.uint32) << 16).view(np.float32)
    s = rand_signs(rng, d)
    a = oracle.sdpa_int4_decode(bits, cache, [T], s, 0.1, 1)
    b = oracle.sdpa_int4_decode(xb, cache, [T], s, 0.1, 1)
    np.testing.assert_array_equal(a, b)


def test_end_to_end_on_grid_rotation_off_is_exact_attention():
    """Quantize-append then decode on inputs already on the int4 grid gives the
    unquantized attention (up to fp64 rounding)."""
    rng = np.random.default_rng(10)
    B, Hkv, G, T, d = 1, 2, 4, 12, 64
    c = rng.integers(-7, 8, (2, B, Hkv, T, d))
    c[..., 3] = 7          # every group needs a full-scale code
    c[..., 35] = -7
    k = (c[0] * 0.25).astype(np.float32)
    v = (c[1] * 0.125).astype(np.float32)
    cache = oracle.empty_cache(B, Hkv, T, d)
    oracle.quantize_append(k, v, [0], None, cache)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    got = oracle.sdpa_int4_decode(q, cache, [T], None, 0.2, Hkv)
    want = oracle.exact_attention(q, k, v, [T], 0.2)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_end_to_end_on_grid_hadamard_rotation_is_exact_attention(d):
    """K and V are built so that their rotated images R x (R = H diag(signs) /
    sqrt(d), H from the Sylvester recursion above, not the oracle's) lie on the
    int4 grid: quantize-append with rotation on must store exactly those codes,
    and decode must give the unquantized attention over the original vectors.
    Catches signs applied after H instead of before, a transposed rotation, a
    missing 1/sqrt(d) in either direction and a query left unrotated."""
    rng = np.random.default_rng(d + 1)
    B, Hkv, G, T = 1, 2, 3, 11
    s = rand_signs(rng, d)
    R = sylvester(d) * s.astype(np.float64)[None, :] / np.sqrt(d)
    c = rng.integers(-7, 8, (2, B, Hkv, T, d))
    c[..., ::32] = 7                      # a full-scale code in every group
    yk, yv = c[0] * 0.25, c[1] * 0.125
    k = (yk @ R).astype(np.float32)       # x = R^T y, so R x = y
    v = (yv @ R).astype(np.float32)
    cache = oracle.empty_cache(B, Hkv, T, d)
    oracle.quantize_append(k, v, [0], s, cache)
    codes_k = oracle.unpack(cache[0].reshape(-1, d // 2), d).reshape(c[0].shape)
    codes_v = oracle.unpack(cache[2].reshape(-1, d // 2), d).reshape(c[1].shape)
    np.testing.assert_array_equal(codes_k, c[0])
    np.testing.assert_array_equal(codes_v, c[1])
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    got = oracle.sdpa_int4_decode(q, cache, [T], s, 0.3, Hkv)
    want = oracle.exact_attention(q, k, v, [T], 0.3)
    np.testing.assert_allclose(got, want, rtol=2e-6, atol=2e-6 * np.abs(want).max())


def test_exact_attention_brute_force():
    rng = np.random.default_rng(13)
    B, Hkv, G, T, d = 1, 2, 2, 9, 32
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    out = oracle.exact_attention(q, k, v, [T], 0.7)
    for h in range(Hkv * G):
        want = _numpy_attention(q[0, h].astype(np.float64), k[0, h // G].astype(np.float64),
                                v[0, h // G].astype(np.float64), 0.7)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-12, atol=1e-14)


def test_oracle_rejects_bad_shapes():
    q = np.zeros((1, 3, 64), np.float32)
    cache = oracle.empty_cache(1, 2, 4, 64)
    with pytest.raises(ValueError):
        oracle.sdpa_int4_decode(q, cache, [4], None, 1.0, 2)      # 3 % 2 != 0
    with pytest.raises(ValueError):
        oracle.sdpa_int4_decode(np.zeros((1, 2, 64), np.float32), cache, [5], None, 1.0, 2)


# ------------------------------------------------------- SRFT variant
# The SRFT post (core method) replaces the Hadamard rotation by a
# sign-randomized Fourier transform that works at widths that are not powers of
# two, followed by a per-coordinate scale lambda.  The oracle's transform is the
# orthonormal discrete Hartley transform; these pins check it against numpy's
# FFT (H = Re X - Im X for X = fft(x)), against the transform's algebra, and
# the whole variant against attention over a cache built exactly on the grid.

def _hartley_from_fft(d):
    X = np.fft.fft(np.eye(d), axis=0)          # column j = DFT of e_j
    return (X.real - X.imag) / np.sqrt(d)


def _rand_lambda(rng, d):
    return np.exp2(rng.uniform(-1.0, 1.0, d)).astype(np.float32)


@pytest.mark.parametrize("d", [1, 2, 3, 5, 12, 32, 96, 160, 256])
def test_dht_matches_numpy_fft(d):
    F = oracle.srft_matrix(d)
    np.testing.assert_allclose(F, _hartley_from_fft(d), rtol=0, atol=1e-14)


def test_dht_hand_values_d4():
    # cas(pi k j / 2) for k, j in 0..3: cos + sin of multiples of 90 degrees
    want = np.array([[1, 1, 1, 1], [1, 1, -1, -1], [1, -1, 1, -1], [1, -1, -1, 1]]) / 2.0
    np.testing.assert_allclose(oracle.srft_matrix(4), want, rtol=0, atol=1e-15)
    assert oracle.dht_entry(4, 1, 1) == pytest.approx(1.0 / 2.0, abs=1e-15)


@pytest.mark.parametrize("d", [32, 96, 160, 224])
def test_dht_is_symmetric_orthogonal_involution(d):
    F = oracle.srft_matrix(d)
    np.testing.assert_array_equal(F, F.T)
    assert np.max(np.abs(F @ F - np.eye(d))) <= 1e-13


@pytest.mark.parametrize("d", [32, 96, 192])
def test_srft_store_map_is_lambda_hartley_signs(d):
    rng = np.random.default_rng(d + 7)
    s, lam = rand_signs(rng, d), _rand_lambda(rng, d)
    A = oracle.srft_matrix(d, s, lam)
    want = lam.astype(np.float64)[:, None] * _hartley_from_fft(d) * s.astype(np.float64)[None, :]
    np.testing.assert_allclose(A, want, rtol=0, atol=1e-13)
    x = rng.standard_normal((5, d)).astype(np.float32)
    y = oracle.srft_rotate(x, s, lam)
    np.testing.assert_allclose(y, (x.astype(np.float64) @ want.T).astype(np.float32), rtol=2e-7,
                               atol=1e-7)


def test_srft_group_uniform_power_of_two_lambda_scales_exactly():
    """lambda = 2^e constant on each group multiplies that group's scale by 2^e
    exactly and leaves its codes unchanged (the quantizer is scale-equivariant)."""
    rng = np.random.default_rng(3)
    d = 96
    s = rand_signs(rng, d)
    e = np.repeat(np.array([-2, 0, 3]), 32)
    lam = np.exp2(e).astype(np.float32)
    x = rng.standard_normal((1, 1, 4, d)).astype(np.float32)
    c1, c2 = oracle.empty_cache(1, 1, 4, d), oracle.empty_cache(1, 1, 4, d)
    oracle.quantize_append_srft(x, x, [0], s, None, None, c1)
    oracle.quantize_append_srft(x, x, [0], s, lam, None, c2)
    np.testing.assert_array_equal(c1[0], c2[0])
    np.testing.assert_array_equal(c1[1] * np.exp2([-2, 0, 3]).astype(np.float32), c2[1])
    np.testing.assert_array_equal(c1[2], c2[2])       # V uses its own (unit) lambda
    np.testing.assert_array_equal(c1[3], c2[3])


@pytest.mark.parametrize("d", [32, 96, 160])
def test_srft_end_to_end_on_grid_is_exact_attention(d):
    """K and V are built so that their SRFT images (with random signs and
    random lambdas) lie on the int4 grid: quantize-append then decode must give
    the unquantized attention over the original vectors.  Catches a query map
    that multiplies by lambda instead of dividing, an output map without the
    inverse transform or without 1/lambda_V, and a transposed sign."""
    rng = np.random.default_rng(d)
    B, Hkv, G, T = 1, 2, 3, 9
    s = rand_signs(rng, d)
    lk, lv = _rand_lambda(rng, d), _rand_lambda(rng, d)
    Fh = _hartley_from_fft(d)
    inv_store = lambda lam: (s.astype(np.float64)[:, None] * Fh) / lam.astype(np.float64)[None, :]
    c = rng.integers(-7, 8, (2, B, Hkv, T, d))
    c[..., ::32] = 7                      # a full-scale code in every group
    yk, yv = c[0] * 0.25, c[1] * 0.125
    k = (yk @ inv_store(lk).T).astype(np.float32)
    v = (yv @ inv_store(lv).T).astype(np.float32)
    cache = oracle.empty_cache(B, Hkv, T, d)
    oracle.quantize_append_srft(k, v, [0], s, lk, lv, cache)
    codes = oracle.unpack(cache[0].reshape(-1, d // 2), d).reshape(c[0].shape)
    np.testing.assert_array_equal(codes, c[0])
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    got = oracle.sdpa_int4_decode_srft(q, cache, [T], s, lk, lv, 0.3, Hkv)
    want = oracle.exact_attention(q, k, v, [T], 0.3)
    np.testing.assert_allclose(got, want, rtol=2e-6, atol=2e-6 * np.abs(want).max())


def test_srft_reduces_to_hartley_when_unit_signs_and_lambda():
    rng = np.random.default_rng(5)
    d = 96
    x = rng.standard_normal((3, d)).astype(np.float32)
    ones = np.ones(d, np.int8)
    np.testing.assert_array_equal(oracle.srft_rotate(x, ones, np.ones(d, np.float32)),
                                  oracle.srft_rotate(x))
    np.testing.assert_allclose(oracle.srft_rotate(x), x.astype(np.float64) @ _hartley_from_fft(d).T,
                               rtol=2e-7, atol=1e-7)


# --------------------------------------------------- codebook variant
# AdapTQ (unified SIMD pipeline; precomputed lookup tables; performance and
# quality): 2/3/4-bit indices into a Max-Lloyd codebook with +-3 sigma
# clipping.  The pins check the Gaussian Max-Lloyd codebook against its closed
# form at 1 bit, its defining conditions by independent numerical integration
# and Max's published distortions; the quantizer against nearest-level
# assignment with an RMS scale computed here; the layout by hand-derived bytes.

from math import erf as _erf, exp as _exp, pi as _pi, sqrt as _sqrt


def _phi(x):
    return _exp(-0.5 * x * x) / _sqrt(2 * _pi)


def _integrate(f, a, b, n=20001):
    """Simpson's rule on [a, b] (a, b finite)."""
    x = np.linspace(a, b, n)
    y = np.array([f(t) for t in x])
    h = (b - a) / (n - 1)
    return h / 3 * (y[0] + y[-1] + 4 * y[1:-1:2].sum() + 2 * y[2:-1:2].sum())


def test_lloyd_max_one_bit_closed_form():
    c = oracle.lloyd_max_gaussian(1)
    np.testing.assert_allclose(c, [-_sqrt(2 / _pi), _sqrt(2 / _pi)], rtol=0, atol=1e-12)


@pytest.mark.parametrize("bits,dist", [(1, 0.3634), (2, 0.1175), (3, 0.03454), (4, 0.009497)])
def test_lloyd_max_distortion_matches_published_table(bits, dist):
    """Mean squared error of the Gaussian Max-Lloyd quantizer (Max, 1960), by
    numerical integration over [-10, 10]."""
    c = oracle.lloyd_max_gaussian(bits)
    t = np.concatenate([[-10.0], 0.5 * (c[1:] + c[:-1]), [10.0]])
    mse = sum(_integrate(lambda x, ci=ci: (x - ci) ** 2 * _phi(x), t[i], t[i + 1])
              for i, ci in enumerate(c))
    assert mse == pytest.approx(dist, rel=2e-3)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_levels_are_cell_means(bits):
    c = oracle.lloyd_max_gaussian(bits)
    np.testing.assert_allclose(c, -c[::-1], atol=1e-12)          # symmetric
    t = np.concatenate([[-12.0], 0.5 * (c[1:] + c[:-1]), [12.0]])
    for i in range(len(c)):
        num = _integrate(lambda x: x * _phi(x), t[i], t[i + 1])
        den = _integrate(_phi, t[i], t[i + 1])
        assert num / den == pytest.approx(c[i], abs=1e-7)


def _rms_sigma(y):
    return np.float32(np.sqrt(np.sum(y.astype(np.float64) ** 2) / 32))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cb_quantizer_is_nearest_level_with_rms_scale(bits):
    rng = np.random.default_rng(bits)
    c = oracle.lloyd_max_gaussian(bits).astype(np.float32)
    y = (rng.standard_normal((200, 64)) * np.exp(rng.uniform(-5, 5, (200, 1)))).astype(np.float32)
    y[:, 7] *= 9                                               # outliers beyond 3 sigma
    idx, sc = oracle.cb_quantize_vectors(y, bits, c)
    for r in range(200):
        for g in range(2):
            yg = y[r, 32 * g:32 * g + 32]
            s = _rms_sigma(yg)
            assert sc[r, g] == s
            u = np.clip((yg / s).astype(np.float32), -3, 3)
            want = np.argmin(np.abs(u[:, None].astype(np.float64) - c[None, :]), axis=1)
            np.testing.assert_array_equal(idx[r, 32 * g:32 * g + 32], want)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cb_quantizer_custom_levels_is_nearest_level(bits):
    """With any increasing levels (here uneven and asymmetric) the index is the
    nearest level to the clipped, rms-scaled coordinate."""
    rng = np.random.default_rng(bits + 70)
    c = np.sort(rng.uniform(-2.6, 2.2, 1 << bits)).astype(np.float32)
    y = (rng.standard_normal((100, 64)) * np.exp(rng.uniform(-3, 3, (100, 1)))).astype(np.float32)
    idx, sc = oracle.cb_quantize_vectors(y, bits, c)
    for r in range(100):
        for g in range(2):
            yg = y[r, 32 * g:32 * g + 32]
            s = _rms_sigma(yg)
            assert sc[r, g] == s
            u = np.clip((yg / s).astype(np.float32), -3, 3).astype(np.float64)
            want = np.argmin(np.abs(u[:, None] - c[None, :].astype(np.float64)), axis=1)
            np.testing.assert_array_equal(idx[r, 32 * g:32 * g + 32], want)


def test_cb_quantizer_tie_and_zero_group_take_the_lower_level():
    c = oracle.lloyd_max_gaussian(2).astype(np.float32)        # middle threshold is exactly 0
    y = np.zeros((2, 32), np.float32)
    y[1, 1:] = 1.0                                             # sigma = sqrt(31/32); y[1,0] = 0 sits on it
    idx, sc = oracle.cb_quantize_vectors(y, 2, c)
    assert sc[0, 0] == 0 and np.all(idx[0] == 1)
    assert idx[1, 0] == 1 and np.all(idx[1, 1:] == 3)


def test_cb_quantizer_scale_equivariance():
    rng = np.random.default_rng(8)
    c = oracle.lloyd_max_gaussian(3).astype(np.float32)
    y = rng.standard_normal((20, 64)).astype(np.float32)
    i1, s1 = oracle.cb_quantize_vectors(y, 3, c)
    i2, s2 = oracle.cb_quantize_vectors(y * np.float32(2.0 ** 7), 3, c)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_array_equal(s1 * np.float32(2.0 ** 7), s2)


def test_cb_pack_hand_layout():
    idx = np.zeros((1, 64), np.uint8)
    idx[0, :4] = [1, 2, 3, 0]
    p2 = oracle.cb_pack(idx, 2)
    assert p2.shape == (1, 16) and p2[0, 0] == 0x39 and not p2[0, 1:].any()
    idx = np.zeros((1, 64), np.uint8)
    idx[0, 0], idx[0, 1] = 5, 3                                # bits 0-2 = 101, bits 3-5 = 011
    idx[0, 10] = 7                                             # bits 30, 31 | 32: straddles bytes 3, 4
    idx[0, 32] = 6                                             # group 1 starts at byte 12
    p3 = oracle.cb_pack(idx, 3)
    assert p3.shape == (1, 24)
    assert p3[0, 0] == 0x1D and p3[0, 3] == 0xC0 and p3[0, 4] == 0x01 and p3[0, 12] == 0x06
    assert p3[0, [1, 2, 5, 6, 7, 8, 9, 10, 11]].sum() == 0
    idx = np.zeros((1, 32), np.uint8)
    idx[0, 0], idx[0, 1], idx[0, 31] = 0xA, 0x3, 0xF
    p4 = oracle.cb_pack(idx, 4)
    assert p4[0, 0] == 0x3A and p4[0, 15] == 0xF0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cb_pack_is_a_bijection(bits):
    rng = np.random.default_rng(bits + 20)
    idx = rng.integers(0, 1 << bits, (50, 128)).astype(np.uint8)
    np.testing.assert_array_equal(oracle.cb_unpack(oracle.cb_pack(idx, bits), 128, bits), idx)


def _random_cb_cache(rng, B, H, T, d, bits, c):
    ik = rng.integers(0, 1 << bits, (B, H, T, d)).astype(np.uint8)
    iv = rng.integers(0, 1 << bits, (B, H, T, d)).astype(np.uint8)
    sk = rng.uniform(0.05, 0.5, (B, H, T, d // 32)).astype(np.float32)
    sv = rng.uniform(0.05, 0.5, (B, H, T, d // 32)).astype(np.float32)
    kp = oracle.cb_pack(ik.reshape(-1, d), bits).reshape(B, H, T, -1)
    vp = oracle.cb_pack(iv.reshape(-1, d), bits).reshape(B, H, T, -1)
    c64 = c.astype(np.float64)
    khat = np.repeat(sk.astype(np.float64), 32, axis=-1) * c64[ik]
    vhat = np.repeat(sv.astype(np.float64), 32, axis=-1) * c64[iv]
    return (kp, sk, vp, sv), khat, vhat


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cb_decode_brute_force_rotation_off(bits):
    rng = np.random.default_rng(bits + 30)
    B, Hkv, G, T, d = 2, 2, 3, 17, 64
    c = oracle.lloyd_max_gaussian(bits).astype(np.float32)
    cache, khat, vhat = _random_cb_cache(rng, B, Hkv, T, d, bits, c)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    out = oracle.sdpa_cb_decode(q, cache, [T, T - 5], None, bits, c, 0.2, Hkv)
    for b, Tb in ((0, T), (1, T - 5)):
        for h in range(Hkv * G):
            want = _numpy_attention(q[b, h].astype(np.float64), khat[b, h // G, :Tb],
                                    vhat[b, h // G, :Tb], 0.2)
            np.testing.assert_allclose(out[b, h], want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("bits,mul,off", [(2, 1e3, 0.3), (3, 1e-3, -0.2), (4, 37.0, 0.05)])
def test_cb_decode_custom_levels_brute_force(bits, mul, off):
    """Levels other than the Gaussian codebook (shifted, far from 1 in
    magnitude): the decode is still attention over sigma * C[index]."""
    rng = np.random.default_rng(bits + 60)
    B, Hkv, G, T, d = 1, 2, 2, 13, 64
    c = ((oracle.lloyd_max_gaussian(bits) + off) * mul).astype(np.float32)
    assert np.all(np.diff(c) > 0)
    cache, khat, vhat = _random_cb_cache(rng, B, Hkv, T, d, bits, c)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    scale = 0.05 / mul
    out = oracle.sdpa_cb_decode(q, cache, [T], None, bits, c, scale, Hkv)
    for h in range(Hkv * G):
        want = _numpy_attention(q[0, h].astype(np.float64), khat[0, h // G], vhat[0, h // G], scale)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-11, atol=1e-12 * max(1.0, mul))


def test_cb_decode_rotation_on_is_attention_in_unrotated_basis():
    rng = np.random.default_rng(44)
    d, Hkv, G, T, bits = 64, 1, 2, 9, 3
    c = oracle.lloyd_max_gaussian(bits).astype(np.float32)
    s = rand_signs(rng, d)
    R = oracle.rotation_matrix(d, s)
    cache, khat_r, vhat_r = _random_cb_cache(rng, 1, Hkv, T, d, bits, c)
    q = rng.standard_normal((1, G, d)).astype(np.float32)
    out = oracle.sdpa_cb_decode(q, cache, [T], s, bits, c, 0.3, Hkv)
    for h in range(G):
        want = _numpy_attention(q[0, h].astype(np.float64), khat_r[0, 0] @ R, vhat_r[0, 0] @ R, 0.3)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-11, atol=1e-12)


def test_cb_append_rotates_then_quantizes_rows_at_pos():
    rng = np.random.default_rng(45)
    d, bits = 128, 2
    c = oracle.lloyd_max_gaussian(bits).astype(np.float32)
    s = rand_signs(rng, d)
    k = rng.standard_normal((1, 2, 3, d)).astype(np.float32)
    v = rng.standard_normal((1, 2, 3, d)).astype(np.float32)
    cache = oracle.empty_cb_cache(1, 2, 8, d, bits)
    oracle.quantize_append_cb(k, v, [4], s, bits, c, cache)
    for h in range(2):
        idx, sc = oracle.cb_quantize_vectors(oracle.rotate(k[0, h], s), bits, c)
        np.testing.assert_array_equal(cache[0][0, h, 4:7], oracle.cb_pack(idx, bits))
        np.testing.assert_array_equal(cache[1][0, h, 4:7], sc)
        assert not cache[0][0, h, :4].any() and not cache[0][0, h, 7:].any()


# ---------------------------------------------------------------------------
# Uniform low-bit variant (Open-TQ-Metal forum summary, future work: int2; read
# as the int4 quantizer at fewer bits): m = 2^(bits-1) - 1, s = fl32(amax / m),
# c = clamp(rne(fl32(y / s)), -m, m), stored as index c + m in the codebook
# layout; the decode-side levels are C[u] = u - m.

def test_uniform_levels_are_the_integer_codes():
    np.testing.assert_array_equal(oracle.uniform_levels(2), [-1, 0, 1, 2])
    np.testing.assert_array_equal(oracle.uniform_levels(3), [-3, -2, -1, 0, 1, 2, 3, 4])
    np.testing.assert_array_equal(oracle.uniform_levels(4), np.arange(16) - 7)


def test_uniform_2bit_hand_values():
    """amax 1 gives s = 1: codes are rne(y), ties to even on both sides of 0."""
    y = np.zeros((1, 32), np.float32)
    y[0, :8] = [1.0, 0.5, -0.5, 0.49999997, -0.50000006, 0.0, 0.75, -1.0]
    idx, sc = oracle.uniform_quantize_vectors(y, 2)
    assert sc[0, 0] == 1.0
    np.testing.assert_array_equal(idx[0, :8], np.array([1, 0, 0, 0, -1, 0, 1, -1]) + 1)
    assert np.all(idx[0, 8:] == 1)


def test_uniform_3bit_hand_values():
    """amax 3 gives s = 3/3 = 1; amax 1.5 gives s = 0.5 exactly."""
    y = np.zeros((2, 32), np.float32)
    y[0, :8] = [3.0, 2.5, 1.5, -2.5, -0.5, 0.4, -3.0, 2.6]
    y[1, :6] = [1.5, 0.25, 0.75, -1.25, 1.0, -0.3]
    idx, sc = oracle.uniform_quantize_vectors(y, 3)
    assert sc[0, 0] == 1.0 and sc[1, 0] == 0.5
    np.testing.assert_array_equal(idx[0, :8], np.array([3, 2, 2, -2, 0, 0, -3, 3]) + 3)
    np.testing.assert_array_equal(idx[1, :6], np.array([3, 0, 2, -2, 2, -1]) + 3)


def test_uniform_4bit_is_the_int4_quantizer():
    """At four bits m = 7: the same scales and codes as the int4 path."""
    rng = np.random.default_rng(70)
    y = (rng.standard_normal((40, 128)) * np.exp(rng.uniform(-6, 6, (40, 1)))).astype(np.float32)
    y[3] = 0.0
    idx, sc = oracle.uniform_quantize_vectors(y, 4)
    codes, sc4 = oracle.quantize_vectors(y)
    np.testing.assert_array_equal(sc.view(np.uint32), sc4.view(np.uint32))
    np.testing.assert_array_equal(idx.astype(np.int64) - 7, codes.astype(np.int64))


@pytest.mark.parametrize("bits", [2, 3])
def test_uniform_quantizer_invariants(bits):
    """Half-step bound, the abs-max element at +-m, sign symmetry, exact
    power-of-two scale equivariance, zero groups."""
    m = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(71 + bits)
    y = (rng.standard_normal((60, 128)) * np.exp(rng.uniform(-8, 8, (60, 1)))).astype(np.float32)
    y[5, 32:64] = 0.0
    idx, sc = oracle.uniform_quantize_vectors(y, bits)
    c = idx.astype(np.int64) - m
    assert c.min() >= -m and c.max() <= m
    s = np.repeat(sc.astype(np.float64), 32, axis=1)
    err = np.abs(y.astype(np.float64) - s * c)
    assert np.all(err <= s * (0.5 + 1e-6))
    g = y.reshape(60, 4, 32)
    top = np.abs(g).argmax(axis=2)
    for r in range(60):
        for k in range(4):
            if sc[r, k] > 0:
                assert abs(c[r, 32 * k + top[r, k]]) == m
    assert sc[5, 1] == 0.0 and np.all(idx[5, 32:64] == m)
    idx_neg, sc_neg = oracle.uniform_quantize_vectors(-y, bits)
    np.testing.assert_array_equal(idx_neg.astype(np.int64) - m, -c)
    np.testing.assert_array_equal(sc_neg, sc)
    idx2, sc2 = oracle.uniform_quantize_vectors(y * np.float32(2.0 ** -5), bits)
    np.testing.assert_array_equal(idx2, idx)
    np.testing.assert_array_equal(sc2, sc * np.float32(2.0 ** -5))


@pytest.mark.parametrize("bits", [2, 3])
def test_uniform_append_rotates_then_quantizes_rows_at_pos(bits):
    rng = np.random.default_rng(72 + bits)
    d = 128
    s = rand_signs(rng, d)
    k = rng.standard_normal((1, 2, 3, d)).astype(np.float32)
    v = rng.standard_normal((1, 2, 3, d)).astype(np.float32)
    cache = oracle.empty_cb_cache(1, 2, 8, d, bits)
    oracle.quantize_append_uniform(k, v, [4], s, bits, cache)
    for h in range(2):
        for src, kp, ks in ((k, cache[0], cache[1]), (v, cache[2], cache[3])):
            idx, sc = oracle.uniform_quantize_vectors(oracle.rotate(src[0, h], s), bits)
            np.testing.assert_array_equal(kp[0, h, 4:7], oracle.cb_pack(idx, bits))
            np.testing.assert_array_equal(ks[0, h, 4:7], sc)
            assert not kp[0, h, :4].any() and not kp[0, h, 7:].any()


@pytest.mark.parametrize("bits", [2, 3])
def test_uniform_decode_is_attention_over_s_times_c(bits):
    """A uniform cache decoded with its integer levels is softmax attention
    over s * c (numpy brute force, rotation off)."""
    m = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(74 + bits)
    B, Hkv, G, T, d = 1, 2, 2, 21, 64
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    cache = oracle.empty_cb_cache(B, Hkv, T, d, bits)
    oracle.quantize_append_uniform(k, v, [0], None, bits, cache)
    ik = oracle.cb_unpack(cache[0].reshape(-1, cache[0].shape[-1]), d, bits).reshape(B, Hkv, T, d)
    iv = oracle.cb_unpack(cache[2].reshape(-1, cache[2].shape[-1]), d, bits).reshape(B, Hkv, T, d)
    khat = np.repeat(cache[1].astype(np.float64), 32, axis=-1) * (ik.astype(np.float64) - m)
    vhat = np.repeat(cache[3].astype(np.float64), 32, axis=-1) * (iv.astype(np.float64) - m)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    out = oracle.sdpa_cb_decode(q, cache, [T], None, bits, oracle.uniform_levels(bits), 0.3, Hkv)
    for h in range(Hkv * G):
        want = _numpy_attention(q[0, h].astype(np.float64), khat[0, h // G], vhat[0, h // G], 0.3)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-12, atol=1e-13)
