"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand) fails it. No GPU needed.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from oracle import bgtq_oracle as OM
from packed_cache_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------------ randomness
def test_philox_known_answers():
    for row in _rows("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in row if x != "->"]
        ctr, key, want = v[:4], v[4:6], v[6:10]
        got = O.philox4x32_10(tuple([c] for c in ctr), tuple(key))
        assert [int(g[0]) for g in got] == want


def test_gaussian_stream_statistics_and_determinism():
    z = O.gaussian_stream(12345, 3, 400001)
    assert z.shape == (400001,)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1) < 0.01
    assert abs(np.mean(z ** 4) - 3) < 0.05          # Gaussian kurtosis
    assert abs(np.corrcoef(z[0:-1:2], z[1::2])[0, 1]) < 0.01  # the cos/sin pair is uncorrelated
    np.testing.assert_array_equal(z[:1000], O.gaussian_stream(12345, 3, 1000))
    assert not np.allclose(z[:100], O.gaussian_stream(12345, 4, 100))
    assert not np.allclose(z[:100], O.gaussian_stream(12346, 3, 100))


def test_haar_rotation_is_the_qr_factor_of_the_seeded_matrix():
    for d in (2, 6, 34, 128):
        r = O.haar_rotation(7, 2, d)
        np.testing.assert_allclose(r @ r.T, np.eye(d), atol=1e-12)
        a = O.gaussian_stream(7, 2, d * d).reshape(d, d)
        t = r.T @ a                                   # must be upper triangular, positive diagonal
        assert np.max(np.abs(np.tril(t, -1))) < 1e-10 * np.max(np.abs(t))
        assert np.all(np.diag(t) > 0)
        x = np.random.default_rng(d).standard_normal((50, d))
        np.testing.assert_allclose(np.linalg.norm(x @ r.T, axis=1) / np.linalg.norm(x, axis=1), 1.0, atol=1e-6)


def test_haar_rotation_first_moment():
    # For Haar-distributed Q, E[Q] = 0 and E[Q_ij^2] = 1/d.
    d = 16
    qs = np.stack([O.haar_rotation(s, 1, d) for s in range(300)])
    assert abs(qs.mean()) < 0.01
    assert abs((qs ** 2).mean() - 1.0 / d) < 0.002


# ------------------------------------------------------------------ Lloyd-Max
def test_lloyd_max_one_bit_closed_form():
    c, t, mse = O.lloyd_max(1)
    assert t.tolist() == [0.0]
    assert c[1] == pytest.approx(math.sqrt(2 / math.pi), rel=1e-14)
    assert mse == pytest.approx(1 - 2 / math.pi, rel=1e-13)


def test_lloyd_max_published_mse():
    for b, want in _rows("gaussian_lloyd_max_mse.txt"):
        assert O.lloyd_max(int(b))[2] == pytest.approx(float(want), rel=1e-3)


def test_lloyd_max_conditions_by_quadrature():
    from scipy import integrate
    from scipy.stats import norm
    for b in (2, 3, 4):
        c, t, mse = O.lloyd_max(b)
        np.testing.assert_allclose(c, -c[::-1], rtol=0, atol=0)
        assert t[len(t) // 2] == 0.0
        np.testing.assert_allclose(t, 0.5 * (c[1:] + c[:-1]), atol=1e-14)
        edges = np.concatenate([[-np.inf], t, [np.inf]])
        tot = 0.0
        for i in range(len(c)):
            p = norm.cdf(edges[i + 1]) - norm.cdf(edges[i])
            m1 = integrate.quad(lambda x: x * norm.pdf(x), edges[i], edges[i + 1])[0]
            assert m1 / p == pytest.approx(c[i], abs=1e-9)
            tot += integrate.quad(lambda x: (x - c[i]) ** 2 * norm.pdf(x), edges[i], edges[i + 1])[0]
        assert tot == pytest.approx(mse, rel=1e-8)


def test_lloyd_max_monte_carlo():
    x = np.random.default_rng(0).standard_normal(2_000_000)
    for b in (1, 2, 3, 4):
        c, t, mse = O.lloyd_max(b)
        xq = c[np.searchsorted(t, x, side="right")]
        assert np.mean((x - xq) ** 2) == pytest.approx(mse, rel=0.01)


def test_diminishing_marginal_gains():
    D = O.lloyd_max_mse_table()
    gains = [D[b] - D[b + 1] for b in (1, 2, 3)]
    assert all(g > 0 for g in gains) and gains[0] > gains[1] > gains[2]


# ------------------------------------------------------------------ energy + allocation
def test_block_energy_constructed_cases():
    n = 5
    # two KV heads, GQA 2: query heads 0,1 -> kv 0; 2,3 -> kv 1
    q = np.zeros((n, 4, 128))
    k = np.zeros((n, 2, 128))
    q[:, 0:2, 3] = 2.0           # kv-0 queries: energy 4 in block 3 (coordinate 3)
    q[:, 2:4, 64 + 10] = 1.0     # kv-1 queries: energy 1 in block 10 (coordinate 74)
    k[:, 0, 3 + 64] = 3.0        # kv-0 keys: energy 9 in block 3 (coordinate 67)
    k[:, 1, 10] = 5.0            # kv-1 keys: energy 25 in block 10
    k[:, 1, 3] = 7.0             # kv-1 key energy in block 3 meets no kv-1 query energy
    s = O.block_energy(q, k)
    want = np.zeros(64)
    want[3] = 4 * 9
    want[10] = 1 * 25
    np.testing.assert_allclose(s, want)


def test_block_energy_is_rope_invariant():
    m = synth.make_layer_model(8, 2, seed=3)
    q = torch.stack([torch.randn(64, 128) for _ in range(8)], 1).double()
    k = torch.stack([torch.randn(64, 128) for _ in range(2)], 1).double()
    pos = torch.arange(64) * 37 + 5
    qr = synth.rope_rotate_half(q.transpose(0, 1), pos, 5e5).transpose(0, 1)
    kr = synth.rope_rotate_half(k.transpose(0, 1), pos, 5e5).transpose(0, 1)
    np.testing.assert_allclose(O.block_energy(qr.numpy(), kr.numpy()), O.block_energy(q.numpy(), k.numpy()), rtol=1e-12)
    assert m.group == 4


def test_greedy_equals_exhaustive_optimum():
    rng = np.random.default_rng(1)
    D = O.lloyd_max_mse_table()
    cases = 0
    for n in (1, 2, 3, 4, 5, 6):
        for trial in range(3 if n < 6 else 1):
            s = rng.exponential(size=n) * rng.choice([1, 10, 100], size=n)
            if trial == 2:
                s[: n // 2] = s[-1]                 # ties
            for budget in range(n, 4 * n + 1):
                g = O.greedy_rates(s, D, 1, 4, budget)
                best, args = O.brute_force_rates(s, D, 1, 4, budget)
                assert g.sum() == budget
                assert O.proxy_objective(s, g, D) == pytest.approx(best, rel=1e-12, abs=1e-15)
                if len(args) == 1:
                    assert tuple(g) == args[0]
                cases += 1
    assert cases > 60


def test_greedy_infeasible_budget():
    D = O.lloyd_max_mse_table()
    with pytest.raises(ValueError):
        O.greedy_rates(np.ones(4), D, 1, 4, 3)
    with pytest.raises(ValueError):
        O.greedy_rates(np.ones(4), D, 1, 4, 17)


def test_greedy_prefers_high_energy_blocks():
    D = O.lloyd_max_mse_table()
    s = np.array([1.0, 100.0, 10.0, 0.01])
    r = O.greedy_rates(s, D, 1, 4, 8)
    assert r[1] >= r[2] >= r[0] >= r[3]


# ------------------------------------------------------------------ layout + format
def _random_rates(rng):
    r = rng.integers(1, 5, 64)
    while r.sum() % 4:
        j = rng.integers(0, 64)
        r[j] = r[j] % 4 + 1
    return r


def test_grouping_and_byte_formula():
    with pytest.raises(ValueError):
        O.make_layout(np.array([1] * 63 + [2]), 2, 0)           # 130 bits: not whole bytes
    lay = O.make_layout(np.array([2] * 64), 2, 0)
    assert lay.n_kgroups == 1 and lay.bytes_per_token == 32 + 32 + 8
    lay = O.make_layout(np.array([4] * 32 + [2] * 32), 2, 0)
    assert [r for r, _ in lay.groups] == [4, 2]
    assert list(lay.groups[0][1][:4]) == [0, 64, 1, 65]
    assert lay.bytes_per_token == 48 + 32 + 12
    mixed = np.array([1] * 16 + [2] * 16 + [3] * 16 + [4] * 16)        # average 2.5 bits
    lay = O.make_layout(mixed, 3, 0)
    assert [r for r, _ in lay.groups] == [4, 3, 2, 1]
    assert lay.k_bits == 2 * (16 + 32 + 48 + 64)
    # K2V2 with four groups: 32 + 32 + 20 = 84 bytes, K3V3 four groups 116, K4V4 one group 136
    k2 = np.array([1] * 22 + [2] * 22 + [3] * 18 + [4] * 2)
    assert k2.sum() == 128
    assert O.make_layout(k2, 2, 0).bytes_per_token == 84
    k3 = np.array([1] * 4 + [2] * 10 + [3] * 32 + [4] * 18)
    assert k3.sum() == 192
    assert O.make_layout(k3, 3, 0).bytes_per_token == 116
    assert O.make_layout(np.full(64, 4), 4, 0).bytes_per_token == 136
    lay = O.make_layout(k2, 2, 0)
    assert O.cache_bytes(lay, 2, 8, 128) == 2 * 8 * 128 * 84
    assert O.cache_bytes(lay, 1, 1, 65) == 128 * 84


def test_pack_places_bits_where_the_format_says():
    """Worked by hand from the fragment-major format: K quad lane i = 4 g + e holds the pair
    e codes of tokens g + 8 m; V lane 4 g + t holds field n = 4 mt + k = (dim 16 g + 2 mt +
    (k & 1), tokens 2 t + 8 (k >> 1) and +1)."""
    lay = O.make_layout(np.array([2] * 32 + [1] * 32), 3, 5)   # packed dims 0..63 rate 2, 64..127 rate 1
    assert [q[1:] for q in lay.k_quads()] == ([(4, 2, 128 * i) for i in range(8)]
                                              + [(4, 1, 1024 + 64 * i) for i in range(8)])
    n = 58
    enc = {"k_codes": np.zeros((n, 128), dtype=np.int64), "v_codes": np.zeros((n, 128), dtype=np.int64),
           "k_norms": np.zeros((n, 2)), "v_norm": np.zeros(n)}
    enc["k_codes"][2, 5] = 3     # quad 0, pair 2 hi; token 2 = (g 2, m 0): lane 10 -> word 10, bits 2-3
    enc["k_codes"][57, 6] = 2    # quad 0, pair 3 lo; token 57 = (g 1, m 7): lane 7 -> word 7, bits 28-29
    enc["k_codes"][1, 64] = 1    # rate-1 quad at 1024, pair 0 lo; token 1 = (g 1, m 0): lane 4 -> halfword 4, bit 0
    enc["k_codes"][0, 127] = 1   # rate-1 quad at 1472, pair 3 hi; token 0: lane 3 -> halfword 3, bit 8
    enc["v_codes"][1, 7] = 5     # chunk 0, dim 7 = (g 0, mt 3, k odd), token 1 = hi of (0, 1): lane 0, field 13
    enc["v_codes"][2, 0] = 6     # dim 0, token 2 = lo of (2, 3): t 1, k 0 -> lane 1, field 0
    enc["v_codes"][9, 127] = 7   # dim 127 = (g 7, mt 7, k odd), token 9 = hi of (8, 9): t 0, k 3 -> lane 28, field 31
    enc["v_codes"][17, 0] = 4    # chunk 1 (tokens 16..31), token 1 of the chunk, dim 0: lane 0, field 0 hi
    enc["k_norms"][1] = [1.5, -2.0]
    enc["v_norm"][2] = 0.25
    buf = O.pack(lay, enc, 64)
    assert lay.k_record_bytes == 24 and lay.tile_bytes == 64 * (24 + 48 + 12) and buf.size == lay.tile_bytes
    assert buf[40] == 0b00001100
    assert buf[31] == 0b00100000
    assert buf[1024 + 8] == 1
    assert buf[1472 + 7] == 1
    vbase = 64 * 24
    lane0 = int.from_bytes(buf[vbase:vbase + 16].tobytes(), "little")
    assert (lane0 >> (6 * 13 + 3)) & 7 == 5
    assert buf[vbase + 16] & 7 == 6
    assert buf[vbase + 512 + 8 * 28 + 7] == 0b11100000        # bits 189-191 of lane 28: its second plane
    assert (buf[vbase + 768] >> 3) & 7 == 4
    nbase = vbase + 64 * 48
    kn = buf[nbase:nbase + 4 * 128].view(np.float32)
    # norms: token t = g + 8 m at entry 8 g + m: token 1 -> entry 8, token 2 -> entry 16
    assert kn[8] == 1.5 and kn[64 + 8] == -2.0
    assert buf[nbase + 512:nbase + 768].view(np.float32)[16] == 0.25
    # nothing else written: one byte per code, and 1.5 / -2.0 / 0.25 have 2 / 1 / 2 nonzero bytes
    assert int(np.count_nonzero(buf)) == 8 + 2 + 1 + 2
    u = O.unpack(lay, buf, n)
    np.testing.assert_array_equal(u["k_codes"], enc["k_codes"])
    np.testing.assert_array_equal(u["v_codes"], enc["v_codes"])


def test_partial_quads_are_packed_densely():
    rates = np.array([4] * 3 + [3] * 5 + [2] * 9 + [1] * 47)     # group dims 6, 10, 18, 94
    assert rates.sum() % 4 == 0
    lay = O.make_layout(rates, 2, 1)
    qs = lay.k_quads()
    assert [(npairs, r) for _, npairs, r, _ in qs] == ([(3, 4), (4, 3), (1, 3), (4, 2), (4, 2), (1, 2)]
                                                       + [(4, 1)] * 11 + [(3, 1)])
    end = qs[-1][3] + 16 * qs[-1][1] * qs[-1][2]
    assert end == 64 * lay.k_record_bytes                      # no padding
    assert all(off % 16 == 0 for *_, off in qs)                # every block starts 16-byte aligned
    assert [p0 for p0, *_ in qs][:4] == [0, 6, 14, 16]


def test_every_code_has_exactly_one_place():
    """Pack codes that name their own (token, dim): a one-to-one format unpacks them back,
    and every code bit of the tile is used (the area sizes are exact)."""
    for rates, vr in ((np.array([4] * 3 + [3] * 5 + [2] * 9 + [1] * 47), 3), (np.full(64, 1), 1),
                      (np.full(64, 4), 4), (np.array([2] * 40 + [1] * 24), 2)):
        lay = O.make_layout(rates, vr, 0)
        rng = np.random.default_rng(int(rates.sum()) + vr)
        prates = lay.packed_rates()
        kc = rng.integers(0, 1 << prates, size=(64, 128))
        vc = rng.integers(0, 1 << vr, size=(64, 128))
        enc = {"k_codes": kc, "v_codes": vc, "k_norms": np.zeros((64, lay.n_kgroups)), "v_norm": np.zeros(64)}
        u = O.unpack(lay, O.pack(lay, enc, 64), 64)
        np.testing.assert_array_equal(u["k_codes"], kc)
        np.testing.assert_array_equal(u["v_codes"], vc)
        full = {"k_codes": (1 << prates)[None, :].repeat(64, 0) - 1, "v_codes": np.full((64, 128), (1 << vr) - 1),
                "k_norms": np.zeros((64, lay.n_kgroups)), "v_norm": np.zeros(64)}
        codes = O.pack(lay, full, 64)[:64 * (lay.k_record_bytes + lay.v_record_bytes)]
        assert np.all(codes == 255)


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(3)
    rates = _random_rates(rng)
    lay = O.make_layout(rates, 2, 11)
    n = 150
    k = rng.standard_normal((n, 128)) * 3
    v = rng.standard_normal((n, 128))
    enc = O.encode(lay, k, v)
    buf = O.pack(lay, enc, 192)
    assert buf.size == O.cache_bytes(lay, 1, 1, 192)
    u = O.unpack(lay, buf, n)
    np.testing.assert_array_equal(u["k_codes"], enc["k_codes"])
    np.testing.assert_array_equal(u["v_codes"], enc["v_codes"])
    np.testing.assert_array_equal(u["k_norms"], enc["k_norms"].astype(np.float32))
    np.testing.assert_array_equal(u["v_norm"], enc["v_norm"].astype(np.float32))


# ------------------------------------------------------------------ encode / decode
def test_codes_are_nearest_centroids():
    rng = np.random.default_rng(4)
    for b in (1, 2, 3, 4):
        lay = O.make_layout(np.full(64, b), b, 9)
        x = rng.standard_normal((40, 128))
        enc = O.encode(lay, x, x)
        y = math.sqrt(128) * (x @ lay.k_rot[0].T) / np.linalg.norm(x, axis=1, keepdims=True)
        c = lay.codebooks[b][0]
        nearest = np.argmin(np.abs(y[..., None] - c[None, None, :]), axis=-1)
        # packed order == group order for a single group: coordinates (0,64,1,65,...)
        y_packed = math.sqrt(128) * (x[:, lay.groups[0][1]] @ lay.k_rot[0].T) / np.linalg.norm(x, axis=1, keepdims=True)
        nearest_p = np.argmin(np.abs(y_packed[..., None] - c[None, None, :]), axis=-1)
        np.testing.assert_array_equal(enc["k_codes"], nearest_p)
        assert nearest.shape == nearest_p.shape


def test_zero_vector_and_threshold_ties():
    lay = O.make_layout(np.full(64, 2), 2, 1)
    enc = O.encode(lay, np.zeros((2, 128)), np.zeros((2, 128)))
    assert np.all(enc["k_codes"] == 2) and np.all(enc["v_codes"] == 2)
    kh, vh = O.reconstruct(lay, enc["k_codes"], enc["k_norms"], enc["v_codes"], enc["v_norm"])
    assert np.all(kh == 0) and np.all(vh == 0)


def test_reconstruction_error_matches_lloyd_max_distortion():
    # After a Haar rotation of a 128-dim vector the coordinates are close to N(0,1)
    # (scaled), so the relative squared error approaches D(b). A transposed rotation
    # or a missing sqrt(d) would give an O(1) error instead.
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3000, 128))
    for b in (1, 2, 3, 4):
        lay = O.make_layout(np.full(64, b), b, 21)
        enc = O.encode(lay, x, x)
        kh, vh = O.reconstruct(lay, enc["k_codes"], enc["k_norms"], enc["v_codes"], enc["v_norm"])
        D = O.lloyd_max(b)[2]
        for xh in (kh, vh):
            rel = np.sum((xh - x) ** 2) / np.sum(x ** 2)
            assert rel == pytest.approx(D, rel=0.05)


def test_mixed_rate_reconstruction_error_by_group():
    rng = np.random.default_rng(6)
    rates = np.array([1] * 16 + [2] * 16 + [3] * 16 + [4] * 16)
    lay = O.make_layout(rates, 2, 8)
    x = rng.standard_normal((4000, 128))
    enc = O.encode(lay, x, x)
    kh, _ = O.reconstruct(lay, enc["k_codes"], enc["k_norms"], enc["v_codes"], enc["v_norm"])
    for r, coords in lay.groups:
        rel = np.sum((kh[:, coords] - x[:, coords]) ** 2) / np.sum(x[:, coords] ** 2)
        # 32-dim groups: the rotated coordinates are only roughly Gaussian; allow 15%
        assert rel == pytest.approx(O.lloyd_max(r)[2], rel=0.15)


# ------------------------------------------------------------------ attention
def test_attention_special_cases():
    rng = np.random.default_rng(7)
    v = rng.standard_normal((9, 128))
    k = rng.standard_normal((9, 128))
    q = rng.standard_normal((3, 128))
    np.testing.assert_allclose(O.attention(q, k[:1], v[:1], 0.1), np.repeat(v[:1], 3, 0), rtol=1e-15)
    np.testing.assert_allclose(O.attention(np.zeros((2, 128)), k, v, 0.1), np.repeat(v.mean(0, keepdims=True), 2, 0), rtol=1e-13)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, :, None, :], torch.tensor(k)[None, None].expand(1, 3, 9, 128),
        torch.tensor(v)[None, None].expand(1, 3, 9, 128), scale=0.1)[0, :, 0].numpy()
    np.testing.assert_allclose(O.attention(q, k, v, 0.1), ref, rtol=1e-12, atol=1e-12)
    assert np.all(O.attention(q, k[:0], v[:0], 0.1) == 0)


def test_decode_attention_equals_rotated_space_form():
    """Scores and values computed from codes in the rotated space (q' = R q per group,
    centroid lookups, inverse rotation of the value sum) equal the original-space result."""
    rng = np.random.default_rng(8)
    rates = _random_rates(rng)
    lay = O.make_layout(rates, 3, 4)
    n, G = 70, 4
    k = rng.standard_normal((n, 128)) * 2
    v = rng.standard_normal((n, 128))
    q = rng.standard_normal((G, 128))
    enc = O.encode(lay, k, v)
    buf = O.pack(lay, enc, 128)
    out = O.decode_attention(lay, q, buf, n, 0.088)
    u = O.unpack(lay, buf, n)
    s = np.zeros((G, n))
    col = 0
    for gi, ((r, coords), rot) in enumerate(zip(lay.groups, lay.k_rot)):
        d = len(coords)
        qp = q[:, coords] @ rot.T
        cv = lay.codebooks[r][0][u["k_codes"][:, col:col + d]]
        s += (qp @ cv.T) * (u["k_norms"][:, gi] / math.sqrt(d))[None, :]
        col += d
    s *= 0.088
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    cv = lay.codebooks[3][0][u["v_codes"]] * (u["v_norm"] / math.sqrt(128))[:, None]
    out_rot = (p @ cv) @ lay.v_rot
    np.testing.assert_allclose(out, out_rot, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ scores and logit error
def test_scores_are_the_logits_of_the_attention():
    """softmax(scores) @ v_hat reproduces the oracle attention: scores are its logits."""
    rng = np.random.default_rng(21)
    lay = O.make_layout(_random_rates(rng), 3, 4)
    k = rng.standard_normal((90, 128)) * 2
    v = rng.standard_normal((90, 128))
    q = rng.standard_normal((3, 128))
    enc = O.encode(lay, k, v)
    buf = O.pack(lay, enc, 128)
    s = O.decode_scores(lay, q, buf, 90, 0.1)
    assert s.shape == (3, 90)
    u = O.unpack(lay, buf, 90)
    _, vh = O.reconstruct(lay, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(p @ vh, O.decode_attention(lay, q, buf, 90, 0.1), rtol=1e-12, atol=1e-12)


def test_logit_mae_matches_the_distortion_closed_form():
    """For Gaussian keys and queries (independent of the rotation), E|q . (k_hat - k)|^2 =
    |q|^2 |k|^2 D(b) / d per coordinate sum, so the mean absolute error of a uniform b-bit
    layout is close to sqrt(2/pi) * sqrt(sum_i q_i^2 E[(k_hat - k)_i^2]) and shrinks with
    b as sqrt(D(b))."""
    rng = np.random.default_rng(22)
    q = rng.standard_normal((4, 128))
    k = rng.standard_normal((3000, 128))
    maes = []
    for b in (1, 2, 3, 4):
        lay = O.make_layout(np.full(64, b), 2, 1)
        maes.append(O.logit_mae(lay, q, k, 1.0))
    D = O.lloyd_max_mse_table()
    for b, m in zip((1, 2, 3, 4), maes):
        # k_hat - k has per-coordinate variance |k|^2 D(b) / d ~ D(b), isotropic after R^T
        want = math.sqrt(2 / math.pi) * np.mean(np.linalg.norm(q, axis=1)) * math.sqrt(D[b])
        assert abs(m / want - 1) < 0.08, (b, m, want)
    assert maes == sorted(maes, reverse=True)


def test_block_allocation_beats_uniform_rates_on_skewed_blocks():
    """The abstract's claim in its simplest form: with energy concentrated in a few RoPE
    blocks, the largest-marginal-gain allocation at the same bit budget gives a lower
    K-only logit error than uniform rates."""
    m = synth.make_layer_model(4, 1, 7)
    q_cal, k_cal = synth.make_calibration(m, 256, 8, 5e5)
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * 2)
    k = synth.key_slice(m, 0, 0, 600, 0, 9, 5e5).double().numpy()
    q = torch.stack([synth.query_slice(m, 0, i, 1, 599, 9, 5e5)[0] for i in range(4)]).double().numpy()
    gtq = O.logit_mae(O.make_layout(rates, 2, 3), q, k, 1 / math.sqrt(128))
    uni = O.logit_mae(O.make_layout(np.full(64, 2), 2, 3), q, k, 1 / math.sqrt(128))
    assert gtq < 0.8 * uni, (gtq, uni)


# ---------------------------------------------------------------- layout variants ----
def test_norm_correction_restores_the_input_norm():
    """NC ("TurboQuant" page, vLLM box "NC"): the decoded group vectors have the norms of the
    inputs, for every group and for V; the codes are those of the plain layout."""
    rates = np.array([3] * 16 + [2] * 24 + [1] * 24)
    plain = O.make_layout(rates, 2, 11)
    nc = O.make_layout(rates, 2, 11, norm_correct=True)
    rng = np.random.default_rng(4)
    k = rng.standard_normal((40, 128)) * rng.uniform(0.1, 10, 128)
    v = rng.standard_normal((40, 128))
    k[3] = 0.0                                   # a zero vector keeps a zero norm
    e0, e1 = O.encode(plain, k, v), O.encode(nc, k, v)
    np.testing.assert_array_equal(e0["k_codes"], e1["k_codes"])
    np.testing.assert_array_equal(e0["v_codes"], e1["v_codes"])
    kh, vh = O.reconstruct(nc, e1["k_codes"], e1["k_norms"], e1["v_codes"], e1["v_norm"])
    for r, coords in nc.groups:
        np.testing.assert_allclose(np.linalg.norm(kh[:, coords], axis=1), np.linalg.norm(k[:, coords], axis=1),
                                   rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(np.linalg.norm(vh, axis=1), np.linalg.norm(v, axis=1), rtol=1e-12)
    # without NC the decoded norms are off by the centroid energy (the distortion NC removes)
    kh0, _ = O.reconstruct(plain, e0["k_codes"], e0["k_norms"], e0["v_codes"], e0["v_norm"])
    r1 = nc.groups[-1][1]
    assert np.max(np.abs(np.linalg.norm(kh0[:, r1], axis=1) / np.maximum(np.linalg.norm(k[:, r1], axis=1), 1e-300)
                         - 1)[np.linalg.norm(k[:, r1], axis=1) > 0]) > 1e-3


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_norm_correction_factor_matches_the_centroid_energy(bits):
    """Centroid condition of a Lloyd-Max quantiser: E[Q(y)^2] = E[y^2] - D(b) = 1 - D(b) for
    y ~ N(0,1). NC stores |x| sqrt(d) / |c|, so the mean of (|x| / stored)^2 = |c|^2 / d
    over many vectors approaches 1 - D(b) (a rotated unit vector times sqrt(d) has
    near-Gaussian coordinates; the sphere's correction is O(1/d))."""
    lay = O.make_layout(np.full(64, bits), bits, 3, norm_correct=True)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((3000, 128))
    enc = O.encode(lay, x, x)
    ratio2 = (np.linalg.norm(x, axis=1) / enc["v_norm"]) ** 2
    d_b = O.lloyd_max_mse_table()[bits]
    assert abs(ratio2.mean() - (1 - d_b)) < 0.01 * (1 - d_b)
    kr = (np.linalg.norm(x, axis=1) / enc["k_norms"][:, 0]) ** 2
    assert abs(kr.mean() - (1 - d_b)) < 0.01 * (1 - d_b)


def test_fp16_norms_are_where_the_format_says():
    """One rate-2 group and V2: K area 64 x 32 bytes, V area 64 x 32, then the K norms fp16
    [1 group][64 entries] at 4096 and the V norms fp16 [64] at 4224; 68 bytes per token.
    Token t = g + 8 m sits at entry 8 g + m: tokens 0, 1, 2, 3 at entries 0, 8, 16, 24.
    fp16 of 3.0 is 0x4200, of 1.5 0x3e00; 1e6 saturates at 65504 (0x7bff); 0.1 rounds to
    nearest (0x2e66)."""
    lay = O.make_layout(np.full(64, 2), 2, 0, norm_fp16=True)
    assert lay.bytes_per_token == 32 + 32 + 2 * 2 and lay.tile_bytes == 64 * 68
    n = 4
    enc = {"k_codes": np.zeros((n, 128), dtype=np.int64), "v_codes": np.zeros((n, 128), dtype=np.int64),
           "k_norms": np.array([[3.0], [1e6], [0.1], [0.0]]), "v_norm": np.array([0.0, 1.5, 0.0, 65519.0])}
    buf = O.pack(lay, enc, 64)
    assert buf.size == 64 * 68
    assert buf[4096:4098].tolist() == [0x00, 0x42] and buf[4112:4114].tolist() == [0xff, 0x7b]
    assert buf[4128:4130].tolist() == [0x66, 0x2e] and buf[4144:4146].tolist() == [0, 0]
    assert buf[4240:4242].tolist() == [0x00, 0x3e] and buf[4272:4274].tolist() == [0xff, 0x7b]
    assert int(np.count_nonzero(buf)) == (1 + 2 + 2) + (1 + 2)   # nonzero bytes of the norms; codes are 0
    u = O.unpack(lay, buf, n)
    assert u["k_norms"][:, 0].tolist() == [3.0, 65504.0, float(np.float16(0.1)), 0.0]
    assert u["v_norm"].tolist() == [0.0, 1.5, 0.0, 65504.0]


def test_resident_bytes_with_fp16_norms():
    """Bytes per (token, KV head) = 128 b_K / 8 + 128 b_V / 8 + 2 (n_gK + 1) with fp16
    norms: K3V3 in one group 48 + 48 + 4 = 100 (5.12x smaller than a 512-byte fp16 K+V
    record); K2V2 over rates 1-4 (four groups) 32 + 32 + 10 = 74 (6.92x)."""
    k3 = O.make_layout(np.full(64, 3), 3, 0, norm_fp16=True)
    assert k3.bytes_per_token == 100 and O.cache_bytes(k3, 2, 4, 65) == 2 * 4 * 2 * 64 * 100
    mixed = O.make_layout(np.array([4] * 8 + [3] * 8 + [2] * 24 + [1] * 24), 2, 0, norm_fp16=True)
    assert mixed.n_kgroups == 4 and mixed.k_record_bytes == 32 and mixed.bytes_per_token == 74
    assert O.make_layout(np.full(64, 3), 3, 0).bytes_per_token == 104           # fp32 norms: 48 + 48 + 8


# ------------------------------------------------------------ multi-token queries ----
def _packed_slice(seed, n, rates=None, v_rate=2):
    rng = np.random.default_rng(seed)
    lay = O.make_layout(np.full(64, 2) if rates is None else rates, v_rate, seed)
    k = rng.standard_normal((n, 128)) * rng.uniform(0.2, 4, 128)
    v = rng.standard_normal((n, 128))
    enc = O.encode(lay, k, v)
    return lay, enc, O.pack(lay, enc, 64 * -(-n // 64))


def test_multi_token_attention_matches_masked_sdpa():
    """Query j of n_q new tokens sits at position L - n_q + j: the result equals PyTorch's
    scaled_dot_product_attention over the decoded cache with the explicit mask
    key <= L - n_q + j (a library routine, not this oracle's attention)."""
    lay, enc, buf = _packed_slice(3, 150)
    L, n_q, G = 150, 5, 3
    q = np.random.default_rng(4).standard_normal((n_q, G, 128))
    got = O.decode_attention_multi(lay, q, buf, L, 0.09)
    kh, vh = O.reconstruct(lay, enc["k_codes"], O.stored_norms(lay, enc["k_norms"]).astype(np.float64),
                           enc["v_codes"], O.stored_norms(lay, enc["v_norm"]).astype(np.float64))
    mask = torch.arange(L)[None, :] <= (L - n_q + torch.arange(n_q))[:, None]       # [n_q, L]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q).permute(1, 0, 2)[None], torch.tensor(kh)[None, None].expand(1, G, L, 128),
        torch.tensor(vh)[None, None].expand(1, G, L, 128), attn_mask=mask[None, None], scale=0.09)
    np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)


def test_multi_token_attention_is_causal_and_reduces_to_one_query():
    lay, enc, buf = _packed_slice(5, 130)
    L, n_q = 130, 4
    q = np.random.default_rng(6).standard_normal((n_q, 2, 128))
    out = O.decode_attention_multi(lay, q, buf, L, 0.1)
    # the last query sees the whole cache: single-token decode attention
    np.testing.assert_allclose(out[-1], O.decode_attention(lay, q[-1], buf, L, 0.1), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.decode_attention_multi(lay, q[-1:], buf, L, 0.1)[0], out[-1], rtol=1e-13)
    # changing the keys and values after query j's position leaves query j alone, and
    # changes the later queries
    enc2 = {kk: vv.copy() for kk, vv in enc.items()}
    enc2["k_codes"][L - 2:] = (enc2["k_codes"][L - 2:] + 1) % 4
    enc2["v_norm"][L - 2:] *= 3.0
    out2 = O.decode_attention_multi(lay, q, O.pack(lay, enc2, 192), L, 0.1)
    np.testing.assert_array_equal(out2[:2], out[:2])
    assert np.all(np.abs(out2[2:] - out[2:]).max(axis=(1, 2)) > 1e-6)


# -------------------------------------------------------------------- rate-0 blocks ----
def test_greedy_with_rate_zero_equals_exhaustive_optimum():
    """With D(0) = 1 (an uncoded N(0,1) coordinate decodes to 0) the gains still diminish
    (1 - D(1) > D(1) - D(2) > ...), so largest-marginal-gain allocation from rate 0 is the
    exhaustive optimum of the proxy [BGTQ sentence 4]."""
    D = O.lloyd_max_mse_table()
    # D(0) is the MSE of decoding an N(0,1) coordinate to 0 (Monte Carlo, 4e5 draws)
    x = np.random.default_rng(21).standard_normal(400_000)
    assert abs(np.mean((x - 0.0) ** 2) - D[0]) < 0.01
    assert D[0] - D[1] > D[1] - D[2] > D[2] - D[3] > D[3] - D[4] > 0
    rng = np.random.default_rng(2)
    cases = 0
    for n in (1, 2, 3, 4, 5):
        s = rng.exponential(size=n) * rng.choice([1, 10, 100], size=n)
        for budget in range(0, 4 * n + 1):
            g = O.greedy_rates(s, D, 0, 4, budget)
            best, args = O.brute_force_rates(s, D, 0, 4, budget)
            assert O.proxy_objective(s, g, D) == pytest.approx(best, rel=1e-12, abs=1e-15)
            if len(args) == 1:
                assert tuple(g) == args[0]
            cases += 1
    assert cases > 40


def test_rate_zero_blocks_are_not_stored_and_decode_to_zero():
    """A rate-0 block is in no group: its two coordinates take no code bits, the group
    norms cover the coded coordinates only, and they decode to exactly 0; the coded
    groups keep the Lloyd-Max distortion of their rate."""
    rates = np.array([0] * 8 + [1] * 16 + [2] * 16 + [3] * 16 + [4] * 8)    # sum 128: K2
    lay = O.make_layout(rates, 2, 9)
    assert [r for r, _ in lay.groups] == [4, 3, 2, 1] and lay.n_packed == 128 - 16
    zero = np.r_[0:8, 64:72]
    assert not set(zero) & set(np.concatenate([c for _, c in lay.groups]))
    assert lay.k_record_bytes == (16 * 2 * 1 + 16 * 2 * 2 + 16 * 2 * 3 + 8 * 2 * 4) // 8 == 32
    rng = np.random.default_rng(10)
    x = rng.standard_normal((3000, 128))
    enc = O.encode(lay, x, x)
    assert enc["k_codes"].shape == (3000, 112)
    c1 = lay.groups[-1][1]
    np.testing.assert_allclose(enc["k_norms"][:, -1], np.linalg.norm(x[:, c1], axis=1), rtol=1e-14)
    kh, _ = O.reconstruct(lay, enc["k_codes"], enc["k_norms"], enc["v_codes"], enc["v_norm"])
    assert np.all(kh[:, zero] == 0.0)
    for r, coords in lay.groups:
        rel = np.sum((kh[:, coords] - x[:, coords]) ** 2) / np.sum(x[:, coords] ** 2)
        assert rel == pytest.approx(O.lloyd_max(r)[2], rel=0.15)
    buf = O.pack(lay, enc, 3008)
    u = O.unpack(lay, buf, 3000)
    np.testing.assert_array_equal(u["k_codes"], enc["k_codes"])
    with pytest.raises(ValueError):
        O.make_layout(np.zeros(64, dtype=int), 2, 0)


# ------------------------------------------------------------ per-KV-head allocation ----
def test_per_head_energy_sums_to_the_layer_score_and_follows_each_head():
    """The per-KV-head scores add up to the layer score, and a head whose keys (and only
    its keys) are scaled by c in block j has its own score for j multiplied by c^2 while
    the other heads' scores stay put."""
    rng = np.random.default_rng(13)
    q = rng.standard_normal((40, 8, 128))
    k = rng.standard_normal((30, 4, 128))
    per = O.block_energy_heads(q, k)
    np.testing.assert_allclose(per.sum(axis=0), O.block_energy(q, k), rtol=1e-13)
    k2 = k.copy()
    k2[:, 2, [5, 69]] *= 3.0
    per2 = O.block_energy_heads(q, k2)
    assert per2[2, 5] == pytest.approx(9.0 * per[2, 5], rel=1e-12)
    np.testing.assert_allclose(np.delete(per2, 2, axis=0), np.delete(per, 2, axis=0), rtol=0, atol=0)
    np.testing.assert_allclose(np.delete(per2[2], 5), np.delete(per[2], 5), rtol=0, atol=0)


def test_random_layouts_with_every_option_pack_one_to_one():
    """Random rate vectors over 0..4 (some blocks uncoded), every value rate and both norm
    types: codes and norms round-trip, and codes at their largest value fill the code
    areas exactly (no bit unused, none shared)."""
    rng = np.random.default_rng(31)
    done = 0
    while done < 12:
        rates = rng.integers(0, 5, size=64)
        if rates.sum() % 4 or rates.max() == 0:
            continue
        vr = int(rng.integers(1, 5))
        fp16 = bool(done % 2)
        lay = O.make_layout(rates, vr, done, norm_fp16=fp16)
        pr = lay.packed_rates()
        n = 100
        kc = rng.integers(0, 1 << pr, size=(n, lay.n_packed))
        vc = rng.integers(0, 1 << vr, size=(n, 128))
        kn = rng.uniform(0, 50, size=(n, lay.n_kgroups))
        vn = rng.uniform(0, 50, size=n)
        buf = O.pack(lay, {"k_codes": kc, "v_codes": vc, "k_norms": kn, "v_norm": vn}, 128)
        assert buf.size == 2 * lay.tile_bytes
        u = O.unpack(lay, buf, n)
        np.testing.assert_array_equal(u["k_codes"], kc)
        np.testing.assert_array_equal(u["v_codes"], vc)
        np.testing.assert_array_equal(u["k_norms"], O.stored_norms(lay, kn).astype(np.float64))
        np.testing.assert_array_equal(u["v_norm"], O.stored_norms(lay, vn).astype(np.float64))
        full = {"k_codes": np.repeat((1 << pr)[None, :] - 1, 128, 0), "v_codes": np.full((128, 128), (1 << vr) - 1),
                "k_norms": np.zeros((128, lay.n_kgroups)), "v_norm": np.zeros(128)}
        tiles = O.pack(lay, full, 128).reshape(2, lay.tile_bytes)
        assert np.all(tiles[:, :64 * (lay.k_record_bytes + lay.v_record_bytes)] == 255)
        done += 1


# ------------------------------------------------------------------ near-threshold mask
def _unit_input_for(y, rot, scale):
    """x with sqrt(d) R x / |x| = y (|y|^2 = d): x = scale R^T y / sqrt(d), |x| = scale."""
    d = len(y)
    return scale * (rot.T @ y) / math.sqrt(d)


@pytest.mark.parametrize("rate", [1, 2, 3, 4])
def test_encode_margin_is_the_distance_to_the_nearest_threshold(rate):
    # Rotated coordinates placed at known offsets from known thresholds: the margin the
    # encoder returns is that offset (an absolute distance, to the nearest threshold, not
    # to a centroid), and the code falls on the side of the threshold the offset says.
    d = 64
    rot = O.haar_rotation(5, rate, d)
    _, t, _ = O.lloyd_max(rate)
    k_mid = len(t) // 2                          # the middle threshold, exactly 0
    k_out = len(t) - 1                           # the largest threshold
    offsets = [(k_out, 0.5e-6), (k_out, -0.5e-6), (k_out, 2e-6), (k_out, -2e-6), (k_mid, 3e-6), (0, -4e-6)]
    y = np.zeros(d)
    for i, (k, off) in enumerate(offsets):
        y[i] = t[k] + off
    # fill the rest with values midway between thresholds (far from every threshold) and
    # close the norm |y|^2 = d with the last coordinate
    inner = 0.5 * (t[k_mid] + t[k_mid + 1]) if len(t) > 1 else 0.8
    for i in range(len(offsets), d - 1):
        y[i] = inner if i % 2 else -inner
    rest = d - np.sum(y[:-1] ** 2)
    assert rest > 0
    y[-1] = math.sqrt(rest)
    x = _unit_input_for(y, rot, 3.7)
    codes, norms, margin = OM._tq_encode_group(x[None, :], rot, t)
    np.testing.assert_allclose(norms, [3.7], rtol=1e-14)
    for i, (k, off) in enumerate(offsets):
        assert abs(margin[0, i] - abs(off)) < 1e-12, (i, margin[0, i], off)
        assert codes[0, i] == (k + 1 if off > 0 else k)
    last = np.min(np.abs(y[-1] - t))
    assert abs(margin[0, -1] - last) < 1e-12
    # a coordinate exactly on the middle threshold codes up and has margin 0
    y0 = np.zeros(d)
    y0[0] = 0.0
    y0[1:] = math.sqrt(d / (d - 1))
    codes0, _, m0 = OM._tq_encode_group(_unit_input_for(y0, rot, 1.0)[None, :], rot, t)
    assert m0[0, 0] < 1e-14
    assert codes0[0, 0] in (k_mid, k_mid + 1)


def test_boundary_mask_covers_exactly_the_near_threshold_codes():
    # Margins set by hand on a mixed-rate layout: the mask must hold all of a coordinate's
    # code bits (1 << rate) - 1 exactly where the margin is below eps (an absolute eps,
    # compared with <), nothing elsewhere, and count those coordinates.
    rates = np.array([4] * 3 + [3] * 4 + [2] * 19 + [1] * 38)
    assert (2 * rates.sum()) % 8 == 0
    lay = O.make_layout(rates, 3, 2)
    n, eps = 70, 1e-6
    rng = np.random.default_rng(3)
    km = rng.uniform(0.01, 1.0, (n, lay.n_packed))
    vm = rng.uniform(0.01, 1.0, (n, 128))
    near_k = [(0, 0), (5, 7), (69, 127), (64, 30), (33, 12)]
    for i, j in near_k:
        km[i, j] = 0.5e-6
    km[1, 1] = 2e-6                       # outside (absolute), inside for a relative eps on |y| ~ 2.4
    km[2, 2] = eps                        # not below eps
    near_v = [(3, 4), (63, 64)]
    for i, j in near_v:
        vm[i, j] = 0.0
    enc = {"k_codes": np.zeros((n, lay.n_packed), dtype=np.int64), "v_codes": np.zeros((n, 128), dtype=np.int64),
           "k_norms": np.ones((n, lay.n_kgroups)), "v_norm": np.ones(n), "k_margin": km, "v_margin": vm}
    cap = 128
    mask, count = O.boundary_mask(lay, enc, cap, eps)
    assert count == len(near_k) + len(near_v)
    u = O.unpack(lay, mask, n)
    want_k = np.zeros((n, lay.n_packed), dtype=np.int64)
    pr = lay.packed_rates()
    for i, j in near_k:
        want_k[i, j] = (1 << pr[j]) - 1
    want_v = np.zeros((n, 128), dtype=np.int64)
    for i, j in near_v:
        want_v[i, j] = (1 << 3) - 1
    np.testing.assert_array_equal(u["k_codes"], want_k)
    np.testing.assert_array_equal(u["v_codes"], want_v)
    # the mask touches no norm byte and no token slot past n
    full = O.unpack(lay, mask, cap)
    assert not full["k_codes"][n:].any() and not full["v_codes"][n:].any()
    assert not full["k_norms"].any() and not full["v_norm"].any()
    # set bits: exactly sum of the masked coordinates' rates
    assert int(np.unpackbits(mask).sum()) == sum(pr[j] for _, j in near_k) + 3 * len(near_v)


# ------------------------------------------------------------------ split attention
def test_merged_partials_equal_attention_over_the_union():
    # The log-sum-exp merge of partial attentions over disjoint token ranges is the
    # softmax attention over all tokens: random split points (empty parts included) and
    # peaked logits (large scale), against attention() computed directly.
    rng = np.random.default_rng(11)
    n, G = 300, 4
    k = rng.standard_normal((n, 128)) * 3
    v = rng.standard_normal((n, 128))
    q = rng.standard_normal((G, 128)) * 2
    full = O.attention(q, k, v, 0.3)
    for cuts in ([0, 300], [0, 0, 300], [0, 1, 299, 300], [0, 64, 64, 200, 300], [0, 150, 300, 300]):
        parts = [O.partial_attention(q, k[a:b], v[a:b], 0.3) for a, b in zip(cuts[:-1], cuts[1:])]
        np.testing.assert_allclose(O.merge_partials(parts), full, rtol=1e-12, atol=1e-12)
    # a merge that dropped the l weights, or kept per-part maxima, would not match
    m, l, o = O.partial_attention(q, k[:10], v[:10], 0.3)
    assert np.all(l >= 1.0) and np.allclose(o, O.attention(q, k[:10], v[:10], 0.3))
    empty = O.partial_attention(q, k[:0], v[:0], 0.3)
    assert np.all(np.isneginf(empty[0])) and not empty[1].any() and not empty[2].any()
    np.testing.assert_array_equal(O.merge_partials([empty, empty]), np.zeros((G, 128)))
