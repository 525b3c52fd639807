"""The C-ABI library's host-side planning against the oracle (no GPU needed), and the
library's exported symbols against include/bgtq.h."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "bgtq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bgtq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(B.EXPORTED) == names


def test_lloyd_max_matches_oracle(lib):
    for b in (1, 2, 3, 4):
        c, t, m = B.lloyd_max(b)
        oc, ot, om = O.lloyd_max(b)
        np.testing.assert_allclose(c, oc, rtol=0, atol=1e-13)
        np.testing.assert_allclose(t, ot, rtol=0, atol=1e-13)
        assert m == pytest.approx(om, rel=1e-12)
        assert t[len(t) // 2] == 0.0
    with pytest.raises(B.BgtqError):
        B.lloyd_max(5)


def _k2_rates():
    return np.array([1] * 22 + [2] * 22 + [3] * 18 + [4] * 2)


@pytest.mark.parametrize("seed", [0, 12345, 2**40 + 7])
def test_layout_matches_oracle(lib, seed):
    rng = np.random.default_rng(seed % 1000)
    rates = rng.permutation(_k2_rates())
    lay = B.Layout(rates, 3, seed)
    ref = O.make_layout(rates, 3, seed)
    assert lay.n_kgroups == ref.n_kgroups
    assert lay.bytes_per_token == ref.bytes_per_token and lay.tile_bytes == ref.tile_bytes
    assert lay.info.k_record_bytes == ref.k_record_bytes
    np.testing.assert_array_equal(lay.coords(), ref.packed_coords())
    for g, (r, coords) in enumerate(ref.groups):
        assert lay.info.group_rate[g] == r and lay.info.group_dim[g] == len(coords)
        np.testing.assert_allclose(lay.rotation(g), ref.k_rot[g], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lay.rotation(lay.n_kgroups), ref.v_rot, rtol=0, atol=1e-12)
    for tokens in (1, 64, 65, 32768):
        assert lay.cache_bytes(2, 8, tokens) == O.cache_bytes(ref, 2, 8, tokens)


def test_rotation_preserves_norms_to_1e6(lib):
    lay = B.Layout(_k2_rates(), 2, 7)
    x = np.random.default_rng(0).standard_normal((100, 128))
    for g in range(lay.n_kgroups + 1):
        r = lay.rotation(g)
        r32 = r.astype(np.float32).astype(np.float64)   # the decode kernels use the fp32 copy
        d = r.shape[0]
        for rr in (r, r32):
            ratio = np.linalg.norm(x[:, :d] @ rr.T, axis=1) / np.linalg.norm(x[:, :d], axis=1)
            assert np.max(np.abs(ratio - 1)) < 1e-6
        assert np.max(np.abs(r32 @ r32.T - np.eye(d))) < 1e-6


def test_layout_rejects_bad_rates(lib):
    with pytest.raises(B.BgtqError):
        B.Layout(np.array([1] * 63 + [2]), 2, 0)          # 130 bits
    with pytest.raises(B.BgtqError):
        B.Layout(np.array([0] * 64), 2, 0)
    with pytest.raises(B.BgtqError):
        B.Layout(np.full(64, 2), 5, 0)


def test_block_energy_matches_oracle(lib):
    m = synth.make_layer_model(32, 8, seed=1)
    q, k = synth.make_calibration(m, 256, 2, 5e5)
    s_lib = B.block_energy(q.numpy(), k.numpy())
    s_ref = O.block_energy(q.numpy().astype(np.float64), k.numpy().astype(np.float64))
    np.testing.assert_allclose(s_lib, s_ref, rtol=1e-12)


def test_allocation_matches_oracle_greedy(lib):
    rng = np.random.default_rng(2)
    D = O.lloyd_max_mse_table()
    for trial in range(20):
        s = rng.exponential(size=64) * rng.choice([0.01, 1, 100], size=64)
        if trial % 5 == 0:
            s[:20] = 3.0                                  # ties
        for avg in (1, 2, 3, 4):
            want = O.greedy_rates(s, D, 1, 4, 64 * avg)
            got = B.allocate_rates(s, 1, 4, 64 * avg)
            np.testing.assert_array_equal(got, want)
        budget = int(rng.integers(64, 257))
        np.testing.assert_array_equal(B.allocate_rates(s, 1, 4, budget), O.greedy_rates(s, D, 1, 4, budget))


def test_allocation_custom_distortion_and_errors(lib):
    s = np.array([5.0, 1.0, 3.0, 0.5])
    D = {1: 1.0, 2: 0.5, 3: 0.3, 4: 0.2}
    np.testing.assert_array_equal(B.allocate_rates(s, 1, 4, 9, D), O.greedy_rates(s, D, 1, 4, 9))
    with pytest.raises(B.BgtqError) as e:
        B.allocate_rates(s, 1, 4, 17)
    assert e.value.status == B.ERR_INFEASIBLE
    with pytest.raises(B.BgtqError) as e:
        B.allocate_rates(s, 2, 1, 6)
    assert e.value.status == B.ERR_INVALID


def test_host_validation_without_device(lib):
    lay = B.Layout(np.full(64, 2), 2, 0)
    assert lib.bgtq_block_energy(None, 1, 1, None, 1, 1, None) == B.ERR_INVALID
    assert lib.bgtq_cache_bytes(None, 1, 1, 1) == -1
    assert lib.bgtq_layout_rotation(lay.handle, 9, None, 0) == B.ERR_INVALID
    # device calls before an upload report DEVICE, never crash
    f = C.c_uint(0)
    assert lib.bgtq_device_status(lay.handle, C.byref(f), 0) == B.ERR_DEVICE
    assert lib.bgtq_encode_append(lay.handle, None, None, 0, 1, 1, 1, None, None, 64, None) == B.ERR_DEVICE
    assert lib.bgtq_decode_attention(lay.handle, None, 0, 1, 1, 1, None, None, 64, 64, 0.1, None, None, 0,
                                     None) == B.ERR_DEVICE
    if not torch.cuda.is_available():
        assert lib.bgtq_layout_upload(lay.handle, 0) in (B.ERR_CUDA, B.ERR_INVALID)


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_layout_options_match_oracle_bytes(lib, flags):
    """bgtq_layout_create_ex: the norm options change the bytes per token as the oracle's
    layout does (2-byte norms with BGTQ_LAYOUT_NORM_FP16); an unknown flag is refused."""
    rates = np.array([4] * 8 + [3] * 8 + [2] * 24 + [1] * 24)
    lay = B.Layout(rates, 3, 9, bool(flags & 1), bool(flags & 2))
    olay = O.make_layout(rates, 3, 9, bool(flags & 1), bool(flags & 2))
    assert lay.info.flags == flags
    assert lay.info.bytes_per_token == olay.bytes_per_token
    assert lay.info.tile_bytes == olay.tile_bytes
    assert lay.cache_bytes(2, 8, 4097) == O.cache_bytes(olay, 2, 8, 4097)
    r = np.ascontiguousarray(rates, dtype=np.int32)
    h = C.c_void_p()
    assert lib.bgtq_layout_create_ex(r.ctypes.data_as(C.c_void_p), 3, 9, 4, C.byref(h)) == B.ERR_INVALID
    assert not h.value


def test_rate_zero_layout_and_allocation_match_oracle(lib):
    """Rate-0 blocks: the allocation from rate 0 equals the oracle's greedy (D(0) = 1), the
    layout stores 128 - 2 x (rate-0 blocks) key dimensions in the oracle's byte count, and
    an all-zero rate vector is refused."""
    rng = np.random.default_rng(12)
    s = rng.exponential(size=64) * rng.choice([0.01, 1, 100], size=64)
    for bits in (1, 2, 3):
        got = B.allocate_rates(s, 0, 4, 64 * bits)
        want = O.greedy_rates(s, O.lloyd_max_mse_table(), 0, 4, 64 * bits)
        np.testing.assert_array_equal(got, want)
        assert (got == 0).any()
        lay, olay = B.Layout(got, 2, 5), O.make_layout(got, 2, 5)
        assert lay.info.n_packed == olay.n_packed == 128 - 2 * int((got == 0).sum())
        assert lay.info.bytes_per_token == olay.bytes_per_token
        assert lay.info.n_kgroups == olay.n_kgroups
        coords = np.zeros(128, dtype=np.int32)
        assert lib.bgtq_layout_coords(lay.handle, coords.ctypes.data_as(C.c_void_p)) == B.OK
        np.testing.assert_array_equal(coords[:olay.n_packed], olay.packed_coords())
    h = C.c_void_p()
    zero = np.zeros(64, dtype=np.int32)
    assert lib.bgtq_layout_create(zero.ctypes.data_as(C.c_void_p), 2, 0, C.byref(h)) == B.ERR_INVALID


def test_per_head_energy_matches_oracle_and_sums_to_layer_score(lib):
    m = synth.make_layer_model(16, 4, 3)
    q_cal, k_cal = synth.make_calibration(m, 64, 4, 5e5)
    per = B.block_energy_heads(q_cal.numpy(), k_cal.numpy())
    np.testing.assert_allclose(per, O.block_energy_heads(q_cal.double().numpy(), k_cal.double().numpy()),
                               rtol=1e-12)
    np.testing.assert_allclose(per.sum(axis=0), B.block_energy(q_cal.numpy(), k_cal.numpy()), rtol=1e-12)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2)
    assert rates.shape == (4, 64) and np.all(rates.sum(axis=1) == 128)
    assert len({tuple(r) for r in rates}) > 1            # the heads' allocations differ


def test_abi_version_and_info_size_agree_with_the_binding(lib):
    """The binding's bgtq_layout_info mirrors the header's (the library fills every field)."""
    assert lib.bgtq_version() == 200
    lay = B.Layout(np.full(64, 2), 2, 0)
    assert lay.info.n_packed == 128 and lay.info.norm_bytes == 4 and lay.info.flags == 0
    assert lay.info.tile_tokens == 64 and lay.info.head_dim == 128


def test_new_host_calls_refuse_bad_arguments(lib):
    q = np.zeros((4, 6, 128), dtype=np.float32)
    k = np.zeros((4, 4, 128), dtype=np.float32)
    out = np.zeros(4 * 64)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    assert lib.bgtq_block_energy_heads(p(q), 4, 6, p(k), 4, 4, p(out)) == B.ERR_INVALID   # 6 % 4 != 0
    assert lib.bgtq_block_energy_heads(None, 4, 8, p(k), 4, 4, p(out)) == B.ERR_INVALID
    s = np.ones(64)
    r = np.zeros(64, dtype=np.int32)
    assert lib.bgtq_allocate_rates(p(s), 64, -1, 4, 64, None, p(r)) == B.ERR_INVALID
    assert lib.bgtq_allocate_rates(p(s), 64, 0, 0, 0, None, p(r)) == B.ERR_INVALID      # max_rate must be >= 1
    assert lib.bgtq_allocate_rates(p(s), 64, 0, 4, 257, None, p(r)) == B.ERR_INFEASIBLE
    assert lib.bgtq_allocate_rates(p(s), 64, 0, 4, 0, None, p(r)) == B.OK and not r.any()
    bad = np.full(64, 5, dtype=np.int32)
    h = C.c_void_p()
    assert lib.bgtq_layout_create(p(bad), 2, 0, C.byref(h)) == B.ERR_INVALID
    neg = np.full(64, 2, dtype=np.int32)
    neg[3] = -1
    assert lib.bgtq_layout_create(p(neg), 2, 0, C.byref(h)) == B.ERR_INVALID


def test_layout_set_refuses_bad_arguments_without_device(lib):
    """bgtq_layout_set_create checks its arguments before touching a device: no output
    pointer, no layouts, and layouts that are not uploaded are refused; the size queries
    of a null set answer 0."""
    h = C.c_void_p()
    assert lib.bgtq_layout_set_create(None, 1, C.byref(h)) == B.ERR_INVALID
    lay = B.Layout(np.full(64, 2), 2, 0)
    arr = (C.c_void_p * 1)(lay.handle)
    assert lib.bgtq_layout_set_create(arr, 0, C.byref(h)) == B.ERR_INVALID
    assert lib.bgtq_layout_set_create(arr, 1, None) == B.ERR_INVALID
    assert lib.bgtq_layout_set_create(arr, 1, C.byref(h)) == B.ERR_DEVICE     # not uploaded
    assert not h.value
    assert lib.bgtq_layout_set_tile_bytes(None) == 0
    assert lib.bgtq_layout_set_cache_bytes(None, 1, 64) == 0
    f = C.c_uint(0)
    assert lib.bgtq_layout_set_status(None, C.byref(f), 0) == B.ERR_INVALID
    assert lib.bgtq_encode_append_heads(None, None, None, 0, 1, 1, None, None, 64, None) == B.ERR_INVALID
    assert lib.bgtq_decode_attention_heads(None, None, 0, 1, 1, None, None, 64, 64, 0.1, None, None, 0,
                                           None) == B.ERR_INVALID
    assert lib.bgtq_decode_attention_multi_heads(None, None, 0, 1, 2, 1, None, None, 64, 64, 0.1, None, None, 0,
                                                 None) == B.ERR_INVALID
    assert lib.bgtq_decode_step_multi_heads(None, None, None, 0, 2, None, 0, 1, 1, None, None, 64, 64, 0.1, None,
                                            None, 0, None) == B.ERR_INVALID
    assert lib.bgtq_decode_step_paged_heads(None, None, None, 0, 1, None, 0, 1, 1, None, 1, None, 1, None, 64, 0.1,
                                            None, None, 0, None) == B.ERR_INVALID
    lib.bgtq_layout_set_destroy(None)                                          # a no-op
