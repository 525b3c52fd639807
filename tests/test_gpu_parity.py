"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Codes: bit-exact except coordinates within 1e-6 of a decision threshold (counted).
Norms: within 1 fp32 ulp. Attention: relative L2 <= 2e-3 per query head, against the
oracle decoding its own packed cache; and the CUDA decode run on the oracle's packed
cache against the same oracle output.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B

from .parity_util import (ATTN_REL_L2, Case, build_inputs, compare_packed, gpu_decode, gpu_encode, oracle_slice,
                          rel_l2, slice_bytes)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32_k2v2": Case(1, 1, 1, 1024, 2, 2, torch.float32, 5e5, 0, scale_v=True),
    "tiny_ragged": Case(1, 1, 1, 1000, 2, 2, torch.float32, 5e5, 0, scale_v=True),
    "gqa4_bf16_k2v2": Case(32, 8, 1, 1000, 2, 2, torch.bfloat16, 5e5, 1),
    "gqa8_bf16_k3v3": Case(16, 2, 1, 2049, 3, 3, torch.bfloat16, 1e6, 2),
    "gqa8_batch3_k2v2": Case(16, 2, 3, 700, 2, 2, torch.bfloat16, 5e5, 3),
    "k4v4_uniform": Case(8, 2, 1, 333, 4, 4, torch.bfloat16, 5e5, 4),
    "k1v1_uniform": Case(8, 2, 1, 333, 1, 1, torch.bfloat16, 5e5, 5),
    "k3v2_f16": Case(4, 4, 2, 129, 3, 2, torch.float16, 5e5, 6),
    "gqa2_len1": Case(2, 1, 1, 1, 2, 2, torch.float32, 5e5, 7),
    "gqa1_len64": Case(1, 1, 2, 64, 2, 3, torch.float32, 5e5, 8),
    "gqa1_len65": Case(3, 3, 1, 65, 2, 1, torch.float32, 5e5, 9),
    # allocations from rate 0: some blocks are not stored
    "gqa4_k2v2_rate0": Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 10, min_rate=0),
    "gqa8_k1v2_rate0": Case(16, 2, 1, 300, 1, 2, torch.bfloat16, 1e6, 11, min_rate=0),
}


def _run_case(case: Case, n_chunks=1):
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v, n_chunks=n_chunks)
    cache_cpu = cache.cpu().numpy()
    out = gpu_decode(lay, case, q, cache)
    G = case.h_q // case.h_kv
    scale = 1.0 / math.sqrt(128)
    total_near, total_near_diff = 0, 0
    for b in range(case.batch):
        for h in range(case.h_kv):
            olay, enc, want = oracle_slice(case, rates, k, v, b, h)
            got = slice_bytes(case, olay.tile_bytes, cache_cpu, b, h)
            n_near, nd = compare_packed(olay, enc, want, got, case.cap)
            total_near += n_near
            total_near_diff += nd
            qs = q[b, h * G:(h + 1) * G].double().numpy()
            ref = O.decode_attention(olay, qs, want, case.length, scale)
            for i in range(G):
                assert rel_l2(out[b, h * G + i], ref[i]) <= ATTN_REL_L2, (b, h, i, rel_l2(out[b, h * G + i], ref[i]))
    assert lay.status() == 0
    return total_near, total_near_diff


@pytest.mark.parametrize("name", list(CASES))
def test_encode_and_decode_match_oracle(name):
    near, near_diff = _run_case(CASES[name])
    print(f"{name}: near-threshold coordinates {near}, of which coded differently {near_diff}")


def test_decode_on_oracle_packed_cache():
    """Same packed bytes on both sides: the decode kernel alone against the oracle."""
    case = Case(32, 8, 1, 1500, 2, 2, torch.bfloat16, 5e5, 11)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    parts = []
    refs = []
    G = case.h_q // case.h_kv
    for h in range(case.h_kv):
        olay, enc, buf = oracle_slice(case, rates, k, v, 0, h)
        parts.append(buf)
        refs.append(O.decode_attention(olay, q[0, h * G:(h + 1) * G].double().numpy(), buf, case.length,
                                       1 / math.sqrt(128)))
    cache = torch.from_numpy(np.concatenate(parts)).cuda()
    out = gpu_decode(lay, case, q, cache)
    errs = [rel_l2(out[0, h * G + i], refs[h][i]) for h in range(case.h_kv) for i in range(G)]
    print(f"decode on the oracle's cache: max rel L2 {max(errs):.2e}, median {np.median(errs):.2e}")
    assert max(errs) <= ATTN_REL_L2


def test_incremental_appends_equal_prefill():
    case = Case(8, 4, 2, 150, 2, 3, torch.bfloat16, 5e5, 12)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    _, c1 = gpu_encode(case, rates, k, v, n_chunks=1, layout=lay)
    _, c2 = gpu_encode(case, rates, k, v, n_chunks=37, layout=lay)
    _, c3 = gpu_encode(case, rates, k, v, n_chunks=150, layout=lay)
    assert torch.equal(c1, c2) and torch.equal(c1, c3)
    # re-appending the last token over itself leaves the cache unchanged
    lens = torch.full((case.batch,), case.length - 1, dtype=torch.int32, device="cuda")
    B.encode_append(lay, k[:, -1:].cuda().contiguous(), v[:, -1:].cuda().contiguous(), lens, c3, case.cap)
    torch.cuda.synchronize()
    assert torch.equal(c1, c3)


def test_ragged_batch_lengths_and_empty_row():
    case = Case(16, 4, 4, 300, 2, 2, torch.bfloat16, 5e5, 13)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.tensor([300, 1, 0, 177], dtype=torch.int32)
    out = gpu_decode(lay, case, q, cache, seq_lens=lens)
    G = case.h_q // case.h_kv
    for b in range(case.batch):
        for h in range(case.h_kv):
            n = int(lens[b])
            olay, enc, buf = oracle_slice(case, rates, k, v, b, h)
            qs = q[b, h * G:(h + 1) * G].double().numpy()
            if n == 0:
                assert np.all(out[b, h * G:(h + 1) * G] == 0)
                continue
            ref = O.decode_attention(olay, qs, buf, n, 1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(out[b, h * G + i], ref[i]) <= ATTN_REL_L2


def test_zero_vectors_code_to_middle_and_zero_norm():
    case = Case(2, 2, 1, 70, 3, 2, torch.float32, 5e5, 14)
    model, rates, q, k, v = build_inputs(case)
    k[0, 5] = 0
    v[0, 9] = 0
    lay, cache = gpu_encode(case, rates, k, v)
    cache_cpu = cache.cpu().numpy()
    for h in range(2):
        olay, enc, want = oracle_slice(case, rates, k, v, 0, h)
        assert np.all(enc["k_norms"][5] == 0) and enc["v_norm"][9] == 0
        compare_packed(olay, enc, want, slice_bytes(case, olay.tile_bytes, cache_cpu, 0, h), case.cap,
                       near_rare=False)
    out = gpu_decode(lay, case, q, cache)
    assert np.all(np.isfinite(out))


def test_capacity_overflow_is_flagged_and_skipped():
    case = Case(1, 1, 1, 64, 2, 2, torch.float32, 5e5, 15)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    before = cache.clone()
    lens = torch.full((1,), 60, dtype=torch.int32, device="cuda")
    kk = torch.randn(1, 8, 1, 128, device="cuda")
    B.encode_append(lay, kk, kk.clone(), lens, cache, 64)
    torch.cuda.synchronize()
    assert lay.status() & B.STATUS_ENCODE_OVERFLOW
    assert lay.status() == 0                           # cleared by the previous read
    # positions 60..63 were written, 64..67 skipped: only tokens 60..63 of the tile changed
    olay = O.make_layout(rates, 2, case.seed)
    u0 = O.unpack(olay, before.cpu().numpy(), 64)
    u1 = O.unpack(olay, cache.cpu().numpy(), 64)
    changed = sorted(set(np.nonzero((u0["k_codes"] != u1["k_codes"]).any(1) | (u0["v_codes"] != u1["v_codes"]).any(1)
                                    | (u0["k_norms"] != u1["k_norms"]).any(1) | (u0["v_norm"] != u1["v_norm"]))[0]))
    assert changed and min(changed) >= 60


def test_decode_clamps_overlong_lengths():
    case = Case(1, 1, 1, 128, 2, 2, torch.float32, 5e5, 16)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    out = gpu_decode(lay, case, q, cache, seq_lens=torch.tensor([128]), max_seq_len=64)
    assert lay.status() & B.STATUS_DECODE_CLAMPED
    olay, enc, buf = oracle_slice(case, rates, k, v, 0, 0)
    ref = O.decode_attention(olay, q[0, :1].double().numpy(), buf, 64, 1 / math.sqrt(128))
    assert rel_l2(out[0, 0], ref[0]) <= ATTN_REL_L2


def test_bad_arguments_are_rejected_before_launch():
    lay = B.Layout(np.full(64, 2), 2, 0).upload(0)
    lib = B.load()
    cache = torch.zeros(lay.cache_bytes(1, 1, 64), dtype=torch.uint8, device="cuda")
    k = torch.zeros(1, 1, 1, 128, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    import ctypes as C
    p = lambda t: C.c_void_p(t.data_ptr())
    assert lib.bgtq_encode_append(lay.handle, p(k), p(k), 9, 1, 1, 1, p(lens), p(cache), 64, None) == B.ERR_INVALID
    assert lib.bgtq_encode_append(lay.handle, p(k), p(k), 0, 1, 1, 1, p(lens), p(cache), 65, None) == B.ERR_CAPACITY
    out = torch.zeros(1, 33, 128, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    assert lib.bgtq_decode_attention(lay.handle, p(out), 0, 1, 33, 1, p(cache), p(lens), 64, 64, 0.1, p(out), p(ws),
                                     ws.numel(), None) == B.ERR_INVALID      # G = 33 > 32
    assert lib.bgtq_decode_attention(lay.handle, p(out), 0, 1, 1, 1, p(cache), p(lens), 64, 128, 0.1, p(out), p(ws),
                                     ws.numel(), None) == B.ERR_CAPACITY     # max_seq_len > capacity
    assert lib.bgtq_decode_attention(lay.handle, p(out), 0, 1, 1, 1, p(cache), p(lens), 64, 64, 0.1, p(out), p(ws),
                                     0, None) == B.ERR_WORKSPACE
    assert lay.status() == 0


def test_cache_bytes_match_what_encode_writes():
    case = Case(8, 2, 2, 640, 2, 2, torch.bfloat16, 5e5, 17)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    olay = O.make_layout(rates, 2, case.seed)
    assert cache.numel() == O.cache_bytes(olay, 2, 2, 640) == 2 * 2 * 640 * olay.bytes_per_token
    # every byte of a full cache belongs to some token's codes or norms: the written
    # cache equals the oracle's packing of all tokens, byte for byte outside thresholds
    assert olay.bytes_per_token == 128 * 2 // 8 * 2 + 4 * (olay.n_kgroups + 1)
