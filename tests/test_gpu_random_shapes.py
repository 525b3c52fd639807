"""Seeded random shapes through the C ABI against the oracle: query heads per KV head,
query tokens per row (up to 32 columns per KV head), batch, ragged lengths, key and value
rates, input dtype, norm correction, fp16 norms, rate-0 blocks, one layout per KV head
(layout sets, with one or several query tokens per row), and appends split into
chunks of random sizes (short appends take the per-token encoder, longer ones the bulk
encoder; a chunk may start anywhere inside a tile). Every packed (row, KV head) slice is
compared with the oracle's bytes, every query column's output with the oracle's
attention."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, Case, build_inputs, compare_packed, rel_l2, slice_bytes

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16, torch.float16]


def _draw(i):
    rng = np.random.default_rng(7000 + i)
    while True:
        G = int(rng.choice([1, 2, 3, 4, 5, 6, 8, 12, 16]))
        n_q = int(rng.choice([1, 2, 3, 4]))
        if G * n_q <= 32:
            break
    h_kv = int(rng.integers(1, 4))
    case = Case(G * h_kv, h_kv, int(rng.integers(1, 4)), int(rng.integers(n_q + 40, 700)), int(rng.choice([2, 3])),
                int(rng.integers(1, 5)), DTYPES[int(rng.integers(0, 3))], 5e5, 100 + i,
                norm_correct=bool(rng.integers(0, 2)), norm_fp16=bool(rng.integers(0, 2)),
                min_rate=int(rng.integers(0, 2)))
    # append chunks: a long one, a short one (per-token encoder), the rest
    a = int(rng.integers(1, case.length - 10))
    b = a + int(rng.integers(1, 8))
    return case, n_q, [0, a, b, case.length]


@pytest.mark.parametrize("i", range(16))
def test_random_shape_matches_oracle(i):
    case, n_q, bounds = _draw(i)
    model, rates, _, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed, case.norm_correct, case.norm_fp16).upload(0)
    cache = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, case.cap), dtype=torch.uint8, device="cuda")
    kd, vd = k.cuda(), v.cuda()
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b > a:
            lens0 = torch.full((case.batch,), a, dtype=torch.int32, device="cuda")
            B.encode_append(lay, kd[:, a:b].contiguous(), vd[:, a:b].contiguous(), lens0, cache, case.cap)
    torch.cuda.synchronize()
    assert lay.status() == 0
    olay = O.make_layout(rates, case.v_bits, case.seed, case.norm_correct, case.norm_fp16)
    cache_cpu = cache.cpu().numpy()
    bufs = {}
    for b in range(case.batch):
        for h in range(case.h_kv):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            want = O.pack(olay, enc, case.cap)
            compare_packed(olay, enc, want, slice_bytes(case, olay.tile_bytes, cache_cpu, b, h), case.cap)
            bufs[b, h] = want
    # ragged rows; the last n_q cached tokens of each row carry its queries
    lens = torch.tensor([max(n_q, case.length - 53 * b) for b in range(case.batch)], dtype=torch.int32)
    q = torch.empty(case.batch, n_q, case.h_q, 128, dtype=case.dtype)
    for b in range(case.batch):
        for hq in range(case.h_q):
            q[b, :, hq] = synth.query_slice(model, b, hq, n_q, int(lens[b]) - n_q, case.seed, case.theta).to(case.dtype)
    out = torch.full((case.batch, n_q, case.h_q, 128), float("nan"), device="cuda")
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q * n_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    B.decode_attention_multi(lay, q.cuda(), cache, lens.cuda(), case.cap, case.length, out, ws, case.h_kv)
    torch.cuda.synchronize()
    assert lay.status() == 0
    got = out.cpu().double().numpy()
    G = case.h_q // case.h_kv
    for b in range(case.batch):
        for h in range(case.h_kv):
            ref = O.decode_attention_multi(olay, q[b, :, h * G:(h + 1) * G].double().numpy(), bufs[b, h],
                                           int(lens[b]), 1 / math.sqrt(128))
            for j in range(n_q):
                for c in range(G):
                    err = rel_l2(got[b, j, h * G + c], ref[j, c])
                    assert err <= ATTN_REL_L2, (case, n_q, b, h, j, c, err)


def _draw_set(i):
    rng = np.random.default_rng(9000 + i)
    G = int(rng.choice([1, 2, 4, 5, 8, 12, 16]))
    h_kv = int(rng.integers(2, 5))
    case = Case(G * h_kv, h_kv, int(rng.integers(1, 3)), int(rng.integers(40, 500)), int(rng.choice([2, 3])),
                int(rng.integers(1, 5)), DTYPES[int(rng.integers(0, 3))], 5e5, 200 + i,
                norm_correct=bool(rng.integers(0, 2)), norm_fp16=bool(rng.integers(0, 2)),
                min_rate=int(rng.integers(0, 2)))
    a = int(rng.integers(1, case.length - 10))
    return case, [0, a, a + int(rng.integers(1, 8)), case.length]


@pytest.mark.parametrize("i", range(6))
def test_random_layout_set_matches_oracle(i):
    """Random shapes with one layout per KV head (the oracle's per-head allocation), coded
    and decoded through a layout set; every head against the oracle with its own layout."""
    case, bounds = _draw_set(i)
    model = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(model, 256, case.seed + 1, case.theta)
    per = O.block_energy_heads(q_cal.double().numpy(), k_cal.double().numpy())
    rates = [O.greedy_rates(per[h], O.lloyd_max_mse_table(), case.min_rate, 4, 64 * case.k_bits)
             for h in range(case.h_kv)]
    q, k, v = synth.make_cache_inputs(model, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed, case.norm_correct, case.norm_fp16).upload(0)
               for h in range(case.h_kv)]
    S = B.LayoutSet(layouts)
    cache = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    kd, vd = k.cuda(), v.cuda()
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b > a:
            lens0 = torch.full((case.batch,), a, dtype=torch.int32, device="cuda")
            B.encode_append_heads(S, kd[:, a:b].contiguous(), vd[:, a:b].contiguous(), lens0, cache, case.cap)
    lens = torch.tensor([max(1, case.length - 31 * b) for b in range(case.batch)], dtype=torch.int32)
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, case.h_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((case.batch, case.h_q, 128), float("nan"), device="cuda")
    B.decode_attention_heads(S, q.cuda(), cache, lens.cuda(), case.cap, case.length, out, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    n_tiles, stride = case.cap // 64, S.tile_bytes
    cv = cache.view(case.batch, case.h_kv, n_tiles, stride).cpu().numpy()
    got = out.cpu().double().numpy()
    G = case.h_q // case.h_kv
    for h in range(case.h_kv):
        olay = O.make_layout(rates[h], case.v_bits, case.seed, case.norm_correct, case.norm_fp16)
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            want = O.pack(olay, enc, case.cap)
            compare_packed(olay, enc, want, np.ascontiguousarray(cv[b, h, :, :olay.tile_bytes]).reshape(-1), case.cap)
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), want, int(lens[b]),
                                     1 / math.sqrt(128))
            for c in range(G):
                err = rel_l2(got[b, h * G + c], ref[c])
                assert err <= ATTN_REL_L2, (case, b, h, c, err)


@pytest.mark.parametrize("i", range(5))
def test_random_layout_set_multi_token_matches_oracle(i):
    """Random shapes with one layout per KV head and n_q query tokens per row (causal among
    them, up to 32 columns per KV head) through decode_attention_multi_heads; every column
    against the oracle's multi-token attention with its head's layout."""
    rng = np.random.default_rng(9500 + i)
    while True:
        G = int(rng.choice([1, 2, 3, 4, 6, 8, 16]))
        n_q = int(rng.choice([2, 3, 4]))
        if G * n_q <= 32:
            break
    h_kv = int(rng.integers(2, 5))
    case = Case(G * h_kv, h_kv, int(rng.integers(1, 3)), int(rng.integers(n_q + 40, 400)), int(rng.choice([2, 3])),
                int(rng.integers(1, 5)), DTYPES[int(rng.integers(0, 3))], 5e5, 300 + i,
                norm_correct=bool(rng.integers(0, 2)), norm_fp16=bool(rng.integers(0, 2)),
                min_rate=int(rng.integers(0, 2)))
    model = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(model, 256, case.seed + 1, case.theta)
    per = O.block_energy_heads(q_cal.double().numpy(), k_cal.double().numpy())
    rates = [O.greedy_rates(per[h], O.lloyd_max_mse_table(), case.min_rate, 4, 64 * case.k_bits)
             for h in range(case.h_kv)]
    _, k, v = synth.make_cache_inputs(model, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed, case.norm_correct, case.norm_fp16).upload(0)
               for h in range(case.h_kv)]
    S = B.LayoutSet(layouts)
    cache = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    a = int(rng.integers(1, case.length - 10))
    kd, vd = k.cuda(), v.cuda()
    for a0, a1 in ((0, a), (a, case.length)):
        lens0 = torch.full((case.batch,), a0, dtype=torch.int32, device="cuda")
        B.encode_append_heads(S, kd[:, a0:a1].contiguous(), vd[:, a0:a1].contiguous(), lens0, cache, case.cap)
    lens = torch.tensor([max(n_q, case.length - 41 * b) for b in range(case.batch)], dtype=torch.int32)
    q = torch.empty(case.batch, n_q, case.h_q, 128, dtype=case.dtype)
    for b in range(case.batch):
        for hq in range(case.h_q):
            q[b, :, hq] = synth.query_slice(model, b, hq, n_q, int(lens[b]) - n_q, case.seed, case.theta).to(case.dtype)
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, case.h_q * n_q, case.h_kv, case.length),
                     dtype=torch.uint8, device="cuda")
    out = torch.full((case.batch, n_q, case.h_q, 128), float("nan"), device="cuda")
    B.decode_attention_multi_heads(S, q.cuda(), cache, lens.cuda(), case.cap, case.length, out, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    n_tiles = case.cap // 64
    cv = cache.view(case.batch, case.h_kv, n_tiles, S.tile_bytes).cpu().numpy()
    got = out.cpu().double().numpy()
    for h in range(case.h_kv):
        olay = O.make_layout(rates[h], case.v_bits, case.seed, case.norm_correct, case.norm_fp16)
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            want = O.pack(olay, enc, case.cap)
            compare_packed(olay, enc, want, np.ascontiguousarray(cv[b, h, :, :olay.tile_bytes]).reshape(-1), case.cap)
            ref = O.decode_attention_multi(olay, q[b, :, h * G:(h + 1) * G].double().numpy(), want, int(lens[b]),
                                           1 / math.sqrt(128))
            for j in range(n_q):
                for c in range(G):
                    err = rel_l2(got[b, j, h * G + c], ref[j, c])
                    assert err <= ATTN_REL_L2, (case, n_q, b, h, j, c, err)
