"""Decode attention split over token ranges, through the C ABI: each range's packed cache
gives partial records (bgtq_decode_attention_partial), bgtq_merge_partials merges them,
and the result must be attention over all tokens. Here the ranges live on one GPU (this
pool gives one GPU per run); across GPUs the records travel by one all-gather
(packed_cache_decode_b200.sharding.split_sequence_decode, tested with gloo ranks in
test_multirank_cpu.py)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import sharding

from .parity_util import ATTN_REL_L2, Case, build_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("parts", [1, 2, 3])
def test_split_ranges_merge_to_the_whole_sequence(parts):
    case = Case(16, 2, 2, 1500, 2, 2, torch.bfloat16, 5e5, 61)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    G = case.h_q // case.h_kv
    recs = torch.empty(parts, case.batch, case.h_q, B.PARTIAL_RECORD, dtype=torch.float32, device="cuda")
    kd, vd, qd = k.cuda(), v.cuda(), q.cuda()
    for r in range(parts):
        t0, t1 = sharding.token_range(case.length, r, parts)
        n = t1 - t0
        cap = max(64, 64 * math.ceil(n / 64))
        cache = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, cap), dtype=torch.uint8, device="cuda")
        lens = torch.zeros(case.batch, dtype=torch.int32, device="cuda")
        B.encode_append(lay, kd[:, t0:t1].contiguous(), vd[:, t0:t1].contiguous(), lens, cache, cap)
        lens.fill_(n)
        ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, n), dtype=torch.uint8, device="cuda")
        B.decode_attention_partial(lay, qd, cache, lens, cap, n, recs[r], ws, case.h_kv)
    out = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    B.merge_partials(lay, recs, out)
    torch.cuda.synchronize()
    assert lay.status() == 0
    got = out.cpu().double().numpy()
    olay = O.make_layout(rates, case.v_bits, case.seed)
    for b in range(case.batch):
        for h in range(case.h_kv):
            buf = O.pack(olay, O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy()), case.cap)
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), buf, case.length,
                                     1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(got[b, h * G + i], ref[i]) <= ATTN_REL_L2, (b, h, i, rel_l2(got[b, h * G + i], ref[i]))


def test_record_of_an_empty_range_is_neutral():
    case = Case(8, 1, 1, 300, 2, 2, torch.bfloat16, 5e5, 62)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    cap = 320
    cache = torch.zeros(lay.cache_bytes(1, 1, cap), dtype=torch.uint8, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.encode_append(lay, k.cuda(), v.cuda(), lens, cache, cap)
    ws = torch.empty(B.workspace_bytes(lay, 1, 8, 1, 300), dtype=torch.uint8, device="cuda")
    recs = torch.empty(2, 1, 8, B.PARTIAL_RECORD, dtype=torch.float32, device="cuda")
    lens.fill_(300)
    B.decode_attention_partial(lay, q.cuda(), cache, lens, cap, 300, recs[0], ws, 1)
    lens.fill_(0)                                   # a range with no token
    B.decode_attention_partial(lay, q.cuda(), cache, lens, cap, 300, recs[1], ws, 1)
    full = torch.empty(1, 8, 128, dtype=torch.float32, device="cuda")
    merged = torch.empty_like(full)
    lens.fill_(300)
    B.decode_attention(lay, q.cuda(), cache, lens, cap, 300, full, ws, 1)
    B.merge_partials(lay, recs, merged)
    torch.cuda.synchronize()
    assert lay.status() == 0
    r1 = recs[1].cpu().numpy()
    assert np.all(np.isneginf(r1[..., 0])) and not r1[..., 1:].any()
    assert torch.allclose(merged, full, rtol=1e-5, atol=1e-6)
