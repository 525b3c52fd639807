"""Paged caches through the C ABI: the same tiles and the same results as a contiguous cache.

Pages of one pool are handed out to the rows in a shuffled order; every tile written by
the paged encode must equal the contiguous encode's tile byte for byte, and attention
over the paged cache must give the contiguous call's output bit for bit (same kernels,
same launch plan).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B

from .parity_util import ATTN_REL_L2, Case, build_inputs, rel_l2

pytestmark = pytest.mark.gpu


def _paged_setup(lay, case, max_pages, extra_pages, seed):
    rng = np.random.default_rng(seed)
    num_pages = case.batch * max_pages + extra_pages
    perm = rng.permutation(num_pages)[:case.batch * max_pages].astype(np.int32)
    table = torch.from_numpy(perm.reshape(case.batch, max_pages)).cuda()
    pool = torch.zeros(B.paged_pool_bytes(lay, case.h_kv, num_pages), dtype=torch.uint8, device="cuda")
    return B.PagedCache(pool, table)


def _tile(pc, lay, h_kv, b, h, i):
    p = int(pc.table[b, i])
    tb = lay.tile_bytes
    return pc.pool[(p * h_kv + h) * tb:(p * h_kv + h + 1) * tb]


@pytest.mark.parametrize("options", [(False, False), (True, True)], ids=["plain", "nc_fp16"])
@pytest.mark.parametrize("shape", [(16, 4, 3, 700, 2, 2), (16, 2, 2, 333, 3, 3)])
def test_paged_equals_contiguous(shape, options):
    h_q, h_kv, batch, length, kb, vb = shape
    case = Case(h_q, h_kv, batch, length, kb, vb, torch.bfloat16, 5e5, 41)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed, *options).upload(0)
    cap = case.cap
    max_pages = cap // 64
    lens = torch.tensor([length - 211 * b for b in range(batch)], dtype=torch.int32)
    kd, vd = k.cuda(), v.cuda()
    # contiguous reference: each row appends its own length (others beyond capacity: skipped)
    cont = torch.zeros(lay.cache_bytes(batch, h_kv, cap), dtype=torch.uint8, device="cuda")
    pc = _paged_setup(lay, case, max_pages, 5, 1)
    for b in range(batch):
        n = int(lens[b])
        lb = torch.full((batch,), cap, dtype=torch.int32, device="cuda")
        lb[b] = 0
        B.encode_append(lay, kd[:, :n].contiguous(), vd[:, :n].contiguous(), lb, cont, cap)
        B.encode_append_paged(lay, kd[:, :n].contiguous(), vd[:, :n].contiguous(), lb, pc)
    torch.cuda.synchronize()
    assert lay.status() & B.STATUS_ENCODE_OVERFLOW     # the rows beyond capacity were skipped
    for b in range(batch):
        for h in range(h_kv):
            for i in range(max_pages):
                c = cont[((b * h_kv + h) * max_pages + i) * lay.tile_bytes:][:lay.tile_bytes]
                assert torch.equal(c, _tile(pc, lay, h_kv, b, h, i)), (b, h, i)
    ws = torch.empty(B.workspace_bytes(lay, batch, h_q, h_kv, length), dtype=torch.uint8, device="cuda")
    o1 = torch.empty(batch, h_q, 128, device="cuda")
    o2 = torch.empty_like(o1)
    B.decode_attention(lay, q.cuda(), cont, lens.cuda(), cap, length, o1, ws, h_kv)
    B.decode_attention_paged(lay, q.cuda(), pc, lens.cuda(), length, o2, ws, h_kv)
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(o1, o2)
    # the paged output against the oracle, per query head: the oracle encodes and packs
    # each row's own tokens and attends over them
    olay = O.make_layout(rates, case.v_bits, case.seed, *options)
    G = h_q // h_kv
    out = o2.cpu().double().numpy()
    for b in range(batch):
        n = int(lens[b])
        for h in range(h_kv):
            enc = O.encode(olay, k[b, :n, h].double().numpy(), v[b, :n, h].double().numpy())
            buf = O.pack(olay, enc, cap)
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), buf, n, 1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(out[b, h * G + i], ref[i]) <= ATTN_REL_L2, (b, h, i, rel_l2(out[b, h * G + i], ref[i]))


def test_paged_steps_equal_contiguous_steps():
    case = Case(8, 2, 2, 200, 2, 2, torch.bfloat16, 5e5, 42, capacity=256)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    cap, max_pages = 256, 4
    kd, vd, qd = k.cuda(), v.cuda(), q.cuda()
    cont = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, cap), dtype=torch.uint8, device="cuda")
    pc = _paged_setup(lay, case, max_pages, 3, 2)
    lens = torch.zeros(case.batch, dtype=torch.int32, device="cuda")
    B.encode_append(lay, kd[:, :150].contiguous(), vd[:, :150].contiguous(), lens, cont, cap)
    B.encode_append_paged(lay, kd[:, :150].contiguous(), vd[:, :150].contiguous(), lens, pc)
    lens.fill_(150)
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, cap), dtype=torch.uint8, device="cuda")
    o1 = torch.empty(case.batch, case.h_q, 128, device="cuda")
    o2 = torch.empty_like(o1)
    for p in range(150, 200):
        kn, vn = kd[:, p:p + 1].contiguous(), vd[:, p:p + 1].contiguous()
        B.decode_step(lay, kn, vn, qd, cont, lens, cap, cap, o1, ws)
        B.decode_step_paged(lay, kn, vn, qd, pc, lens, cap, o2, ws)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2), p
        lens += 1
    assert lay.status() == 0


def test_page_outside_the_pool_is_flagged_and_left_out():
    case = Case(4, 1, 2, 128, 2, 2, torch.float32, 5e5, 43)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    pc = _paged_setup(lay, case, 2, 0, 3)
    lens = torch.zeros(2, dtype=torch.int32, device="cuda")
    B.encode_append_paged(lay, k.cuda(), v.cuda(), lens, pc)
    torch.cuda.synchronize()
    assert lay.status() == 0
    good = B.PagedCache(pc.pool, pc.table.clone())
    pc.table[1, 1] = 1 << 20                       # row 1's second tile: no such page
    lens.fill_(128)
    ws = torch.empty(B.workspace_bytes(lay, 2, 4, 1, 128), dtype=torch.uint8, device="cuda")
    o_bad = torch.empty(2, 4, 128, device="cuda")
    o_ref = torch.empty_like(o_bad)
    B.decode_attention_paged(lay, q.cuda(), pc, lens, 128, o_bad, ws, 1)
    torch.cuda.synchronize()
    assert lay.status() & B.STATUS_BAD_PAGE
    # row 0 is untouched; row 1 equals attention over its first 64 tokens only
    short = torch.tensor([128, 64], dtype=torch.int32, device="cuda")
    B.decode_attention_paged(lay, q.cuda(), good, short, 128, o_ref, ws, 1)
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(o_bad[0], o_ref[0])
    assert torch.allclose(o_bad[1], o_ref[1], rtol=1e-5, atol=1e-6)
