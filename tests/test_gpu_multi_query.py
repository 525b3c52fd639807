"""Multi-token decode attention through the C ABI against the oracle: n_q query tokens per
row, the last n_q of the row's cached tokens, causal among themselves (speculative
verification, a prefill chunk). The G query heads x n_q tokens of a KV head are the
columns of tensor-core tiles of 8, so the cases cover both q' fragment forms (G n_q <= 4
and 5..8 columns), several column tiles per KV head (up to 32 columns, a last tile with a
single column) and ragged rows.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, Case, build_inputs, gpu_encode, oracle_slice, rel_l2, slice_bytes

pytestmark = pytest.mark.gpu

CASES = {   # (case, n_q)
    "gqa4_nq2_8cols": (Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 51), 2),
    "gqa2_nq2_4cols": (Case(8, 4, 2, 333, 2, 2, torch.bfloat16, 5e5, 52), 2),
    "gqa1_nq8": (Case(2, 2, 1, 260, 3, 3, torch.bfloat16, 1e6, 53), 8),
    "gqa1_nq3_f32_k1v4": (Case(2, 2, 3, 130, 1, 4, torch.float32, 5e5, 54), 3),
    "gqa8_nq1": (Case(16, 2, 1, 500, 3, 3, torch.bfloat16, 1e6, 55), 1),
    "gqa8_nq2_16cols": (Case(16, 2, 2, 500, 2, 2, torch.bfloat16, 5e5, 58), 2),
    "gqa8_nq4_32cols": (Case(16, 2, 1, 300, 3, 3, torch.bfloat16, 1e6, 59), 4),
    "gqa3_nq3_9cols": (Case(6, 2, 2, 400, 2, 2, torch.float16, 5e5, 60), 3),
    "gqa16_nq1": (Case(32, 2, 2, 260, 2, 3, torch.bfloat16, 5e5, 61), 1),
}


def _multi_queries(model, case, n_q, lens):
    """q [B, n_q, h_q, 128]: row b's queries at positions lens[b] - n_q .. lens[b] - 1."""
    q = torch.empty(case.batch, n_q, case.h_q, 128, dtype=case.dtype)
    for b in range(case.batch):
        for hq in range(case.h_q):
            q[b, :, hq] = synth.query_slice(model, b, hq, n_q, int(lens[b]) - n_q, case.seed, case.theta).to(case.dtype)
    return q


def _ws(lay, case, n_q, msl):
    return torch.empty(B.workspace_bytes(lay, case.batch, case.h_q * n_q, case.h_kv, msl), dtype=torch.uint8,
                       device="cuda")


@pytest.mark.parametrize("name", list(CASES))
def test_multi_query_attention_matches_oracle(name):
    case, n_q = CASES[name]
    model, rates, _, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.tensor([case.length - 37 * b for b in range(case.batch)], dtype=torch.int32)
    q = _multi_queries(model, case, n_q, lens)
    out = torch.full((case.batch, n_q, case.h_q, 128), float("nan"), dtype=torch.float32, device="cuda")
    B.decode_attention_multi(lay, q.cuda(), cache, lens.cuda(), case.cap, case.length, out,
                             _ws(lay, case, n_q, case.length), case.h_kv)
    torch.cuda.synchronize()
    assert lay.status() == 0
    got = out.cpu().double().numpy()
    G = case.h_q // case.h_kv
    for b in range(case.batch):
        n = int(lens[b])
        for h in range(case.h_kv):
            olay, enc, buf = oracle_slice(case, rates, k, v, b, h)
            qs = q[b, :, h * G:(h + 1) * G].double().numpy()                   # [n_q, G, 128]
            ref = O.decode_attention_multi(olay, qs, buf, n, 1 / math.sqrt(128))
            for j in range(n_q):
                for i in range(G):
                    err = rel_l2(got[b, j, h * G + i], ref[j, i])
                    assert err <= ATTN_REL_L2, (b, h, j, i, err)


def test_one_query_token_equals_decode_attention():
    case = Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 56)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.tensor([700, 650], dtype=torch.int32, device="cuda")
    o1 = torch.empty(case.batch, case.h_q, 128, device="cuda")
    o2 = torch.empty(case.batch, 1, case.h_q, 128, device="cuda")
    B.decode_attention(lay, q.cuda(), cache, lens, case.cap, case.length, o1, _ws(lay, case, 1, case.length),
                       case.h_kv)
    B.decode_attention_multi(lay, q.cuda()[:, None].contiguous(), cache, lens, case.cap, case.length, o2,
                             _ws(lay, case, 1, case.length), case.h_kv)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2[:, 0])


@pytest.mark.parametrize("h_q", [8, 16], ids=["8cols", "16cols"])
@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
def test_step_multi_equals_append_then_attend(paged, h_q):
    """decode_step_multi appends the n_new draft tokens and attends with their queries in one
    chain: same cache bytes and outputs as encode_append + decode_attention_multi, and the
    oracle's multi-token attention over the grown rows (h_q / h_kv x n_new = 8 or 16 query
    columns per KV head: one or two column tiles)."""
    case = Case(h_q, 4, 3, 600, 2, 2, torch.bfloat16, 5e5, 57, capacity=640)
    n_new = 4
    model, rates, _, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    lens0 = torch.tensor([590, 401, 3], dtype=torch.int32)
    kd, vd = k.cuda(), v.cuda()
    base = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, case.cap), dtype=torch.uint8, device="cuda")
    for b in range(case.batch):
        lb = torch.full((case.batch,), case.cap, dtype=torch.int32, device="cuda")
        lb[b] = 0
        n = int(lens0[b])
        B.encode_append(lay, kd[:, :n].contiguous(), vd[:, :n].contiguous(), lb, base, case.cap)
    torch.cuda.synchronize()
    lay.status()                                   # the skipped rows flagged an overflow: clear it
    # row b's new tokens are k[b, lens0[b] .. lens0[b] + n_new)
    k_new = torch.stack([k[b, int(lens0[b]):int(lens0[b]) + n_new] for b in range(case.batch)]).cuda().contiguous()
    v_new = torch.stack([v[b, int(lens0[b]):int(lens0[b]) + n_new] for b in range(case.batch)]).cuda().contiguous()
    q = _multi_queries(model, case, n_new, lens0 + n_new).cuda()
    msl = int(lens0.max()) + n_new
    lens_d = lens0.cuda()
    c_sep = base.clone()
    o_sep = torch.empty(case.batch, n_new, case.h_q, 128, device="cuda")
    o_fus = torch.empty_like(o_sep)
    B.encode_append(lay, k_new, v_new, lens_d, c_sep, case.cap)
    B.decode_attention_multi(lay, q, c_sep, lens_d + n_new, case.cap, msl, o_sep, _ws(lay, case, n_new, msl),
                             case.h_kv)
    if paged:
        n_tiles = case.cap // 64
        perm = np.random.default_rng(3).permutation(case.batch * n_tiles + 2)[:case.batch * n_tiles].astype(np.int32)
        table = torch.from_numpy(perm.reshape(case.batch, n_tiles)).cuda()
        pool = torch.zeros(B.paged_pool_bytes(lay, case.h_kv, case.batch * n_tiles + 2), dtype=torch.uint8,
                           device="cuda")
        tb = lay.tile_bytes
        src = base.view(case.batch, case.h_kv, n_tiles, tb)
        pv = pool.view(-1, case.h_kv, tb)
        for b in range(case.batch):
            for i in range(n_tiles):
                pv[int(perm[b * n_tiles + i])] = src[b, :, i]
        pc = B.PagedCache(pool, table)
        B.decode_step_multi_paged(lay, k_new, v_new, q, pc, lens_d, msl, o_fus, _ws(lay, case, n_new, msl))
        torch.cuda.synchronize()
        c_fus = torch.stack([torch.stack([pv[int(perm[b * n_tiles + i])] for i in range(n_tiles)], 1)
                             for b in range(case.batch)]).contiguous().view(-1)
    else:
        c_fus = base.clone()
        B.decode_step_multi(lay, k_new, v_new, q, c_fus, lens_d, case.cap, msl, o_fus, _ws(lay, case, n_new, msl))
        torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)
    got = o_fus.cpu().double().numpy()
    cache_cpu = c_fus.cpu().numpy()
    G = case.h_q // case.h_kv
    olay = O.make_layout(rates, case.v_bits, case.seed)
    for b in range(case.batch):
        n = int(lens0[b]) + n_new
        for h in range(case.h_kv):
            buf = slice_bytes(case, olay.tile_bytes, cache_cpu, b, h)
            ref = O.decode_attention_multi(olay, q[b, :, h * G:(h + 1) * G].double().cpu().numpy(), buf, n,
                                           1 / math.sqrt(128))
            for j in range(n_new):
                for i in range(G):
                    assert rel_l2(got[b, j, h * G + i], ref[j, i]) <= ATTN_REL_L2, (b, h, j, i)


def test_multi_query_rejects_bad_shapes():
    lay = B.Layout(np.full(64, 2), 2, 0).upload(0)
    lib = B.load()
    cache = torch.zeros(lay.cache_bytes(1, 1, 64), dtype=torch.uint8, device="cuda")
    q = torch.zeros(1, 8, 4, 128, device="cuda")
    lens = torch.full((1,), 10, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, 8, 4, 128, device="cuda")
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    call = lambda n_q, h_q: lib.bgtq_decode_attention_multi(lay.handle, p(q), 0, 1, n_q, h_q, 1, p(cache), p(lens), 64,
                                                            64, 0.1, p(out), p(ws), ws.numel(), None)
    assert call(9, 4) == B.ERR_INVALID      # 4 heads x 9 tokens = 36 columns > 32 (rejected before any launch)
    assert call(0, 1) == B.ERR_INVALID
    assert call(2, 4) == B.OK
    assert call(3, 4) == B.OK               # 12 columns: two column tiles
    assert lib.bgtq_decode_step_multi(lay.handle, p(q), p(q), 0, 0, p(q), 0, 1, 1, 1, p(cache), p(lens), 64, 64, 0.1,
                                      p(out), p(ws), ws.numel(), None) == B.ERR_INVALID   # n_new = 0
    torch.cuda.synchronize()
    assert lay.status() == 0
