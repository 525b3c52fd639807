"""bgtq_decode_step (append + attend in one kernel chain) through the C ABI.

A step must give exactly what the two separate calls give (the same encode arithmetic
and the same split plan, so caches and outputs are compared bit for bit), and a run of
steps that generates tokens one at a time must match the oracle after every step.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, Case, build_inputs, compare_packed, gpu_encode, oracle_slice, rel_l2, slice_bytes

pytestmark = pytest.mark.gpu


def _queries(model, case, pos):
    """q [B, h_q, 128] of every row at token position pos."""
    q = torch.empty(case.batch, case.h_q, 128, dtype=case.dtype)
    for b in range(case.batch):
        for hq in range(case.h_q):
            q[b, hq] = synth.query_slice(model, b, hq, 1, pos, case.seed, case.theta)[0].to(case.dtype)
    return q


def _separate(lay, case, k_new, v_new, q, cache, lens, msl):
    B.encode_append(lay, k_new, v_new, lens, cache, case.cap)
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, msl), dtype=torch.uint8, device="cuda")
    out = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    B.decode_attention(lay, q, cache, lens + k_new.shape[1], case.cap, msl, out, ws, case.h_kv)
    return out


def _fused(lay, case, k_new, v_new, q, cache, lens, msl):
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, msl), dtype=torch.uint8, device="cuda")
    out = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    B.decode_step(lay, k_new, v_new, q, cache, lens, case.cap, msl, out, ws)
    return out


@pytest.mark.parametrize("n_new", [0, 1, 5, 64])
def test_step_equals_append_then_attend(n_new):
    case = Case(16, 4, 3, 700, 2, 2, torch.bfloat16, 5e5, 21, capacity=832)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    pre = case.length - 64
    base = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, case.cap), dtype=torch.uint8, device="cuda")
    lens0 = torch.tensor([pre, pre - 61, 3], dtype=torch.int32, device="cuda")  # ragged rows, one near a tile start
    kd, vd = k.cuda(), v.cuda()
    for b in range(case.batch):
        n = int(lens0[b])
        lb = torch.full((case.batch,), case.cap, dtype=torch.int32, device="cuda")
        lb[b] = 0
        B.encode_append(lay, kd[:, :n].contiguous(), vd[:, :n].contiguous(), lb, base, case.cap)
    torch.cuda.synchronize()
    lay.status()                                  # the skipped rows flagged an overflow: clear it
    k_new = kd[:, pre:pre + n_new].contiguous()
    v_new = vd[:, pre:pre + n_new].contiguous()
    qd = q.cuda()
    msl = pre + n_new
    c_sep, c_fus = base.clone(), base.clone()
    o_sep = _separate(lay, case, k_new, v_new, qd, c_sep, lens0, msl)
    o_fus = _fused(lay, case, k_new, v_new, qd, c_fus, lens0, msl)
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)


def test_token_by_token_generation_matches_oracle():
    case = Case(8, 2, 2, 200, 3, 2, torch.bfloat16, 5e5, 22, capacity=256)
    model, rates, q, k, v = build_inputs(case)
    pre, steps = 130, 70                          # crosses the tile boundary at 192
    short = Case(**{**case.__dict__, "length": pre})
    lay, cache = gpu_encode(short, rates, k[:, :pre], v[:, :pre])
    assert cache.numel() == lay.cache_bytes(case.batch, case.h_kv, case.cap)
    kd, vd = k.cuda(), v.cuda()
    lens = torch.full((case.batch,), pre, dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, case.cap), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    G = case.h_q // case.h_kv
    olay = O.make_layout(rates, case.v_bits, case.seed)
    for s in range(steps):
        p = pre + s
        qp = _queries(model, case, p)
        B.decode_step(lay, kd[:, p:p + 1].contiguous(), vd[:, p:p + 1].contiguous(), qp.cuda(), cache, lens,
                      case.cap, case.cap, out, ws)
        lens += 1
        if s % 23 == 0 or s == steps - 1:         # the oracle on every 23rd step and the last
            got = out.cpu().double().numpy()
            for b in range(case.batch):
                for h in range(case.h_kv):
                    _, _, buf = oracle_slice(case, rates, k, v, b, h, n=p + 1)
                    ref = O.decode_attention(olay, qp[b, h * G:(h + 1) * G].double().numpy(), buf, p + 1,
                                             1 / math.sqrt(128))
                    for i in range(G):
                        assert rel_l2(got[b, h * G + i], ref[i]) <= ATTN_REL_L2, (s, b, h, i)
    torch.cuda.synchronize()
    assert lay.status() == 0
    cache_cpu = cache.cpu().numpy()
    for b in range(case.batch):
        for h in range(case.h_kv):
            olay, enc, want = oracle_slice(case, rates, k, v, b, h)
            compare_packed(olay, enc, want, slice_bytes(case, olay.tile_bytes, cache_cpu, b, h), case.cap)


def test_step_past_capacity_is_flagged():
    case = Case(4, 1, 1, 64, 2, 2, torch.float32, 5e5, 23)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.full((1,), 62, dtype=torch.int32, device="cuda")
    kk = torch.randn(1, 4, 1, 128, device="cuda")
    ws = torch.empty(B.workspace_bytes(lay, 1, 4, 1, 64), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, 4, 128, dtype=torch.float32, device="cuda")
    B.decode_step(lay, kk, kk.clone(), q.cuda(), cache, lens, 64, 64, out, ws)
    torch.cuda.synchronize()
    st = lay.status()
    assert st & B.STATUS_ENCODE_OVERFLOW and st & B.STATUS_DECODE_CLAMPED
    assert torch.isfinite(out).all()


def test_step_rejects_bad_arguments():
    lay = B.Layout(np.full(64, 2), 2, 0).upload(0)
    lib = B.load()
    cache = torch.zeros(lay.cache_bytes(1, 1, 64), dtype=torch.uint8, device="cuda")
    k = torch.zeros(1, 1, 1, 128, device="cuda")
    q = torch.zeros(1, 1, 128, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, 1, 128, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    call = lambda kd, n, hq, cap, msl, wsb: lib.bgtq_decode_step(lay.handle, p(k), p(k), kd, n, p(q), 0, 1, hq, 1,
                                                                 p(cache), p(lens), cap, msl, 0.1, p(out), p(ws),
                                                                 wsb, None)
    assert call(7, 1, 1, 64, 64, ws.numel()) == B.ERR_INVALID       # bad dtype
    assert call(0, -1, 1, 64, 64, ws.numel()) == B.ERR_INVALID      # negative n_new
    assert call(0, 1, 33, 64, 64, ws.numel()) == B.ERR_INVALID      # G = 33 > 32 (rejected before any launch)
    assert call(0, 1, 1, 65, 64, ws.numel()) == B.ERR_CAPACITY      # capacity not a multiple of 64
    assert call(0, 1, 1, 64, 128, ws.numel()) == B.ERR_CAPACITY     # max_seq_len > capacity
    assert call(0, 1, 1, 64, 64, 0) == B.ERR_WORKSPACE
    assert lib.bgtq_decode_step(lay.handle, None, None, 0, 1, p(q), 0, 1, 1, 1, p(cache), p(lens), 64, 64, 0.1,
                                p(out), p(ws), ws.numel(), None) == B.ERR_INVALID
    assert lay.status() == 0
