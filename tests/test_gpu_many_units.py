"""Many short (batch row, KV head) units: far more units than split CTAs, so every CTA's
slice runs through several units (segments of a few tiles, some empty after clipping to
a short row), with ragged rows of 1 to 100 tokens (1, 64 and 65 among them). Every unit
is compared with the oracle: one layout with one query token, one layout with three query
tokens per row (12 columns per KV head: two column tiles, twice the units), and a layout
set (one layout per KV head, a head change at most segment starts)."""
import math

import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, Case, build_inputs, rel_l2

pytestmark = pytest.mark.gpu

H_Q, H_KV, BATCH, LENGTH, CAP = 16, 4, 80, 100, 128


def _lens(n_min):
    lens = [(b * 29) % LENGTH + 1 for b in range(BATCH)]
    lens[:3] = [1, 64, 65]
    return torch.tensor([max(n_min, x) for x in lens], dtype=torch.int32)


def _queries(model, case, lens, n_q):
    q = torch.empty(BATCH, n_q, H_Q, 128, dtype=case.dtype)
    for b in range(BATCH):
        for hq in range(H_Q):
            q[b, :, hq] = synth.query_slice(model, b, hq, n_q, int(lens[b]) - n_q, case.seed, case.theta).to(case.dtype)
    return q


@pytest.fixture(scope="module")
def single_layout():
    case = Case(H_Q, H_KV, BATCH, LENGTH, 2, 2, torch.bfloat16, 5e5, 81, capacity=CAP)
    model, rates, _, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed).upload(0)
    cache = torch.zeros(lay.cache_bytes(BATCH, H_KV, CAP), dtype=torch.uint8, device="cuda")
    B.encode_append(lay, k.cuda(), v.cuda(), torch.zeros(BATCH, dtype=torch.int32, device="cuda"), cache, CAP)
    torch.cuda.synchronize()
    assert lay.status() == 0
    olay = O.make_layout(rates, case.v_bits, case.seed)
    packed = {(b, h): O.pack(olay, O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy()), CAP)
              for b in range(BATCH) for h in range(H_KV)}
    return case, model, lay, cache, olay, packed


@pytest.mark.parametrize("n_q", [1, 3])
def test_many_units_match_oracle(single_layout, n_q):
    case, model, lay, cache, olay, packed = single_layout
    lens = _lens(n_q)
    q = _queries(model, case, lens, n_q)
    ws = torch.empty(B.workspace_bytes(lay, BATCH, H_Q * n_q, H_KV, LENGTH), dtype=torch.uint8, device="cuda")
    out = torch.full((BATCH, n_q, H_Q, 128), float("nan"), device="cuda")
    B.decode_attention_multi(lay, q.cuda(), cache, lens.cuda(), CAP, LENGTH, out, ws, H_KV)
    torch.cuda.synchronize()
    assert lay.status() == 0
    got = out.cpu().double().numpy()
    G = H_Q // H_KV
    for b in range(BATCH):
        for h in range(H_KV):
            ref = O.decode_attention_multi(olay, q[b, :, h * G:(h + 1) * G].double().numpy(), packed[b, h],
                                           int(lens[b]), 1 / math.sqrt(128))
            for j in range(n_q):
                for c in range(G):
                    assert rel_l2(got[b, j, h * G + c], ref[j, c]) <= ATTN_REL_L2, (n_q, b, h, j, c)


def test_many_units_layout_set_match_oracle():
    case = Case(H_Q, H_KV, BATCH, LENGTH, 2, 2, torch.float16, 5e5, 82, capacity=CAP)
    model = synth.make_layer_model(H_Q, H_KV, case.seed)
    q_cal, k_cal = synth.make_calibration(model, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2, min_rate=0)
    q, k, v = synth.make_cache_inputs(model, BATCH, LENGTH, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(H_KV)]
    S = B.LayoutSet(layouts)
    cache = torch.zeros(S.cache_bytes(BATCH, CAP), dtype=torch.uint8, device="cuda")
    B.encode_append_heads(S, k.cuda(), v.cuda(), torch.zeros(BATCH, dtype=torch.int32, device="cuda"), cache, CAP)
    lens = _lens(1)
    ws = torch.empty(B.workspace_bytes(layouts[0], BATCH, H_Q, H_KV, LENGTH), dtype=torch.uint8, device="cuda")
    out = torch.full((BATCH, H_Q, 128), float("nan"), device="cuda")
    B.decode_attention_heads(S, q.cuda(), cache, lens.cuda(), CAP, LENGTH, out, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    got = out.cpu().double().numpy()
    G = H_Q // H_KV
    for h in range(H_KV):
        olay = O.make_layout(rates[h], case.v_bits, case.seed)
        for b in range(BATCH):
            want = O.pack(olay, O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy()), CAP)
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), want, int(lens[b]),
                                     1 / math.sqrt(128))
            for c in range(G):
                assert rel_l2(got[b, h * G + c], ref[c]) <= ATTN_REL_L2, (b, h, c)


def test_many_units_step_equals_append_then_attend(single_layout):
    """bgtq_decode_step over the 320 units (one new token per row at a ragged position):
    the cache bytes and outputs of encode_append followed by decode_attention, bit for bit
    (both of those are checked against the oracle above)."""
    case, model, lay, cache, olay, packed = single_layout
    gen = torch.Generator().manual_seed(83)
    lens0 = (_lens(1) - 1).cuda()  # rows of 0 .. 99 tokens before the step
    k_new = torch.randn(BATCH, 1, H_KV, 128, generator=gen).to(case.dtype).cuda()
    v_new = torch.randn(BATCH, 1, H_KV, 128, generator=gen).to(case.dtype).cuda()
    q = torch.randn(BATCH, H_Q, 128, generator=gen).to(case.dtype).cuda()
    ws = torch.empty(B.workspace_bytes(lay, BATCH, H_Q, H_KV, LENGTH), dtype=torch.uint8, device="cuda")
    c_sep, c_fus = cache.clone(), cache.clone()
    o_sep = torch.empty(BATCH, H_Q, 128, device="cuda")
    o_fus = torch.empty_like(o_sep)
    B.encode_append(lay, k_new, v_new, lens0, c_sep, CAP)
    B.decode_attention(lay, q, c_sep, lens0 + 1, CAP, LENGTH, o_sep, ws, H_KV)
    B.decode_step(lay, k_new, v_new, q, c_fus, lens0, CAP, LENGTH, o_fus, ws)
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)
    assert not torch.isnan(o_fus).any()
