"""Rate allocation per KV head through the C ABI: every KV head gets its own energy score,
rates and layout (its own groups, rotations and tile format). Each head is cached and
decoded either by its own calls (h_kv = 1) or, through a layout set, together with the
other heads in one call; each head matches the oracle with that head's layout."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, Case, compare_packed, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("min_rate", [1, 0])
def test_per_head_layouts_match_oracle(min_rate):
    case = Case(16, 4, 2, 500, 2, 2, torch.bfloat16, 5e5, 61)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    per = O.block_energy_heads(q_cal.double().numpy(), k_cal.double().numpy())
    rates = np.stack([O.greedy_rates(per[h], O.lloyd_max_mse_table(), min_rate, 4, 128) for h in range(case.h_kv)])
    np.testing.assert_array_equal(rates, B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2, min_rate=min_rate))
    q, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    G = case.h_q // case.h_kv
    lens = torch.tensor([500, 433], dtype=torch.int32, device="cuda")
    for h in range(case.h_kv):
        lay = B.Layout(rates[h], case.v_bits, case.seed).upload(0)
        cache = torch.zeros(lay.cache_bytes(case.batch, 1, case.cap), dtype=torch.uint8, device="cuda")
        B.encode_append(lay, k[:, :, h:h + 1].contiguous().cuda(), v[:, :, h:h + 1].contiguous().cuda(),
                        torch.zeros(case.batch, dtype=torch.int32, device="cuda"), cache, case.cap)
        ws = torch.empty(B.workspace_bytes(lay, case.batch, G, 1, case.length), dtype=torch.uint8, device="cuda")
        out = torch.empty(case.batch, G, 128, device="cuda")
        B.decode_attention(lay, q[:, h * G:(h + 1) * G].contiguous().cuda(), cache, lens, case.cap, case.length,
                           out, ws, 1)
        torch.cuda.synchronize()
        assert lay.status() == 0
        olay = O.make_layout(rates[h], case.v_bits, case.seed)
        cache_cpu = cache.cpu().numpy().reshape(case.batch, -1)
        got = out.cpu().double().numpy()
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            want = O.pack(olay, enc, case.cap)
            compare_packed(olay, enc, want, cache_cpu[b], case.cap)
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), want, int(lens[b]),
                                     1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(got[b, i], ref[i]) <= ATTN_REL_L2, (h, b, i)


def _head_tiles(cache, batch, h_kv, n_tiles, stride, tile_bytes, b, h):
    """The first tile_bytes of every tile of (row b, head h) in a cache of tile stride `stride`."""
    return cache.view(batch, h_kv, n_tiles, stride)[b, h, :, :tile_bytes]


@pytest.mark.parametrize("shape", [(16, 4, 0), (16, 2, 1), (32, 2, 1)], ids=["gqa4_min0", "gqa8_min1", "gqa16_two_column_tiles"])
def test_layout_set_one_call_matches_oracle(shape):
    """A layout set: one encode and one attention call for every KV head, each head with its
    own layout. The tiles equal those of the head's own single-layout cache byte for byte,
    the outputs match the oracle per query head, the logits equal the single-head calls'."""
    h_q, h_kv, min_rate = shape
    case = Case(h_q, h_kv, 2, 500, 2, 2, torch.bfloat16, 5e5, 62)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2, min_rate=min_rate)
    assert len({tuple(r) for r in rates}) > 1                      # the heads' layouts differ
    q, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(h_kv)]
    S = B.LayoutSet(layouts)
    stride, n_tiles = S.tile_bytes, case.cap // 64
    assert stride == max(lay.tile_bytes for lay in layouts)
    cache = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    kd, vd = k.cuda(), v.cuda()
    # bulk appends (>= 4 tokens) and a 3-token append (the per-token encoder)
    for a0, a1 in ((0, 300), (300, 303), (303, 500)):
        lens0 = torch.full((case.batch,), a0, dtype=torch.int32, device="cuda")
        B.encode_append_heads(S, kd[:, a0:a1].contiguous(), vd[:, a0:a1].contiguous(), lens0, cache, case.cap)
    torch.cuda.synchronize()
    assert S.status() == 0
    G = h_q // h_kv
    lens = torch.tensor([500, 433], dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, h_q, h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((case.batch, h_q, 128), float("nan"), device="cuda")
    B.decode_attention_heads(S, q.cuda(), cache, lens, case.cap, case.length, out, ws)
    ld = case.length + 5
    sc = torch.full((case.batch, h_q, ld), float("nan"), device="cuda")
    B.decode_scores_heads(S, q.cuda(), cache, lens, case.cap, case.length, sc, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    got = out.cpu().double().numpy()
    for h, lay in enumerate(layouts):
        # the head's own cache, written and read through the single-layout calls
        own = torch.zeros(lay.cache_bytes(case.batch, 1, case.cap), dtype=torch.uint8, device="cuda")
        B.encode_append(lay, kd[:, :, h:h + 1].contiguous(), vd[:, :, h:h + 1].contiguous(),
                        torch.zeros(case.batch, dtype=torch.int32, device="cuda"), own, case.cap)
        ws1 = torch.empty(B.workspace_bytes(lay, case.batch, G, 1, case.length), dtype=torch.uint8, device="cuda")
        sc1 = torch.full((case.batch, G, ld), float("nan"), device="cuda")
        B.decode_scores(lay, q[:, h * G:(h + 1) * G].contiguous().cuda(), own, lens, case.cap, case.length, sc1, ws1, 1)
        torch.cuda.synchronize()
        assert lay.status() == 0
        for b in range(case.batch):
            mine = own.view(case.batch, n_tiles, lay.tile_bytes)[b]
            assert torch.equal(_head_tiles(cache, case.batch, h_kv, n_tiles, stride, lay.tile_bytes, b, h), mine), (h, b)
        assert torch.equal(sc[:, h * G:(h + 1) * G].isnan(), sc1.isnan())
        assert torch.equal(sc[:, h * G:(h + 1) * G].nan_to_num(), sc1.nan_to_num()), h
        olay = O.make_layout(rates[h], case.v_bits, case.seed)
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), O.pack(olay, enc, case.cap),
                                     int(lens[b]), 1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(got[b, h * G + i], ref[i]) <= ATTN_REL_L2, (h, b, i)


def test_layout_set_rejects_mixed_layouts():
    a = B.Layout(np.full(64, 2), 2, 0).upload(0)
    b = B.Layout(np.full(64, 2), 3, 0).upload(0)          # another value rate
    c = B.Layout(np.full(64, 2), 2, 1).upload(0)          # another seed (value rotation)
    for pair in ((a, b), (a, c)):
        with pytest.raises(B.BgtqError) as e:
            B.LayoutSet(pair)
        assert e.value.status == B.ERR_INVALID
    with pytest.raises(B.BgtqError):
        B.LayoutSet([a, B.Layout(np.full(64, 2), 2, 0)])   # not uploaded


@pytest.mark.parametrize("n_new", [1, 5])
def test_layout_set_step_equals_append_then_attend(n_new):
    """bgtq_decode_step_heads: the fused append + attend over a layout set gives the cache
    bytes and outputs of encode_append_heads followed by decode_attention_heads, and each
    head's outputs match the oracle over the grown rows."""
    case = Case(16, 4, 2, 400, 2, 2, torch.bfloat16, 5e5, 63, capacity=448)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2)
    q, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(case.h_kv)]
    S = B.LayoutSet(layouts)
    pre = case.length - n_new
    kd, vd = k.cuda(), v.cuda()
    base = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    B.encode_append_heads(S, kd[:, :pre].contiguous(), vd[:, :pre].contiguous(),
                          torch.zeros(case.batch, dtype=torch.int32, device="cuda"), base, case.cap)
    lens0 = torch.full((case.batch,), pre, dtype=torch.int32, device="cuda")
    k_new, v_new = kd[:, pre:].contiguous(), vd[:, pre:].contiguous()
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, case.h_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    c_sep, c_fus = base.clone(), base.clone()
    o_sep = torch.empty(case.batch, case.h_q, 128, device="cuda")
    o_fus = torch.empty_like(o_sep)
    B.encode_append_heads(S, k_new, v_new, lens0, c_sep, case.cap)
    B.decode_attention_heads(S, q.cuda(), c_sep, lens0 + n_new, case.cap, case.length, o_sep, ws)
    B.decode_step_heads(S, k_new, v_new, q.cuda(), c_fus, lens0, case.cap, case.length, o_fus, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)
    G = case.h_q // case.h_kv
    got = o_fus.cpu().double().numpy()
    for h in range(case.h_kv):
        olay = O.make_layout(rates[h], case.v_bits, case.seed)
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), O.pack(olay, enc, case.cap),
                                     case.length, 1 / math.sqrt(128))
            for i in range(G):
                assert rel_l2(got[b, h * G + i], ref[i]) <= ATTN_REL_L2, (h, b, i)


def test_layout_set_paged_equals_contiguous():
    """A layout set over a paged cache (pages handed out in shuffled order): the same tiles
    as the contiguous layout-set cache, byte for byte, and the same outputs, bit for bit."""
    case = Case(16, 4, 2, 300, 2, 2, torch.bfloat16, 5e5, 64)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2)
    q, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(case.h_kv)]
    S = B.LayoutSet(layouts)
    n_tiles = case.cap // 64
    num_pages = case.batch * n_tiles + 3
    perm = np.random.default_rng(5).permutation(num_pages)[:case.batch * n_tiles].astype(np.int32)
    pc = B.PagedCache(torch.zeros(S.paged_pool_bytes(num_pages), dtype=torch.uint8, device="cuda"),
                      torch.from_numpy(perm.reshape(case.batch, n_tiles)).cuda())
    cont = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    kd, vd = k.cuda(), v.cuda()
    for a0, a1 in ((0, 250), (250, 252), (252, 300)):
        lens0 = torch.full((case.batch,), a0, dtype=torch.int32, device="cuda")
        B.encode_append_heads(S, kd[:, a0:a1].contiguous(), vd[:, a0:a1].contiguous(), lens0, cont, case.cap)
        B.encode_append_paged_heads(S, kd[:, a0:a1].contiguous(), vd[:, a0:a1].contiguous(), lens0, pc)
    torch.cuda.synchronize()
    assert S.status() == 0
    tb = S.tile_bytes
    pv = pc.pool.view(num_pages, case.h_kv, tb)
    cv = cont.view(case.batch, case.h_kv, n_tiles, tb)
    for b in range(case.batch):
        for i in range(n_tiles):
            assert torch.equal(pv[int(perm[b * n_tiles + i])], cv[b, :, i]), (b, i)
    lens = torch.tensor([300, 241], dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, case.h_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    o1 = torch.empty(case.batch, case.h_q, 128, device="cuda")
    o2 = torch.empty_like(o1)
    B.decode_attention_heads(S, q.cuda(), cont, lens, case.cap, case.length, o1, ws)
    B.decode_attention_paged_heads(S, q.cuda(), pc, lens, case.length, o2, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("shape", [(16, 4, 2), (12, 4, 3), (32, 2, 2)], ids=["gqa4_nq2", "gqa3_nq3", "gqa16_nq2_32cols"])
def test_layout_set_multi_token_matches_oracle(shape):
    """decode_attention_multi_heads: n_q query tokens per row (causal among them) over a
    layout set, each KV head against the oracle's multi-token attention with its own layout."""
    h_q, h_kv, n_q = shape
    case = Case(h_q, h_kv, 2, 400, 2, 2, torch.float16, 5e5, 65)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2, min_rate=0)
    _, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    layouts = [B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(h_kv)]
    S = B.LayoutSet(layouts)
    cache = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    B.encode_append_heads(S, k.cuda(), v.cuda(), torch.zeros(case.batch, dtype=torch.int32, device="cuda"), cache,
                          case.cap)
    lens = torch.tensor([400, 317], dtype=torch.int32)
    q = torch.empty(case.batch, n_q, h_q, 128, dtype=case.dtype)
    for b in range(case.batch):
        for hq in range(h_q):
            q[b, :, hq] = synth.query_slice(m, b, hq, n_q, int(lens[b]) - n_q, case.seed, case.theta).to(case.dtype)
    ws = torch.empty(B.workspace_bytes(layouts[0], case.batch, h_q * n_q, h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((case.batch, n_q, h_q, 128), float("nan"), device="cuda")
    B.decode_attention_multi_heads(S, q.cuda(), cache, lens.cuda(), case.cap, case.length, out, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    G = h_q // h_kv
    n_tiles = case.cap // 64
    cv = cache.view(case.batch, h_kv, n_tiles, S.tile_bytes).cpu().numpy()
    got = out.cpu().double().numpy()
    for h in range(h_kv):
        olay = O.make_layout(rates[h], case.v_bits, case.seed)
        for b in range(case.batch):
            enc = O.encode(olay, k[b, :, h].double().numpy(), v[b, :, h].double().numpy())
            want = O.pack(olay, enc, case.cap)
            compare_packed(olay, enc, want, np.ascontiguousarray(cv[b, h, :, :olay.tile_bytes]).reshape(-1), case.cap)
            ref = O.decode_attention_multi(olay, q[b, :, h * G:(h + 1) * G].double().numpy(), want, int(lens[b]),
                                           1 / math.sqrt(128))
            for j in range(n_q):
                for c in range(G):
                    assert rel_l2(got[b, j, h * G + c], ref[j, c]) <= ATTN_REL_L2, (h, b, j, c)


def _set_with_prefix(h_q, h_kv, pre, seed, capacity):
    case = Case(h_q, h_kv, 2, pre + 8, 2, 2, torch.bfloat16, 5e5, seed, capacity=capacity)
    m = synth.make_layer_model(case.h_q, case.h_kv, case.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, case.seed + 1, case.theta)
    rates = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), 2)
    _, k, v = synth.make_cache_inputs(m, case.batch, case.length, case.seed, case.theta, case.dtype)
    S = B.LayoutSet([B.Layout(rates[h], case.v_bits, case.seed).upload(0) for h in range(h_kv)])
    return case, S, k.cuda(), v.cuda()


@pytest.mark.parametrize("n_new", [2, 3])
def test_layout_set_multi_step_equals_append_then_attend(n_new):
    """decode_step_multi_heads: the new tokens' own queries over a layout set (12 columns per
    KV head at n_new = 3: two column tiles) give the cache bytes and outputs of
    encode_append_heads followed by decode_attention_multi_heads (oracle-checked above)."""
    case, S, kd, vd = _set_with_prefix(16, 4, 300, 66, 320)
    pre = 300
    base = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    B.encode_append_heads(S, kd[:, :pre].contiguous(), vd[:, :pre].contiguous(),
                          torch.zeros(case.batch, dtype=torch.int32, device="cuda"), base, case.cap)
    lens0 = torch.tensor([pre, pre - 37], dtype=torch.int32, device="cuda")
    k_new, v_new = kd[:, pre:pre + n_new].contiguous(), vd[:, pre:pre + n_new].contiguous()
    q = torch.randn(case.batch, n_new, case.h_q, 128, generator=torch.Generator().manual_seed(7)).to(case.dtype).cuda()
    ws = torch.empty(B.workspace_bytes(S.layouts[0], case.batch, case.h_q * n_new, case.h_kv, case.length),
                     dtype=torch.uint8, device="cuda")
    c_sep, c_fus = base.clone(), base.clone()
    o_sep = torch.empty(case.batch, n_new, case.h_q, 128, device="cuda")
    o_fus = torch.empty_like(o_sep)
    B.encode_append_heads(S, k_new, v_new, lens0, c_sep, case.cap)
    B.decode_attention_multi_heads(S, q, c_sep, lens0 + n_new, case.cap, case.length, o_sep, ws)
    B.decode_step_multi_heads(S, k_new, v_new, q, c_fus, lens0, case.cap, case.length, o_fus, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)
    assert not torch.isnan(o_fus).any()


def test_layout_set_paged_step_equals_contiguous_step():
    """decode_step_paged_heads on a paged cache (shuffled pages) against decode_step_heads on
    the contiguous cache: the same tiles byte for byte and the same outputs bit for bit."""
    case, S, kd, vd = _set_with_prefix(16, 4, 250, 67, 320)
    pre = 250
    n_tiles = case.cap // 64
    num_pages = case.batch * n_tiles + 2
    perm = np.random.default_rng(9).permutation(num_pages)[:case.batch * n_tiles].astype(np.int32)
    pc = B.PagedCache(torch.zeros(S.paged_pool_bytes(num_pages), dtype=torch.uint8, device="cuda"),
                      torch.from_numpy(perm.reshape(case.batch, n_tiles)).cuda())
    cont = torch.zeros(S.cache_bytes(case.batch, case.cap), dtype=torch.uint8, device="cuda")
    zero = torch.zeros(case.batch, dtype=torch.int32, device="cuda")
    B.encode_append_heads(S, kd[:, :pre].contiguous(), vd[:, :pre].contiguous(), zero, cont, case.cap)
    B.encode_append_paged_heads(S, kd[:, :pre].contiguous(), vd[:, :pre].contiguous(), zero, pc)
    lens0 = torch.tensor([pre, 191], dtype=torch.int32, device="cuda")  # 191: the new token opens tile 2
    k_new, v_new = kd[:, pre:pre + 1].contiguous(), vd[:, pre:pre + 1].contiguous()
    q = torch.randn(case.batch, case.h_q, 128, generator=torch.Generator().manual_seed(8)).to(case.dtype).cuda()
    ws = torch.empty(B.workspace_bytes(S.layouts[0], case.batch, case.h_q, case.h_kv, case.length),
                     dtype=torch.uint8, device="cuda")
    o1 = torch.empty(case.batch, case.h_q, 128, device="cuda")
    o2 = torch.empty_like(o1)
    B.decode_step_heads(S, k_new, v_new, q, cont, lens0, case.cap, case.length, o1, ws)
    B.decode_step_paged_heads(S, k_new, v_new, q, pc, lens0, case.length, o2, ws)
    torch.cuda.synchronize()
    assert S.status() == 0
    tb = S.tile_bytes
    pv = pc.pool.view(num_pages, case.h_kv, tb)
    cv = cont.view(case.batch, case.h_kv, n_tiles, tb)
    for b in range(case.batch):
        for i in range(n_tiles):
            assert torch.equal(pv[int(perm[b * n_tiles + i])], cv[b, :, i]), (b, i)
    assert torch.equal(o1, o2)
    assert not torch.isnan(o1).any()
