"""Parity at the benchmark's full sizes, sampled.

The whole layer is encoded and attended on the GPU with the same shapes (and so the
same split-K launch plan) as bench.py; the oracle then checks a few sampled
(batch row, KV head) units completely: every code byte of their caches and the
attention output of every query head that reads them.
"""
import math

import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B
from packed_cache_decode_b200 import synth

from .parity_util import ATTN_REL_L2, compare_packed, rel_l2

pytestmark = pytest.mark.gpu

FULL = {
    "llama8b_32k_k2v2": ("llama8b", [(0, 1), (0, 6)]),
    "qwen3b_128k_k3v3": ("qwen3b", [(0, 1)]),
    "llama70b_b4_128k_k2v2": ("llama70b", [(1, 3), (3, 7)]),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled_units(name):
    wl_name, samples = FULL[name]
    wl = synth.WORKLOADS[wl_name]
    m = synth.make_layer_model(wl.h_q, wl.h_kv, wl.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, wl.seed + 1, wl.theta)
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * wl.k_bits)
    L, Bt, G = wl.length, wl.batch, wl.h_q // wl.h_kv
    cap = 64 * math.ceil(L / 64)
    lay = B.Layout(rates, wl.v_bits, wl.seed).upload(0)
    cache = torch.zeros(lay.cache_bytes(Bt, wl.h_kv, cap), dtype=torch.uint8, device="cuda")
    q = torch.empty(Bt, wl.h_q, 128, dtype=wl.dtype)
    lens = torch.zeros(Bt, dtype=torch.int32, device="cuda")
    for b in range(Bt):                   # one batch row at a time keeps host memory small
        kb = torch.stack([synth.key_slice(m, b, h, L, 0, wl.seed, wl.theta) for h in range(wl.h_kv)], 1)
        vb = torch.stack([synth.value_slice(m, b, h, L, wl.seed) for h in range(wl.h_kv)], 1)
        for hq in range(wl.h_q):
            q[b, hq] = synth.query_slice(m, b, hq, 1, L - 1, wl.seed, wl.theta)[0].to(wl.dtype)
        kd = torch.zeros(Bt, L, wl.h_kv, 128, dtype=wl.dtype, device="cuda")
        vd = torch.zeros_like(kd)
        kd[b] = kb.to(wl.dtype).cuda()
        vd[b] = vb.to(wl.dtype).cuda()
        lens_b = torch.full((Bt,), cap, dtype=torch.int32, device="cuda")   # other rows: beyond capacity, skipped
        lens_b[b] = 0
        B.encode_append(lay, kd, vd, lens_b, cache, cap)
        torch.cuda.synchronize()
        del kd, vd
    if Bt > 1:
        assert lay.status() & B.STATUS_ENCODE_OVERFLOW   # the skipped rows were flagged, nothing written there
    lens.fill_(L)
    ws = torch.empty(B.workspace_bytes(lay, Bt, wl.h_q, wl.h_kv, L), dtype=torch.uint8, device="cuda")
    out = torch.empty(Bt, wl.h_q, 128, dtype=torch.float32, device="cuda")
    B.decode_attention(lay, q.cuda(), cache, lens, cap, L, out, ws, wl.h_kv)
    torch.cuda.synchronize()
    assert lay.status() == 0
    out = out.cpu().double().numpy()
    olay = O.make_layout(rates, wl.v_bits, wl.seed)
    per_unit = cap // 64 * olay.tile_bytes
    for b, h in samples:
        k = synth.key_slice(m, b, h, L, 0, wl.seed, wl.theta).to(wl.dtype).double().numpy()
        v = synth.value_slice(m, b, h, L, wl.seed).to(wl.dtype).double().numpy()
        enc = O.encode(olay, k, v)
        want = O.pack(olay, enc, cap)
        u = b * wl.h_kv + h
        got = cache[u * per_unit:(u + 1) * per_unit].cpu().numpy()
        near, near_diff = compare_packed(olay, enc, want, got, cap)
        ref = O.decode_attention(olay, q[b, h * G:(h + 1) * G].double().numpy(), want, L, 1 / math.sqrt(128))
        errs = [rel_l2(out[b, h * G + i], ref[i]) for i in range(G)]
        print(f"{name} unit ({b},{h}): near-threshold {near} (coded differently {near_diff}), "
              f"max rel L2 {max(errs):.2e}")
        assert max(errs) <= ATTN_REL_L2
