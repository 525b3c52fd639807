"""Rate allocation per KV head through the C ABI: every KV head gets its own energy score,
rates and layout (its own groups, rotations and tile format), is cached in its own buffer
and decoded by its own call (h_kv = 1); each head matches the oracle with that head's
layout."""
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
