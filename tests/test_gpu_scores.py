"""bgtq_decode_scores (logits over the packed cache) through the C ABI against the oracle.

The logits use the attention's key path (q' hi + lo fragments, exact centroids, fp32
accumulation), so they agree with the fp64 oracle to about 2^-20 of their scale.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B

from .parity_util import Case, build_inputs, gpu_encode, oracle_slice

pytestmark = pytest.mark.gpu

SCORE_TOL = 2e-5   # max |gpu - oracle| / max |oracle| per (row, KV head)

CASES = {
    "gqa4_bf16_k2": Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 31),
    "gqa8_bf16_k3": Case(16, 2, 1, 1000, 3, 3, torch.bfloat16, 1e6, 32),
    "gqa1_f32_k4": Case(2, 2, 1, 129, 4, 1, torch.float32, 5e5, 33),
    "k1_uniform": Case(8, 2, 1, 300, 1, 1, torch.bfloat16, 5e5, 34),
    "gqa12_two_column_tiles": Case(24, 2, 2, 400, 2, 2, torch.bfloat16, 5e5, 35),
}


def _gpu_scores(lay, case, q, cache, lens, msl, ld):
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, msl), dtype=torch.uint8, device="cuda")
    out = torch.full((case.batch, case.h_q, ld), float("nan"), dtype=torch.float32, device="cuda")
    B.decode_scores(lay, q.cuda().contiguous(), cache, lens.to(torch.int32).cuda(), case.cap, msl, out, ws, case.h_kv)
    torch.cuda.synchronize()
    return out.cpu().double().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_scores_match_oracle(name):
    case = CASES[name]
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.tensor([case.length - 37 * b for b in range(case.batch)], dtype=torch.int32)
    ld = case.length + 3
    got = _gpu_scores(lay, case, q, cache, lens, case.length, ld)
    G = case.h_q // case.h_kv
    worst = 0.0
    for b in range(case.batch):
        n = int(lens[b])
        for h in range(case.h_kv):
            olay, enc, buf = oracle_slice(case, rates, k, v, b, h)
            ref = O.decode_scores(olay, q[b, h * G:(h + 1) * G].double().numpy(), buf, n, 1 / math.sqrt(128))
            g = got[b, h * G:(h + 1) * G]
            err = np.max(np.abs(g[:, :n] - ref)) / np.max(np.abs(ref))
            worst = max(worst, err)
            assert err <= SCORE_TOL, (b, h, err)
            assert np.all(np.isnan(g[:, n:]))          # nothing written past the row's length
    assert lay.status() == 0
    print(f"{name}: max relative score error {worst:.2e}")


def test_scores_give_the_attention_output():
    """softmax of the GPU logits times the oracle's decoded values reproduces the GPU
    attention output of the same call (to the attention tolerance)."""
    case = Case(8, 2, 1, 400, 2, 2, torch.bfloat16, 5e5, 35)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.full((1,), case.length, dtype=torch.int32)
    s = _gpu_scores(lay, case, q, cache, lens, case.length, case.length)
    G = case.h_q // case.h_kv
    ws = torch.empty(B.workspace_bytes(lay, 1, case.h_q, case.h_kv, case.length), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, case.h_q, 128, dtype=torch.float32, device="cuda")
    B.decode_attention(lay, q.cuda(), cache, lens.cuda(), case.cap, case.length, out, ws, case.h_kv)
    out = out.cpu().double().numpy()
    for h in range(case.h_kv):
        olay, enc, buf = oracle_slice(case, rates, k, v, 0, h)
        u = O.unpack(olay, buf, case.length)
        _, vh = O.reconstruct(olay, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
        sh = s[0, h * G:(h + 1) * G]
        p = np.exp(sh - sh.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        want = p @ vh
        for i in range(G):
            err = np.linalg.norm(out[0, h * G + i] - want[i]) / np.linalg.norm(want[i])
            assert err <= 2e-3, (h, i, err)


def test_scores_reject_short_rows():
    lay = B.Layout(np.full(64, 2), 2, 0).upload(0)
    cache = torch.zeros(lay.cache_bytes(1, 1, 64), dtype=torch.uint8, device="cuda")
    q = torch.zeros(1, 1, 128, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, 1, 32, device="cuda")
    with pytest.raises(B.BgtqError):
        B.decode_scores(lay, q, cache, lens, 64, 64, s, ws, 1)      # scores_ld 32 < max_seq_len 64
