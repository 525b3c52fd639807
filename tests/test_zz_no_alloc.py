"""The no-allocation decode entry point against the regular one.

Some callers cannot call cudaMalloc (servers that give all device memory to their own
pool, plugins whose framework forbids allocation while they execute), so the library
offers bgtq_decode_attention_noalloc, which keeps its split-K scratch in a fixed
device array instead of a caller workspace. This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from packed_cache_decode_b200 import binding as B

from .parity_util import ATTN_REL_L2, Case, build_inputs, gpu_encode, rel_l2

pytestmark = pytest.mark.gpu


def _regular(lay, case, q, cache, lens):
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    B.decode_attention(lay, q, cache, lens, case.cap, case.length, out, ws, case.h_kv)
    return out


def test_noalloc_matches_regular_decode_twice():
    lib = B.load()
    assert lib.bgtq_noalloc_scratch_capacity() == 8 << 20
    case = Case(16, 4, 2, 1500, 2, 2, torch.bfloat16, 5e5, 21)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    qd = q.cuda().contiguous()
    lens = torch.full((case.batch,), case.length, dtype=torch.int32, device="cuda")
    want = _regular(lay, case, qd, cache, lens).cpu().double().numpy()
    for call in range(2):              # the second call reuses the scratch the first left behind
        out = torch.full((case.batch, case.h_q, 128), float("nan"), dtype=torch.float32, device="cuda")
        B.decode_attention_noalloc(lay, qd, cache, lens, case.cap, case.length, out, case.h_kv)
        torch.cuda.synchronize()
        got = out.cpu().double().numpy()
        for b in range(case.batch):
            for h in range(case.h_q):
                assert rel_l2(got[b, h], want[b, h]) <= ATTN_REL_L2, (call, b, h)
    assert lay.status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lay = B.Layout(np.full(64, 2), 2, 0).upload(0)
    cap = 64
    cache = torch.zeros(lay.cache_bytes(1024, 8, cap), dtype=torch.uint8, device="cuda")
    q = torch.zeros(1024, 64, 128, device="cuda")
    lens = torch.zeros(1024, dtype=torch.int32, device="cuda")
    out = torch.zeros(1024, 64, 128, device="cuda")
    need = B.workspace_bytes(lay, 1024, 64, 8, cap)
    assert need > 8 << 20
    with pytest.raises(B.BgtqError) as e:
        B.decode_attention_noalloc(lay, q, cache, lens, cap, cap, out, 8)
    assert e.value.status == B.ERR_WORKSPACE
    assert "scratch" in str(e.value)
