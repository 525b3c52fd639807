"""Layout variants through the C ABI against the oracle: norm correction ("TurboQuant:
paper algorithm and vLLM engineering implementation", vLLM column, box "NC": the stored
norm is |x| sqrt(d) / |c|) and fp16 norms.

The encode of a norm-corrected layout runs the four parts of a token as one thread-block
cluster (in the append kernel and in the first kernel of a decode step), so both launch
paths are covered; the decode reads fp16 norms in its own kernel variant.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle as O
from packed_cache_decode_b200 import binding as B

from .parity_util import Case, build_inputs, compare_packed, gpu_encode, oracle_slice, slice_bytes
from .test_gpu_parity import _run_case

pytestmark = pytest.mark.gpu

OPTIONS = {"nc": (True, False), "fp16": (False, True), "nc_fp16": (True, True)}
CASES = {
    "gqa4_bf16_k2v2": Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 41),
    "gqa8_bf16_k3v3": Case(16, 2, 1, 1000, 3, 3, torch.bfloat16, 1e6, 42),
    "gqa2_f32_k1v4_ragged": Case(4, 2, 1, 130, 1, 4, torch.float32, 5e5, 43),
}


def _with(case: Case, opt: str) -> Case:
    nc, fp16 = OPTIONS[opt]
    return dataclasses.replace(case, norm_correct=nc, norm_fp16=fp16)


@pytest.mark.parametrize("opt", list(OPTIONS))
@pytest.mark.parametrize("name", list(CASES))
def test_codes_norms_and_attention_match_oracle(name, opt):
    """Appended in three calls; codes bit-exact away from thresholds, norms to 1 ulp of
    their type, attention to the usual tolerance."""
    n_near, n_diff = _run_case(_with(CASES[name], opt), n_chunks=3)
    assert n_diff <= n_near


def test_layout_info_and_cache_bytes_follow_the_options():
    rates = np.array([4] * 8 + [3] * 8 + [2] * 24 + [1] * 24)
    for nc, fp16 in [(False, False), *OPTIONS.values()]:
        lay = B.Layout(rates, 2, 0, nc, fp16)
        olay = O.make_layout(rates, 2, 0, nc, fp16)
        assert lay.info.bytes_per_token == olay.bytes_per_token
        assert lay.info.tile_bytes == olay.tile_bytes
        assert lay.info.norm_bytes == (2 if fp16 else 4)
        assert lay.cache_bytes(3, 8, 1000) == O.cache_bytes(olay, 3, 8, 1000)


@pytest.mark.parametrize("opt", ["nc", "nc_fp16"])
def test_norm_corrected_cache_decodes_to_the_input_norms(opt):
    """The oracle's decode of the GPU-written cache restores each key group's and each
    value's input norm (to the rounding of the stored norm)."""
    case = _with(Case(4, 2, 1, 200, 2, 2, torch.float32, 5e5, 44), opt)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    cache_cpu = cache.cpu().numpy()
    olay = O.make_layout(rates, case.v_bits, case.seed, case.norm_correct, case.norm_fp16)
    tol = 2e-3 if case.norm_fp16 else 1e-6
    for h in range(case.h_kv):
        u = O.unpack(olay, slice_bytes(case, olay.tile_bytes, cache_cpu, 0, h), case.length)
        kh, vh = O.reconstruct(olay, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
        kk, vv = k[0, :, h].double().numpy(), v[0, :, h].double().numpy()
        for _, coords in olay.groups:
            np.testing.assert_allclose(np.linalg.norm(kh[:, coords], axis=1), np.linalg.norm(kk[:, coords], axis=1),
                                       rtol=tol)
        np.testing.assert_allclose(np.linalg.norm(vh, axis=1), np.linalg.norm(vv, axis=1), rtol=tol)


@pytest.mark.parametrize("n_new", [1, 5])
def test_step_with_options_equals_append_then_attend(n_new):
    """The decode step's first kernel runs the norm-corrected encode as clusters next to
    the q' blocks: same cache bytes and same outputs as the two separate calls."""
    case = Case(16, 4, 3, 700, 2, 2, torch.bfloat16, 5e5, 45, capacity=832, norm_correct=True, norm_fp16=True)
    model, rates, q, k, v = build_inputs(case)
    lay = B.Layout(rates, case.v_bits, case.seed, True, True).upload(0)
    pre = case.length - 64
    lens0 = torch.tensor([pre, pre - 61, 3], dtype=torch.int32, device="cuda")
    base = torch.zeros(lay.cache_bytes(case.batch, case.h_kv, case.cap), dtype=torch.uint8, device="cuda")
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
    ws = lambda: torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, msl), dtype=torch.uint8,
                             device="cuda")
    c_sep, c_fus = base.clone(), base.clone()
    o_sep = torch.empty(case.batch, case.h_q, 128, dtype=torch.float32, device="cuda")
    o_fus = torch.empty_like(o_sep)
    B.encode_append(lay, k_new, v_new, lens0, c_sep, case.cap)
    B.decode_attention(lay, qd, c_sep, lens0 + n_new, case.cap, msl, o_sep, ws(), case.h_kv)
    B.decode_step(lay, k_new, v_new, qd, c_fus, lens0, case.cap, msl, o_fus, ws())
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert torch.equal(c_sep, c_fus)
    assert torch.equal(o_sep, o_fus)
    # and the step's cache holds what the oracle writes for those rows
    cache_cpu = c_fus.cpu().numpy()
    for b in range(case.batch):
        n = int(lens0[b]) + n_new
        for h in range(case.h_kv):
            kk = torch.cat([k[b, :int(lens0[b]), h], k[b, pre:pre + n_new, h]]).double().numpy()
            vv = torch.cat([v[b, :int(lens0[b]), h], v[b, pre:pre + n_new, h]]).double().numpy()
            olay = O.make_layout(rates, case.v_bits, case.seed, True, True)
            enc = O.encode(olay, kk, vv)
            compare_packed(olay, enc, O.pack(olay, enc, case.cap), slice_bytes(case, olay.tile_bytes, cache_cpu, b, h),
                           case.cap)


def test_scores_with_fp16_norms_match_oracle():
    case = Case(16, 4, 2, 700, 2, 2, torch.bfloat16, 5e5, 46, norm_correct=True, norm_fp16=True)
    model, rates, q, k, v = build_inputs(case)
    lay, cache = gpu_encode(case, rates, k, v)
    lens = torch.tensor([case.length, case.length - 37], dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_bytes(lay, case.batch, case.h_q, case.h_kv, case.length), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((case.batch, case.h_q, case.length), float("nan"), dtype=torch.float32, device="cuda")
    B.decode_scores(lay, q.cuda().contiguous(), cache, lens, case.cap, case.length, out, ws, case.h_kv)
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    G = case.h_q // case.h_kv
    for b in range(case.batch):
        n = int(lens[b])
        for h in range(case.h_kv):
            olay, enc, buf = oracle_slice(case, rates, k, v, b, h)
            ref = O.decode_scores(olay, q[b, h * G:(h + 1) * G].double().numpy(), buf, n, 1 / math.sqrt(128))
            err = np.max(np.abs(got[b, h * G:(h + 1) * G, :n] - ref)) / np.max(np.abs(ref))
            assert err <= 2e-5, (b, h, err)
    assert lay.status() == 0

