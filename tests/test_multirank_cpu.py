"""Multi-rank host logic on CPU: world-size-2 gloo process groups.

Each rank computes (with the CPU oracle) decode attention for the units its shard owns;
rank 0 gathers and checks the union against one process doing every unit. The timing
reduction (sum of keys, max of time) is checked the same way. No GPU involved.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from packed_cache_decode_b200 import sharding, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_shards_partition_every_unit():
    for batch in (1, 2, 3, 4, 7, 8, 32):
        for h_kv in (1, 2, 8):
            for world in (1, 2, 3, 4, 8):
                seen = np.zeros((batch, h_kv), dtype=int)
                for r in range(world):
                    s = sharding.shard_units(batch, h_kv, r, world)
                    seen[s.b0:s.b1, s.h0:s.h1] += 1
                if batch * h_kv >= world or batch >= world:
                    assert np.all(seen == 1), (batch, h_kv, world)
                else:
                    assert np.all(seen >= 1)
    with pytest.raises(ValueError):
        sharding.shard_units(2, 2, 2, 2)


CASE = dict(h_q=8, h_kv=2, batch=3, length=150, k_bits=2, v_bits=2, theta=5e5, seed=5)


def _unit_outputs(shard):
    c = CASE
    m = synth.make_layer_model(c["h_q"], c["h_kv"], c["seed"])
    q_cal, k_cal = synth.make_calibration(m, 64, c["seed"] + 1, c["theta"])
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * c["k_bits"])
    lay = O.make_layout(rates, c["v_bits"], c["seed"])
    G = c["h_q"] // c["h_kv"]
    out = {}
    for b in range(shard.b0, shard.b1):
        for h in range(shard.h0, shard.h1):
            k = synth.key_slice(m, b, h, c["length"], 0, c["seed"], c["theta"]).double().numpy()
            v = synth.value_slice(m, b, h, c["length"], c["seed"]).double().numpy()
            q = torch.stack([synth.query_slice(m, b, h * G + i, 1, c["length"] - 1, c["seed"], c["theta"])[0]
                             for i in range(G)]).double().numpy()
            buf = O.pack(lay, O.encode(lay, k, v), 192)
            out[(b, h)] = O.decode_attention(lay, q, buf, c["length"], 1 / math.sqrt(128))
    return out


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shard = sharding.shard_units(CASE["batch"], CASE["h_kv"], rank, world)
        res = _unit_outputs(shard)
        gathered = [None] * world
        dist.all_gather_object(gathered, res)
        keys, ms = sharding.aggregate(shard.units * CASE["length"], 10.0 + rank, dist)
        if rank == 0:
            merged = {}
            for g in gathered:
                merged.update(g)
            q.put((merged, keys, ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_cover_the_batch_and_match_one_process():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    merged, keys, ms = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = _unit_outputs(sharding.Shard(0, CASE["batch"], 0, CASE["h_kv"]))
    assert set(merged) == set(full)
    for key in full:
        np.testing.assert_array_equal(merged[key], full[key])
    assert keys == CASE["batch"] * CASE["h_kv"] * CASE["length"]
    assert ms == 11.0


# ------------------------------------------------------------------ one sequence split over ranks
SEQ = dict(h_q=8, h_kv=2, length=333, k_bits=2, v_bits=2, theta=5e5, seed=9)


def _seq_setup():
    c = SEQ
    m = synth.make_layer_model(c["h_q"], c["h_kv"], c["seed"])
    q_cal, k_cal = synth.make_calibration(m, 64, c["seed"] + 1, c["theta"])
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * c["k_bits"])
    lay = O.make_layout(rates, c["v_bits"], c["seed"])
    G = c["h_q"] // c["h_kv"]
    units = []
    for h in range(c["h_kv"]):
        k = synth.key_slice(m, 0, h, c["length"], 0, c["seed"], c["theta"]).double().numpy()
        v = synth.value_slice(m, 0, h, c["length"], c["seed"]).double().numpy()
        q = torch.stack([synth.query_slice(m, 0, h * G + i, 1, c["length"] - 1, c["seed"], c["theta"])[0]
                         for i in range(G)]).double().numpy()
        enc = O.encode(lay, k, v)
        kh, vh = O.reconstruct(lay, enc["k_codes"], enc["k_norms"], enc["v_codes"], enc["v_norm"])
        units.append((q, kh, vh))
    return units


def _records(units, t0, t1):
    """Partial records [1, h_q, 130] of tokens [t0, t1): m in base-2 units, l, o'."""
    rec = []
    for q, kh, vh in units:
        m, l, o = O.partial_attention(q, kh[t0:t1], vh[t0:t1], 1 / math.sqrt(128))
        rec.append(np.concatenate([(m / math.log(2))[:, None], l[:, None], o], axis=1))
    return torch.from_numpy(np.concatenate(rec)[None])


def _merge_records(stacked):
    out = []
    for i in range(stacked.shape[2]):
        parts = [(stacked[r, 0, i, 0].item() * math.log(2) * np.ones(1), stacked[r, 0, i, 1].item() * np.ones(1),
                  stacked[r, 0, i, 2:].numpy()[None]) for r in range(stacked.shape[0])]
        out.append(O.merge_partials(parts)[0])
    return np.stack(out)


def _seq_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        units = _seq_setup()
        t0, t1 = sharding.token_range(SEQ["length"], rank, world)
        out = sharding.split_sequence_decode(lambda: _records(units, t0, t1), _merge_records, dist)
        q.put((rank, (t0, t1), out))
    finally:
        dist.destroy_process_group()


def test_token_ranges_cover_the_sequence_in_tiles():
    for length in (0, 1, 63, 64, 65, 333, 4096, 131072):
        for world in (1, 2, 3, 8):
            rs = [sharding.token_range(length, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == length
            for (a0, a1), (b0, b1) in zip(rs[:-1], rs[1:]):
                assert a1 == b0 and a0 <= a1
            assert all(a % 64 == 0 or a == length for a, _ in rs)
    with pytest.raises(ValueError):
        sharding.token_range(10, 2, 2)


def test_sequence_split_over_two_ranks_matches_one_process():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_seq_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    units = _seq_setup()
    full = np.concatenate([O.attention(qq, kh, vh, 1 / math.sqrt(128)) for qq, kh, vh in units])
    ranges = sorted(r[1] for r in results)
    assert ranges[0][0] == 0 and ranges[-1][1] == SEQ["length"] and ranges[0][1] == ranges[1][0]
    for _, _, out in results:                      # every rank ends with the whole result
        np.testing.assert_allclose(out, full, rtol=1e-10, atol=1e-12)
