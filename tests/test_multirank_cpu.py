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
