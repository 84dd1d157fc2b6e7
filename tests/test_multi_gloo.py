"""Host-side multi-rank logic on CPU (gloo, world size 2): token sharding, pooling the raw
calibration accumulators across ranks, and the max-over-ranks timing reduction.

Each rank takes a contiguous token shard of one seeded batch, accumulates the oracle's
raw moments of its shard, and pools them with ``pool_moments``; the pooled accumulators
and the angles solved from them must equal the oracle on the whole batch.
"""
import datetime
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, T, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import synth
    from oracle import bitspec as B
    from oracle import definition as D
    from transform_rope_head_b200.distributed import max_over_ranks, pool_moments, token_shard
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = synth.make_inputs("llama32_1b", T=T, threads=1)
        w = inp["workload"]
        a, b = token_shard(T, rank, world)
        r = B.transform_quantize(inp["q"][a:b], inp["k"][a:b], inp["pos"][a:b], w.d_h,
                                 theta=w.theta, max_pos=w.max_pos, mode="rope_only",
                                 group=w.group, want_f32=True)
        m = torch.from_numpy(D.moments(r["q_f32"], r["k_f32"]))
        pool_moments(m)
        phi = D.solve_angles(m.numpy(), "pooled")
        tmax = max_over_ranks(0.5 + rank)
        out_q.put((rank, (a, b), m.numpy(), phi, tmax))
    finally:
        dist.destroy_process_group()


def test_token_shard_covers_every_token_once():
    from transform_rope_head_b200.distributed import token_shard
    for T in (0, 1, 7, 256, 131072, 131073):
        for world in (1, 2, 3, 8):
            spans = [token_shard(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        token_shard(10, 2, 2)


def test_two_rank_calibration_pooling_matches_whole_batch():
    import multiprocessing as mp

    import synth
    from oracle import bitspec as B
    from oracle import definition as D
    T, world = 301, 2                 # odd: the shards differ in size
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    inp = synth.make_inputs("llama32_1b", T=T, threads=1)
    w = inp["workload"]
    r = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta,
                             max_pos=w.max_pos, mode="rope_only", group=w.group, want_f32=True)
    m_all = D.moments(r["q_f32"], r["k_f32"])
    phi_all = D.solve_angles(m_all, "pooled")
    assert [x[1] for x in res] == [(0, 151), (151, 301)]
    for _, _, m, phi, tmax in res:
        np.testing.assert_allclose(m, m_all, rtol=1e-12, atol=1e-9)
        np.testing.assert_allclose(phi, phi_all, atol=1e-12)
        assert tmax == 1.5
