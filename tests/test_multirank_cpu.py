"""The multi-GPU path's host logic on CPU: world_size 2 over gloo.

Each rank drafts its shard of the request rows with the oracle (the rows are
independent) and the gathered result equals one process drafting all rows;
the job time is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_draft_model_dspark_b200.sharding import max_over_ranks, shard_rows


def test_shard_rows_cover_disjoint():
    for A in (0, 1, 3, 4, 32, 33, 64):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(A, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == A
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0 and a0 <= a1
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(4, 2, 2)


def _tiny_round(rows):
    from oracle import dspark as O
    from synthetic import ModelShape, make_weights
    m = ModelShape(hidden_size=32, num_hidden_layers=1, num_attention_heads=4, global_head_dim=16,
                   num_global_key_value_heads=2, intermediate_size=48, vocab_size=64, block_size=3,
                   mask_token_id=63, markov_rank=8, rope_theta=1e4, partial_rotary_factor=0.5, dtype="fp32")
    W = O.OracleWeights(make_weights(m, 3, markov_scale=30.0), m)
    g = torch.Generator().manual_seed(1)
    A = 5
    hid = torch.randn(A, 6, m.hidden_size, generator=g)
    lens = [6, 2, 5, 1, 4]
    anchors = [3, 9, 12, 40, 7]
    kv = O.project_context_kv(W, hid[rows[0]:rows[1]], [0] * (rows[1] - rows[0]), lengths=lens[rows[0]:rows[1]])
    out = O.draft_rows(W, kv, anchors[rows[0]:rows[1]], lens[rows[0]:rows[1]])
    return out["tokens"], out["conf"]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = shard_rows(5, world, rank)
        toks, conf = _tiny_round((lo, hi))
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi, toks, conf))
        slowest = max_over_ranks(0.5 + rank)
        if rank == 0:
            q.put((gathered, slowest))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gloo_match_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered, slowest = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert slowest == 1.5
    toks = np.concatenate([g[2] for g in sorted(gathered)])
    conf = np.concatenate([g[3] for g in sorted(gathered)])
    ref_t, ref_c = _tiny_round((0, 5))
    np.testing.assert_array_equal(toks, ref_t)
    np.testing.assert_allclose(conf, ref_c, rtol=1e-12)
