"""Request sharding of a batch over ranks (request b -> rank b mod G, chunks
gathered back in request order), on CPU: the index logic, and a world-size-2
gloo run in which each rank denoises its share with the oracle (standing in
for that rank's GPU call) and the gathered batch equals the unsharded one.
The oracle is the check here, not part of the sharding code."""
import os
import socket

import numpy as np
import pytest

from vla_flow_matching_denoise_b200 import shard, synth

torch = pytest.importorskip("torch")

SHAPE = synth.ExpertShape(1, 64, 2, 1, 32, 128, 6, 5, 2, batch=5)


def test_rank_requests_partition_the_batch():
    for B in (0, 1, 5, 64):
        for G in (1, 2, 3, 8):
            parts = [shard.rank_requests(B, r, G) for r in range(G)]
            flat = sorted(i for p in parts for i in p)
            assert flat == list(range(B))
            assert all(i % G == r for r, p in enumerate(parts) for i in p)
            assert max(len(p) for p in parts) - min(len(p) for p in parts) <= 1
    with pytest.raises(ValueError):
        shard.rank_requests(4, 2, 2)


def test_single_rank_gather_is_identity():
    a = np.arange(12.0).reshape(3, 2, 2)
    assert shard.gather_in_order(a, 3, 0, 1, None) is a
    with pytest.raises(ValueError):
        shard.gather_in_order(a, 4, 0, 1, None)


def _inputs():
    raw = synth.make_weights(SHAPE)
    kp, vp = synth.make_prefix(SHAPE)
    x0 = synth.make_x0(SHAPE)
    return raw, kp, vp, x0


def _oracle_run(raw, x, k, v):
    from oracle import fm_oracle as O
    s = synth.ExpertShape(**{**SHAPE.__dict__, "batch": x.shape[0]})
    return O.denoise(x, s.steps, raw, list(k), list(v), s)


def _worker(rank, ws, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    raw, kp, vp, x0 = _inputs()
    out = shard.denoise_sharded(lambda x, k, v: _oracle_run(raw, x, k, v), x0, kp, vp, rank, ws, dist)
    q.put((rank, out))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_batch_in_request_order():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp = torch.multiprocessing.get_context("spawn")
    q = mp.Queue()
    ps = [mp.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(2))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    raw, kp, vp, x0 = _inputs()
    ref = _oracle_run(raw, x0, kp, vp)
    for r in (0, 1):
        assert res[r].shape == ref.shape
        assert np.array_equal(res[r], ref)      # same per-request arithmetic, same order
