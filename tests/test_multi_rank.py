"""The N > 1 benchmark path on CPU: world-size-2 gloo ranks take disjoint
shards of the sequences and reduce only their elapsed times (max over ranks)
into the whole-job token rate.  No GPU."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WL = dict(name="t", batch=3, heads=2, d_k=64, d_v=64, steps=4, window=4, n_comp=1, gate="scalar",
          io="bf16", smoothing=True, outlier_rows=1, outlier_cols=1, outlier_scale=30.0)


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from linear_attention_recurrent_int8_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = bench._dist()
        seqs = list(bench.shard(r, w, 5))
        elapsed = 10.0 * (rank + 1)          # rank 1 is the slow one
        ms, rate = bench.aggregate(elapsed, 5 * 16, w)
        tok = bench.shard_tokens(synth.DecodeWorkload(**WL), r, w, 4, 8, "cpu")
        out.put((rank, seqs, ms, rate, {k: v.float().numpy() for k, v in tok.items()}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res = sorted(res, key=lambda r: r[0])
    shards = [r[1] for r in res]
    assert shards == [[0, 1, 2, 3, 4], [5, 6, 7, 8, 9]]
    for _, _, ms, rate, _ in res:
        assert ms == 20.0                      # max over ranks
        assert rate == pytest.approx(2 * 5 * 16 / 0.020)   # all ranks' tokens / max time
    # the two ranks' inputs are the two halves of one rank's draw over the global batch
    from linear_attention_recurrent_int8_b200 import synth
    wl = synth.DecodeWorkload(**WL)
    one = bench.shard_tokens(synth.DecodeWorkload(**dict(WL, batch=2 * WL["batch"])), 0, 1, 4, 8, "cpu")
    for rank, *_, tok in res:
        sl = slice(rank * wl.batch, (rank + 1) * wl.batch)
        for key, val in tok.items():
            np.testing.assert_array_equal(val, one[key][sl].float().numpy(), err_msg=key)


def test_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        bench.shard(2, 2, 4)
    with pytest.raises(ValueError):
        bench.shard(0, 1, 0)
    assert list(bench.shard(0, 1, 3)) == [0, 1, 2]
