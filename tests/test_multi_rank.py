"""The N > 1 path on CPU: two gloo ranks run bench.py's rank plumbing
(barrier, max over ranks, whole-job rate) and decode disjoint canvas shards
with the oracle (replicas need no collective on the data path)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from oracle import dlm_oracle as O
    import workloads as W
    w, r, local, pg = bench.dist_init(world, backend="gloo")
    dev = torch.device("cpu")
    bench.barrier(pg, dev)
    # per-rank "elapsed ms": the slowest rank decides
    ms = 10.0 * (rank + 1)
    ms_max = bench.max_over_ranks(pg, ms, dev)
    rate = bench.aggregate_rate(w, 100, ms_max)
    # each rank decodes its own shard of canvases (mask corruption: no RNG)
    wl = W.small_workload("mr", d_model=64, n_heads=2, n_kv_heads=1, head_dim=16, vocab=200,
                          dtype="f32", prefix_kind="tokens", prefix_len=(8, 20), batch=4,
                          canvas=8, steps=4, quota=2)
    weights = W.make_weights(wl.shape, seed=1)
    lens, toks, _, _ = W.make_prefix(wl, seed=1)
    mine = [b for b in range(wl.batch) if b % w == r]
    om = O.OracleModel(O.ModelDims.of(wl.shape), weights)
    for i, b in enumerate(mine):
        om.kv_append_tokens(i, toks[b])
    p = O.SamplerParams(canvas=8, steps=4, quota=2)
    st = O.init_canvas(len(mine), p, wl.shape.mask_id, wl.shape.vocab)
    O.decode_block(om, st, p)
    np.savez(os.path.join(out_dir, "r%d.npz" % r), rate=rate, ms_max=ms_max,
             tokens=st.tokens, mine=np.array(mine))
    bench.barrier(pg, dev)
    pg.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = np.load(tmp_path / "r0.npz")
    r1 = np.load(tmp_path / "r1.npz")
    assert float(r0["ms_max"]) == float(r1["ms_max"]) == 20.0
    assert abs(float(r0["rate"]) - 2 * 100 / 0.020) < 1e-6
    # the shards together equal one process decoding every canvas
    import sys
    sys.path.insert(0, ROOT)
    from oracle import dlm_oracle as O
    import workloads as W
    wl = W.small_workload("mr", d_model=64, n_heads=2, n_kv_heads=1, head_dim=16, vocab=200,
                          dtype="f32", prefix_kind="tokens", prefix_len=(8, 20), batch=4,
                          canvas=8, steps=4, quota=2)
    weights = W.make_weights(wl.shape, seed=1)
    lens, toks, _, _ = W.make_prefix(wl, seed=1)
    om = O.OracleModel(O.ModelDims.of(wl.shape), weights)
    for b in range(4):
        om.kv_append_tokens(b, toks[b])
    p = O.SamplerParams(canvas=8, steps=4, quota=2)
    st = O.init_canvas(4, p, wl.shape.mask_id, wl.shape.vocab)
    O.decode_block(om, st, p)
    for r in (r0, r1):
        for i, b in enumerate(r["mine"]):
            assert np.array_equal(r["tokens"][i], st.tokens[b])
