"""The multi-GPU host logic with two gloo ranks on the CPU.

Each rank owns a disjoint block of sequences (no data exchange); the only collectives
are the barrier and the max of per-rank times.  Here every rank runs the oracle's
state updates on its own sequences, and the gathered result must equal one process
running all sequences.  A second test drives the benchmark's own per-rank plan (the
residual seeds each rank runs, the max-over-ranks device time, the whole-job
throughput) on two ranks and checks it against one process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hybrid_deltanet_attention_kva_b200 import multi


def test_rank_sequences_partition():
    for n_seq in (1, 5, 8, 13):
        for world in (1, 2, 3, 8):
            owned = [multi.rank_sequences(n_seq, r, world) for r in range(world)]
            flat = [s for o in owned for s in o]
            assert flat == list(range(n_seq))          # disjoint, contiguous, complete
            assert max(map(len, owned)) - min(map(len, owned)) <= 1
    assert len({multi.rank_seed(1003, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n_seq, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import kva_inputs as KI
    from oracle import kva_ref as R
    multi.init("gloo", timeout_s=60)
    geom = KI.TINY
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, 31).items()}
    st = KI.make_states(geom, n_seq, 32, std=0.1)
    mix = KI.make_mixer_inputs(geom, n_seq, 40, 33)
    res = {}
    for s in multi.rank_sequences(n_seq, rank, world):
        kc = [np.zeros((geom.attn_n_kv, 96, geom.attn_d_h))]
        vc = [np.zeros_like(kc[0])]
        S, tail = R.update_states(mix[s].double().numpy(), geom, P, st["state"][s].double().numpy(),
                                  st["conv_tail"][s].double().numpy(), kc, vc, 7 * s)
        res[s] = (S, tail, kc[0])
    multi.barrier()
    mx = multi.max_over_ranks(float(rank + 1) * 0.5)
    gathered = [None] * world
    dist.all_gather_object(gathered, res)
    if rank == 0:
        merged = {}
        for g in gathered:
            assert not set(g) & set(merged)          # no sequence computed twice
            merged.update(g)
        torch.save({"merged": merged, "max": mx}, os.path.join(out_dir, "result.pt"))
    multi.finish()


def test_two_gloo_ranks_equal_one_process(tmp_path):
    n_seq, world = 5, 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, n_seq, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    out = torch.load(os.path.join(tmp_path, "result.pt"), weights_only=False)
    assert out["max"] == 1.0
    merged = out["merged"]
    assert sorted(merged) == list(range(n_seq))

    import kva_inputs as KI
    from oracle import kva_ref as R
    geom = KI.TINY
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, 31).items()}
    st = KI.make_states(geom, n_seq, 32, std=0.1)
    mix = KI.make_mixer_inputs(geom, n_seq, 40, 33)
    for s in range(n_seq):
        kc = [np.zeros((geom.attn_n_kv, 96, geom.attn_d_h))]
        vc = [np.zeros_like(kc[0])]
        S, tail = R.update_states(mix[s].double().numpy(), geom, P, st["state"][s].double().numpy(),
                                  st["conv_tail"][s].double().numpy(), kc, vc, 7 * s)
        np.testing.assert_array_equal(merged[s][0], S)
        np.testing.assert_array_equal(merged[s][1], tail)
        np.testing.assert_array_equal(merged[s][2], kc[0])


def _bench_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import kva_inputs as KI
    from oracle import kva_ref as R
    multi.init("gloo", timeout_s=60)
    geom, T = KI.TINY, 12
    W = R.weights_to_f64(KI.make_projector_weights(geom, 1001))
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, 1002).items()}
    seeds = bench.rank_residual_seeds(1001, rank)
    S = np.zeros((geom.n_gdn, geom.gdn_n_v, geom.gdn_d_v, geom.gdn_d_k))
    tail = np.zeros((geom.n_gdn, 3, geom.gdn_conv_ch))
    kc = [np.zeros((geom.attn_n_kv, T * len(seeds), geom.attn_d_h))]
    vc = [np.zeros_like(kc[0])]
    for i, sd in enumerate(seeds):           # the rank's own sequence, ubatch after ubatch
        res = KI.make_residual(geom, T, sd, dtype=torch.float32, n_outliers=0).double().numpy()
        _, S, tail = R.prefill_ubatch(res, W, geom, P, S, tail, kc, vc, i * T)
    multi.barrier()
    local_ms = 10.0 * (rank + 1)             # a stand-in for this rank's device time
    ms = multi.max_over_ranks(local_ms)
    value = bench.job_throughput(world, 3, T, ms)
    gathered = [None] * world
    dist.all_gather_object(gathered, {"rank": rank, "seeds": seeds, "S": S, "tail": tail, "k": kc[0],
                                      "ms": ms, "value": value})
    if rank == 0:
        torch.save(gathered, os.path.join(out_dir, "bench_ranks.pt"))
    multi.finish()


def test_bench_per_rank_plan_on_two_gloo_ranks(tmp_path):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import kva_inputs as KI
    from oracle import kva_ref as R
    world = 2
    mp.start_processes(_bench_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = torch.load(os.path.join(tmp_path, "bench_ranks.pt"), weights_only=False)
    # every rank runs its own sequence: the seeds differ between ranks
    assert not set(got[0]["seeds"]) & set(got[1]["seeds"])
    # the job's time is the slowest rank's, and the value counts every rank's tokens
    for g in got:
        assert g["ms"] == 20.0
        assert g["value"] == world * 3 * 12 / 0.020
    # each rank's result equals one process running that rank's plan
    geom, T = KI.TINY, 12
    W = R.weights_to_f64(KI.make_projector_weights(geom, 1001))
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, 1002).items()}
    for g in got:
        assert g["seeds"] == bench.rank_residual_seeds(1001, g["rank"])
        S = np.zeros((geom.n_gdn, geom.gdn_n_v, geom.gdn_d_v, geom.gdn_d_k))
        tail = np.zeros((geom.n_gdn, 3, geom.gdn_conv_ch))
        kc = [np.zeros((geom.attn_n_kv, T * len(g["seeds"]), geom.attn_d_h))]
        vc = [np.zeros_like(kc[0])]
        for i, sd in enumerate(g["seeds"]):
            res = KI.make_residual(geom, T, sd, dtype=torch.float32, n_outliers=0).double().numpy()
            _, S, tail = R.prefill_ubatch(res, W, geom, P, S, tail, kc, vc, i * T)
        np.testing.assert_array_equal(g["S"], S)
        np.testing.assert_array_equal(g["tail"], tail)
        np.testing.assert_array_equal(g["k"], kc[0])
