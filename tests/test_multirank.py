"""The N > 1 data-parallel path on the CPU with the gloo backend (world size 2):
sequences are sharded across ranks by token count, each rank computes its
shard (here with the fp64 oracle, standing in for one GPU's gdn_chunk_fwd), and
the gathered results equal one run over the whole batch.  The benchmark's
max-over-ranks timing reduction is exercised the same way."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_140_b200.shard import local_batch, shard_sequences


def test_shard_sequences_balances_and_covers():
    lens = [256, 4096, 1000, 3000, 77, 2048, 2048, 500]
    for world in (1, 2, 3, 8):
        parts = shard_sequences(lens, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(lens)))  # every sequence exactly once
        loads = [sum(lens[i] for i in p) for p in parts]
        # LPT bound: max load <= mean + max sequence
        assert max(loads) <= sum(lens) / world + max(lens)
    assert shard_sequences(lens, 2) == shard_sequences(list(lens), 2)  # deterministic
    with pytest.raises(ValueError):
        shard_sequences(lens, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from gated_delta_rule_140_b200.inputs import prefill_inputs
        g = torch.Generator().manual_seed(51)
        lens = [37, 130, 64, 5, 90]
        x = prefill_inputs(1, 0, 2, 16, 16, dtype=torch.float32, seed=51, init_std=0.1,
                           lengths=lens, gen=g)
        seqs = shard_sequences(lens, world)[rank]
        xl = local_batch(x, seqs)
        o, sf = oracle.recurrent(xl["q"], xl["k"], xl["v"], xl["log_alpha"], xl["beta"],
                                 xl["initial_state"], xl["cu_seqlens"], nthreads=1)
        # gather every rank's (sequence ids, outputs, final states)
        obj = (seqs, o, sf, xl["cu_seqlens"].tolist())
        gathered = [None] * world
        dist.all_gather_object(gathered, obj)
        # max over ranks, as the benchmark reduces its timings
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            np.save(os.path.join(result_dir, "max.npy"), t.numpy())
            ro, rs = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      x["initial_state"], x["cu_seqlens"], nthreads=1)
            cu = x["cu_seqlens"].tolist()
            ok = True
            for seqs_r, o_r, sf_r, cu_r in gathered:
                for j, i in enumerate(seqs_r):
                    a = o_r[0, cu_r[j]:cu_r[j + 1]]
                    b = ro[0, cu[i]:cu[i + 1]]
                    ok &= bool(np.allclose(a, b, atol=1e-12)) and bool(
                        np.allclose(sf_r[j], rs[i], atol=1e-12))
            np.save(os.path.join(result_dir, "ok.npy"), np.array([ok]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_shards_match_the_whole_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    assert bool(np.load(tmp_path / "ok.npy")[0])
    assert float(np.load(tmp_path / "max.npy")[0]) == 2.0
