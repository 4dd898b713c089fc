"""Sequence sharding on the CPU: the segment-map decomposition against the fp64
oracle on the whole sequence, and the exchange itself (gated_delta_rule_140_b200.seqshard)
on gloo ranks with the oracle standing in for each rank's GPU.

The decomposition: over a segment the recurrence is affine in its starting state,
S_end = S_start M + B, with B the final state from a zero state and M the final
state from the identity with v = 0 (FG2-GDN section 1's transition A_t =
Diag(alpha_t)(I - beta_t k_t k_t^T), composed over the segment); the outputs of a
segment run from its true start are the whole sequence's outputs there."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_140_b200 import seqshard
from gated_delta_rule_140_b200.inputs import prefill_inputs


def _problem(decay, T=150, B=2, H=2, d=8, seed=5):
    g = torch.Generator().manual_seed(seed)
    return prefill_inputs(B, T, H, d, d, dtype=torch.float32, decay=decay, seed=seed,
                          init_std=0.3, gen=g, alpha_shift=1.0 if decay == "scalar" else 1.5)


def _ops():
    """The three operations of the exchange in fp64 on the CPU: the oracle's
    recurrence, a plain matrix product and an identity."""
    def prefill(q, k, v, log_alpha, beta, s0):
        o, sf = oracle.recurrent(q, k, v, log_alpha, beta, s0)
        return torch.from_numpy(o), torch.from_numpy(sf)

    def compose(s, m, b):
        return s @ m + b

    def identity(n, h, d, like):
        return torch.eye(d, dtype=torch.float64).expand(n, h, d, d).clone()

    return prefill, compose, identity


def _seg(x, a, b):
    return {k: x[k][:, a:b] for k in ("q", "k", "v", "log_alpha", "beta")}


@pytest.mark.parametrize("decay,bounds", [("scalar", [0, 37, 64, 121, 150]),
                                          ("channel", [0, 37, 64, 121, 150]),
                                          ("scalar", [0, 50, 50, 150])])  # an empty segment
def test_segment_maps_compose_to_the_whole_sequence(decay, bounds):
    x = _problem(decay)
    ro, rs = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    prefill, compose, identity = _ops()
    maps, outs = [], []
    for r in range(len(bounds) - 1):
        s = _seg(x, bounds[r], bounds[r + 1])
        if r == 0:
            o, se = prefill(**s, s0=x["initial_state"])
            maps.append((torch.zeros_like(se), se))
            outs.append(o)
        else:
            maps.append(seqshard.segment_map(**s, prefill=prefill, identity=identity))
    for r in range(1, len(bounds) - 1):
        s0 = seqshard.start_state(maps, r, compose=compose)
        o, se = prefill(**_seg(x, bounds[r], bounds[r + 1]), s0=s0)
        outs.append(o)
    o = torch.cat(outs, dim=1).numpy()
    assert np.abs(o - ro).max() <= 1e-10 * max(1.0, np.abs(ro).max())
    assert np.abs(se.numpy() - rs).max() <= 1e-10 * max(1.0, np.abs(rs).max())
    # the map itself: S_end = S_start M + B for an arbitrary start (a short
    # segment, so that M is far from zero)
    s = _seg(x, 64, 68)
    m_map, b_map = seqshard.segment_map(**s, prefill=prefill, identity=identity)
    s_any = torch.randn(2, 2, 8, 8, dtype=torch.float64, generator=torch.Generator().manual_seed(9))
    _, se = prefill(**s, s0=s_any)
    assert torch.allclose(se, s_any @ m_map + b_map, atol=1e-12, rtol=0)
    # and the order matters: M S + B is not the map
    assert m_map.abs().max() > 1e-2
    assert not torch.allclose(se, m_map @ s_any + b_map, atol=1e-6)


def test_balanced_bounds():
    # rank 0 takes three shares (one pass), every other rank one share (three passes)
    b = seqshard.balanced_bounds(65536, 8)
    assert b[0] == 0 and b[-1] == 65536 and len(b) == 9
    lens = np.diff(b)
    assert all(x % 64 == 0 for x in b[:-1])
    assert abs(lens[0] - 3 * 65536 / 10) <= 64 and all(abs(x - 65536 / 10) <= 128 for x in lens[1:])
    # per-rank passes x tokens are balanced: max / min close to 1
    work = [lens[0]] + [3 * x for x in lens[1:]]
    assert max(work) / min(work) < 1.05
    assert seqshard.balanced_bounds(100, 1) == [0, 100]
    assert seqshard.balanced_bounds(0, 3) == [0, 0, 0, 0]
    small = seqshard.balanced_bounds(130, 3)
    assert small[0] == 0 and small[-1] == 130 and list(small) == sorted(small)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, decay, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = _problem(decay, T=130)
        edges = np.linspace(0, 130, world + 1).astype(int)
        edges[1] += 7  # ragged
        s = _seg(x, edges[rank], edges[rank + 1])
        prefill, compose, identity = _ops()
        o, se = seqshard.sequence_sharded_prefill(**s, initial_state=x["initial_state"],
                                                  prefill=prefill, compose=compose,
                                                  identity=identity)
        got = [None] * world
        dist.all_gather_object(got, (o.numpy(), se.numpy()))
        if rank == 0:
            ro, rs = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      x["initial_state"])
            o_all = np.concatenate([g[0] for g in got], axis=1)
            ok = (np.abs(o_all - ro).max() <= 1e-10 * max(1.0, np.abs(ro).max()) and
                  np.abs(got[-1][1] - rs).max() <= 1e-10 * max(1.0, np.abs(rs).max()))
            np.save(os.path.join(result_dir, "ok.npy"), np.array([ok]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,decay", [(1, "scalar"), (2, "scalar"), (3, "channel")])
def test_sequence_sharded_prefill_on_gloo_ranks(tmp_path, world, decay):
    mp.start_processes(_worker, args=(world, _free_port(), decay, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    assert bool(np.load(tmp_path / "ok.npy")[0])
