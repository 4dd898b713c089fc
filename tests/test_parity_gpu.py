"""GPU parity: gdn_chunk_fwd and gdn_recurrent_step (through the C ABI) against
the fp64 oracle on the same seeded inputs.

Reduced cases span several 64-token chunks and a ragged tail and are compared
element by element over every head; the full-size workloads run on the GPU in
the launch configuration the benchmark times and are compared on sampled
(sequence, head) chains, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_140_b200 import _native as nat
from gated_delta_rule_140_b200 import chunk_fwd, recurrent_step
from gated_delta_rule_140_b200.inputs import (WORKLOADS, decode_inputs, prefill_inputs,
                                              workload_inputs)
from tests.parity_util import TOL, gpu_head, oracle_heads, record_margin, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _run(x, **kw):
    d = to_dev(x)
    o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                      d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o, sf


def _full_compare(x, o, sf, dtype):
    ro, rs = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              x["initial_state"], x["cu_seqlens"])
    to, ts = TOL[dtype]
    eo, es = rel_err(o, ro), rel_err(sf, rs)
    assert eo <= to, f"o error {eo:.3g} > {to}"
    assert es <= ts, f"final-state error {es:.3g} > {ts}"
    return eo, es


# --------------------------------------------------------------------------- #
# reduced cases, every element                                                #
# --------------------------------------------------------------------------- #
def test_tiny_fp32_workload(cuda_ok):
    """B=1, H=2, T=256, d=64, fp32, chunk 64, zero initial state, seed 0."""
    x = workload_inputs("gdn_tiny_fp32")
    o, sf = _run(x)
    _full_compare(x, o, sf, torch.float32)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("decay", ["scalar", "channel"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("path", ["default", "pool", "pair", "cuda_cores"])
def test_reduced_ragged(cuda_ok, dtype, decay, d, path):
    """Several chunks and a ragged tail (T = 3*64 + 37), with an initial state,
    on each prefill kernel that takes the shape (the pool kernel is GDN only)."""
    if path == "pool" and decay == "channel":
        pytest.skip("the pool kernel takes scalar decay")
    x = prefill_inputs(2, 229, 3, d, d, dtype=dtype, decay=decay, seed=21,
                       alpha_shift=2.0 if decay == "scalar" else 3.0, init_std=0.05)
    o, sf = _run(x, cuda_cores=path == "cuda_cores", pair=path == "pair", pool=path == "pool")
    _full_compare(x, o, sf, dtype)


@pytest.mark.parametrize("decay", ["scalar", "channel"])
def test_varlen_with_empty_and_short_sequences(cuda_ok, decay):
    lens = [0, 1, 63, 64, 65, 200, 0, 130]
    g = torch.Generator().manual_seed(22)
    x = prefill_inputs(1, 0, 4, 128, 128, dtype=torch.bfloat16, decay=decay,
                       alpha_shift=2.0 if decay == "scalar" else 3.0, init_std=0.02,
                       lengths=lens, gen=g)
    o, sf = _run(x)
    _full_compare(x, o, sf, torch.bfloat16)
    # empty sequences: the final state is the initial state, bit for bit
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(sf[n].cpu(), x["initial_state"][n])


def test_final_state_may_alias_initial_state(cuda_ok):
    x = prefill_inputs(2, 150, 2, 128, 128, dtype=torch.bfloat16, seed=23, init_std=0.05)
    d = to_dev(x)
    o_ref, sf_ref = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                              d["initial_state"].clone())
    s = d["initial_state"].clone()
    o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], s, final_state=s)
    torch.cuda.synchronize()
    assert sf.data_ptr() == s.data_ptr()
    assert torch.equal(o, o_ref) and torch.equal(s, sf_ref)


def test_no_final_state_and_deterministic(cuda_ok):
    x = prefill_inputs(1, 300, 2, 128, 128, dtype=torch.bfloat16, seed=24)
    d = to_dev(x)
    o1, sf1 = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                        output_final_state=False)
    o2, _ = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"])
    torch.cuda.synchronize()
    assert sf1 is None
    assert torch.equal(o1, o2), "two runs differ"


def test_segment_chaining_on_device(cuda_ok):
    """prefill(T1) then prefill(T2, S0 = final) agrees with prefill(T1 + T2)."""
    x = prefill_inputs(1, 320, 2, 128, 128, dtype=torch.bfloat16, seed=25, init_std=0.02)
    d = to_dev(x)
    o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"])
    a, b = slice(0, 128), slice(128, 320)
    cut = lambda t, s: t[:, s].contiguous()
    oa, sa = chunk_fwd(*(cut(d[n], a) for n in ("q", "k", "v", "log_alpha", "beta")),
                       d["initial_state"])
    ob, sb = chunk_fwd(*(cut(d[n], b) for n in ("q", "k", "v", "log_alpha", "beta")), sa)
    torch.cuda.synchronize()
    assert rel_err(torch.cat([oa, ob], 1).float(), o.float().cpu().numpy()) < 1e-2
    assert rel_err(sb, sf.cpu().numpy()) < 1e-2


def test_bad_cu_seqlens_reported_by_workspace_status(cuda_ok):
    x = prefill_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, seed=26)
    d = to_dev(x)
    cu = torch.tensor([0, 200, 100, 256], dtype=torch.int32, device="cuda")  # not monotone
    ws = nat.Workspace()
    chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, cu, workspace=ws)
    assert ws.status() == nat.GDN_ERR_DEVICE_INPUT
    assert ws.status() == nat.GDN_OK  # the word is cleared by the read
    cu = torch.tensor([0, 100, 200, 256], dtype=torch.int32, device="cuda")
    chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, cu, workspace=ws)
    assert ws.status() == nat.GDN_OK


def test_check_flag_raises_on_bad_cu_seqlens(cuda_ok):
    """chunk_fwd(check=True) turns the sticky device word into an exception."""
    x = prefill_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, seed=26)
    d = to_dev(x)
    bad = torch.tensor([0, 200, 100, 256], dtype=torch.int32, device="cuda")
    with pytest.raises(nat.GdnError) as ei:
        chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, bad, check=True)
    assert ei.value.status == nat.GDN_ERR_DEVICE_INPUT
    good = torch.tensor([0, 100, 200, 256], dtype=torch.int32, device="cuda")
    o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, good, check=True)
    x["cu_seqlens"] = good.cpu()
    _full_compare(x, o, sf, torch.bfloat16)
    recurrent_step(d["q"][0, :2], d["k"][0, :2], d["v"][0, :2], d["log_alpha"][0, :2],
                   d["beta"][0, :2], torch.zeros(2, 2, 128, 128, device="cuda"), check=True)


TC_KERNELS = [("one_cta", "scalar"), ("pair", "scalar"), ("pair", "channel"),
              ("pool", "scalar")]


@pytest.mark.parametrize("kind,decay", TC_KERNELS)
def test_bounded_waits_expire_cleanly(cuda_ok, kind, decay):
    """The test-only header word shortens every data wait to 200 SM cycles, so
    the waits run out: the kernel records GDN_ERR_TIMEOUT, drains its own copies
    and MMAs, frees its tensor memory and returns.  A normal call on the same
    workspace, process and GPU right after is exact again (nothing left hung or
    allocated)."""
    x = prefill_inputs(2, 600, 2, 128, 128, dtype=torch.bfloat16, decay=decay,
                       alpha_shift=2.0 if decay == "scalar" else 3.0, seed=33, init_std=0.05)
    d = to_dev(x)
    kw = {kind: True}
    ws = nat.Workspace()
    ws.get(nat.workspace_size(nat.prefill_dims(d["q"], d["v"], d["log_alpha"], **kw)))
    ws.set_wait_limit(200)
    chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
              workspace=ws, **kw)
    assert ws.status() == nat.GDN_ERR_TIMEOUT
    ws.set_wait_limit(0)
    for _ in range(2):
        o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                          workspace=ws, check=True, **kw)
        _full_compare(x, o, sf, torch.bfloat16)


def test_tensor_core_and_cuda_core_paths_agree(cuda_ok):
    x = prefill_inputs(2, 512, 4, 128, 128, dtype=torch.bfloat16, seed=27, init_std=0.02)
    d = to_dev(x)
    assert nat.chunk_fwd_path(nat.prefill_dims(d["q"], d["v"], d["log_alpha"])) == "tensor_core"
    assert nat.chunk_fwd_path(nat.prefill_dims(d["q"], d["v"], d["log_alpha"], pair=True)) == \
        "tensor_core_pair"
    o1, s1 = _run(x)
    for kw in ({"cuda_cores": True}, {"pair": True}):
        o2, s2 = _run(x, **kw)
        assert rel_err(o1, o2.float().cpu().numpy()) < 2e-2
        assert rel_err(s1, s2.cpu().numpy()) < 1e-2


def test_kda_pair_kernel_is_exact_for_any_decay_in_one_launch(cuda_ok):
    """KDA runs on the two-CTA tensor-core kernel for every decay, in one launch.
    Off the diagonal 16-token blocks the products are referenced at the row
    block's start (both factors <= 1); inside a diagonal block a channel whose
    decay over the block passes e^-80 is left out of the factored product and its
    exact terms are added from a correction table.  Cases: mild decay; the KDA
    workload's (log alpha ~ -3); -30 per token on 8 channels of head 0 (e^-480
    over a block); -30 on every channel of head 0; channels straddling the
    block-decay limit (-4.9 and -5.1 per token: 16 tokens give -78 and -82)."""
    cases = [((-2.0, 31), None), ((3.0, 30), None), ((3.0, 30), ("ch8", -30.0)),
             ((3.0, 34), ("all", -30.0)), ((3.0, 35), ("edge", None))]
    for (shift, seed), strong in cases:
        x = prefill_inputs(2, 200, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                           alpha_shift=shift, seed=seed, init_std=0.05)
        if strong is not None:
            kind, val = strong
            if kind == "ch8":
                x["log_alpha"][:, :, 0, :8] = val
            elif kind == "all":
                x["log_alpha"][:, :, 0, :] = val
            else:
                x["log_alpha"][:, :, 0, 0:4] = -4.9
                x["log_alpha"][:, :, 0, 4:8] = -5.1
                x["log_alpha"][:, :, 1, 8:12] = -100.0
        d = to_dev(x)
        assert nat.chunk_fwd_path(nat.prefill_dims(d["q"], d["v"], d["log_alpha"])) == \
            "tensor_core_pair"
        n0 = nat.launch_count()
        o, sf = _run(x)
        assert nat.launch_count() - n0 == 1, "one launch, no re-run"
        _full_compare(x, o, sf, torch.bfloat16)
    # final state aliasing the initial state, with fast-decaying channels
    x = prefill_inputs(2, 200, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                       alpha_shift=3.0, seed=30, init_std=0.05)
    x["log_alpha"][:, :, 0, :8] = -30.0
    d = to_dev(x)
    ref_o, ref_s = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                             d["initial_state"].clone(), cuda_cores=True)
    s = d["initial_state"].clone()
    o2, _ = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], s, final_state=s)
    torch.cuda.synchronize()
    assert rel_err(o2, ref_o.float().cpu().numpy()) < 2e-2
    assert rel_err(s, ref_s.cpu().numpy()) < 1e-2


def _fg2_compare(x, o, sf):
    ro, rs = oracle.fg2_recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None,
                                  x["initial_state"], x["cu_seqlens"])
    to, ts = TOL[torch.bfloat16]
    eo, es = rel_err(o, ro), rel_err(sf, rs)
    assert eo <= to, f"o error {eo:.3g} > {to}"
    assert es <= ts, f"final-state error {es:.3g} > {ts}"


@pytest.mark.parametrize("case", ["ragged", "packed", "fast_channels"])
def test_fg2_rate_per_key_channel_matches_oracle(cuda_ok, case):
    """FG2-GDN: beta [B,T,H,d_k], keys scaled by sqrt(beta) in the two-CTA
    kernel's gate pass, unit rate in the delta-rule step; against the oracle's
    FG2 recurrence (which its pins tie to KDA and to KDA's chunkwise form).
    Ragged sequences, a packed batch with empty ones, and fast-forgetting
    channels (the exact diagonal-block correction with scaled keys)."""
    if case == "packed":
        x = prefill_inputs(1, 0, 3, 128, 128, dtype=torch.bfloat16, decay="channel",
                           alpha_shift=3.0, init_std=0.05, lengths=[0, 1, 65, 200, 0, 130],
                           gen=torch.Generator().manual_seed(81), beta_channel=True)
    else:
        x = prefill_inputs(2, 229, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                           alpha_shift=3.0, seed=82, init_std=0.05, beta_channel=True)
        if case == "fast_channels":
            x["log_alpha"][:, :, 0, :8] = -30.0
    d = to_dev(x)
    assert nat.chunk_fwd_path(nat.prefill_dims(d["q"], d["v"], d["log_alpha"],
                                               beta_channel=True)) == "tensor_core_pair"
    o, sf = _run(x, check=True)
    _fg2_compare(x, o, sf)


@pytest.mark.parametrize("case", ["ragged", "packed"])
def test_fg2plus_value_rate_matches_oracle(cuda_ok, case):
    """FG2-GDN+: a value-side rate beta_v [B,T,H,d_v] with FG2-GDN's key-side one;
    v is scaled by sqrt(beta_v) into the workspace (gdn_chunk_fwd_value_rate) and
    the FG2-GDN prefill runs on it.  Against the oracle's FG2 recurrence with the
    value gate; rates of exactly 1 leave the FG2-GDN result unchanged."""
    g = torch.Generator().manual_seed(84)
    if case == "packed":
        x = prefill_inputs(1, 0, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                           alpha_shift=3.0, init_std=0.05, lengths=[0, 70, 200, 1, 129],
                           gen=g, beta_channel=True)
    else:
        x = prefill_inputs(2, 229, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                           alpha_shift=3.0, init_std=0.05, gen=g, beta_channel=True)
    bv = torch.sigmoid(torch.randn(x["v"].shape, generator=g) + 1.0)
    d = to_dev(x)
    o, sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                      d["cu_seqlens"], beta_v=bv.cuda(), check=True)
    torch.cuda.synchronize()
    ro, rs = oracle.fg2_recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], bv,
                                  x["initial_state"], x["cu_seqlens"])
    to, ts = TOL[torch.bfloat16]
    eo, es = rel_err(o, ro), rel_err(sf, rs)
    assert eo <= to and es <= ts, (eo, es)
    # unit value rates: FG2-GDN bit for bit (sqrt(1) = 1, the same bf16 values)
    o1, s1 = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                       d["cu_seqlens"], beta_v=torch.ones_like(bv).cuda(), check=True)
    o0, s0 = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                       d["cu_seqlens"], check=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o0) and torch.equal(s1, s0)


def test_kda_log_alpha_4_byte_aligned_gives_identical_results(cuda_ok):
    """The ABI asks 4-byte alignment of log alpha; the KDA gate pass loads channel
    pairs as float2 when the pointer allows and one float at a time otherwise.
    Both read the same values and sum them in the same order: bit-identical."""
    x = prefill_inputs(2, 200, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                       alpha_shift=3.0, seed=32, init_std=0.05)
    d = to_dev(x)
    o1, s1 = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"])
    n = d["log_alpha"].numel()
    buf = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    la = buf[1:].view(d["log_alpha"].shape)
    la.copy_(d["log_alpha"])
    assert la.data_ptr() % 8 == 4
    o2, s2 = chunk_fwd(d["q"], d["k"], d["v"], la, d["beta"], d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("decay", ["scalar", "channel"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 128, 129, 640])
def test_pair_kernel_chunk_counts(cuda_ok, T, decay):
    """The two-CTA kernel with 1..10 chunks per sequence: both local groups (GDN)
    or the one group on both ring slots (KDA), odd and even chunk counts, a
    one-token sequence."""
    x = prefill_inputs(2, T, 2, 128, 128, dtype=torch.bfloat16, decay=decay,
                       alpha_shift=2.0 if decay == "scalar" else 3.0, seed=28 + T,
                       init_std=0.05)
    o, sf = _run(x, pair=True)
    _full_compare(x, o, sf, torch.bfloat16)


def test_pair_kernel_strong_and_zero_decay(cuda_ok):
    """log alpha from -20 to 0 per token: block decays that underflow, chunks
    with no decay at all."""
    x = prefill_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, seed=29, init_std=0.05)
    la = x["log_alpha"]
    la[:, :64] = -20.0
    la[:, 64:128] = 0.0
    for kw in ({}, {"pair": True}, {"pool": True}, {"one_cta": True}):
        o, sf = _run(x, **kw)
        _full_compare(x, o, sf, torch.bfloat16)


# --------------------------------------------------------------------------- #
# the pool kernel: chunk-local work on a pool of SMs, chains on chain SMs     #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("T", [1, 63, 64, 65, 128, 129, 640, 1000])
def test_pool_kernel_chunk_counts(cuda_ok, T):
    """1..16 chunks per sequence: both local groups, every ring slot, partial
    last chunks, a one-token sequence."""
    x = prefill_inputs(2, T, 2, 128, 128, dtype=torch.bfloat16, seed=60 + T, init_std=0.05)
    o, sf = _run(x, pool=True)
    _full_compare(x, o, sf, torch.bfloat16)


@pytest.mark.parametrize("nch", ["1", "3", "7"])
def test_pool_kernel_chain_rounds(cuda_ok, monkeypatch, nch):
    """Fewer chain CTAs than chains: each chain CTA runs several chains one after
    another (rounds), the ring slots are reused across chains."""
    monkeypatch.setenv("GDN_POOL_CHAIN_CTAS", nch)
    x = prefill_inputs(3, 300, 4, 128, 128, dtype=torch.bfloat16, seed=70, init_std=0.05)
    o, sf = _run(x, pool=True)
    _full_compare(x, o, sf, torch.bfloat16)


@pytest.mark.parametrize("nch", ["0", "2", "5"])
def test_pool_kernel_packed_batch(cuda_ok, monkeypatch, nch):
    """Packed sequences of 0..700 tokens (empty ones too), initial states; rounds
    padded to their longest chain (empty padding tasks)."""
    if nch != "0":
        monkeypatch.setenv("GDN_POOL_CHAIN_CTAS", nch)
    lens = [0, 1, 63, 64, 65, 200, 0, 130, 700, 5, 0]
    g = torch.Generator().manual_seed(71)
    x = prefill_inputs(1, 0, 3, 128, 128, dtype=torch.bfloat16, init_std=0.02, lengths=lens,
                       gen=g)
    d = to_dev(x)
    assert nat.chunk_fwd_path(nat.prefill_dims(d["q"], d["v"], d["log_alpha"], d["cu_seqlens"],
                                               pool=True)) == "tensor_core_pool"
    o, sf = _run(x, pool=True, check=True)
    _full_compare(x, o, sf, torch.bfloat16)
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(sf[n].cpu(), x["initial_state"][n])


def test_pool_kernel_matches_pair_kernel_bitwise_in_local_products(cuda_ok):
    """The pool and two-CTA kernels share the chunk-local arithmetic; their state
    passes differ (one product per chunk against two), so results agree within
    rounding, and each run of the pool kernel is deterministic."""
    x = prefill_inputs(2, 700, 3, 128, 128, dtype=torch.bfloat16, seed=72, init_std=0.05)
    o1, s1 = _run(x, pool=True)
    o2, s2 = _run(x, pool=True)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    o3, s3 = _run(x, pair=True)
    assert rel_err(o1, o3.float().cpu().numpy()) < 2e-2
    assert rel_err(s1, s3.cpu().numpy()) < 1e-2


# --------------------------------------------------------------------------- #
# full-size workloads, sampled chains                                         #
# --------------------------------------------------------------------------- #
FULL = {
    "gdn_prefill_bf16": [(0, 0), (3, 15), (1, 7)],
    "gdn_varlen_bf16": [(0, 0), (31, 15), (17, 5)],
    "kda_prefill_bf16": [(0, 0), (1, 31)],
    "kda_fast8_prefill_bf16": [(0, 0), (1, 17)],
    "fg2_prefill_bf16": [(0, 0), (1, 29)],
    "gdn_long_prefill_bf16": [(0, 0), (0, 31)],
}


@pytest.mark.parametrize("kernel", ["default", "pool"])
@pytest.mark.parametrize("name", list(FULL))
def test_full_workload_sampled(cuda_ok, name, kernel):
    if kernel == "pool" and WORKLOADS[name].decay == "channel":
        pytest.skip("the pool kernel takes scalar decay")
    x = workload_inputs(name)
    o, sf = _run(x, pool=kernel == "pool", check=True)
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    to, ts = TOL[WORKLOADS[name].dtype]
    worst_o = worst_s = 0.0
    for n, h, ro, rs in oracle_heads(x, FULL[name]):
        go, gs = gpu_head(x, o, sf, n, h)
        eo, es = rel_err(go, ro), rel_err(gs, rs)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
        assert eo <= to, f"{name} (n={n}, h={h}) o error {eo:.3g}"
        assert es <= ts, f"{name} (n={n}, h={h}) final-state error {es:.3g}"
    record_margin(f"{name} [{kernel}]", worst_o, to, worst_s, ts)


# --------------------------------------------------------------------------- #
# decode                                                                      #
# --------------------------------------------------------------------------- #
def _verify_inputs(N, K, H, d, dtype, decay, seed):
    g = torch.Generator().manual_seed(seed)
    x = prefill_inputs(N, K, H, d, d, dtype=dtype, decay=decay, init_std=0.3, gen=g,
                       alpha_shift=2.0 if decay == "scalar" else 3.0)
    return x


@pytest.mark.parametrize("decay,dtype,d", [("scalar", torch.bfloat16, 128),
                                           ("channel", torch.bfloat16, 128),
                                           ("scalar", torch.float32, 64)])
def test_recurrent_verify_outputs_and_commit_match_oracle(cuda_ok, decay, dtype, d):
    """Multi-token verification: the outputs of all K drafts equal the oracle's
    recurrence over the K tokens from the state; the committed state equals the
    oracle's state after each sequence's first n_commit tokens (0 .. K, 0 leaves it
    as it was); a peek (no commit) leaves the state bit for bit untouched."""
    from gated_delta_rule_140_b200 import recurrent_verify
    N, K, H = 6, 7, 3
    x = _verify_inputs(N, K, H, d, dtype, decay, 91)
    d_ = to_dev(x)
    s0 = d_["initial_state"].contiguous()
    commit = torch.tensor([0, 1, 3, 7, 5, 2], dtype=torch.int32)
    to, ts = TOL[dtype]
    ro, _ = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    # peek
    st = s0.clone()
    o = recurrent_verify(d_["q"], d_["k"], d_["v"], d_["log_alpha"], d_["beta"], st, check=True)
    assert torch.equal(st, s0)
    assert rel_err(o, ro) <= to
    # commit with and without outputs
    for outputs in (True, False):
        st = s0.clone()
        o2 = recurrent_verify(d_["q"], d_["k"], d_["v"], d_["log_alpha"], d_["beta"], st,
                              commit.cuda(), outputs=outputs, check=True)
        if outputs:
            assert torch.equal(o2, o)
        for n in range(N):
            j = int(commit[n])
            if j == 0:
                assert torch.equal(st[n], s0[n])
                continue
            sl = lambda t: t[n:n + 1, :j]
            _, rs = oracle.recurrent(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["log_alpha"]),
                                     sl(x["beta"]), x["initial_state"][n:n + 1])
            assert rel_err(st[n], rs[0]) <= ts, (n, j)


@pytest.mark.parametrize("decay,dtype,d", [("scalar", torch.bfloat16, 128),
                                           ("channel", torch.bfloat16, 128),
                                           ("scalar", torch.float32, 64)])
def test_recurrent_verify_tree_matches_oracle_paths(cuda_ok, decay, dtype, d):
    """Tree-shaped drafts: node j's output equals the oracle's recurrence over the
    tokens on the path from the state to j; committing node c - 1 leaves the
    oracle's state after that path.  Sequence 0 is a chain (its outputs equal the
    chain verification's bit for bit), sequence 1 branches, sequence 2 has
    out-of-range parents, which count as -1 (children of the state)."""
    from gated_delta_rule_140_b200 import recurrent_verify
    N, K, H = 3, 10, 2
    x = _verify_inputs(N, K, H, d, dtype, decay, 93)
    dd = to_dev(x)
    s0 = dd["initial_state"].contiguous()
    parent = torch.tensor([[-1, 0, 1, 2, 3, 4, 5, 6, 7, 8],
                           [-1, 0, 0, 1, 1, 2, -1, 6, 7, 3],
                           [-1, 5, 0, 9, 2, -7, 4, 6, 6, 12]], dtype=torch.int32)
    commit = torch.tensor([7, 10, 9], dtype=torch.int32)  # nodes 6, 9, 8

    def path(n, j):
        p = []
        while j >= 0:
            p.append(j)
            q_ = int(parent[n, j])
            j = q_ if 0 <= q_ < j else -1
        return p[::-1]

    to, ts = TOL[dtype]
    st = s0.clone()
    o = recurrent_verify(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], st,
                         commit.cuda(), parent=parent.cuda(), check=True)
    for n in range(N):
        for j in range(K):
            pj = path(n, j)
            sl = lambda t: t[n:n + 1, pj]
            ro, rs = oracle.recurrent(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["log_alpha"]),
                                      sl(x["beta"]), x["initial_state"][n:n + 1])
            assert rel_err(o[n, j], ro[0, -1]) <= to, (n, j)
            if j == int(commit[n]) - 1:
                assert rel_err(st[n], rs[0]) <= ts, (n, j)
    # the chain-shaped sequence: the chain kernel's outputs bit for bit
    s_chain = s0.clone()
    o_chain = recurrent_verify(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], s_chain,
                               check=True)
    assert torch.equal(o[0], o_chain[0])
    # a peek leaves the state untouched
    st2 = s0.clone()
    recurrent_verify(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], st2,
                     parent=parent.cuda(), check=True)
    assert torch.equal(st2, s0)


def test_recurrent_verify_tree_of_64_nodes(cuda_ok):
    """The largest tree (64 nodes, random parents, bf16 KDA): every node's output and
    the commit of the deepest node against the oracle's recurrence over its path."""
    from gated_delta_rule_140_b200 import recurrent_verify
    N, K, H, d = 2, 64, 2, 128
    x = _verify_inputs(N, K, H, d, torch.bfloat16, "channel", 95)
    dd = to_dev(x)
    g = torch.Generator().manual_seed(96)
    parent = torch.stack([torch.tensor([-1] + [int(torch.randint(-1, j, (1,), generator=g))
                                               for j in range(1, K)], dtype=torch.int32)
                          for _ in range(N)])

    def path(n, j):
        p = []
        while j >= 0:
            p.append(j)
            j = int(parent[n, j])
        return p[::-1]

    deepest = [max(range(K), key=lambda j: len(path(n, j))) for n in range(N)]
    commit = torch.tensor([c + 1 for c in deepest], dtype=torch.int32)
    st = dd["initial_state"].clone()
    o = recurrent_verify(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], st,
                         commit.cuda(), parent=parent.cuda(), check=True)
    to, ts = TOL[torch.bfloat16]
    for n in range(N):
        for j in range(K):
            pj = path(n, j)
            sl = lambda t: t[n:n + 1, pj]
            ro, rs = oracle.recurrent(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["log_alpha"]),
                                      sl(x["beta"]), x["initial_state"][n:n + 1])
            assert rel_err(o[n, j], ro[0, -1]) <= to, (n, j)
            if j == deepest[n]:
                assert rel_err(st[n], rs[0]) <= ts, n


def test_recurrent_verify_commit_all_equals_decode_steps(cuda_ok):
    """Committing all K tokens is K decode steps: the same recurrence in fp32, with
    the row sums reduced in another order (a transposed butterfly over eight rows
    against the decode kernel's per-row reduction), so equal to rounding."""
    from gated_delta_rule_140_b200 import recurrent_verify
    N, K, H = 5, 4, 2
    for decay in ("scalar", "channel"):
        x = to_dev(_verify_inputs(N, K, H, 128, torch.bfloat16, decay, 92))
        st = x["initial_state"].clone()
        o = recurrent_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], st,
                             torch.full((N,), K, dtype=torch.int32, device="cuda"), check=True)
        st2 = x["initial_state"].clone()
        outs = [recurrent_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                               x["v"][:, t].contiguous(), x["log_alpha"][:, t].contiguous(),
                               x["beta"][:, t].contiguous(), st2) for t in range(K)]
        torch.cuda.synchronize()
        assert rel_err(st, st2.double().cpu().numpy()) <= 1e-5
        assert rel_err(o, torch.stack(outs, 1).double().cpu().numpy()) <= 1e-2 / 4  # bf16 o

def _decode_check(x, picks, dtype):
    steps = x["q"].shape[0]
    d = to_dev(x)
    state = d["state"].clone()
    outs = []
    for t in range(steps):
        outs.append(recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["log_alpha"][t],
                                   d["beta"][t], state))
    torch.cuda.synchronize()
    o = torch.stack(outs)  # [S,N,H,dv]
    to, ts = TOL[dtype]
    worst_o = worst_s = 0.0
    for n, h in picks:
        # the oracle sees the same tokens as one sequence of `steps` tokens
        seq = lambda t: t[:, n:n + 1, h:h + 1].transpose(0, 1)  # [1,S,1,...]
        ro, rs = oracle.recurrent(seq(x["q"]), seq(x["k"]), seq(x["v"]),
                                  seq(x["log_alpha"]), seq(x["beta"]),
                                  x["state"][n:n + 1, h:h + 1])
        eo, es = rel_err(o[:, n, h], ro[0, :, 0]), rel_err(state[n, h], rs[0, 0])
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
        assert eo <= to
        assert es <= ts
    return worst_o, worst_s


@pytest.mark.parametrize("decay", ["scalar", "channel"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_reduced(cuda_ok, decay, d, dtype):
    x = decode_inputs(5, 3, d, d, 20, dtype=dtype, decay=decay, seed=31,
                      alpha_shift=2.0 if decay == "scalar" else 3.0)
    _decode_check(x, [(n, h) for n in range(5) for h in range(3)], dtype)


def test_decode_full_workload_sampled(cuda_ok):
    """N=256, H=32, d=128, fp32 state in place, 64 steps."""
    x = workload_inputs("gdn_decode")
    eo, es = _decode_check(x, [(0, 0), (255, 31), (100, 17)], torch.bfloat16)
    record_margin("gdn_decode [decode, 64 steps]", eo, TOL[torch.bfloat16][0], es,
                  TOL[torch.bfloat16][1])


def test_decode_matches_prefill(cuda_ok):
    """64 decode steps from S0 equal one 64-token prefill from S0 (same tokens)."""
    x = decode_inputs(4, 2, 128, 128, 64, seed=32)
    d = to_dev(x)
    state = d["state"].clone()
    outs = [recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["log_alpha"][t], d["beta"][t],
                           state) for t in range(64)]
    seq = lambda t: t.transpose(0, 1).contiguous()  # [N,64,H,...]
    o, sf = chunk_fwd(seq(d["q"]), seq(d["k"]), seq(d["v"]), seq(d["log_alpha"]),
                      seq(d["beta"]), d["state"])
    torch.cuda.synchronize()
    assert rel_err(torch.stack(outs).transpose(0, 1), o.float().cpu().numpy()) < 2e-2
    assert rel_err(state, sf.cpu().numpy()) < 1e-2


# --------------------------------------------------------------------------- #
# the fused input prologue (gdn_chunk_fwd_raw)                                #
# --------------------------------------------------------------------------- #
def _raw_problem(B, T, H, seed, lengths=None, zero_key=False):
    """Unnormalised q, k (per-token scales 0.5..3.5), v, decay and writing-rate
    logits ~ N(0,1), a per-head decay bias, an initial state."""
    g = torch.Generator().manual_seed(seed)
    cu = None
    if lengths is not None:
        B, T = 1, int(sum(lengths))
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths), 0).to(torch.int32)
    n = B if cu is None else len(lengths)
    scale = lambda: 0.5 + 3.0 * torch.rand(B, T, H, 1, generator=g)
    q = (torch.randn(B, T, H, 128, generator=g) * scale()).to(torch.bfloat16)
    k = (torch.randn(B, T, H, 128, generator=g) * scale()).to(torch.bfloat16)
    if zero_key:
        k[0, min(5, T - 1), 0] = 0
    v = torch.randn(B, T, H, 128, generator=g).to(torch.bfloat16)
    a = torch.randn(B, T, H, generator=g)
    b = torch.randn(B, T, H, generator=g)
    bias = torch.linspace(1.0, 3.0, H)
    s0 = torch.randn(n, H, 128, 128, generator=g) * 0.05
    return dict(q_raw=q, k_raw=k, v=v, a=a, b=b, bias=bias, s0=s0, cu=cu)


@pytest.mark.parametrize("case", ["ragged", "packed", "zero_key", "no_bias"])
def test_fused_prologue_matches_oracle(cuda_ok, case):
    """chunk_fwd_raw against the oracle's prologue (FG2-GDN section 3.5: unit
    q and k, sigmoid beta, -softplus decay with a bias) followed by its
    recurrence; and against gdn_chunk_fwd on the prologue's outputs."""
    from gated_delta_rule_140_b200 import chunk_fwd_raw
    if case == "packed":
        r = _raw_problem(0, 0, 3, 91, lengths=[0, 1, 63, 64, 65, 200, 0, 130, 700])
    else:
        r = _raw_problem(2, 229 if case != "no_bias" else 700, 3, 90, zero_key=case == "zero_key")
    bias = None if case == "no_bias" else r["bias"]
    q, k, la, beta = oracle.prologue(r["q_raw"], r["k_raw"], r["a"], r["b"], bias)
    ro, rs = oracle.recurrent(q, k, r["v"], la, beta, r["s0"], r["cu"])
    dv = lambda t: None if t is None else t.cuda()
    o, sf = chunk_fwd_raw(dv(r["q_raw"]), dv(r["k_raw"]), dv(r["v"]), dv(r["a"]), dv(r["b"]),
                          dv(bias), dv(r["s0"]), dv(r["cu"]), check=True)
    torch.cuda.synchronize()
    to, ts = TOL[torch.bfloat16]
    eo, es = rel_err(o, ro), rel_err(sf, rs)
    assert eo <= to and es <= ts, (eo, es)
    # the unfused path on the prologue's outputs (q, k rounded to bf16 there)
    t = lambda x, dt: torch.from_numpy(x).to(dt).cuda()
    o2, sf2 = chunk_fwd(t(q, torch.bfloat16), t(k, torch.bfloat16), dv(r["v"]),
                        t(la, torch.float32), t(beta, torch.float32), dv(r["s0"]), dv(r["cu"]),
                        pool=True)
    torch.cuda.synchronize()
    assert rel_err(o, o2.double().cpu().numpy()) < 2e-2
    assert rel_err(sf, sf2.cpu().numpy()) < 1e-2


def test_fused_prologue_rejects_other_shapes(cuda_ok):
    from gated_delta_rule_140_b200 import chunk_fwd_raw
    r = _raw_problem(1, 64, 2, 92)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in r.items()}
    with pytest.raises(nat.GdnError) as ei:  # channel decay
        chunk_fwd_raw(d["q_raw"], d["k_raw"], d["v"], d["a"][..., None].expand(1, 64, 2, 128)
                      .contiguous(), d["b"])
    assert ei.value.status == nat.GDN_ERR_UNSUPPORTED
    with pytest.raises(nat.GdnError) as ei:  # fp32
        chunk_fwd_raw(d["q_raw"].float(), d["k_raw"].float(), d["v"].float(), d["a"], d["b"])
    assert ei.value.status == nat.GDN_ERR_UNSUPPORTED


# --------------------------------------------------------------------------- #
# segment state maps (sequence sharding)                                      #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("dv,dk", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_state_compose_and_identity(cuda_ok, dv, dk):
    """gdn_state_compose: out = s m + b per (sequence, head), against an fp64
    matrix product; with b null; with out aliasing b.  gdn_state_identity: I."""
    g = torch.Generator().manual_seed(71)
    N, H = 3, 2
    s = torch.randn(N, H, dv, dk, generator=g)
    m = torch.randn(N, H, dk, dk, generator=g) / dk ** 0.5
    b = torch.randn(N, H, dv, dk, generator=g)
    ref = s.double() @ m.double() + b.double()
    sd, md, bd = s.cuda(), m.cuda(), b.cuda()
    out = nat.state_compose(sd, md, bd)
    assert rel_err(out, ref.numpy()) <= 1e-5
    out0 = nat.state_compose(sd, md)
    assert rel_err(out0, (s.double() @ m.double()).numpy()) <= 1e-5
    nat.state_compose(sd, md, bd, out=bd)  # in place over b
    torch.cuda.synchronize()
    assert torch.equal(bd, out)
    if dv == dk:
        eye = nat.state_identity(N, H, dk, "cuda")
        assert torch.equal(eye.cpu(), torch.eye(dk).expand(N, H, dk, dk))
        assert torch.equal(nat.state_compose(sd, eye), sd)


@pytest.mark.parametrize("decay", ["scalar", "channel"])
def test_sequence_sharding_emulated_on_one_gpu(cuda_ok, decay):
    """One 1200-token sequence as four ragged segments, each run as its rank would:
    segment 0 from the initial state, segments >= 1 reduced to their state maps
    (two prefills each), the maps composed into every segment's start, and each
    segment rerun from it; the concatenated outputs and the last segment's state
    equal the oracle's whole-sequence recurrence within the parity bounds."""
    from gated_delta_rule_140_b200 import seqshard
    g = torch.Generator().manual_seed(73)
    x = prefill_inputs(1, 1200, 2, 128, 128, dtype=torch.bfloat16, decay=decay, seed=73,
                       init_std=0.3, gen=g, alpha_shift=3.0 if decay == "scalar" else 4.0)
    d = to_dev(x)
    bounds = [0, 337, 587, 651, 1200]
    seg = lambda t, r: t[:, bounds[r]:bounds[r + 1]].contiguous()
    names = ("q", "k", "v", "log_alpha", "beta")
    outs, maps = [], []
    for r in range(4):
        s = {n_: seg(d[n_], r) for n_ in names}
        if r == 0:
            o, se = chunk_fwd(**s, initial_state=d["initial_state"], check=True)
            outs.append(o)
            maps.append((torch.zeros_like(se), se))
        else:
            maps.append(seqshard.segment_map(**s))
    for r in range(1, 4):
        s = {n_: seg(d[n_], r) for n_ in names}
        o, se = chunk_fwd(**s, initial_state=seqshard.start_state(maps, r), check=True)
        outs.append(o)
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=1)
    ro, rs = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    to, ts = TOL[torch.bfloat16]
    eo, es = rel_err(o, ro), rel_err(se, rs)
    assert eo <= to and es <= ts, (eo, es)
    record_margin(f"sequence sharding, 4 segments of 1200 tokens [{decay}]", eo, to, es, ts)
