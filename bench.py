"""Throughput of the gated delta rule hot path on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--decode-workload NAME]
                    [--legs all|none|NAME,NAME,...] [--leg-seconds S]
                    [--prefill-kernel default|pool|pair|one_cta|cuda_cores]

A step is one pass of the whole hot path on one GPU:
  * prefill leg: gdn_chunk_fwd over one batch of the prefill workload
    (default: GDN bf16, B=4, H=16, T=4096, d_k=d_v=128; cumulative decay, A,
    T=(I+A)^-1, W/U, inter-chunk state pass, output), then
  * decode leg: one gdn_recurrent_step over the decode workload (N=256
    sequences, H=32, d=128, fp32 state updated in place).
``value`` is prefill tokens/s over all ranks: tokens processed by all ranks
divided by the max over ranks of the summed prefill-leg device time (CUDA
events on the launching stream) over exactly K timed steps.  ``ms_per_step``
is the device time of whole steps, barrier to barrier, max over ranks.  Under
torchrun (N > 1) every rank runs its own independent batch (the problems shard
with no data-path collective): weak scaling.  Inputs are larger than L2
(prefill 275 MB, decode state 537 MB), so no flush is needed between steps.

``legs`` (rank 0 of a 1-GPU run, or every rank with --legs on N GPUs) times
each workload on its own for at least --leg-seconds of device time: the six
bf16 prefill workloads (GDN B4 H16 T4096; packed varlen, 32 sequences of
256-4096 tokens with initial states; KDA B2 H32 T8192, the same with 8 key
channels per head forgetting at log alpha = -30 per token, and with FG2-GDN's
writing rate per key channel; GDN B1 H32 T65536)
and the decode step (N256 H32, fp32 state in place).  Each leg carries its own
roofline (max of FLOPs / bf16 peak and algorithmic bytes / HBM bandwidth, the
measured peaks), end-to-end rate through host buffers, and a bounded CPU
baseline of the fp64 oracle.  A clock sampler runs across the timed regions.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of the same prefill workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule prefill tokens/s and decode steps/s; % of roofline on 1 B200"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CHUNK = 64
PREFILL_LEGS = ("gdn_prefill_bf16", "gdn_varlen_bf16", "kda_prefill_bf16",
                "kda_fast8_prefill_bf16", "fg2_prefill_bf16", "gdn_long_prefill_bf16")
RAW_LEG = "gdn_prefill_bf16_raw"  # the config-2 shapes through the fused input prologue
DECODE_LEG = "gdn_decode"
DECODE_LEGS = (DECODE_LEG, "kda_decode")  # the scalar- and channel-decay decode steps
FIG3_LEGS = tuple(f"fig3_{T // 1024}kx{32768 // T}" for T in (2048, 4096, 8192, 16384, 32768))
KERNEL_SRC = {
    "tensor_core_pool": ("chunk_pool_kernel", "gdn_chunk_pool.cu"),
    "tensor_core_pair": ("chunk_pair_kernel", "gdn_chunk_pair.cu"),
    "tensor_core": ("chunk_tc_kernel", "gdn_chunk_tc.cu"),
    "cuda_core": ("chunk_simt_kernel", "gdn_chunk_simt.cu"),
}


# --------------------------------------------------------------------------- #
# helpers                                                                     #
# --------------------------------------------------------------------------- #
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def prefill_bytes(es, channel, tok_heads, dk, dv, n_states, beta_channel=False):
    """Algorithmic HBM bytes of one prefill: q, k, v read and o written once
    (element size ``es``), fp32 log alpha (per key channel for KDA) and beta (per
    key channel for FG2-GDN) read once, and ``n_states`` fp32 states of d_v x d_k
    read or written once."""
    per_tok = es * (2 * dk + 2 * dv) + 4 * (dk if channel else 1) + 4 * (dk if beta_channel else 1)
    return tok_heads * per_tok + n_states * dv * dk * 4


def prefill_flops(tok_heads, dk, dv, C=CHUNK):
    """Algorithmic FLOPs of one chunkwise prefill per token-head: the three
    d_k x d_v products (W S^T, Q S^T, the state update) 6 d_k d_v; the chunk
    products K K^T, Q K^T, W, U and the causal P V' 2C(3 d_k + 2 d_v); the
    triangular inverse C^2 / 3."""
    return tok_heads * (6 * dk * dv + 2 * C * (3 * dk + 2 * dv) + C * C / 3)


def decode_bytes(N, H, dk, dv, es=2, channel=False):
    """Per step: fp32 state read + written, q/k/v read and o written, gates read."""
    return N * H * (2 * 4 * dv * dk + es * (2 * dk + 2 * dv) + 4 * (dk if channel else 1) + 4)


def decode_flops(N, H, dk, dv):
    """Per step and head: S k, S q, the rank-1 update and the decay, ~8 d_k d_v."""
    return N * H * 8 * dk * dv


def roofline(flops, nbytes, seconds, pk, pk_kind, traffic=None, kernel=None):
    """Roofline of one launch: the bound is the larger of FLOPs / bf16 peak and
    bytes / HBM bandwidth; ``frac`` is that time over the measured time."""
    hbm, tf = pk["hbm_gbs"], pk["bf16_tflops"]
    t_b, t_f = nbytes / (hbm * 1e9), flops / (tf * 1e12)
    if t_f > t_b:
        ach, peak, unit, bound = flops / seconds / 1e12, tf, "TFLOP/s", "tensor"
    else:
        ach, peak, unit, bound = nbytes / seconds / 1e9, hbm, "GB/s", "hbm"
    return {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
            "traffic": traffic, "kernel": kernel, "alg_bytes": nbytes, "alg_flops": flops,
            "t_hbm_us": t_b * 1e6, "t_flop_us": t_f * 1e6, "peak_source": pk_kind}


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, rows=None):
        rows = self.rows if rows is None else rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = sorted(float(r[0]) for r in rows if r[0].replace(".", "").isdigit())
        mx = max((float(r[1]) for r in rows if r[1].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if len(r) > 4 + i and r[4 + i].lower().startswith("active")})
        power = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def traffic_for(kernel: str, src: str, workload: str = ""):
    """DRAM bytes per launch from a committed ncu capture of this kernel on this
    workload (entry "kernel:workload", else "kernel"), if the kernel source is
    unchanged since the counters were taken (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    recs = json.load(open(p))
    rec = recs.get(f"{kernel}:{workload}") or recs.get(kernel)
    if not rec:
        return None
    path = os.path.join(ROOT, src)
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    return rec.get("bytes_per_launch") if rec.get("src_sha") == sha else None


def headline_config(workload, decode_workload, world):
    """The ``config`` object of the JSON line, identical in both arms."""
    from gated_delta_rule_140_b200.inputs import WORKLOADS
    w, wd = WORKLOADS[workload], WORKLOADS[decode_workload]
    return {"workload": workload, "B": w.B, "T": w.T, "H": w.H, "d_k": w.d, "d_v": w.d,
            "decay": w.decay, "chunk": CHUNK, "parallelism": f"dp{world} (independent batches)",
            "l2": "inputs larger than L2 (no flush)",
            "decode_workload": f"{decode_workload}: N={wd.B}, H={wd.H}, d={wd.d}, "
                               "fp32 state in place"}


# --------------------------------------------------------------------------- #
# distributed plumbing                                                        #
# --------------------------------------------------------------------------- #
def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return rank, world, local


def init_pg(backend, world):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- #
# the fp64 oracle on the host cores (reference arm and CPU baselines)         #
# --------------------------------------------------------------------------- #
SAMPLE_TOKEN_HEADS = 262144  # about 10 s of one host core for the fp64 oracle at d = 128


def oracle_sample(workload, budget_token_heads=SAMPLE_TOKEN_HEADS):
    """A bounded sample of the workload for the oracle: whole sequences from the
    start of the batch (all heads) until about ``budget_token_heads``
    token-heads, cut to the first tokens of one sequence when a single one is
    larger."""
    from gated_delta_rule_140_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS[workload]
    x = workload_inputs(workload)
    H = w.H
    budget = max(1, budget_token_heads // H)  # tokens
    cu = x["cu_seqlens"]
    names = ("q", "k", "v", "log_alpha", "beta")
    if cu is None:
        nseq = max(1, min(w.B, budget // w.T))
        ntok_seq = min(w.T, budget)
        s = {n: x[n][:nseq, :ntok_seq] for n in names}
        s0 = None if x["initial_state"] is None else x["initial_state"][:nseq]
        desc = f"{nseq} x {ntok_seq} tokens x {H} heads of {workload}"
        return s, s0, None, nseq * ntok_seq, desc
    ends = cu[1:].tolist()
    nseq = max(1, sum(1 for e in ends if e <= budget))
    end = int(cu[nseq])
    s = {n: x[n][:, :end] for n in names}
    s0 = None if x["initial_state"] is None else x["initial_state"][:nseq]
    desc = f"first {nseq} sequences ({end} tokens) x {H} heads of {workload}"
    return s, s0, cu[:nseq + 1].clone(), end, desc


def _oracle_pass(s, s0, cu, nthreads=0):
    import oracle
    if s["beta"].dim() == 4:  # FG2-GDN's rate per key channel
        oracle.fg2_recurrent(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], None, s0, cu,
                             nthreads=nthreads)
        return nthreads if nthreads > 0 else (os.cpu_count() or 1)
    _, _, used = oracle.recurrent(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], s0, cu,
                                  nthreads=nthreads, return_threads=True)
    return used


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores, each
    step one pass over the bounded sample of the workload (rank 0 only)."""
    if rank != 0:
        return 0
    s, s0, cu, ntok, desc = oracle_sample(args.workload)
    used = 1
    for _ in range(args.warmup):
        used = _oracle_pass(s, s0, cu)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        used = _oracle_pass(s, s0, cu)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = args.steps * ntok / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(args.workload, args.decode_workload, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": desc + ", fp64, one pass per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(workload, budget=SAMPLE_TOKEN_HEADS, nthreads=0):
    """The oracle timed on the host cores on the bounded sample, one pass."""
    s, s0, cu, ntok, desc = oracle_sample(workload, budget)
    t0 = time.perf_counter()
    used = _oracle_pass(s, s0, cu, nthreads)
    dt = time.perf_counter() - t0
    return {"value": ntok / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": desc + ", fp64, one pass"}


def cpu_baseline_decode(xd_cpu, n_seqs=64):
    """The oracle on one decode step of the first ``n_seqs`` sequences (all
    heads): a T = 1 prefill from the decode state."""
    import oracle
    s = {k: xd_cpu[k][0, :n_seqs].unsqueeze(1) for k in ("q", "k", "v", "log_alpha", "beta")}
    s0 = xd_cpu["state"][:n_seqs]
    t0 = time.perf_counter()
    _, _, used = oracle.recurrent(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], s0,
                                  return_threads=True)
    dt = time.perf_counter() - t0
    return {"value": n_seqs / dt / xd_cpu["q"].shape[1], "unit": "steps/s", "cores": used,
            "kind": "oracle", "sample": f"one step of {n_seqs} of {xd_cpu['q'].shape[1]} "
                                        "sequences (all heads), fp64; rate scaled to all"}


# --------------------------------------------------------------------------- #
# our arm                                                                     #
# --------------------------------------------------------------------------- #
def _kflags(kind):
    return {"pool": kind == "pool", "pair": kind == "pair", "one_cta": kind == "one_cta",
            "cuda_cores": kind == "cuda_cores"}


class PrefillLeg:
    """One prefill workload resident on the device, with its output buffers."""

    def __init__(self, name, dev, kflags, ws):
        import torch
        from gated_delta_rule_140_b200.inputs import WORKLOADS, workload_inputs
        self.name, self.w, self.kflags, self.ws = name, WORKLOADS[name], kflags, ws
        if self.w.decay == "channel":  # the pool and single-CTA kernels take scalar decay
            self.kflags = {k: (v and k not in ("pool", "one_cta")) for k, v in kflags.items()}
        self.cpu = workload_inputs(name)
        self.x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.cpu.items()}
        x = self.x
        self.B, self.T, self.H, self.dk = x["q"].shape
        self.dv = x["v"].shape[-1]
        self.n_seqs = self.B if x["cu_seqlens"] is None else len(x["cu_seqlens"]) - 1
        self.tokens = self.B * self.T
        self.o = torch.empty_like(x["v"])
        self.sf = torch.empty(self.n_seqs, self.H, self.dv, self.dk, dtype=torch.float32,
                              device=dev)

    def run(self, x=None, o=None, sf=None):
        from gated_delta_rule_140_b200 import chunk_fwd
        x = self.x if x is None else x
        chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"],
                  x["cu_seqlens"], o=self.o if o is None else o,
                  final_state=self.sf if sf is None else sf, workspace=self.ws, **self.kflags)

    def work(self):
        import torch
        es = 2 if self.w.dtype == torch.bfloat16 else 4
        th = self.tokens * self.H
        n_states = self.n_seqs * (int(self.x["initial_state"] is not None) + 1)
        return (prefill_flops(th, self.dk, self.dv),
                prefill_bytes(es, self.w.decay == "channel", th, self.dk, self.dv,
                              n_states * self.H, self.w.beta_channel))

    def kernel(self):
        from gated_delta_rule_140_b200 import _native as nat
        path = nat.chunk_fwd_path(nat.prefill_dims(self.x["q"], self.x["v"],
                                                   self.x["log_alpha"], self.x["cu_seqlens"],
                                                   **self.kflags))
        k, src = KERNEL_SRC.get(path, KERNEL_SRC["cuda_core"])
        return k, "gated_delta_rule_140_b200/csrc/" + src


def time_loop(fn, reps, stream):
    """Device time (ms) of ``reps`` back-to-back calls, CUDA events on ``stream``."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def e2e_prefill(leg, n, stream):
    """n end-to-end steps through the public API with host buffers: every step
    copies its inputs in from pinned host memory, runs the call, and copies o
    and the final state back.  As in a serving loop, consecutive steps overlap
    on three streams (copy-in, compute, copy-out) with double-buffered device
    inputs and outputs.  Returns (ms, h2d bytes per step, d2h bytes per step)."""
    import torch
    dev = leg.o.device
    pin = {k: (v.cpu().pin_memory() if isinstance(v, torch.Tensor) else None)
           for k, v in leg.x.items()}
    if leg.x["cu_seqlens"] is not None:
        pin["cu_seqlens"] = leg.cpu["cu_seqlens"].pin_memory()
    o_h = torch.empty(leg.o.shape, dtype=leg.o.dtype).pin_memory()
    sf_h = torch.empty(leg.sf.shape, dtype=leg.sf.dtype).pin_memory()
    dbuf = [{k: (torch.empty_like(v) if isinstance(v, torch.Tensor) else None)
             for k, v in leg.x.items()} for _ in range(2)]
    obuf = [(torch.empty_like(leg.o), torch.empty_like(leg.sf)) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = o_h.numel() * o_h.element_size() + sf_h.numel() * sf_h.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def go(n):
        ev = {key: [torch.cuda.Event() for _ in range(n)] for key in ("in", "comp", "out")}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for t in range(n):
            b, ib = t % 2, dbuf[t % 2]
            with torch.cuda.stream(s_in):
                if t >= 2:
                    s_in.wait_event(ev["comp"][t - 2])  # step t-2 has read these inputs
                for k2, v in pin.items():
                    if v is not None:
                        ib[k2].copy_(v, non_blocking=True)
                ev["in"][t].record(s_in)
            stream.wait_event(ev["in"][t])
            if t >= 2:
                stream.wait_event(ev["out"][t - 2])  # step t-2's outputs are downloaded
            leg.run(ib, obuf[b][0], obuf[b][1])
            ev["comp"][t].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp"][t])
                o_h.copy_(obuf[b][0], non_blocking=True)
                sf_h.copy_(obuf[b][1], non_blocking=True)
                ev["out"][t].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    go(2)
    ms = go(n)
    del dbuf, obuf
    return ms, h2d, d2h


def e2e_decode(xd, state, od, wd, n, stream):
    """n decode steps through the public API with host buffers: each step copies
    its token inputs in from pinned host memory and o back (the state stays
    resident, as in serving)."""
    import torch
    from gated_delta_rule_140_b200 import recurrent_step
    names = ("q", "k", "v", "log_alpha", "beta")
    pin = {k: xd[k].cpu().pin_memory() for k in names}
    dbuf = {k: torch.empty_like(xd[k][0]) for k in names}
    o_h = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    h2d = sum(pin[k][0].numel() * pin[k][0].element_size() for k in names)
    d2h = o_h.numel() * o_h.element_size()
    steps_d = xd["q"].shape[0]

    def go(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t in range(n):
            i = t % steps_d
            for k in names:
                dbuf[k].copy_(pin[k][i], non_blocking=True)
            recurrent_step(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"],
                           state, o=od)
            o_h.copy_(od, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    go(2)
    return go(n), h2d, d2h


def raw_leg(head, dev, ws, stream, pk, pk_kind, args, K):
    """The headline workload's shapes through gdn_chunk_fwd_raw: unnormalised q,
    k and gate logits in, the L2 norms, sigmoid and -softplus applied inside the
    kernel.  Beside it, the unfused route a caller would take otherwise: torch
    element-wise passes (normalise q and k, sigmoid, -softplus) that read the raw
    inputs and write the prepared ones, then the same call on the pool kernel."""
    import torch
    import torch.nn.functional as F
    from gated_delta_rule_140_b200 import chunk_fwd, chunk_fwd_raw
    from gated_delta_rule_140_b200.inputs import raw_prefill_inputs
    w = head.w
    r = {k: v.to(dev) for k, v in raw_prefill_inputs(w.B, w.T, w.H, w.d, seed=11).items()}
    o = torch.empty_like(r["v"])
    sf = torch.empty(w.B, w.H, w.d, w.d, dtype=torch.float32, device=dev)

    def fused():
        chunk_fwd_raw(r["q_raw"], r["k_raw"], r["v"], r["alpha_logit"], r["beta_logit"],
                      r["alpha_bias"], o=o, final_state=sf, workspace=ws)

    def unfused():
        q = (r["q_raw"].float() / r["q_raw"].float().norm(dim=-1, keepdim=True)).to(r["v"].dtype)
        k = (r["k_raw"].float() / r["k_raw"].float().norm(dim=-1, keepdim=True)).to(r["v"].dtype)
        la = -F.softplus(r["alpha_logit"] + r["alpha_bias"])
        be = torch.sigmoid(r["beta_logit"])
        chunk_fwd(q, k, r["v"], la, be, o=o, final_state=sf, workspace=ws, pool=True)

    for _ in range(3):
        fused()
        unfused()
    t1 = time_loop(fused, 3, stream) / 3 / 1e3
    reps = max(K, math.ceil(args.leg_seconds / max(t1, 1e-6)))
    sec = time_loop(fused, reps, stream) / reps / 1e3
    reps_u = max(K, math.ceil(0.5 * args.leg_seconds / max(t1, 1e-6)))
    sec_u = time_loop(unfused, reps_u, stream) / reps_u / 1e3
    fl, by = head.work()
    th = head.tokens * head.H
    extra = th * (2 * 2 * 2 * w.d + 4 * 4)  # q, k read + written (bf16), 2 gates read + written
    return {"value": head.tokens / sec, "unit": "tokens/s", "ms": sec * 1e3, "reps": reps,
            "roofline": roofline(fl, by, sec, pk, pk_kind, None, "chunk_pool_kernel"),
            "unfused_ms": sec_u * 1e3, "unfused_extra_hbm_bytes": extra,
            "config": {"B": w.B, "T": w.T, "H": w.H, "d_k": w.d, "d_v": w.d,
                       "inputs": "q, k unnormalised; decay and rate logits; bias 2 per head"}}


def run_ours(args, rank, world, local):
    import torch
    from gated_delta_rule_140_b200 import _native as nat
    from gated_delta_rule_140_b200 import recurrent_step
    from gated_delta_rule_140_b200.inputs import WORKLOADS, workload_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_pg("nccl", world)
    nat.lib()
    pk, pk_kind = peaks()
    kflags = _kflags(args.prefill_kernel)
    ws = nat.Workspace(dev)
    stream = torch.cuda.current_stream()

    head = PrefillLeg(args.workload, dev, kflags, ws)
    wd = WORKLOADS[args.decode_workload]
    xd_cpu = workload_inputs(args.decode_workload)
    xd = {k: v.to(dev) for k, v in xd_cpu.items()}
    state = xd["state"].clone()
    od = torch.empty(wd.B, wd.H, wd.d, dtype=wd.dtype, device=dev)
    steps_d = xd["q"].shape[0]

    def decode(t):
        i = t % steps_d
        recurrent_step(xd["q"][i], xd["k"][i], xd["v"][i], xd["log_alpha"][i], xd["beta"][i],
                       state, o=od)

    for t in range(args.warmup):
        head.run()
        decode(t)
    torch.cuda.synchronize()
    if ws.status() != nat.GDN_OK:
        raise SystemExit("device-side error in warm-up")

    # ---- the headline: exactly K steps of (prefill + decode) ----------------
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    launches0 = nat.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.__enter__()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for t in range(K):
        ev[t][0].record(stream)
        head.run()
        ev[t][1].record(stream)
        decode(args.warmup + t)
        ev[t][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = nat.launch_count() - launches0
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    total_ms = t_start.elapsed_time(t_end)
    pre_ms = max_over_ranks(pre_ms, world, dev)
    dec_ms = max_over_ranks(dec_ms, world, dev)
    total_ms = max_over_ranks(total_ms, world, dev)
    if ws.status() != nat.GDN_OK:
        raise SystemExit("device-side error in the timed region")
    pre_s, dec_s = pre_ms / K / 1e3, dec_ms / K / 1e3

    # ---- every workload on its own, >= leg_seconds of device time each -------
    want = PREFILL_LEGS + (RAW_LEG,) + DECODE_LEGS if args.legs == "all" else \
        tuple() if args.legs == "none" else tuple(args.legs.split(","))
    if args.fig3:
        want = want + FIG3_LEGS
    legs = {}
    n_leg_launches = 0
    if rank == 0 or world > 1:
        for name in want:
            rows0 = len(clocks.rows)
            if name == RAW_LEG:
                legs[name] = raw_leg(head, dev, ws, stream, pk, pk_kind, args, K)
                legs[name]["clocks"] = clocks.summary(clocks.rows[rows0:])
                continue
            if name in DECODE_LEGS:
                if name == args.decode_workload:
                    wl, xl_cpu, xl, st_l, od_l, dec_fn, dl_s = wd, xd_cpu, xd, state, od, decode, dec_s
                else:
                    wl = WORKLOADS[name]
                    xl_cpu = workload_inputs(name)
                    xl = {k: v.to(dev) for k, v in xl_cpu.items()}
                    st_l = xl["state"].clone()
                    od_l = torch.empty(wl.B, wl.H, wl.d, dtype=wl.dtype, device=dev)

                    def dec_fn(t, xl=xl, st_l=st_l, od_l=od_l, n=xl["q"].shape[0]):
                        i = t % n
                        recurrent_step(xl["q"][i], xl["k"][i], xl["v"][i], xl["log_alpha"][i],
                                       xl["beta"][i], st_l, o=od_l)
                    for t in range(3):
                        dec_fn(t)
                    dl_s = time_loop(lambda it=iter(range(10 ** 9)): dec_fn(next(it)), 3, stream) / 3 / 1e3
                dec_reps = max(K, math.ceil(args.leg_seconds / max(dl_s, 1e-6)))
                l0 = nat.launch_count()
                ms = time_loop(lambda it=iter(range(10 ** 9)): dec_fn(next(it)), dec_reps, stream)
                n_leg_launches += nat.launch_count() - l0
                sec = ms / dec_reps / 1e3
                fl = decode_flops(wl.B, wl.H, wl.d, wl.d)
                by = decode_bytes(wl.B, wl.H, wl.d, wl.d, 2 if wl.dtype == torch.bfloat16 else 4,
                                  wl.decay == "channel")
                e2e_ms, h2d, d2h = e2e_decode(xl, st_l, od_l, wl, max(64, min(dec_reps, 2000)),
                                              stream)
                n_e2e = max(64, min(dec_reps, 2000))
                legs[name] = {
                    "value": 1.0 / sec, "unit": "steps/s", "ms": sec * 1e3, "reps": dec_reps,
                    "tokens_per_s": wl.B / sec,
                    "roofline": roofline(fl, by, sec, pk, pk_kind,
                                         traffic_for("decode_kernel",
                                                     "gated_delta_rule_140_b200/csrc/gdn_decode.cu",
                                                     name),
                                         "decode_kernel"),
                    "e2e": {"value": n_e2e / (e2e_ms / 1e3), "unit": "steps/s",
                            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                    "config": {"N": wl.B, "H": wl.H, "d_k": wl.d, "d_v": wl.d,
                               "decay": wl.decay, "state": "fp32, in place"},
                }
                if world == 1 and not args.no_cpu_baseline:
                    legs[name]["cpu_baseline"] = cpu_baseline_decode(xl_cpu)
            else:
                leg = head if name == args.workload else PrefillLeg(name, dev, kflags, ws)
                for _ in range(3):
                    leg.run()
                t1 = time_loop(leg.run, 3, stream) / 3 / 1e3
                reps = max(K, math.ceil(args.leg_seconds / max(t1, 1e-6)))
                l0 = nat.launch_count()
                ms = time_loop(leg.run, reps, stream)
                n_leg_launches += nat.launch_count() - l0
                if ws.status() != nat.GDN_OK:
                    raise SystemExit(f"device-side error in leg {name}")
                sec = ms / reps / 1e3
                fl, by = leg.work()
                kern, src = leg.kernel()
                n_e2e = max(4, min(reps, math.ceil(2.0 / max(sec, 1e-6)), 200))
                e2e_ms, h2d, d2h = e2e_prefill(leg, n_e2e, stream)
                legs[name] = {
                    "value": leg.tokens / sec, "unit": "tokens/s", "ms": sec * 1e3,
                    "reps": reps,
                    "roofline": roofline(fl, by, sec, pk, pk_kind, traffic_for(kern, src, name),
                                         kern),
                    "e2e": {"value": leg.tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s",
                            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                    "config": {"B": leg.B, "T": leg.T, "H": leg.H, "d_k": leg.dk, "d_v": leg.dv,
                               "n_seqs": leg.n_seqs, "decay": leg.w.decay,
                               "initial_state": leg.x["initial_state"] is not None},
                }
                if world == 1 and not args.no_cpu_baseline:
                    legs[name]["cpu_baseline"] = cpu_baseline(name, SAMPLE_TOKEN_HEADS // 2)
                if leg is not head:
                    del leg
                    torch.cuda.empty_cache()
            legs[name]["clocks"] = clocks.summary(clocks.rows[rows0:])
    clocks.__exit__(None, None, None)
    barrier(world)

    if rank == 0:
        fl, by = head.work()
        kern, src = head.kernel()
        roof_pre = roofline(fl, by, pre_s, pk, pk_kind, traffic_for(kern, src, args.workload),
                            kern)
        dbytes = decode_bytes(wd.B, wd.H, wd.d, wd.d, 2 if wd.dtype == torch.bfloat16 else 4,
                              wd.decay == "channel")
        roof_dec = roofline(decode_flops(wd.B, wd.H, wd.d, wd.d), dbytes, dec_s, pk, pk_kind,
                            traffic_for("decode_kernel",
                                        "gated_delta_rule_140_b200/csrc/gdn_decode.cu",
                                        args.decode_workload),
                            "decode_kernel")
        dominant = roof_pre if pre_s >= dec_s else roof_dec
        hl = legs.get(args.workload)
        if hl is not None:
            e2e = dict(hl["e2e"])
            e2e["value"] *= world
        else:
            e2e_ms, h2d, d2h = e2e_prefill(head, max(K, 4), stream)
            e2e = {"value": world * head.tokens * max(K, 4) / (e2e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        line = {
            "metric": METRIC, "value": world * head.tokens / pre_s, "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if head.w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": headline_config(args.workload, args.decode_workload, world),
            "prefill": {"value": world * head.tokens / pre_s, "unit": "tokens/s",
                        "ms": pre_s * 1e3, "kernel": kern, "roofline": roof_pre},
            "decode": {"value": 1.0 / dec_s, "unit": "steps/s", "ms": dec_s * 1e3,
                       "tokens_per_s": world * wd.B / dec_s, "roofline": roof_dec},
            "roofline": {k: dominant[k] for k in
                         ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel")},
            "e2e": e2e,
            "gpu_launches": launches,
            "gpu_launches_legs": n_leg_launches,
            "clocks": clocks.summary(),
            "legs": legs,
        }
        if all(n in legs for n in FIG3_LEGS):
            # FG2-GDN Fig. 3's comparison: throughput of 32k x 1 over 2k x 16
            line["fig3_ratio_32kx1_over_2kx16"] = legs["fig3_32kx1"]["value"] / legs["fig3_2kx16"]["value"]
        if world == 1 and not args.no_cpu_baseline:
            if args.workload in legs and "cpu_baseline" in legs[args.workload]:
                line["cpu_baseline"] = legs[args.workload]["cpu_baseline"]
            else:
                line["cpu_baseline"] = cpu_baseline(args.workload)
            one = cpu_baseline(args.workload, SAMPLE_TOKEN_HEADS // 4, nthreads=1)
            one["sample"] += ", one thread"
            line["cpu_baseline_one_core"] = one
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def profile_once(args):
    """Run one prefill workload ``warmup + steps`` times (no timing, one GPU): the
    command the committed ncu captures profile, with -s/-c picking one launch."""
    import torch
    from gated_delta_rule_140_b200 import _native as nat
    from gated_delta_rule_140_b200 import chunk_fwd
    from gated_delta_rule_140_b200.inputs import workload_inputs
    name, _, tok = args.profile_once.partition(":")
    ov = {"T": int(tok)} if tok else {}
    x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
         for k, v in workload_inputs(name, **ov).items()}
    kw = {k: v for k, v in _kflags(args.prefill_kernel).items() if v}
    ws = nat.Workspace()
    for _ in range(args.warmup + args.steps):
        chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"],
                  x["cu_seqlens"], workspace=ws, **kw)
    torch.cuda.synchronize()
    st = ws.status()
    path = nat.chunk_fwd_path(nat.prefill_dims(x["q"], x["v"], x["log_alpha"], x["cu_seqlens"],
                                               beta_channel=x["beta"].dim() == 4, **kw))
    print(f"{name} {ov} [{path}] x{args.warmup + args.steps}: status {st}")
    return 0 if st == nat.GDN_OK else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gdn_prefill_bf16")
    ap.add_argument("--decode-workload", default="gdn_decode")
    ap.add_argument("--legs", default="all",
                    help="'all', 'none' or a comma-separated list of workloads timed on their own")
    ap.add_argument("--leg-seconds", type=float, default=1.0,
                    help="minimum device time of each leg's timed loop")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-kernel", choices=["default", "pool", "pair", "one_cta",
                                                 "cuda_cores"],
                    default="default",
                    help="prefill kernel: the library's choice, or force one of the "
                         "tensor-core kernels or the fp32 CUDA-core kernel")
    ap.add_argument("--fig3", action="store_true",
                    help="add the FG2-GDN Fig. 3 shape sweep to the legs: 32k tokens as 2k x 16, "
                         "4k x 8, 8k x 4, 16k x 2 and 32k x 1 (GDN, 16 heads, d = 128)")
    ap.add_argument("--profile-once", default=None, metavar="WORKLOAD[:T]",
                    help="no timing: run one prefill workload (optionally with T tokens per "
                         "sequence) warmup + steps times through the library and exit, for a "
                         "profiler capture of one launch")
    args = ap.parse_args()
    if args.profile_once:
        return profile_once(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1 and args.legs == "all":
        args.legs = "none"  # scaling runs time the headline step only
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
