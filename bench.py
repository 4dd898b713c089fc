"""Throughput of the gated delta rule hot path on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--decode-workload NAME]
                    [--prefill-kernel default|pair|one_cta|cuda_cores]

A step is one pass of the whole hot path on one GPU:
  * prefill leg: gdn_chunk_fwd over one batch of the prefill workload
    (default: GDN bf16, B=4, H=16, T=4096, d_k=d_v=128; cumulative decay, A,
    T=(I+A)^-1, W/U, inter-chunk state pass, output), then
  * decode leg: one gdn_recurrent_step over the decode workload (N=256
    sequences, H=32, d=128, fp32 state updated in place).
``value`` is prefill tokens/s over all ranks: tokens processed by all ranks
divided by the max over ranks of the summed prefill-leg device time (CUDA
events on the launching stream).  The decode leg is reported in ``decode``
(steps/s).  ``ms_per_step`` is the device time of whole steps, barrier to
barrier, max over ranks.  Under torchrun (N > 1) every rank runs its own
independent batch (the problems shard with no data-path collective): weak
scaling.  Inputs are larger than L2 (prefill 275 MB, decode state 537 MB), so
no flush is needed between steps.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of the same prefill workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule prefill tokens/s and decode steps/s; % of roofline on 1 B200"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- #
# helpers                                                                     #
# --------------------------------------------------------------------------- #
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def prefill_bytes(w, B, T, H, dk, dv, n_seqs, has_s0, has_sf):
    """Algorithmic HBM bytes of one prefill: q, k, v read and o written once
    (element size of the dtype), fp32 log alpha (per key channel for KDA) and
    beta read once, and the fp32 states read/written once where present."""
    import torch
    es = 2 if w.dtype == torch.bfloat16 else 4
    tok = B * T * H
    per_tok = es * (2 * dk + 2 * dv) + 4 * (dk if w.decay == "channel" else 1) + 4
    state = n_seqs * H * dv * dk * 4
    return tok * per_tok + state * (int(has_s0) + int(has_sf))


def decode_bytes(N, H, dk, dv, es=2, channel=False):
    """Per step: fp32 state read + written, q/k/v read and o written, gates read."""
    return N * H * (2 * 4 * dv * dk + es * (2 * dk + 2 * dv) + 4 * (dk if channel else 1) + 4)


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

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = sorted(float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit())
        mx = max((float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if len(r) > 4 + i and r[4 + i].lower().startswith("active")})
        power = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(self.rows),
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
    sha = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    return rec.get("bytes_per_launch") if rec.get("src_sha") == sha else None


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
# the reference arm: the fp64 oracle on the host cores                        #
# --------------------------------------------------------------------------- #
SAMPLE_TOKEN_HEADS = 262144  # about 10 s of one host core for the fp64 oracle at d = 128


def oracle_sample(workload):
    """A bounded sample of the workload for the oracle: whole sequences from the
    start of the batch (all heads) until about SAMPLE_TOKEN_HEADS token-heads,
    cut to the first tokens of one sequence when a single one is larger."""
    from gated_delta_rule_140_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS[workload]
    x = workload_inputs(workload)
    H = w.H
    budget = max(1, SAMPLE_TOKEN_HEADS // H)  # tokens
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


def _oracle_pass(s, s0, cu):
    import oracle
    _, _, used = oracle.recurrent(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], s0, cu,
                                  return_threads=True)
    return used


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores, each
    step one pass over the bounded sample of the workload (rank 0 only)."""
    if rank != 0:
        return 0
    from gated_delta_rule_140_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
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
        "config": {"workload": args.workload, "B": w.B, "T": w.T, "H": w.H, "d": w.d},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": desc + ", fp64, one pass per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(workload):
    """The oracle timed on the host cores on the bounded sample, one pass."""
    s, s0, cu, ntok, desc = oracle_sample(workload)
    t0 = time.perf_counter()
    used = _oracle_pass(s, s0, cu)
    dt = time.perf_counter() - t0
    return {"value": ntok / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": desc + ", fp64, one pass"}


# --------------------------------------------------------------------------- #
# our arm                                                                     #
# --------------------------------------------------------------------------- #
def run_ours(args, rank, world, local):
    import torch
    from gated_delta_rule_140_b200 import _native as nat
    from gated_delta_rule_140_b200 import chunk_fwd, recurrent_step
    from gated_delta_rule_140_b200.inputs import WORKLOADS, workload_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_pg("nccl", world)
    nat.lib()

    wp, wd = WORKLOADS[args.workload], WORKLOADS[args.decode_workload]
    xp = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
          for k, v in workload_inputs(args.workload).items()}
    xd = {k: v.to(dev) for k, v in workload_inputs(args.decode_workload).items()}
    B, T, H, dk = xp["q"].shape
    dv = xp["v"].shape[-1]
    n_seqs = B if xp["cu_seqlens"] is None else len(xp["cu_seqlens"]) - 1
    tokens = B * T
    o = torch.empty_like(xp["v"])
    sf = torch.empty(n_seqs, H, dv, dk, dtype=torch.float32, device=dev)
    ws = nat.Workspace(dev)
    state = xd["state"].clone()
    od = torch.empty(wd.B, wd.H, wd.d, dtype=wd.dtype, device=dev)
    steps_d = xd["q"].shape[0]
    stream = torch.cuda.current_stream()

    kflags = {"pair": args.prefill_kernel == "pair",
              "one_cta": args.prefill_kernel == "one_cta",
              "cuda_cores": args.prefill_kernel == "cuda_cores"}

    def prefill():
        chunk_fwd(xp["q"], xp["k"], xp["v"], xp["log_alpha"], xp["beta"], xp["initial_state"],
                  xp["cu_seqlens"], o=o, final_state=sf, workspace=ws, **kflags)

    def decode(t):
        i = t % steps_d
        recurrent_step(xd["q"][i], xd["k"][i], xd["v"][i], xd["log_alpha"][i], xd["beta"][i],
                       state, o=od)

    for t in range(args.warmup):
        prefill()
        decode(t)
    torch.cuda.synchronize()
    if ws.status() != nat.GDN_OK:
        raise SystemExit("device-side error in warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    launches0 = nat.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for t in range(K):
            ev[t][0].record(stream)
            prefill()
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

    # end-to-end through the public API with host buffers: every step copies its
    # inputs in from pinned host memory, runs the call, and copies o and the final
    # state back.  As in a serving loop, consecutive steps overlap on three streams
    # (copy-in, compute, copy-out) with double-buffered device inputs and outputs:
    # step t + 1's inputs upload while step t computes and downloads.
    pin = {k: (v.cpu().pin_memory() if isinstance(v, torch.Tensor) else None)
           for k, v in xp.items()}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    sf_h = torch.empty(sf.shape, dtype=sf.dtype).pin_memory()
    dbuf = [{k: (torch.empty_like(v) if isinstance(v, torch.Tensor) else None)
             for k, v in xp.items()} for _ in range(2)]
    obuf = [(torch.empty_like(o), torch.empty_like(sf)) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = o_h.numel() * o_h.element_size() + sf_h.numel() * sf_h.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        """n overlapped end-to-end steps; returns their device time in ms."""
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
            chunk_fwd(ib["q"], ib["k"], ib["v"], ib["log_alpha"], ib["beta"],
                      ib["initial_state"], ib["cu_seqlens"], o=obuf[b][0],
                      final_state=obuf[b][1], workspace=ws, **kflags)
            ev["comp"][t].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp"][t])
                o_h.copy_(obuf[b][0], non_blocking=True)
                sf_h.copy_(obuf[b][1], non_blocking=True)
                ev["out"][t].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    e2e_run(2)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_run(K), world, dev)
    barrier(world)
    if ws.status() != nat.GDN_OK:
        raise SystemExit("device-side error in the timed region")

    if rank == 0:
        pk, pk_kind = peaks()
        hbm = pk["hbm_gbs"]
        has_s0 = xp["initial_state"] is not None
        pbytes = prefill_bytes(wp, B, T, H, dk, dv, n_seqs, has_s0, True)
        dbytes = decode_bytes(wd.B, wd.H, wd.d, wd.d, 2 if wd.dtype == torch.bfloat16 else 4,
                              wd.decay == "channel")
        pre_s, dec_s = pre_ms / K / 1e3, dec_ms / K / 1e3
        path = nat.chunk_fwd_path(nat.prefill_dims(xp["q"], xp["v"], xp["log_alpha"],
                                                   xp["cu_seqlens"], **kflags))
        pre_kernel, pre_src = {
            "tensor_core_pair": ("chunk_pair_kernel", "gdn_chunk_pair.cu"),
            "tensor_core": ("chunk_tc_kernel", "gdn_chunk_tc.cu"),
        }.get(path, ("chunk_simt_kernel", "gdn_chunk_simt.cu"))
        pre_src = "gated_delta_rule_140_b200/csrc/" + pre_src
        roof_pre = {"bound": "hbm", "achieved": pbytes / pre_s / 1e9, "peak": hbm,
                    "unit": "GB/s", "frac": pbytes / pre_s / 1e9 / hbm,
                    "traffic": traffic_for(pre_kernel, pre_src, args.workload), "kernel": pre_kernel,
                    "alg_bytes": pbytes, "peak_source": pk_kind}
        roof_dec = {"bound": "hbm", "achieved": dbytes / dec_s / 1e9, "peak": hbm,
                    "unit": "GB/s", "frac": dbytes / dec_s / 1e9 / hbm,
                    "traffic": traffic_for("decode_kernel",
                                           "gated_delta_rule_140_b200/csrc/gdn_decode.cu"),
                    "kernel": "decode_kernel", "alg_bytes": dbytes, "peak_source": pk_kind}
        dominant = roof_pre if pre_s >= dec_s else roof_dec
        cfg = {"workload": args.workload, "B": B, "T": T, "H": H, "d_k": dk, "d_v": dv,
               "decay": wp.decay, "chunk": 64, "prefill_kernel": pre_kernel, "parallelism": f"dp{world} (independent batches)",
               "l2": "inputs larger than L2 (no flush)",
               "decode_workload": f"{args.decode_workload}: N={wd.B}, H={wd.H}, d={wd.d}, "
                                  "fp32 state in place"}
        line = {
            "metric": METRIC, "value": world * tokens / pre_s, "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wp.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": cfg,
            "prefill": {"value": world * tokens / pre_s, "unit": "tokens/s",
                        "ms": pre_s * 1e3, "roofline": roof_pre},
            "decode": {"value": 1.0 / dec_s, "unit": "steps/s", "ms": dec_s * 1e3,
                       "tokens_per_s": world * wd.B / dec_s, "roofline": roof_dec},
            "roofline": {k: dominant[k] for k in
                         ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel")},
            "e2e": {"value": world * tokens * K / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gdn_prefill_bf16")
    ap.add_argument("--decode-workload", default="gdn_decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-kernel", choices=["default", "pair", "one_cta", "cuda_cores"],
                    default="default",
                    help="prefill kernel: the library's choice, the two-CTA tensor-core "
                         "kernel (GDN_FLAG_PAIR) or the fp32 CUDA-core kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
