"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
the benchmark.

This module holds no arithmetic of the gated delta rule: it only draws the
inputs the method consumes, with the distributions of the workloads (the
1.3B-scale linear-attention layers of the FG2-GDN paper, section 3.5: d_k =
d_v = 128, L2-normalised queries and keys, beta from a sigmoid, decay from a
negative softplus).  Everything is drawn on the CPU from
``torch.Generator().manual_seed(seed)`` in fp32, in a fixed order, then cast.

Draw order for one prefill problem: [varlen lengths], q, k, v, beta logits,
decay logits, initial state.  The decode problem draws the state first, then
for each step q, k, v, beta logits, decay logits.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.nn.functional as F

__all__ = ["WORKLOADS", "Workload", "prefill_inputs", "decode_inputs", "varlen_lengths",
           "raw_prefill_inputs"]


@dataclass(frozen=True)
class Workload:
    """One named problem: shapes, dtype, decay kind and the seed."""
    name: str
    kind: str                 # "prefill" or "decode"
    H: int
    d: int
    dtype: torch.dtype
    decay: str = "scalar"     # "scalar" (GDN) or "channel" (KDA)
    B: int = 1
    T: int = 0
    seed: int = 0
    alpha_shift: float = 2.0  # log alpha = -softplus(N(0,1) + alpha_shift)
    init_std: float | None = None
    n_seqs: int = 0           # > 0: variable-length packed batch
    len_range: tuple = field(default=(0, 0))
    steps: int = 0            # decode steps
    beta_channel: bool = False  # FG2-GDN: beta per key channel [B,T,H,dk]
    fast_channels: int = 0    # KDA: the first n key channels of every head decay at
    fast_log_alpha: float = -30.0  # this log alpha per token (fast-forgetting channels)


WORKLOADS = {
    w.name: w for w in (
        Workload("gdn_tiny_fp32", "prefill", H=2, d=64, dtype=torch.float32, B=1, T=256, seed=0),
        Workload("gdn_prefill_bf16", "prefill", H=16, d=128, dtype=torch.bfloat16, B=4, T=4096,
                 seed=1),
        Workload("gdn_varlen_bf16", "prefill", H=16, d=128, dtype=torch.bfloat16, seed=2,
                 init_std=0.02, n_seqs=32, len_range=(256, 4096)),
        Workload("kda_prefill_bf16", "prefill", H=32, d=128, dtype=torch.bfloat16, B=2, T=8192,
                 decay="channel", alpha_shift=3.0, seed=3),
        Workload("gdn_decode", "decode", H=32, d=128, dtype=torch.bfloat16, B=256, steps=64,
                 init_std=0.02, seed=4),
        Workload("kda_decode", "decode", H=32, d=128, dtype=torch.bfloat16, B=256, steps=64,
                 decay="channel", alpha_shift=3.0, init_std=0.02, seed=7),
        Workload("gdn_long_prefill_bf16", "prefill", H=32, d=128, dtype=torch.bfloat16, B=1,
                 T=65536, seed=5),
        Workload("kda_fast8_prefill_bf16", "prefill", H=32, d=128, dtype=torch.bfloat16, B=2,
                 T=8192, decay="channel", alpha_shift=3.0, seed=3, fast_channels=8),
        Workload("fg2_prefill_bf16", "prefill", H=32, d=128, dtype=torch.bfloat16, B=2,
                 T=8192, decay="channel", alpha_shift=3.0, seed=6, beta_channel=True),
        # FG2-GDN section 4.5, Fig. 3: prefill shapes of 32k tokens, sequence length x batch
        # from 2k x 16 to 32k x 1 (GDN layers of the 1.3B models: 16 heads of d = 128)
        *(Workload(f"fig3_{T // 1024}kx{32768 // T}", "prefill", H=16, d=128,
                   dtype=torch.bfloat16, B=32768 // T, T=T, seed=8)
          for T in (2048, 4096, 8192, 16384, 32768)),
    )
}


def varlen_lengths(n: int, lo: int, hi: int, gen: torch.Generator) -> torch.Tensor:
    """n integer lengths uniform on [lo, hi] inclusive."""
    return torch.randint(lo, hi + 1, (n,), generator=gen, dtype=torch.int64)


def _unit(x: torch.Tensor) -> torch.Tensor:
    """L2-normalise the last axis (per token and head), in fp32."""
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                   decay: str = "scalar", seed: int = 0, alpha_shift: float = 2.0,
                   init_std: float | None = None, lengths=None, gen=None,
                   beta_channel: bool = False) -> dict:
    """Draw one prefill problem on the CPU.

    Returns a dict with q, k [B,T,H,dk] and v [B,T,H,dv] in ``dtype``;
    log_alpha [B,T,H] (scalar decay) or [B,T,H,dk] (channel decay) and beta
    [B,T,H] (or [B,T,H,dk] with ``beta_channel``: FG2-GDN's rate per key
    channel) in fp32; initial_state [N,H,dv,dk] fp32 or None; cu_seqlens int32
    [N+1] or None.  With ``lengths`` the batch is packed (B = 1, T = sum).
    """
    g = gen if gen is not None else torch.Generator().manual_seed(seed)
    cu = None
    if lengths is not None:
        lengths = torch.as_tensor(lengths, dtype=torch.int64)
        B, T = 1, int(lengths.sum())
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lengths, 0).to(torch.int32)
    n_seqs = B if cu is None else len(cu) - 1
    q = _unit(torch.randn(B, T, H, dk, generator=g)).to(dtype)
    k = _unit(torch.randn(B, T, H, dk, generator=g)).to(dtype)
    v = torch.randn(B, T, H, dv, generator=g).to(dtype)
    beta = torch.sigmoid(torch.randn(*((B, T, H, dk) if beta_channel else (B, T, H)), generator=g))
    la_shape = (B, T, H) if decay == "scalar" else (B, T, H, dk)
    log_alpha = -F.softplus(torch.randn(*la_shape, generator=g) + alpha_shift)
    s0 = None
    if init_std is not None:
        s0 = torch.randn(n_seqs, H, dv, dk, generator=g) * init_std
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, initial_state=s0, cu_seqlens=cu)


def decode_inputs(N: int, H: int, dk: int, dv: int, steps: int, *, dtype=torch.bfloat16,
                  decay: str = "scalar", seed: int = 0, alpha_shift: float = 2.0,
                  init_std: float = 0.02) -> dict:
    """Draw a decode problem: state [N,H,dv,dk] fp32 and per-step q, k [S,N,H,dk],
    v [S,N,H,dv] (``dtype``), beta [S,N,H] and log_alpha [S,N,H] or [S,N,H,dk]."""
    g = torch.Generator().manual_seed(seed)
    state = torch.randn(N, H, dv, dk, generator=g) * init_std
    q = _unit(torch.randn(steps, N, H, dk, generator=g)).to(dtype)
    k = _unit(torch.randn(steps, N, H, dk, generator=g)).to(dtype)
    v = torch.randn(steps, N, H, dv, generator=g).to(dtype)
    beta = torch.sigmoid(torch.randn(steps, N, H, generator=g))
    la_shape = (steps, N, H) if decay == "scalar" else (steps, N, H, dk)
    log_alpha = -F.softplus(torch.randn(*la_shape, generator=g) + alpha_shift)
    return dict(state=state, q=q, k=k, v=v, beta=beta, log_alpha=log_alpha)


def workload_inputs(name: str, **overrides) -> dict:
    """Inputs of a named workload (overrides change shapes, e.g. for a reduced case)."""
    w = WORKLOADS[name]
    H = overrides.get("H", w.H)
    d = overrides.get("d", w.d)
    if w.kind == "decode":
        return decode_inputs(overrides.get("B", w.B), H, d, d, overrides.get("steps", w.steps),
                             dtype=w.dtype, decay=w.decay, seed=w.seed,
                             alpha_shift=w.alpha_shift, init_std=w.init_std)
    g = torch.Generator().manual_seed(w.seed)
    lengths = None
    if w.n_seqs:
        n = overrides.get("n_seqs", w.n_seqs)
        lo, hi = overrides.get("len_range", w.len_range)
        lengths = varlen_lengths(n, lo, hi, g)
    x = prefill_inputs(overrides.get("B", w.B), overrides.get("T", w.T), H, d, d,
                       dtype=w.dtype, decay=w.decay, alpha_shift=w.alpha_shift,
                       init_std=w.init_std, lengths=lengths, gen=g, beta_channel=w.beta_channel)
    if w.fast_channels:
        x["log_alpha"][..., :w.fast_channels] = w.fast_log_alpha
    return x


def raw_prefill_inputs(B: int, T: int, H: int, d: int, *, seed: int = 0, bias: float = 2.0,
                       dtype=torch.bfloat16) -> dict:
    """Inputs of the fused entry point (gdn_chunk_fwd_raw) before any
    normalisation: q_raw, k_raw ~ N(0,1) times a per-token scale in [0.5, 3.5];
    v ~ N(0,1); decay and writing-rate logits ~ N(0,1); a per-head decay bias
    (``bias``, so that the decay has the distribution of the prefill workloads).
    Draw order: q scale, q, k scale, k, v, decay logits, rate logits."""
    g = torch.Generator().manual_seed(seed)
    qs = 0.5 + 3.0 * torch.rand(B, T, H, 1, generator=g)
    q = (torch.randn(B, T, H, d, generator=g) * qs).to(dtype)
    ks = 0.5 + 3.0 * torch.rand(B, T, H, 1, generator=g)
    k = (torch.randn(B, T, H, d, generator=g) * ks).to(dtype)
    v = torch.randn(B, T, H, d, generator=g).to(dtype)
    a = torch.randn(B, T, H, generator=g)
    b = torch.randn(B, T, H, generator=g)
    return dict(q_raw=q, k_raw=k, v=v, alpha_logit=a, beta_logit=b,
                alpha_bias=torch.full((H,), float(bias)))
