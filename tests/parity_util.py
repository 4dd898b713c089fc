"""Helpers for the GPU-vs-oracle parity tests.

Error measure (the stated tolerance): max |gpu - oracle| divided by the max
|oracle| of the same tensor.  Bounds: 2e-2 on o and 1e-2 on the final state
for bf16 inputs with fp32 accumulation; 1e-4 on both for fp32 inputs.
"""
import json
import os

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}


def rel_err(gpu, ref) -> float:
    g = gpu.detach().to("cpu", torch.float64).numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite values in the GPU result"
    scale = np.abs(r).max()
    return float(np.abs(g - r).max() / (scale if scale > 0 else 1.0))


def record_margin(case: str, err_o: float, tol_o: float, err_s: float, tol_s: float) -> None:
    """Append one case's achieved worst errors and its bounds as a JSON line to the
    file named by GDN_PARITY_MARGINS (nothing is written when it is unset), so that
    a run can report how much of each tolerance a configuration uses."""
    path = os.environ.get("GDN_PARITY_MARGINS")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"case": case, "o_err": err_o, "o_tol": tol_o, "state_err": err_s,
                            "state_tol": tol_s}) + "\n")


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def oracle_heads(x: dict, picks, nthreads=0):
    """Run the oracle on sampled (sequence, head) chains only.  Chains are
    independent, so slicing the inputs to one chain is exact.  Returns a list
    of (n, h, o [L,dv], S_final [dv,dk]) in fp64."""
    out = []
    cu = x.get("cu_seqlens")
    for n, h in picks:
        if cu is None:
            sl = (slice(n, n + 1), slice(None), slice(h, h + 1))
        else:
            s, e = int(cu[n]), int(cu[n + 1])
            sl = (slice(0, 1), slice(s, e), slice(h, h + 1))
        args = [x[name][sl] for name in ("q", "k", "v", "log_alpha", "beta")]
        s0 = None if x.get("initial_state") is None else x["initial_state"][n:n + 1, h:h + 1]
        if x["beta"].dim() == 4:  # FG2-GDN: rate per key channel
            o, sf = oracle.fg2_recurrent(*args, None, s0, nthreads=nthreads)
        else:
            o, sf = oracle.recurrent(*args, s0, nthreads=nthreads)
        out.append((n, h, o[0, :, 0], sf[0, 0]))
    return out


def gpu_head(x: dict, o_gpu, sf_gpu, n, h):
    cu = x.get("cu_seqlens")
    if cu is None:
        o = o_gpu[n, :, h]
    else:
        o = o_gpu[0, int(cu[n]):int(cu[n + 1]), h]
    return o, (None if sf_gpu is None else sf_gpu[n, h])
