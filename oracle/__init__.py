"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never links, loads
or calls it, and it shares no code with the CUDA path.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64); this module compiles
it with gcc on first use and marshals numpy / torch-CPU arrays through ctypes.

Functions
---------
recurrent(...)   the plain token-by-token definition (Gated DeltaNet scalar
                 decay, or KDA channel-wise decay), FG2-GDN paper section 1 and
                 section 5; o_t = S_t q_t with S in R^{d_v x d_k}.
chunkwise(...)   the chunkwise WY / UT-transform form of FG2-GDN section 3.6,
                 with explicit per-chunk matrices; equal to ``recurrent`` in
                 exact arithmetic.
chunk_stage(...) one chunk's intermediates (g, A, T, W, U, V', O, S_out).
prologue(...)    the input prologue of the fused entry point (FG2-GDN section
                 3.5): L2-normalised q and k, beta = sigmoid(b),
                 log alpha = -softplus(a + bias).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so next to it (gcc, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    common = [ctypes.c_int, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
              _D, _D, _D, _D, _D, _D, _D, _D]
    lib.oracle_gdn_recurrent.argtypes = common + [ctypes.c_int]
    lib.oracle_gdn_recurrent.restype = ctypes.c_int
    lib.oracle_gdn_chunkwise.argtypes = common + [ctypes.c_int, ctypes.c_int]
    lib.oracle_gdn_chunkwise.restype = ctypes.c_int
    lib.oracle_gdn_chunk_stage.argtypes = [ctypes.c_int] * 3 + [_D] * 14
    lib.oracle_gdn_chunk_stage.restype = None
    lib.oracle_gdn_prologue.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _D, _D, _D, _D, _D, _D, _D, _D, _D]
    lib.oracle_gdn_prologue.restype = ctypes.c_int
    lib.oracle_fg2_recurrent.argtypes = [ctypes.c_int, _I64, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int] + [_D] * 9 + [ctypes.c_int]
    lib.oracle_fg2_recurrent.restype = ctypes.c_int
    return lib


def build_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of the oracle source (used by the mutation tests
    to show that the pins catch planted mistakes)."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-shared", "-fPIC",
                           "-o", out_path, c_path, "-lm", "-lpthread"])
    return out_path


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _f64(x):
    """Any array-like (numpy, torch CPU in any float dtype) -> C-contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast exactly (bf16/fp32 -> fp64)
        import torch
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return a.ctypes.data_as(_D) if a is not None else None


def _problem(q, k, v, log_alpha, beta, initial_state, cu_seqlens):
    """Normalise to packed token-major arrays and sequence offsets.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; log_alpha: [B,T,H] or [B,T,H,dk];
    beta: [B,T,H].  With ``cu_seqlens`` (N+1 offsets) B must be 1 and the
    sequences are packed along T.
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    channel = la.ndim == 4
    if cu_seqlens is None:
        starts = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("cu_seqlens requires B == 1")
        starts = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens), dtype=np.int64)
    n = len(starts) - 1
    s0 = _f64(initial_state)
    if s0 is not None and s0.shape != (n, H, dv, dk):
        raise ValueError(f"initial_state must be {(n, H, dv, dk)}, got {s0.shape}")
    return q, k, v, la, b, s0, starts, (B, T, H, dk, dv, n, channel)


def recurrent(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, nthreads=0,
              return_threads=False):
    """Token-by-token recurrence in fp64.  Returns (o [B,T,H,dv], S_final [N,H,dv,dk])."""
    q, k, v, la, b, s0, starts, (B, T, H, dk, dv, n, channel) = _problem(
        q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    o = np.zeros((B, T, H, dv), np.float64)
    sf = np.zeros((n, H, dv, dk), np.float64)
    used = _load().oracle_gdn_recurrent(n, starts.ctypes.data_as(_I64), H, dk, dv, int(channel),
                                        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                        _ptr(o), _ptr(sf), int(nthreads))
    if used < 0:
        raise ValueError("oracle rejected its arguments")
    return (o, sf, used) if return_threads else (o, sf)


def chunkwise(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk=64,
              nthreads=0):
    """Chunkwise WY/UT form in fp64.  Returns (o, S_final) like ``recurrent``."""
    q, k, v, la, b, s0, starts, (B, T, H, dk, dv, n, channel) = _problem(
        q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    o = np.zeros((B, T, H, dv), np.float64)
    sf = np.zeros((n, H, dv, dk), np.float64)
    used = _load().oracle_gdn_chunkwise(n, starts.ctypes.data_as(_I64), H, dk, dv, int(channel),
                                        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                        _ptr(o), _ptr(sf), int(chunk), int(nthreads))
    if used < 0:
        raise ValueError("oracle rejected its arguments")
    return o, sf


def fg2_recurrent(q, k, v, log_alpha, beta_k, beta_v=None, initial_state=None, cu_seqlens=None,
                  nthreads=0):
    """FG2-GDN (FG2-GDN paper, sections 3.2, 3.4, 3.6; the update's equations are
    lost from the page): channel decay log_alpha [B,T,H,dk], key-side writing rate
    beta_k [B,T,H,dk] and, for FG2-GDN+, a value-side rate beta_v [B,T,H,dv]
    (None: FG2-GDN, no value gate).  Keys and values are scaled by the square
    roots of their rates, k~ = sqrt(beta_k) . k and v~ = sqrt(beta_v) . v, and
    S_t = S_{t-1} Diag(alpha_t) (I - k~ k~^T) + v~ k~^T,  o_t = S_t q_t, token by
    token in fp64.  Returns (o, S_final) like ``recurrent``."""
    bk = _f64(beta_k)
    bv = _f64(beta_v)
    dummy_beta = np.zeros(np.asarray(bk).shape[:3], np.float64)
    q, k, v, la, _, s0, starts, (B, T, H, dk, dv, n, channel) = _problem(
        q, k, v, log_alpha, dummy_beta, initial_state, cu_seqlens)
    if not channel:
        raise ValueError("FG2-GDN takes channel decay (log_alpha [B,T,H,dk])")
    if bk.shape != (B, T, H, dk):
        raise ValueError(f"beta_k must be {(B, T, H, dk)}, got {bk.shape}")
    if bv is not None and bv.shape != (B, T, H, dv):
        raise ValueError(f"beta_v must be {(B, T, H, dv)}, got {bv.shape}")
    o = np.zeros((B, T, H, dv), np.float64)
    sf = np.zeros((n, H, dv, dk), np.float64)
    used = _load().oracle_fg2_recurrent(n, starts.ctypes.data_as(_I64), H, dk, dv, _ptr(q),
                                        _ptr(k), _ptr(v), _ptr(la), _ptr(bk), _ptr(bv),
                                        _ptr(s0), _ptr(o), _ptr(sf), int(nthreads))
    if used < 0:
        raise ValueError("oracle rejected its arguments")
    return o, sf


def chunk_stage(q, k, v, log_alpha, beta, S):
    """One chunk of one head.  q,k [L,dk]; v [L,dv]; log_alpha [L] or [L,dk];
    beta [L]; S [dv,dk].  Returns a dict of the intermediates G, A, T, W, U, Vp,
    O and S_out (all fp64)."""
    q, k, v, la, b, S = (_f64(x) for x in (q, k, v, log_alpha, beta, S))
    L, dk = q.shape
    dv = v.shape[1]
    if la.ndim == 1:  # scalar decay: every key channel carries the same log decay
        la = np.ascontiguousarray(np.repeat(la[:, None], dk, axis=1))
    out = {name: np.zeros(shape, np.float64) for name, shape in
           (("G", (L, dk)), ("A", (L, L)), ("T", (L, L)), ("W", (L, dk)), ("U", (L, dv)),
            ("Vp", (L, dv)), ("O", (L, dv)), ("S_out", (dv, dk)))}
    _load().oracle_gdn_chunk_stage(L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
                                   _ptr(S), *(_ptr(out[x]) for x in
                                              ("G", "A", "T", "W", "U", "Vp", "O", "S_out")))
    return out


def prologue(q_raw, k_raw, a_logit, b_logit, a_bias=None):
    """The fused entry point's input prologue in fp64.  q_raw, k_raw [...,H,dk];
    a_logit [...,H] (scalar decay) or [...,H,dk] (channel decay); b_logit
    [...,H]; a_bias [H] or [H,dk] or None.  Returns (q, k, log_alpha, beta) as
    float64 arrays of the input shapes."""
    qr, kr, al, bl = (_f64(x) for x in (q_raw, k_raw, a_logit, b_logit))
    H, dk = qr.shape[-2], qr.shape[-1]
    ntok = qr.size // (H * dk)
    channel = al.shape == qr.shape
    ab = _f64(a_bias)
    if ab is not None and ab.size != (H * dk if channel else H):
        raise ValueError("a_bias must be [H] (scalar decay) or [H, d_k] (channel decay)")
    q, k = np.zeros_like(qr), np.zeros_like(kr)
    la, b = np.zeros_like(al), np.zeros_like(bl)
    r = _load().oracle_gdn_prologue(ntok, H, dk, int(channel), _ptr(qr), _ptr(kr), _ptr(al),
                                    _ptr(ab), _ptr(bl), _ptr(q), _ptr(k), _ptr(la), _ptr(b))
    if r != 0:
        raise ValueError("oracle rejected its arguments")
    return q, k, la, b
