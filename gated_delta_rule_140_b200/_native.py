"""ctypes binding of libgdn.so (include/gdn.h).

Argument marshalling only: shapes and dtypes of torch tensors are turned into a
``gdn_dims`` struct and raw device pointers, and the call is enqueued on the
current torch CUDA stream.  Every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if the library is missing the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdn.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "gdn.h")

GDN_OK, GDN_ERR_INVALID, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, \
    GDN_ERR_DEVICE_INPUT = range(6)
GDN_BF16, GDN_FP32 = 0, 1
GDN_DECAY_SCALAR, GDN_DECAY_CHANNEL = 0, 1
GDN_FLAG_CUDA_CORES, GDN_FLAG_PAIR, GDN_FLAG_ONE_CTA, GDN_FLAG_POOL = 1, 2, 4, 8
GDN_FLAG_BETA_CHANNEL = 16
GDN_FLAG_VALUE_RATE = 32


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "T", "H", "d_k", "d_v", "n_seqs", "dtype", "decay", "flags")]


_lib = None


def lib():
    """Load libgdn.so (built in-tree by ``python -m gated_delta_rule_140_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m gated_delta_rule_140_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    D = ctypes.POINTER(Dims)
    L.gdn_chunk_fwd_workspace_size.argtypes = [D]
    L.gdn_chunk_fwd_workspace_size.restype = sz
    L.gdn_chunk_fwd.argtypes = [D, vp, vp, vp, fp, fp, fp, vp, vp, fp, vp, sz, vp]
    L.gdn_chunk_fwd.restype = ctypes.c_int
    L.gdn_chunk_fwd_value_rate.argtypes = [D, vp, vp, vp, fp, fp, fp, fp, vp, vp, fp, vp, sz, vp]
    L.gdn_chunk_fwd_value_rate.restype = ctypes.c_int
    L.gdn_chunk_fwd_noalloc.argtypes = [D, vp, vp, vp, fp, fp, fp, vp, vp, fp, vp]
    L.gdn_chunk_fwd_noalloc.restype = ctypes.c_int
    L.gdn_recurrent_step.argtypes = [D, vp, vp, vp, fp, fp, fp, vp, vp]
    L.gdn_recurrent_step.restype = ctypes.c_int
    L.gdn_recurrent_verify.argtypes = [D, vp, vp, vp, fp, fp, fp, vp, vp, vp]
    L.gdn_recurrent_verify.restype = ctypes.c_int
    L.gdn_recurrent_verify_tree.argtypes = [D, vp, vp, vp, fp, fp, fp, vp, vp, vp, vp]
    L.gdn_recurrent_verify_tree.restype = ctypes.c_int
    L.gdn_state_compose.argtypes = [D, fp, fp, fp, fp, vp]
    L.gdn_state_compose.restype = ctypes.c_int
    L.gdn_state_identity.argtypes = [D, fp, vp]
    L.gdn_state_identity.restype = ctypes.c_int
    L.gdn_chunk_fwd_raw.argtypes = [D, vp, vp, vp, fp, fp, fp, fp, vp, vp, fp, vp, sz, vp]
    L.gdn_chunk_fwd_raw.restype = ctypes.c_int
    L.gdn_noalloc_status.argtypes = [vp]
    L.gdn_noalloc_status.restype = ctypes.c_int
    L.gdn_workspace_init.argtypes = [vp, sz, vp]
    L.gdn_workspace_init.restype = ctypes.c_int
    L.gdn_workspace_status.argtypes = [vp, vp]
    L.gdn_workspace_status.restype = ctypes.c_int
    L.gdn_chunk_fwd_path.argtypes = [D]
    L.gdn_chunk_fwd_path.restype = ctypes.c_char_p
    L.gdn_status_string.argtypes = [ctypes.c_int]
    L.gdn_status_string.restype = ctypes.c_char_p
    L.gdn_launch_count.argtypes = []
    L.gdn_launch_count.restype = ctypes.c_uint64
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of the functions include/gdn.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def launch_count() -> int:
    return int(lib().gdn_launch_count())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt):
    import torch
    if dt == torch.bfloat16:
        return GDN_BF16
    if dt == torch.float32:
        return GDN_FP32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {dt}")


def _check_dev(name, t, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def prefill_dims(q, v, log_alpha, cu_seqlens=None, cuda_cores=False, pair=False,
                 one_cta=False, pool=False, beta_channel=False, value_rate=False) -> Dims:
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    return Dims(B, T, H, dk, dv, (len(cu_seqlens) - 1) if cu_seqlens is not None else B,
                _dtype_code(q.dtype),
                GDN_DECAY_CHANNEL if log_alpha.dim() == 4 else GDN_DECAY_SCALAR,
                (GDN_FLAG_CUDA_CORES if cuda_cores else 0) | (GDN_FLAG_PAIR if pair else 0)
                | (GDN_FLAG_ONE_CTA if one_cta else 0) | (GDN_FLAG_POOL if pool else 0)
                | (GDN_FLAG_BETA_CHANNEL if beta_channel else 0)
                | (GDN_FLAG_VALUE_RATE if value_rate else 0))


def chunk_fwd_path(dims: Dims) -> str:
    """"tensor_core_pool", "tensor_core_pair", "tensor_core" or "cuda_core": the
    prefill kernel gdn_chunk_fwd selects."""
    r = lib().gdn_chunk_fwd_path(ctypes.byref(dims))
    if r is None:
        raise GdnError(GDN_ERR_INVALID, "gdn_chunk_fwd_path")
    return r.decode()


def workspace_size(dims: Dims) -> int:
    n = int(lib().gdn_chunk_fwd_workspace_size(ctypes.byref(dims)))
    if n == 0:
        raise GdnError(GDN_ERR_INVALID, "gdn_chunk_fwd_workspace_size")
    return n


class Workspace:
    """A zeroed device workspace that grows on demand (one per stream)."""

    def __init__(self, device=None):
        self.buf = None
        self.device = device

    def get(self, nbytes: int, stream=None):
        import torch
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device or "cuda")
        return self.buf

    def status(self, stream=None) -> int:
        """Synchronise the stream, read and clear the sticky device error word."""
        if self.buf is None:
            return GDN_OK
        return int(lib().gdn_workspace_status(_ptr(self.buf), _stream(stream)))

    def set_wait_limit(self, cycles: int, stream=None):
        """Test-only: the second header word replaces the tensor-core kernels'
        bounded-wait limit on data waits (0 restores the default)."""
        import torch
        if self.buf is None:
            self.get(256, stream)
        word = torch.tensor([int(cycles)], dtype=torch.int32).view(torch.uint8)
        self.buf[4:8].copy_(word.to(self.buf.device), non_blocking=False)


def noalloc_status(stream=None) -> int:
    """gdn_noalloc_status: the device errors of the last gdn_chunk_fwd_noalloc call."""
    return int(lib().gdn_noalloc_status(_stream(stream)))


def _raise_on_status(st: int, where: str):
    if st != GDN_OK:
        raise GdnError(st, where)


_default_ws = {}


def _workspace_for(device, stream) -> Workspace:
    key = (str(device), None if stream is None else stream.cuda_stream)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, *,
              output_final_state=True, o=None, final_state=None, workspace: Workspace = None,
              cuda_cores=False, pair=False, one_cta=False, pool=False, check=False,
              stream=None, beta_v=None):
    """Chunkwise prefill (gdn_chunk_fwd).  Returns (o, final_state or None).
    A ``beta`` of shape [B,T,H,d_k] (with channel decay) is FG2-GDN's writing rate
    per key channel (GDN_FLAG_BETA_CHANNEL); [B,T,H] is the usual scalar rate.
    ``beta_v`` [B,T,H,d_v] adds FG2-GDN+'s value-side rate (with a per-channel
    ``beta``; gdn_chunk_fwd_value_rate).
    ``cuda_cores`` / ``pool`` / ``pair`` / ``one_cta`` select the fp32
    CUDA-core kernel or one of the tensor-core kernels instead of the default
    (GDN_FLAG_*).  With ``check`` the call synchronises the stream afterwards
    and raises GdnError if the device recorded an error (bad cu_seqlens
    contents, an expired bounded wait, an internal error): without it such
    errors stay in the workspace's sticky word until ``workspace.status()``."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(name, t, q.dtype)
    _check_dev("log_alpha", log_alpha, torch.float32)
    _check_dev("beta", beta, torch.float32)
    _check_dev("initial_state", initial_state, torch.float32)
    _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    _check_dev("beta_v", beta_v, torch.float32)
    beta_channel = beta is not None and beta.dim() == 4
    dims = prefill_dims(q, v, log_alpha, cu_seqlens, cuda_cores, pair, one_cta, pool,
                        beta_channel, beta_v is not None)
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(dims.n_seqs, dims.H, dims.d_v, dims.d_k, dtype=torch.float32,
                                  device=q.device)
    ws = workspace if workspace is not None else _workspace_for(q.device, stream)
    nbytes = workspace_size(dims)
    buf = ws.get(nbytes, stream)
    if beta_v is not None:
        st = lib().gdn_chunk_fwd_value_rate(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(log_alpha), _ptr(beta), _ptr(beta_v),
                                            _ptr(initial_state), _ptr(cu_seqlens), _ptr(o),
                                            _ptr(final_state), _ptr(buf),
                                            ctypes.c_size_t(buf.numel()), _stream(stream))
    else:
        st = lib().gdn_chunk_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                 _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), _ptr(o),
                                 _ptr(final_state), _ptr(buf), ctypes.c_size_t(buf.numel()),
                                 _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_value_rate" if beta_v is not None else "gdn_chunk_fwd")
    if check:
        _raise_on_status(ws.status(stream), "gdn_chunk_fwd (device)")
    return o, final_state


def chunk_fwd_raw(q_raw, k_raw, v, alpha_logit, beta_logit, alpha_bias=None,
                  initial_state=None, cu_seqlens=None, *, output_final_state=True, o=None,
                  final_state=None, workspace: Workspace = None, check=False, stream=None):
    """Chunkwise prefill with the input prologue fused in (gdn_chunk_fwd_raw):
    q_raw, k_raw unnormalised, alpha_logit [B,T,H] and beta_logit [B,T,H]
    logits, alpha_bias [H] or None.  The kernel L2-normalises q and k, takes
    beta = sigmoid(beta_logit) and log alpha = -softplus(alpha_logit + bias).
    Returns (o, final_state or None)."""
    import torch
    for name, t in (("q_raw", q_raw), ("k_raw", k_raw), ("v", v)):
        _check_dev(name, t, q_raw.dtype)
    _check_dev("alpha_logit", alpha_logit, torch.float32)
    _check_dev("beta_logit", beta_logit, torch.float32)
    _check_dev("alpha_bias", alpha_bias, torch.float32)
    _check_dev("initial_state", initial_state, torch.float32)
    _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    dims = prefill_dims(q_raw, v, alpha_logit, cu_seqlens, pool=True)
    if o is None:
        o = torch.empty(v.shape, dtype=q_raw.dtype, device=q_raw.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(dims.n_seqs, dims.H, dims.d_v, dims.d_k, dtype=torch.float32,
                                  device=q_raw.device)
    ws = workspace if workspace is not None else _workspace_for(q_raw.device, stream)
    # (a shape the fused path does not take has no workspace size: the call
    # itself then returns its status)
    buf = ws.get(max(256, int(lib().gdn_chunk_fwd_workspace_size(ctypes.byref(dims)))), stream)
    st = lib().gdn_chunk_fwd_raw(ctypes.byref(dims), _ptr(q_raw), _ptr(k_raw), _ptr(v),
                                 _ptr(alpha_logit), _ptr(alpha_bias), _ptr(beta_logit),
                                 _ptr(initial_state), _ptr(cu_seqlens), _ptr(o),
                                 _ptr(final_state), _ptr(buf), ctypes.c_size_t(buf.numel()),
                                 _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_raw")
    if check:
        _raise_on_status(ws.status(stream), "gdn_chunk_fwd_raw (device)")
    return o, final_state


def recurrent_verify(q, k, v, log_alpha, beta, state, n_commit=None, *, outputs=True, o=None,
                     check=False, stream=None, parent=None):
    """Multi-token verification (gdn_recurrent_verify): K draft tokens per sequence
    from ``state`` [N,H,dv,dk] fp32.  q, k [N,K,H,dk]; v [N,K,H,dv]; log_alpha
    [N,K,H] or [N,K,H,dk]; beta [N,K,H]; ``n_commit`` int32 [N] on the device or
    None.  Returns o [N,K,H,dv] (None with ``outputs=False``); the state becomes
    the state after the first n_commit[n] tokens of each sequence (untouched for
    None or 0).  With ``parent`` int32 [N,K] on the device the drafts form a tree
    (gdn_recurrent_verify_tree): node j follows node parent[n][j] (-1: the state),
    its output is read after the path to it, and n_commit[n] = c commits the state
    after node c - 1's path."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(name, t, q.dtype)
    _check_dev("log_alpha", log_alpha, torch.float32)
    _check_dev("beta", beta, torch.float32)
    _check_dev("state", state, torch.float32)
    _check_dev("n_commit", n_commit, torch.int32)
    _check_dev("parent", parent, torch.int32)
    N, K, H, dk = q.shape
    dv = v.shape[-1]
    dims = Dims(N, K, H, dk, dv, N, _dtype_code(q.dtype),
                GDN_DECAY_CHANNEL if log_alpha.dim() == 4 else GDN_DECAY_SCALAR, 0)
    if outputs and o is None:
        o = torch.empty(N, K, H, dv, dtype=q.dtype, device=q.device)
    if not outputs:
        o = None
    if parent is not None:
        st = lib().gdn_recurrent_verify_tree(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v),
                                             _ptr(log_alpha), _ptr(beta), _ptr(state),
                                             _ptr(parent), _ptr(n_commit), _ptr(o),
                                             _stream(stream))
    else:
        st = lib().gdn_recurrent_verify(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(log_alpha), _ptr(beta), _ptr(state), _ptr(n_commit),
                                        _ptr(o), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_recurrent_verify_tree" if parent is not None else
                       "gdn_recurrent_verify")
    if check:
        s = stream if stream is not None else torch.cuda.current_stream()
        try:
            s.synchronize()
        except RuntimeError as e:
            raise GdnError(GDN_ERR_CUDA, f"gdn_recurrent_verify (device): {e}") from e
    return o


def _state_dims(N, H, dk, dv):
    return Dims(N, 0, H, dk, dv, N, GDN_FP32, GDN_DECAY_SCALAR, 0)


def state_compose(s, m, b=None, *, out=None, stream=None):
    """out = s m (+ b) per (sequence, head) through gdn_state_compose: s, b
    [N,H,dv,dk] and m [N,H,dk,dk] fp32 on the device.  Composes segment state
    maps (S_start M + B); ``out`` may be ``b``, not ``s`` or ``m``."""
    import torch
    for name, t in (("s", s), ("m", m), ("b", b), ("out", out)):
        _check_dev(name, t, torch.float32)
    N, H, dv, dk = s.shape
    if tuple(m.shape) != (N, H, dk, dk) or (b is not None and tuple(b.shape) != tuple(s.shape)):
        raise ValueError("state_compose: s [N,H,dv,dk], m [N,H,dk,dk], b like s")
    if out is None:
        out = torch.empty_like(s)
    st = lib().gdn_state_compose(ctypes.byref(_state_dims(N, H, dk, dv)), _ptr(s), _ptr(m),
                                 _ptr(b), _ptr(out), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_state_compose")
    return out


def state_identity(N, H, d, device, *, out=None, stream=None):
    """An identity state per (sequence, head), fp32 [N,H,d,d] (gdn_state_identity):
    the initial state from which a prefill with v = 0 returns a segment's
    transition matrix."""
    import torch
    if out is None:
        out = torch.empty(N, H, d, d, dtype=torch.float32, device=device)
    _check_dev("out", out, torch.float32)
    st = lib().gdn_state_identity(ctypes.byref(_state_dims(N, H, d, d)), _ptr(out), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_state_identity")
    return out


def recurrent_step(q, k, v, log_alpha, beta, state, *, o=None, check=False, stream=None):
    """One decode step (gdn_recurrent_step); ``state`` [N,H,dv,dk] fp32 is updated
    in place.  q, k [N,H,dk]; v [N,H,dv]; log_alpha [N,H] or [N,H,dk]; beta [N,H].
    Returns o [N,H,dv].  The decode kernel has no device-detected errors (no
    waits, no offsets); with ``check`` the call synchronises the stream and
    raises if the launch or the kernel failed."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(name, t, q.dtype)
    _check_dev("log_alpha", log_alpha, torch.float32)
    _check_dev("beta", beta, torch.float32)
    _check_dev("state", state, torch.float32)
    N, H, dk = q.shape
    dv = v.shape[-1]
    dims = Dims(N, 1, H, dk, dv, N, _dtype_code(q.dtype),
                GDN_DECAY_CHANNEL if log_alpha.dim() == 3 else GDN_DECAY_SCALAR, 0)
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    st = lib().gdn_recurrent_step(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(log_alpha), _ptr(beta), _ptr(state), _ptr(o),
                                  _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_recurrent_step")
    if check:
        s = stream if stream is not None else torch.cuda.current_stream()
        try:
            s.synchronize()
        except RuntimeError as e:
            raise GdnError(GDN_ERR_CUDA, f"gdn_recurrent_step (device): {e}") from e
    return o
