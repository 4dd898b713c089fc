"""The C ABI of libgdn.so on the host, without a GPU: the library loads, exports
every function include/gdn.h declares, and rejects bad arguments with a status
code before touching the device."""
import ctypes
import os
import subprocess

import pytest

from gated_delta_rule_140_b200 import _native as nat
from gated_delta_rule_140_b200 import build as B


@pytest.fixture(scope="module")
def L():
    B.build()
    return nat.lib()


def test_library_exports_every_declared_symbol(L):
    names = nat.header_functions()
    assert {"gdn_chunk_fwd", "gdn_recurrent_step", "gdn_chunk_fwd_workspace_size",
            "gdn_workspace_status", "gdn_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libgdn.so does not export {n}"
    out = subprocess.run(["nm", "-D", "--defined-only", nat.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_library_links_no_oracle_and_no_torch(L):
    out = subprocess.run(["ldd", nat.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out and "torch" not in out and "libc10" not in out
    syms = subprocess.run(["nm", "-D", nat.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle_" not in syms


def test_status_strings(L):
    for s in range(6):
        assert nat.status_string(s).startswith("GDN_")
    assert "unknown" in nat.status_string(99)


def _dims(**kw):
    d = dict(B=2, T=128, H=4, d_k=128, d_v=128, n_seqs=2, dtype=nat.GDN_BF16,
             decay=nat.GDN_DECAY_SCALAR, flags=0)
    d.update(kw)
    return nat.Dims(*(d[f] for f, _ in nat.Dims._fields_))


def test_workspace_size(L):
    n = L.gdn_chunk_fwd_workspace_size(ctypes.byref(_dims()))
    assert n >= 256 and n % 256 == 0
    assert L.gdn_chunk_fwd_workspace_size(ctypes.byref(_dims(d_k=96))) == 0
    assert L.gdn_chunk_fwd_workspace_size(None) == 0


def test_prefill_kernel_choice(L):
    """The library's choice for bf16 d = 128: channel decay on the two-CTA
    kernel; scalar decay on the pool kernel when the sequences average 2048
    tokens or more and the (sequence, head) chains number at most a quarter of
    the SMs (148 without a device), else on the two-CTA kernel from a mean of
    2048 tokens (B * T / n_seqs) and on the single-CTA kernel below; the flags
    override it, GDN_FLAG_ONE_CTA only for scalar decay and not with
    GDN_FLAG_PAIR; other shapes on CUDA cores."""
    path = lambda **kw: nat.chunk_fwd_path(_dims(**kw))
    # few long sequences: the pool kernel (chains <= 37)
    assert path(B=4, T=2048, n_seqs=4) == "tensor_core_pool"        # 16 chains
    assert path(B=4, T=2048, n_seqs=0) == "tensor_core_pool"        # n_seqs 0: B sequences
    assert path(B=1, T=65536, n_seqs=1, H=32) == "tensor_core_pool"  # 32 chains
    assert path(B=1, T=65536, n_seqs=9) == "tensor_core_pool"       # 36 chains
    # many: the two-CTA kernel from 2048 tokens, the single-CTA one below
    assert path(B=4, T=4096, n_seqs=4, H=16) == "tensor_core_pair"   # 64 chains
    assert path(B=1, T=65536, n_seqs=10) == "tensor_core_pair"      # 40 chains
    assert path(B=1, T=65536, n_seqs=32, H=16) == "tensor_core_pair"
    assert path(B=4, T=2047, n_seqs=0) == "tensor_core"
    assert path(B=1, T=65536, n_seqs=64) == "tensor_core"           # packed, mean 1024
    assert path(B=1, T=65536, n_seqs=1, flags=nat.GDN_FLAG_ONE_CTA) == "tensor_core"
    assert path(B=1, T=65536, n_seqs=1, flags=nat.GDN_FLAG_PAIR) == "tensor_core_pair"
    assert path(B=4, T=128, n_seqs=4, flags=nat.GDN_FLAG_PAIR) == "tensor_core_pair"
    assert path(B=4, T=128, n_seqs=4, flags=nat.GDN_FLAG_CUDA_CORES) == "cuda_core"
    assert path(decay=nat.GDN_DECAY_CHANNEL) == "tensor_core_pair"
    assert path(decay=nat.GDN_DECAY_CHANNEL, B=1, T=65536, n_seqs=1) == "tensor_core_pair"
    assert path(dtype=nat.GDN_FP32) == "cuda_core"
    assert path(d_k=64, d_v=64, flags=nat.GDN_FLAG_ONE_CTA) == "cuda_core"
    assert path(B=4, T=4096, n_seqs=4, flags=nat.GDN_FLAG_POOL) == "tensor_core_pool"
    assert path(B=4, T=128, n_seqs=4, flags=nat.GDN_FLAG_POOL) == "tensor_core_pool"
    assert path(dtype=nat.GDN_FP32, flags=nat.GDN_FLAG_POOL) == "cuda_core"
    for flags, decay in ((nat.GDN_FLAG_ONE_CTA | nat.GDN_FLAG_PAIR, nat.GDN_DECAY_SCALAR),
                         (nat.GDN_FLAG_POOL | nat.GDN_FLAG_PAIR, nat.GDN_DECAY_SCALAR),
                         (nat.GDN_FLAG_POOL | nat.GDN_FLAG_ONE_CTA, nat.GDN_DECAY_SCALAR),
                         (nat.GDN_FLAG_POOL, nat.GDN_DECAY_CHANNEL),
                         (nat.GDN_FLAG_ONE_CTA, nat.GDN_DECAY_CHANNEL), (32, nat.GDN_DECAY_SCALAR)):
        with pytest.raises(nat.GdnError):
            path(flags=flags, decay=decay)


def test_fg2_rate_per_key_channel_runs_on_the_two_cta_kernel_only(L):
    """GDN_FLAG_BETA_CHANNEL (FG2-GDN's writing rate per key channel) needs channel
    decay and the two-CTA kernel's shapes; it is a prefill-only option."""
    fg2 = nat.GDN_FLAG_BETA_CHANNEL
    ch = nat.GDN_DECAY_CHANNEL
    assert nat.chunk_fwd_path(_dims(decay=ch, flags=fg2)) == "tensor_core_pair"
    assert nat.chunk_fwd_path(_dims(decay=ch, flags=fg2 | nat.GDN_FLAG_PAIR)) == "tensor_core_pair"
    assert _call_fwd(L, _dims(flags=fg2)) == nat.GDN_ERR_INVALID                       # scalar decay
    assert _call_fwd(L, _dims(decay=ch, flags=fg2 | nat.GDN_FLAG_POOL)) == nat.GDN_ERR_INVALID
    assert _call_fwd(L, _dims(decay=ch, flags=fg2 | nat.GDN_FLAG_ONE_CTA)) == nat.GDN_ERR_INVALID
    assert _call_fwd(L, _dims(decay=ch, flags=fg2 | nat.GDN_FLAG_CUDA_CORES)) == \
        nat.GDN_ERR_UNSUPPORTED
    assert _call_fwd(L, _dims(decay=ch, flags=fg2, dtype=nat.GDN_FP32)) == nat.GDN_ERR_UNSUPPORTED
    assert _call_fwd(L, _dims(decay=ch, flags=fg2, d_k=64, d_v=64)) == nat.GDN_ERR_UNSUPPORTED
    d = _dims(B=8, T=1, n_seqs=8, decay=ch, flags=fg2)
    v = ctypes.c_void_p(FAKE)
    assert L.gdn_recurrent_step(ctypes.byref(d), v, v, v, v, v, v, v, None) == nat.GDN_ERR_UNSUPPORTED


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def _call_fwd(L, dims, **kw):
    p = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, cu=None, o=FAKE, sf=None,
             ws=FAKE, wsb=1 << 20)
    p.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.gdn_chunk_fwd(ctypes.byref(dims), v(p["q"]), v(p["k"]), v(p["v"]), v(p["la"]),
                           v(p["beta"]), v(p["s0"]), v(p["cu"]), v(p["o"]), v(p["sf"]),
                           v(p["ws"]), ctypes.c_size_t(p["wsb"]), None)


@pytest.mark.parametrize("case,kw,dims_kw,expect", [
    ("null q", dict(q=None), {}, nat.GDN_ERR_INVALID),
    ("null o", dict(o=None), {}, nat.GDN_ERR_INVALID),
    ("null workspace", dict(ws=None), {}, nat.GDN_ERR_INVALID),
    ("workspace too small", dict(wsb=16), {}, nat.GDN_ERR_INVALID),
    ("misaligned k", dict(k=FAKE + 2), {}, nat.GDN_ERR_INVALID),
    ("misaligned state", dict(s0=FAKE + 4), {}, nat.GDN_ERR_INVALID),
    ("misaligned beta", dict(beta=FAKE + 2), {}, nat.GDN_ERR_INVALID),
    ("d_k = 96", {}, dict(d_k=96), nat.GDN_ERR_UNSUPPORTED),
    ("d_v = 0", {}, dict(d_v=0), nat.GDN_ERR_INVALID),
    ("negative T", {}, dict(T=-1), nat.GDN_ERR_INVALID),
    ("H = 0", {}, dict(H=0), nat.GDN_ERR_INVALID),
    ("bad dtype", {}, dict(dtype=7), nat.GDN_ERR_INVALID),
    ("bad decay", {}, dict(decay=3), nat.GDN_ERR_INVALID),
    ("bad flags", {}, dict(flags=32), nat.GDN_ERR_INVALID),
    ("FG2 rate with scalar decay", {}, dict(flags=16), nat.GDN_ERR_INVALID),
    ("n_seqs != B", {}, dict(n_seqs=3), nat.GDN_ERR_INVALID),
    ("cu_seqlens with B > 1", dict(cu=FAKE), dict(n_seqs=2), nat.GDN_ERR_INVALID),
    ("cu_seqlens with no sequences", dict(cu=FAKE), dict(B=1, n_seqs=0), nat.GDN_ERR_INVALID),
])
def test_chunk_fwd_rejects_bad_arguments(L, case, kw, dims_kw, expect):
    assert _call_fwd(L, _dims(**dims_kw), **kw) == expect, case


def test_null_dims(L):
    assert L.gdn_chunk_fwd(None, *([None] * 10), ctypes.c_size_t(0), None) == nat.GDN_ERR_INVALID
    assert L.gdn_recurrent_step(None, *([None] * 8)) == nat.GDN_ERR_INVALID


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), nat.GDN_ERR_INVALID),
    (dict(state=FAKE + 8), nat.GDN_ERR_INVALID),
    (dict(v=FAKE + 2), nat.GDN_ERR_INVALID),
    (dict(la=FAKE + 1), nat.GDN_ERR_INVALID),
])
def test_recurrent_step_rejects_bad_arguments(L, kw, expect):
    p = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, state=FAKE, o=FAKE)
    p.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    d = _dims(B=8, T=1, n_seqs=8)
    assert L.gdn_recurrent_step(ctypes.byref(d), v(p["q"]), v(p["k"]), v(p["v"]), v(p["la"]),
                                v(p["beta"]), v(p["state"]), v(p["o"]), None) == expect


@pytest.mark.parametrize("kw,dims_kw,expect", [
    (dict(q=None), {}, nat.GDN_ERR_INVALID),
    (dict(state=FAKE + 8), {}, nat.GDN_ERR_INVALID),
    (dict(k=FAKE + 2), {}, nat.GDN_ERR_INVALID),
    (dict(n_commit=FAKE + 2), {}, nat.GDN_ERR_INVALID),
    ({}, dict(flags=nat.GDN_FLAG_BETA_CHANNEL, decay=nat.GDN_DECAY_CHANNEL), nat.GDN_ERR_UNSUPPORTED),
    ({}, dict(d_k=96), nat.GDN_ERR_UNSUPPORTED),
])
def test_recurrent_verify_rejects_bad_arguments(L, kw, dims_kw, expect):
    p = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, state=FAKE, n_commit=FAKE, o=FAKE)
    p.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    d = _dims(**{**dict(B=8, T=5, n_seqs=8), **dims_kw})
    assert L.gdn_recurrent_verify(ctypes.byref(d), v(p["q"]), v(p["k"]), v(p["v"]), v(p["la"]),
                                  v(p["beta"]), v(p["state"]), v(p["n_commit"]), v(p["o"]),
                                  None) == expect


def test_recurrent_verify_without_tokens_is_a_noop_without_device(L):
    for dims_kw in (dict(B=0, T=5, n_seqs=0), dict(B=8, T=0, n_seqs=8)):
        d = _dims(**dims_kw)
        assert L.gdn_recurrent_verify(ctypes.byref(d), *([None] * 8), None) == nat.GDN_OK


def test_empty_batch_is_a_noop_without_device(L):
    # B = 0: nothing to launch, nothing touched -- succeeds even without a GPU
    d = _dims(B=0, n_seqs=0)
    assert _call_fwd(L, d, q=None, k=None, v=None, la=None, beta=None, o=None) == nat.GDN_OK
    d = _dims(B=0, T=1, n_seqs=0)
    assert L.gdn_recurrent_step(ctypes.byref(d), *([None] * 8)) == nat.GDN_OK


def test_value_rate_flags_and_workspace(L):
    f = ctypes.c_void_p(FAKE)
    fg2 = dict(decay=nat.GDN_DECAY_CHANNEL, flags=nat.GDN_FLAG_BETA_CHANNEL)
    both = dict(decay=nat.GDN_DECAY_CHANNEL,
                flags=nat.GDN_FLAG_BETA_CHANNEL | nat.GDN_FLAG_VALUE_RATE)
    # the value rate needs the key-side rate; gdn_chunk_fwd refuses it
    assert L.gdn_chunk_fwd_workspace_size(ctypes.byref(_dims(flags=nat.GDN_FLAG_VALUE_RATE))) == 0
    n_fg2 = L.gdn_chunk_fwd_workspace_size(ctypes.byref(_dims(**fg2)))
    n_both = L.gdn_chunk_fwd_workspace_size(ctypes.byref(_dims(**both)))
    assert n_both - n_fg2 == 2 * 128 * 4 * 128 * 2  # v~: B T H d_v bf16
    d = _dims(**both)
    assert _call_fwd(L, d) == nat.GDN_ERR_INVALID
    args = [f, f, f, f, f]  # q k v log_alpha beta
    assert L.gdn_chunk_fwd_value_rate(ctypes.byref(_dims(**fg2)), *args, f, None, None, f, None, f,
                                      n_both, None) == nat.GDN_ERR_INVALID
    assert L.gdn_chunk_fwd_value_rate(ctypes.byref(d), *args, None, None, None, f, None, f,
                                      n_both, None) == nat.GDN_ERR_INVALID
    assert L.gdn_chunk_fwd_value_rate(ctypes.byref(d), *args, f, None, None, f, None, f,
                                      n_fg2, None) == nat.GDN_ERR_INVALID


def test_recurrent_verify_tree_rejects_bad_arguments(L):
    f = ctypes.c_void_p(FAKE)
    args = [f, f, f, f, f, f]  # q k v log_alpha beta state
    d = _dims(T=8)
    assert L.gdn_recurrent_verify_tree(ctypes.byref(d), *args, None, None, f, None) == \
        nat.GDN_ERR_INVALID  # no parent
    assert L.gdn_recurrent_verify_tree(ctypes.byref(_dims(T=65)), *args, f, None, f, None) == \
        nat.GDN_ERR_UNSUPPORTED  # more than 64 nodes
    assert L.gdn_recurrent_verify_tree(None, *args, f, None, f, None) == nat.GDN_ERR_INVALID
    # no drafts: nothing to do, succeeds without a device
    assert L.gdn_recurrent_verify_tree(ctypes.byref(_dims(T=0)), *([None] * 6), None, None, None,
                                       None) == nat.GDN_OK


def test_state_maps_reject_bad_arguments(L):
    f = ctypes.c_void_p(FAKE)
    d = _dims(dtype=nat.GDN_FP32)
    # null operands, an output that aliases s or m, misalignment, unsupported sizes
    assert L.gdn_state_compose(ctypes.byref(d), None, f, None, f, None) == nat.GDN_ERR_INVALID
    assert L.gdn_state_compose(ctypes.byref(d), f, f, None, f, None) == nat.GDN_ERR_INVALID
    odd = ctypes.c_void_p(FAKE + 4)
    assert L.gdn_state_compose(ctypes.byref(d), f, ctypes.c_void_p(FAKE + 4096), None, odd,
                               None) == nat.GDN_ERR_INVALID
    assert L.gdn_state_compose(ctypes.byref(_dims(d_k=96)), f, f, None, f, None) == \
        nat.GDN_ERR_UNSUPPORTED
    assert L.gdn_state_compose(None, f, f, None, f, None) == nat.GDN_ERR_INVALID
    assert L.gdn_state_identity(ctypes.byref(_dims(d_v=64)), f, None) == nat.GDN_ERR_UNSUPPORTED
    assert L.gdn_state_identity(ctypes.byref(d), None, None) == nat.GDN_ERR_INVALID
    # no sequences: nothing to launch, succeeds without a device
    d0 = _dims(B=0, n_seqs=0)
    assert L.gdn_state_compose(ctypes.byref(d0), None, None, None, None, None) == nat.GDN_OK
    assert L.gdn_state_identity(ctypes.byref(d0), None, None) == nat.GDN_OK


def test_workspace_init_rejects_bad_arguments(L):
    assert L.gdn_workspace_init(None, 256, None) == nat.GDN_ERR_INVALID
    assert L.gdn_workspace_init(ctypes.c_void_p(FAKE), 16, None) == nat.GDN_ERR_INVALID
    assert L.gdn_workspace_status(None, None) == nat.GDN_ERR_INVALID


def test_python_api_refuses_host_tensors():
    """No CPU fallback: every entry of the binding refuses host tensors before any call."""
    import torch
    from gated_delta_rule_140_b200 import (chunk_fwd, recurrent_step, recurrent_verify,
                                           state_compose)
    q = torch.zeros(1, 4, 2, 64)
    la, b = torch.zeros(1, 4, 2), torch.zeros(1, 4, 2)
    for call in (lambda: chunk_fwd(q, q, q, la, b),
                 lambda: chunk_fwd(q, q, q, la, b, beta_v=torch.zeros(1, 4, 2, 64)),
                 lambda: recurrent_step(q[:, 0], q[:, 0], q[:, 0], la[:, 0], b[:, 0],
                                        torch.zeros(1, 2, 64, 64)),
                 lambda: recurrent_verify(q, q, q, la, b, torch.zeros(1, 2, 64, 64),
                                          parent=torch.zeros(1, 4, dtype=torch.int32)),
                 lambda: state_compose(torch.zeros(1, 2, 64, 64), torch.zeros(1, 2, 64, 64))):
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_python_api_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(nat, "_lib", None)
    monkeypatch.setattr(nat, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        nat.lib()


def test_build_uses_sm100a_flags():
    assert "arch=compute_100a,code=sm_100a" in " ".join(B.NVCC_FLAGS)
    assert os.path.exists(B.LIB)
