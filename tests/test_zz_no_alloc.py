"""gdn_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (a plugin handed only its input and output buffers, a serving loop that
forbids allocation after start-up, a process whose device memory another
allocator already owns).  It runs the same kernels as gdn_chunk_fwd with a
fixed array inside the library as scratch.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it passes alone in a fresh process
as well.  The entry point is called through the C ABI (ctypes), once per
problem on four problems in a row, and each result is checked against
gdn_chunk_fwd's within the parity tolerances; a call with bad cu_seqlens
contents is then reported by gdn_noalloc_status."""
import ctypes

import pytest
import torch

from gated_delta_rule_140_b200 import _native as nat
from gated_delta_rule_140_b200 import chunk_fwd
from gated_delta_rule_140_b200.inputs import prefill_inputs
from tests.parity_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(d):
    """Call gdn_chunk_fwd_noalloc through the C ABI on device inputs ``d``."""
    L = nat.lib()
    q, v, la, cu = d["q"], d["v"], d["log_alpha"], d["cu_seqlens"]
    dims = nat.prefill_dims(q, v, la, cu)
    o = torch.full(v.shape, float("nan"), dtype=q.dtype, device=q.device)
    sf = torch.full((dims.n_seqs, dims.H, dims.d_v, dims.d_k), float("nan"),
                    dtype=torch.float32, device=q.device)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = L.gdn_chunk_fwd_noalloc(ctypes.byref(dims), p(q), p(d["k"]), p(v), p(la),
                                 p(d["beta"]), p(d["initial_state"]), p(cu), p(o), p(sf),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nat.GDN_OK, nat.status_string(st)
    return o, sf


def _problems():
    a = prefill_inputs(2, 229, 3, 128, 128, dtype=torch.bfloat16, seed=41, init_std=0.05)
    g = torch.Generator().manual_seed(42)
    b = prefill_inputs(1, 0, 4, 64, 64, dtype=torch.float32, decay="channel", alpha_shift=3.0,
                       init_std=0.02, lengths=[70, 0, 129, 5], gen=g)
    # KDA bf16 d = 128: the default two-CTA kernel's ring does not fit, so the
    # entry point runs the CUDA-core kernel; compared with the default path
    c = prefill_inputs(2, 150, 2, 128, 128, dtype=torch.bfloat16, decay="channel",
                       alpha_shift=3.0, seed=43, init_std=0.05)
    # GDN bf16 d = 128 with a sequence of 2048+ tokens: the default is the two-CTA
    # kernel, whose ring does not fit; the entry point runs the single-CTA kernel
    e = prefill_inputs(1, 2048 + 37, 2, 128, 128, dtype=torch.bfloat16, seed=44, init_std=0.05)
    return [(a, torch.bfloat16), (b, torch.float32), (c, torch.bfloat16), (e, torch.bfloat16)]


def test_noalloc_matches_chunk_fwd_on_calls_in_a_row(cuda_ok):
    for x, dtype in _problems():
        d = to_dev(x)
        o, sf = _noalloc(d)
        o_ref, sf_ref = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                  d["initial_state"], d["cu_seqlens"])
        torch.cuda.synchronize()
        to, ts = TOL[dtype]
        assert rel_err(o, o_ref.double().cpu().numpy()) <= to
        assert rel_err(sf, sf_ref.cpu().numpy()) <= ts


def test_noalloc_fits_its_array_or_refuses(cuda_ok):
    L = nat.lib()
    # the two-CTA kernel's ring never fits in the fixed array (the entry point
    # then runs the default kernel); the default kernels need the header alone
    for n_seqs in (1, 1 << 10, 1 << 16):
        dims = nat.Dims(1, n_seqs * 64, 16, 128, 128, n_seqs, nat.GDN_BF16,
                        nat.GDN_DECAY_SCALAR, nat.GDN_FLAG_PAIR)
        assert L.gdn_chunk_fwd_workspace_size(ctypes.byref(dims)) > 256 * 1024
        dims.flags = 0
        assert L.gdn_chunk_fwd_workspace_size(ctypes.byref(dims)) <= 256 * 1024
    # invalid dims are still invalid
    bad = nat.Dims(1, 64, 16, 96, 128, 1, nat.GDN_BF16, nat.GDN_DECAY_SCALAR, 0)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(bad), *([None] * 9), None) != nat.GDN_OK


def test_noalloc_status_reports_bad_cu_seqlens(cuda_ok):
    """Errors only the device can see land in the array's header; the caller
    reads them with gdn_noalloc_status (the next call clears them)."""
    x = prefill_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, seed=45)
    d = to_dev(x)
    d["cu_seqlens"] = torch.tensor([0, 200, 100, 256], dtype=torch.int32, device="cuda")
    _noalloc(d)
    assert nat.noalloc_status() == nat.GDN_ERR_DEVICE_INPUT
    assert nat.noalloc_status() == nat.GDN_OK  # cleared by the read
    d["cu_seqlens"] = torch.tensor([0, 100, 200, 256], dtype=torch.int32, device="cuda")
    o, sf = _noalloc(d)
    assert nat.noalloc_status() == nat.GDN_OK
    o_ref, sf_ref = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None,
                              d["cu_seqlens"])
    torch.cuda.synchronize()
    assert rel_err(o, o_ref.double().cpu().numpy()) <= TOL[torch.bfloat16][0]
    assert rel_err(sf, sf_ref.cpu().numpy()) <= TOL[torch.bfloat16][1]
