"""B200-native gated delta rule (Gated DeltaNet and KDA) sequence mixer.

    from gated_delta_rule_140_b200 import chunk_fwd, recurrent_step

``chunk_fwd`` is the chunkwise WY / UT-transform prefill (``chunk_fwd_raw`` the
same with the input normalisation and gate transforms fused in), ``recurrent_step``
the in-place single-token decode step and ``recurrent_verify`` the multi-token
draft verification with commit of the accepted prefix; ``state_compose`` and
``state_identity`` build the per-segment state maps with which ``seqshard`` runs
one long sequence over several GPUs; all call the C ABI of libgdn.so
(include/gdn.h), whose CUDA kernels do all of the work.  Importing the package
does not load the library; the first call does, and raises if it is missing.
"""
from ._native import (GdnError, Workspace, chunk_fwd, chunk_fwd_raw, launch_count,
                      recurrent_step, recurrent_verify, state_compose, state_identity,
                      status_string, workspace_size)

__all__ = ["chunk_fwd", "chunk_fwd_raw", "recurrent_step", "recurrent_verify", "state_compose",
           "state_identity", "Workspace", "GdnError", "launch_count", "status_string",
           "workspace_size"]
