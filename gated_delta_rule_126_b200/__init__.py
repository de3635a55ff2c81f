"""B200-native Kimi Delta Attention (KDA) operator.

The operator runs in hand-written sm_100a CUDA kernels behind the C ABI declared
in ``include/kda.h`` (library ``lib/libkda_b200.so``, built by
``python -m gated_delta_rule_126_b200.build``).  This package is the thin Python
binding over that ABI, with the same names:

* ``kda_prefill``     -- chunked prefill over packed variable-length sequences;
* ``kda_prefill_gated`` -- the same with the layer's output epilogue (sigmoid gate
  and RMSNorm) applied to o;
* ``kda_prologue``    -- the layer's input prologue (short conv, Swish, L2Norm, gates)
  that makes the prefill's inputs from the projections;
* ``kda_decode_step`` -- one recurrent decode step for a batch of sequences;
* ``kda_decode_tokens`` -- n tokens per sequence with states in a slot pool;
* ``kda_backward``    -- gradients of the recurrence with respect to every input;
* ``prefill_workspace_size``, ``backward_workspace_size``, ``workspace_status``, ``KdaError``;
* ``wait_timeout_selftest`` -- runs the kernels' bounded-wait error path on events
  that never come, leaving the flag ``workspace_status`` reads.

``inputs`` holds the seeded synthetic input generators.  Importing the package
does not load the CUDA library; the first call does, and raises if it is missing.
"""
from ._binding import (KdaError, backward_workspace_size, kda_backward, kda_decode_step,
                       kda_decode_tokens, kda_prefill, kda_prefill_gated, kda_prologue, load,
                       prefill_workspace_size, wait_timeout_selftest, workspace_status)

__all__ = ["KdaError", "backward_workspace_size", "kda_backward", "kda_decode_step", "kda_decode_tokens",
           "kda_prefill", "kda_prefill_gated", "kda_prologue", "load", "prefill_workspace_size",
           "wait_timeout_selftest", "workspace_status"]
