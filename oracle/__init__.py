"""CPU oracle for PHOTON's hierarchical prefill and HierGen/RecGen decode.

THIS PACKAGE IS TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test
suite (tests/), the smoke check in __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import, call or execute anything in it.  The
library in hierarchical_autoregressive_lm_b200/ never imports it, and it
never imports the library: the two share no code.  The only common module
is synth_inputs, which generates seeded prompt ids and holds none of the
model's arithmetic.

Contents:
  weights.py -- the counter-based N(0, 0.02^2) weight generator, written
                from its definition (SplitMix64 + polar method), fp64.
  photon.py  -- the model in plain fp64 NumPy, one sequence at a time,
                following the PHOTON pages step by step.
  sampling.py -- temperature sampling by the Gumbel-max rule with a
                counter-based generator (SplitMix64 + MurmurHash3 fmix32).
  vanilla.py -- a vanilla token-level Transformer of the same width, the
                baseline of the pages' TPM comparison, built from the same
                pinned blocks.
  aggregate.py -- multi-query aggregation (majority vote, best-of-N by
                teacher-forced log-likelihood) over groups of sampled rows.
  hierarchy.py -- the same model for any number of levels L (L = 1: a
                single-level block model; L = 2 reduces to photon.py; L >= 3:
                deeper hierarchies), HierGen and RecGen.

Every oracle function is pinned by CPU tests (tests/test_oracle_*.py) to
facts that do not come from the oracle itself: published SplitMix64 test
vectors, closed forms, library routines for special cases (PyTorch's
scaled-dot-product attention, RMSNorm, GELU and linear layers in fp64),
invariants the pages state (chunk-local decoder, causal coarse stream,
cache-equals-recompute, Theorem A.6) and brute force on tiny inputs.  The
model's output values themselves are not printed anywhere on the pages
("parity unpinned" by a worked example); they are pinned only through those
component and invariant checks.
"""
from .photon import (Config, PhotonOracle, SeqState, StepResult, LayerKV,  # noqa: F401
                     rmsnorm, rope, gelu, attention, block, stack, chunker,
                     converter, decode_attention, tpm)
from .weights import (make_weights, tensor_specs, draw_tensor, mix64,  # noqa: F401
                      splitmix64_stream, round_fp32_to_bf16)
