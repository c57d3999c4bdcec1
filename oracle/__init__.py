"""CPU oracle for the looped-transformer decode path (float64 NumPy).

THIS PACKAGE IS TEST INFRASTRUCTURE.  Only the tests, the smoke check and the
CPU-baseline leg of the benchmark may import it.  The CUDA library never calls
it and it never calls the CUDA library: the two share no code.  The only module
both sides use is `synthetic`, which draws the seeded random inputs and holds
none of the model's arithmetic.

It is written to be read against the pages, not to be fast:
  quant.py   symmetric per-group INT4 quantiser / nibble packing / dequant,
             BF16 rounding of float64 masters.
  model.py   RMSNorm, RoPE, causal attention over a per-iteration KV cache,
             the transformer block, embed -> pre blocks -> loop x L -> head.
  decode.py  greedy decode with per-lane L, hidden-state relative-L2 early exit,
             monotonic L clamp, and an iteration-granularity (continuous depth
             batching) scheduler over many lanes; per lane also logit-margin
             early exit, an L-warmup schedule (with KVCache's deepest-iteration
             reading) and self-speculative decoding.

Parity status: every function is pinned by the `-m "not gpu"` tests in
tests/test_oracle_*.py against closed forms, invariants, brute force on tiny
inputs, and hand-derived fixtures in tests/golden/.  The whole model has no
worked numeric example on the pages; its pins are the invariants the pages
state (L = k equals k applications of one block; a batch with per-lane L equals
each lane alone; INT4 dequant round-trips) plus the textbook definitions of
each step.
"""
from . import quant, model, decode  # noqa: F401
from .model import build_weights, Weights  # noqa: F401
from .decode import EarlyExit, generate_lane, generate_cdb, speculative_lane  # noqa: F401
