"""CPU oracle for the uniform-state text-diffusion denoise step.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg import this package. The CUDA library never
imports, links or executes it, and it shares no code with the library: it has
its own counter-based hash, schedule, stand-in, softmax/entropy, sampler and
stop test, written from the pages' description in plain numpy, fp64 for all
floating-point work except where a decision is taken in the kernel's fp32
precision (argmax over logits, the entropy sort, the acceptance prefix sums and
the confidence threshold), which is stated at each such place.

Modules:
  rng     -- SplitMix64 counter hash, uniform tokens, Gaussian draws.
  method  -- temperature schedule, stand-in hidden state, vocabulary
             softmax/entropy/argmax/self-conditioning, the self-conditioning
             feed-forward network, entropy-bounded sampler, re-noise,
             adaptive stop, the step and the block loop.
  fp8     -- e4m3/e5m2 rounding, per-row power-of-two scaling and the step's
             vocabulary attention with a narrow (e4m3) embedding.

Parity status: every function is pinned by tests/test_oracle_*.py against
closed forms, brute force in long double, a published SplitMix64 vector, a
hand-worked acceptance example, every code of the 8-bit formats and a library
conversion. The pages' end-to-end quality behaviour
(quality versus step count, the Sudoku experiment) needs the trained model and
is not part of this oracle.
"""
from . import rng, method, fp8  # noqa: F401
