"""Plain CPU oracle of the TTT-Linear scan (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. It shares no code with the CUDA path.
"""

from .ttt_oracle import (GATE_CHANNEL, GRAD_ABLATE, GRAD_LNJAC, GRAD_NORM_MATCH,  # noqa: F401
                         KQ_SILU, MINIBATCH, NO_LN, backward, build, decode_step, forward,
                         forward_heads, lngrad, max_threads)
