"""CPU oracle for the chunked Gated DeltaNet (GDN) scan.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import, call, link or run anything
in this package.  The product path (``gated_deltanet_linear_chunked_b200``)
never does, and the two share no code: they meet only through the seeded
input generators, which hold none of the method's arithmetic.

Contents
  * ``cpu``        -- ctypes front end of ``gdn_oracle.c``: the token-by-token
                      recurrence in double (and long double), threaded over
                      (batch, head).  The reference for every parity test.
                      Its ``*_logits`` variants take the gate layer's logits
                      and form g = -softplus(x), beta = sigmoid(y) themselves.
  * ``numpy_ref``  -- the same recurrence in numpy (a second, independent
                      transcription for tiny cases) and the chunked (WY / UT)
                      form of the scan in fp64, used only to pin that the
                      chunked algebra reaches the recurrence exactly;
                      reverse mode through that chunked form, pinned to the
                      autograd gradients the same way; and
                      ``gates_from_logits``, the gate activations in numpy.
  * ``backward``   -- the forward definition in plain PyTorch CPU float64,
                      differentiated by autograd: the reference gradients of
                      the scan.
  * ``sink_window_attn`` -- the softmax blocks' attention over a persistent
                      sink and a sliding window of chunks, in numpy float64.

Parity is pinned, not assumed: ``tests/test_oracle_pins.py`` and
``tests/test_oracle_sink_window.py`` check these
functions against closed forms, invariants, a hand-derived example and brute
force (see each test's docstring).
"""
from .cpu import (  # noqa: F401
    build,
    online_cores,
    oracle_bidir,
    oracle_bidir_logits,
    oracle_fwd,
    oracle_fwd_logits,
)
from . import backward  # noqa: F401
from . import sink_window_attn  # noqa: F401
from .numpy_ref import (  # noqa: F401
    chunked_bidir,
    chunked_fwd,
    gates_from_logits,
    recurrence_bidir,
    recurrence_fwd,
)
