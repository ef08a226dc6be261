"""fp64 CPU oracle for the Simple GLA mixer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``linear_attention_simple_b200``) never imports it and shares
no code with it.

Contents
  - ``recurrent``: ctypes front end to ``gla_oracle.c`` (token-by-token fp64
    recurrence, its hand-derived reverse recurrence, the decode step and the
    LayerNorm -> causal conv -> SiLU front end).
  - ``closed_form``: an independent NumPy restatement of the same forward as
    a quadratic sum over token pairs, plus the textbook causal linear
    attention special case (a == 0).
  - ``chunked``: an independent NumPy chunked evaluation with an arbitrary
    chunk size, used to show that results do not depend on chunking.

Parity status of each function is listed in the module docstrings.
"""
