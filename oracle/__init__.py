"""Oracle for the gated-delta-rule forward: plain, slow, obviously correct CPU code.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / ``--impl reference`` leg may import, call, link
or run anything under ``oracle/``. The product library
(``linear_attention_recurrent_chunked_b200``) never does, and this package
never imports it: the two share no code. The only shared module is the seeded
input generator ``linear_attention_recurrent_chunked_b200.workloads``, which
holds none of the method's arithmetic.

Contents (each cites the passage it follows in its own docstring):

* ``scan``        -- fp64 sequential scan in C with OpenMP (the oracle proper).
* ``decode_step`` -- the scan over B sequences of one token each.
* ``transition_products`` -- second formulation: explicit products of the
  transition matrices M_t = alpha_t (I - beta_t k_t k_t^T); small T only.
* ``chunked``     -- third formulation: fp64 chunked (intra/inter-chunk) form
  with per-stage dumps; a stage reference, pinned by equality with ``scan``.

Pins (``tests/test_oracle.py``): the three formulations agree to ~1e-12; the
invariants the rule fixes (beta=0 & alpha=1 leaves S unchanged; alpha=1,
beta=1 with orthonormal keys stores and retrieves v exactly; alpha=0 resets
the state); closed forms (beta=0 => S_T = exp(sum g) S0; a repeated unit key
makes S k a scalar exponential moving average); the norm bound
||S_t||_F <= alpha_t ||S_{t-1}||_F + beta_t ||v_t||; brute force at d=2 against
hand-expanded 2x2 algebra and a hand-derived golden example in
``tests/golden/``; mutation tests showing that planted mistakes fail the pins.
"""
from .scan import scan, decode_step, as_f64, num_threads, set_num_threads  # noqa: F401
from .products import transition_products  # noqa: F401
from .chunked import chunked, chunk_step  # noqa: F401
