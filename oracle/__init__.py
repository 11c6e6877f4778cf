"""CPU oracle for exact scaled dot-product attention with optional dropout.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
link this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, tables or helpers with the CUDA library in ``exact_io_aware_49_b200``
and never imports it.

What it computes (fp64 NumPy, inputs given as bf16-rounded values upcast
exactly to fp64):

* ``attention.forward`` / ``attention.backward`` -- the plain materialising
  definition of attention: scores, softmax, weighted sum of values ("Flash
  Attention" glossary, section "Why Regular Attention Becomes a Bottleneck";
  "DL0056 FlashAttention", Answer and the "Where:" definition of S_ij), with
  the causal mask and the inverted-scaling attention dropout, and the
  analytic gradients of that definition.
* ``online.forward_online`` -- the tile-by-tile online-softmax recurrence
  ("DL0056 FlashAttention", Mathematical Formulation) written out step by
  step; it exists only so the tests can show that it equals the two-pass
  definition above.
* ``paged.decode_forward`` -- attention over a paged key/value cache:
  gathers each sequence's pages back into contiguous keys and values and
  applies ``attention.forward`` (grouped-query heads share a key/value head).
* ``philox`` -- Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random
  Numbers: As Easy as 1, 2, 3", SC'11) and the dropout keep-mask built on it.

Pins (tests/test_oracle_*.py, tests/test_philox_oracle.py): rows of P sum to
one; Q = 0 closed forms; a hand-derived two-token example under
tests/golden/; online recurrence == two-pass; gradients against central
finite differences; shift / permutation / N = 1 / p = 0 invariants; Philox
against its authors' published known-answer vectors (tests/golden/) and an
independent library implementation (ATen's header-only ``philox_engine``),
plus keep-rate and lag-1 correlation statistics.  No
function here is "parity unpinned".
"""

from . import philox, attention, online, paged  # noqa: F401

__all__ = ["philox", "attention", "online", "paged"]
