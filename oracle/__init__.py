"""CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct fp64 implementations of what the hot path
computes, written from the pages:

* "PagedAttention" (devoured.fyi digest), sections "PagedAttention in one
  picture", "Copy-on-write: when two requests share a prefix", "Why the
  attention kernel works at all" and "Misconceptions";
* "PagedAttention, Visualized", Parts 2 and 3;
* "LLM Inference Visualizer", lesson 06 "PagedAttention", "How paging grows".

Two independent implementations: ``reference.py`` (NumPy) and ``pa_oracle.c``
(plain C, loaded through ctypes by ``c_oracle.py``).  Neither shares code with
the CUDA library, and neither imports it.  Only ``tests/``, the package-level
``smoke()`` check and the CPU-baseline leg of the benchmark may use this
package; the product path never does.

Pins (what fixes each function independently of itself) live in
``tests/test_oracle_pins.py`` and ``tests/test_oracle_mutants.py``.
"""

from . import reference  # noqa: F401
