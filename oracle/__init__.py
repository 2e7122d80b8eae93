"""Float64 CPU oracle for the CSA2 decode step (test infrastructure).

This package is the reference that the CUDA path is checked against. It is
test infrastructure, not part of the product:

* only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
  ``--impl reference`` legs of ``bench.py`` may import it;
* it shares no code, table or constant with the CUDA library
  (``kv_cache_decode_index_b200``) and imports nothing from it;
* every function is written from the definitions on the pages (cited in its
  docstring) or, where the pages are silent, from the reading stated there.

Modules:
    formats  -- E2M1 / E4M3 codecs, FP4 main-KV and FP8 indexer quantisation.
    csa2     -- indexer score, block max, pool, top-k, Reuse, sparse attention,
                the decode layer group and the causal prefill indexer.

Pins (checked by ``tests/test_oracle_*.py``, marker ``not gpu``) tie each
function to something other than itself: the printed format limits, library
routines on special cases, brute force on tiny inputs and closed forms.
Parity of the score, block and group-order functions against DeepSeek's own
model is unpinned: the pages never give them (see the per-function notes).
"""
