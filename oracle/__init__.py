"""CPU oracle of the quantized linear layer: test infrastructure only.

Imported by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``; never by the library itself."""
