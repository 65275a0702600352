"""CPU oracle of the ZAYA1 decoder block -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA path never does.
"""
