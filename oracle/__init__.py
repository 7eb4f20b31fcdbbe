"""CPU oracle of the displaced-patch block step: test infrastructure only.

Imported only by tests/, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg; the product path never imports it.
"""
