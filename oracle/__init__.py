"""CPU oracle of the BasisKV decode-attention block (test infrastructure only).

Importable by the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg; the product path never imports it."""
