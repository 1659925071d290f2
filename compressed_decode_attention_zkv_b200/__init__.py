"""RVQ KV-cache encode and compressed decode attention for B200 (sm_100a).

``compressed_decode_attention_zkv_b200.zkv`` is the thin ctypes binding of the C-ABI library
``libzkv.so`` (built from ``csrc/``).  ``inputs`` holds the seeded synthetic input generators.
Nothing is imported eagerly so that CPU-only users (input generation) do not need the library.
"""
