"""TurboQuant KV-cache compression for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libtq.so`` built from ``csrc/``;
``kv_cache_vector_12_b200.tq`` is its thin Python binding (argument
marshalling only).  Importing this package loads nothing; importing ``tq``
loads the library and raises if it is missing.
"""
