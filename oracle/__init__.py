"""Oracle for the DuoLM multi-item-scoring forward -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU restatement of what the ranker computes, written from the
pages (see ``oracle.ranker`` for the definitions followed and the readings
taken).  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import it; the CUDA library never does.
"""
