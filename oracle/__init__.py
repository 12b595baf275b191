"""Float64 CPU oracle for exact RoPE / LeRoPE attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.  It
shares no code with the CUDA path.  Every function is pinned by a CPU test in
``tests/test_oracle_pins.py``; no function is parity-unpinned.
"""
