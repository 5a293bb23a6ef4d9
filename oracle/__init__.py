"""CPU oracle for the GCA hot path — TEST INFRASTRUCTURE.

Plain, slow, fp64 restatement of what the GCA path computes, written from the
LingBot-Map pages: ``gca`` (visibility rule, streaming simulator, brute force,
closed forms, fp64 attention core in C and numpy, the 3D rotary position
encoding as explicit rotation matrices) and ``allocator`` (page-table
simulator).  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
cpu_baseline leg and reference arm may import, call, link or execute anything
here.  It shares no code with the CUDA library and never imports it.
"""
