"""Oracle for exact scaled-dot-product attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct CPU implementations of what the CUDA library
computes, used to prove the CUDA path right.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline / reference arm may
import, call, link or execute anything in this package.  The product path never
does, and this package imports nothing from the product package: the two sides
share only the seeded input generators in ``attn_inputs``.

Contents
--------
``reference``  numpy fp64: ``ref_fwd`` / ``ref_bwd`` materialise S and P (per
               head, or per row block), straight from the definition
               O = softmax(Q K^T / sqrt(d)) V.  ``online_fwd_head`` restates the
               pages' blockwise online-softmax recurrence (used only to pin the
               exactness claim).
``brute.c``    plain C, long double, triple loops, no BLAS: forward and backward
               for tiny shapes, an independent second implementation.
``build``      compiles ``brute.c`` with gcc into ``_brute.so``.

Pins (``tests/test_oracle.py``) tie every function to something other than
itself: brute force in C, torch's fp64 CPU scaled-dot-product attention and
autograd, central finite differences, closed forms (constant V, Q = 0, a
dominant score, N = 1, V = I), shift invariance and the blockwise = full claim.
No function here is "parity unpinned".
"""
