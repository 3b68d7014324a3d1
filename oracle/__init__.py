"""Float64 CPU oracle for MFA decode attention and the MFA query projection.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg. The product package never imports it.
"""
