"""MoE token dispatch and combine on one B200 (sm_100a).

The compute path is the C-ABI library ``libmoe_dispatch.so`` built from
``csrc/``; this package only marshals arguments to it (``api``), chains the
calls into an autograd Function (``autograd``) and draws seeded synthetic
inputs (``inputs``).  The library is loaded on first use; a missing or
unloadable library raises instead of falling back to anything else.
"""
