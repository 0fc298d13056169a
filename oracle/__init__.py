"""Plain fp64 CPU oracle of one streaming pyramid denoising round.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports or calls
anything here; only the tests, `__graft_entry__.smoke()` and the bench's CPU
baseline leg do. See `oracle/personalive.py` for the definitions and the
passages each one follows.
"""
from .personalive import *  # noqa: F401,F403
