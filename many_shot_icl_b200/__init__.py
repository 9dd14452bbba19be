"""DBSA attention engine for B200 (sm_100a).

The compute path lives in the C-ABI library ``libdbsa.so`` (built from
``many_shot_icl_b200/csrc``); :mod:`many_shot_icl_b200.dbsa` is its thin
ctypes binding.  Importing the package does not load the library; the first
call into :mod:`many_shot_icl_b200.dbsa` does, and raises if it is missing.
"""
__all__ = ["dbsa", "inputs"]
