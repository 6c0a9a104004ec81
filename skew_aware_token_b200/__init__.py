"""Skew-aware MoE forward layer on one B200 (sm_100a).

The layer's work runs in the CUDA library ``libmoeskew.so`` behind a C ABI
(``include/moeskew.h``); ``skew_aware_token_b200.native`` is its thin ctypes binding and
``skew_aware_token_b200.layer`` strings the calls together.  ``synth`` draws seeded
synthetic inputs.  Importing the package loads nothing native; the binding loads the
library on first use and raises if it is missing.
"""
