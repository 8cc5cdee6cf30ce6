"""B200-native activation-sparse gated FFN (TwELL format) for sm_100a.

The compute path is the C-ABI library ``libtwell.so`` built from ``csrc/``;
``twell`` is its thin ctypes binding.  Importing this package loads nothing;
``twell`` loads the library on first use and raises if it is missing.
"""
