"""B200-native jagged candidate-isolated attention.

The compute path lives in ``libjca.so`` (hand-written sm_100a CUDA behind a C ABI declared in
``include/jca.h``); ``candidate_isolated_jagged_b200.jca`` is the thin ctypes binding over it.
Importing this package does not load the library; ``jca.lib()`` does, and fails loudly when the
library is missing.
"""
