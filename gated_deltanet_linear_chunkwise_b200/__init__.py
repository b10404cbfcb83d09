"""B200-native (sm_100a) chunkwise gated delta rule.

The computation lives in ``libgdn_b200.so`` (C ABI declared in
``include/gdn.h``); this package re-exports a thin ctypes binding of it and
the named synthetic workloads.  Importing the package does not load the
library; the first call does, and fails loudly if it has not been built.
"""
from .binding import (GdnError, bidirectional, gdn_fwd, gdn_fwd_host, gdn_step, last_error,
                      load_library, workspace_bytes)

__all__ = ["GdnError", "bidirectional", "gdn_fwd", "gdn_fwd_host", "gdn_step", "last_error",
           "load_library", "workspace_bytes"]
