"""Graph views used by the oracle (plain numpy).

Sobek, section 4: "cached stable CSR views give receiver and source reductions fixed
ownership".  The receiver CSR (row_ptr, src) is the input; the source view groups the
same edge ids by source, keeping receiver order inside each source row (a stable
sort by source), and records each edge's receiver.
"""

import numpy as np


def source_view(row_ptr, src, n_nodes):
    """Return (t_ptr[N+1], t_eid[E], t_dst[E]) as int32 (stable grouping by source)."""
    src = np.asarray(src, dtype=np.int64)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    order = np.argsort(src, kind="stable")
    counts = np.bincount(src, minlength=n_nodes) if src.size else np.zeros(n_nodes, np.int64)
    t_ptr = np.zeros(n_nodes + 1, dtype=np.int64)
    t_ptr[1:] = np.cumsum(counts)
    dst = np.repeat(np.arange(n_nodes), np.diff(row_ptr))
    return t_ptr.astype(np.int32), order.astype(np.int32), dst[order].astype(np.int32)
