"""Oracle: group permute and varlen boundaries.

The pages (note, key design 2) permute tokens so the members of each group
sit together, describe the group boundaries with cu_seqlens / max_seqlen for a
varlen attention call, and repermute afterwards.  They do not state the order
inside a group; this build takes the stable order (ascending token index),
which is the one order that makes perm a unique, bit-comparable result.

  counts[i]     = #{t : g_t = i}
  cu_seqlens    = exclusive prefix sum of counts, cu[0] = 0, cu[M] = N
  perm          = the tokens of group 0 in ascending order, then group 1, ...
  max_seqlen    = max_i counts[i]

Pinned by: perm o perm^-1 = id, sum counts = N, g[perm[j]] equal to the
segment index, strictly ascending tokens inside a segment, and equality with
Python's stable sort on tiny inputs.
"""
from __future__ import annotations

import numpy as np


def permute(g: np.ndarray, M: int):
    """Returns (perm [N] int64, cu_seqlens [M+1] int64, counts [M] int64, max_seqlen int)."""
    g = np.asarray(g)
    members = [np.nonzero(g == i)[0] for i in range(M)]
    counts = np.array([len(m) for m in members], dtype=np.int64)
    cu = np.zeros(M + 1, dtype=np.int64)
    cu[1:] = np.cumsum(counts)
    perm = np.concatenate(members) if len(g) else np.zeros(0, dtype=np.int64)
    return perm.astype(np.int64), cu, counts, int(counts.max()) if M else 0
