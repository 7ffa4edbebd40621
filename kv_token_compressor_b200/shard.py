"""Host-side plan for splitting one compressor problem across ranks (one process per GPU).

The compressor shards with no exchange of results: every entry depends only on its own
window ("序列压缩注意力", table attn-seqcomp-overlap).  A rank that owns the contiguous
entries [e0, e1) of a sequence needs the token rows [m e0, m e1) of the a-streams and,
with the CSA overlap, also the b-rows of entry e0, i.e. the m rows [m (e0 - 1), m e0):
a halo of one block read from the previous rank's range.  The rank runs the ordinary
compressor on its local rows [m (e0 - 1), m e1) and drops local entry 0 (that entry is
the halo block, which the local problem sees with no predecessor).  Ranks owning entry 0
of a sequence keep the true boundary of eq. attn-seqcomp-overlap-bound.

Only planning lives here; the data path is the same C-ABI call on each rank.
"""

from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    rank: int
    e0: int          # first entry owned (global index within the sequence)
    e1: int          # one past the last entry owned
    row0: int        # first token row the rank must read (halo included)
    row1: int        # one past the last token row it must read
    drop_first: bool  # the local problem's entry 0 is the halo, not an owned entry

    @property
    def entries(self) -> int:
        return self.e1 - self.e0


def plan(n: int, m: int, world: int, overlap: bool = True) -> list[Shard]:
    """Balanced contiguous entry ranges of an n-token sequence over `world` ranks."""
    if m < 1 or n < 0 or world < 1:
        raise ValueError("need m >= 1, n >= 0, world >= 1")
    ne = n // m
    out = []
    for r in range(world):
        e0 = (r * ne) // world
        e1 = ((r + 1) * ne) // world
        halo = overlap and e0 > 0 and e1 > e0
        row0 = m * (e0 - 1) if halo else m * e0
        out.append(Shard(rank=r, e0=e0, e1=e1, row0=row0, row1=m * e1, drop_first=halo))
    return out
