"""Host-side split of one ragged batch over data-parallel ranks (one process per GPU).

The layer has no exchange step when its work is split by query rows: every query row
needs only its own sequence's cache up to its position, so ranks that hold the caches they
read compute their rows independently and no collective touches the data path.  This
module decides who computes what:

  - ``split_sequences``: whole sequences dealt to ranks, balanced on their cost (a serving
    batch of many sequences, each cache living on one GPU);
  - ``split_rows``: the query rows of one long sequence cut into contiguous ranges of about
    equal cost (one long prefill over several GPUs that each hold the whole cache);
  - ``shard``: the rank's pieces as a ragged batch of its own, with rebased offsets, plus
    where each piece's rows and cache rows sit in the global arrays.

Cost of a query row that sees n positions: min(K, n) gathered K/V rows (the attention,
which dominates) plus n / 64 for the indexer's scores (the measured per-position cost ratio
of the two stages at K = 2048 is about 1:57).  Planning arithmetic only: nothing here
computes any part of the layer.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

import numpy as np

INDEXER_WEIGHT = 1.0 / 64.0


def row_costs(q_len: int, kv_len: int, K: int) -> np.ndarray:
    """Cost of each query row of one sequence (query i sees n = kv_len - q_len + i + 1)."""
    n = np.arange(kv_len - q_len + 1, kv_len + 1, dtype=np.float64)
    return np.minimum(n, K) + INDEXER_WEIGHT * n


def seq_cost(q_len: int, kv_len: int, K: int) -> float:
    return float(row_costs(q_len, kv_len, K).sum())


def split_sequences(q_lens: Sequence[int], kv_lens: Sequence[int], K: int,
                    world: int) -> List[List[int]]:
    """Sequences per rank: longest-processing-time-first assignment of whole sequences to
    the least loaded rank (ties to the lower rank); each rank's list is kept in batch order."""
    costs = [seq_cost(q, l, K) for q, l in zip(q_lens, kv_lens)]
    order = sorted(range(len(costs)), key=lambda b: (-costs[b], b))
    load = [0.0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for b in order:
        r = min(range(world), key=lambda i: (load[i], i))
        out[r].append(b)
        load[r] += costs[b]
    return [sorted(x) for x in out]


def split_rows(q_len: int, kv_len: int, K: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous query-row ranges [i0, i1) of one sequence, one per rank, cut where the
    running cost crosses r / world of the total (causal rows grow in cost along the
    sequence, so the later ranges hold fewer rows)."""
    c = np.cumsum(row_costs(q_len, kv_len, K))
    total = c[-1] if len(c) else 0.0
    cuts = [0]
    for r in range(1, world):
        cuts.append(int(np.searchsorted(c, total * r / world, side="left")))
    cuts.append(q_len)
    cuts = [min(max(x, 0), q_len) for x in cuts]
    for i in range(1, len(cuts)):
        cuts[i] = max(cuts[i], cuts[i - 1])
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


@dataclass
class Piece:
    seq: int      # global sequence index
    q0: int       # first query of the sequence in this piece (0-based within the sequence)
    q1: int       # one past the last
    kv_len: int   # cache positions the piece's rows can see (its last query's position + 1)


@dataclass
class RankShard:
    """The pieces of one rank as a ragged batch of its own."""
    pieces: List[Piece] = field(default_factory=list)
    q_lens: List[int] = field(default_factory=list)
    kv_lens: List[int] = field(default_factory=list)

    @property
    def q_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int64)

    @property
    def kv_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.kv_lens)]).astype(np.int64)

    def global_rows(self, q_offsets: Sequence[int]) -> np.ndarray:
        """Global packed query rows of this shard, in its local order."""
        rows = [np.arange(int(q_offsets[p.seq]) + p.q0, int(q_offsets[p.seq]) + p.q1)
                for p in self.pieces]
        return np.concatenate(rows).astype(np.int64) if rows else np.zeros(0, np.int64)

    def global_cache_rows(self, kv_offsets: Sequence[int]) -> List[Tuple[int, int]]:
        """Per piece, the global cache rows [start, end) it reads (a prefix of its sequence)."""
        return [(int(kv_offsets[p.seq]), int(kv_offsets[p.seq]) + p.kv_len) for p in self.pieces]

    def cost(self, K: int) -> float:
        return float(sum(seq_cost(q, l, K) for q, l in zip(self.q_lens, self.kv_lens)))


def shard(q_lens: Sequence[int], kv_lens: Sequence[int], K: int, world: int, rank: int,
          by: str = "auto") -> RankShard:
    """Rank `rank`'s share of the batch.  by = "sequences" deals whole sequences, "rows" cuts
    every sequence's query rows into `world` ranges, "auto" takes "sequences" when there are
    at least as many sequences as ranks and "rows" otherwise."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    if by == "auto":
        by = "sequences" if len(q_lens) >= world else "rows"
    sh = RankShard()
    if by == "sequences":
        for b in split_sequences(q_lens, kv_lens, K, world)[rank]:
            q, l = int(q_lens[b]), int(kv_lens[b])
            sh.pieces.append(Piece(b, 0, q, l))
    elif by == "rows":
        for b, (q, l) in enumerate(zip(q_lens, kv_lens)):
            i0, i1 = split_rows(int(q), int(l), K, world)[rank]
            if i1 > i0:
                sh.pieces.append(Piece(b, i0, i1, int(l) - int(q) + i1))
    else:
        raise ValueError(by)
    sh.q_lens = [p.q1 - p.q0 for p in sh.pieces]
    sh.kv_lens = [p.kv_len for p in sh.pieces]
    return sh
