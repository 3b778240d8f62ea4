"""Dynamic block-size scheduling, plain reference (test infrastructure, like the
rest of oracle/; the library's own C++ policy shares no code with it).

Source: "DFlash – 플래시 추측적 디코딩을 위한 블록 확산" §3 item 4 and §4: the drafter
is trained with block size 16 and can be run with smaller blocks; the block size
is scheduled dynamically. The pages give no formula; the reading taken here:

* acceptance model: alpha_i = P(draft i accepted | drafts 1..i-1 accepted) for
  block position i >= 1, estimated from verify results. A cycle run with block B
  that accepted a drafts tested positions 1 .. min(a+1, B-1) and accepted
  positions 1 .. a. Counts decay by a factor per observation window and carry a
  Beta(1, 1) prior: alpha_i = (A_i + 1) / (T_i + 2);
* expected tokens committed by a cycle with block B (the accepted drafts plus
  the correction or bonus token): 1 + sum_{i=1}^{B-1} prod_{j=1}^{i} alpha_j;
* choice: among the candidate block sizes, the one that maximises expected
  tokens per unit of cycle cost, cost(B) given by the caller (for example the
  measured cycle time at the current concurrency, or c0 + c1 * bs * B); on an
  exact tie the smaller block.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np


def acceptance_counts(accepted: Sequence[int], B: int, n_pos: int) -> Tuple[np.ndarray, np.ndarray]:
    """(tested, accepted) counts per block position 0..n_pos-1 (position 0 unused)
    from the accepted lengths of one cycle's requests run with block B."""
    tested = np.zeros(n_pos, dtype=np.int64)
    acc = np.zeros(n_pos, dtype=np.int64)
    for a in accepted:
        a = int(a)
        for i in range(1, B):
            if i <= a + 1:
                tested[i] += 1
            if i <= a:
                acc[i] += 1
    return tested, acc


class BlockPolicy:
    def __init__(self, candidates: Sequence[int], decay: float, n_pos: int):
        self.candidates = sorted(int(b) for b in candidates)
        self.decay = float(decay)
        self.T = np.zeros(n_pos)
        self.A = np.zeros(n_pos)

    def observe(self, tested, accepted) -> None:
        self.T = self.decay * self.T + np.asarray(tested, dtype=np.float64)
        self.A = self.decay * self.A + np.asarray(accepted, dtype=np.float64)

    def alpha(self) -> np.ndarray:
        return (self.A + 1.0) / (self.T + 2.0)

    def expected_tokens(self, B: int) -> float:
        al = self.alpha()
        total, run = 1.0, 1.0
        for i in range(1, B):
            run *= al[i]
            total += run
        return total

    def choose(self, costs: Sequence[float]) -> int:
        """costs[k]: the cycle cost at candidates[k] (sorted ascending)."""
        best, best_v = self.candidates[0], -1.0
        for B, c in zip(self.candidates, costs):
            v = self.expected_tokens(B) / float(c)
            if v > best_v:
                best, best_v = B, v
        return best

    def choose_linear(self, bs: int, c0: float, c1: float) -> int:
        return self.choose([c0 + c1 * bs * B for B in self.candidates])
