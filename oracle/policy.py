"""Per-step policy of the block-sparse attention node -- TEST INFRASTRUCTURE ONLY.

A plain restatement, for the tests, of when one attention call stays dense
instead of taking the sparse path.  Sources (cited by title and section):

  "BlockSparseAttention - ComfyUI Built-in Node Documentation", general inputs
  (start_percent: the point in the sampling schedule where sparse attention
  starts, dense before it, default 0.2; end_percent: where it ends, dense
  after it, default 1.0; dense_blocks: transformer blocks always run dense,
  written like '0, 1, 47-49', default empty; min_tokens: shorter sequences
  stay dense, default 12288) and "constraints and limitations" (those cases
  fall back to dense attention; dense_blocks is ignored for a model that
  reports no block index).
  "minimax-h3-chunk-star7" README, "Hybrid": attention switches between whole
  sampling steps; the guard steps at the front and back run dense, the middle
  ones sparse (in a four-step run the first and fourth steps are dense); the
  run stops with an error when the step cannot be determined.

Readings where the pages leave a point open: the window is inclusive at both
ends; a guard region is one step at each end unless told otherwise; the reasons
are reported in the order short sequence, listed block, hybrid guard, window.
"""
from __future__ import annotations

from dataclasses import dataclass

SPARSE, SHORT, BLOCK, HYBRID, WINDOW = 0, 1, 2, 3, 4


@dataclass
class Policy:
    start_percent: float = 0.2
    end_percent: float = 1.0
    min_tokens: int = 12288
    hybrid: bool = False
    hybrid_guard_steps: int = 1
    dense_blocks: str = ""


def listed_blocks(spec: str) -> list:
    """The (low, high) inclusive ranges of a dense_blocks string; ValueError if malformed."""
    out = []
    for part in spec.split(","):
        part = part.strip()
        if not part:
            continue
        if "-" in part:
            lo, _, hi = part.partition("-")
            lo, hi = lo.strip(), hi.strip()
            if not lo.isdigit() or not hi.isdigit() or int(hi) < int(lo):
                raise ValueError(f"malformed range {part!r}")
            out.append((int(lo), int(hi)))
        else:
            if not part.isdigit():
                raise ValueError(f"malformed block index {part!r}")
            out.append((int(part), int(part)))
    return out


def decide(pol: Policy, n_tokens: int, block_index: int, progress: float, step: int = -1, n_steps: int = 0) -> int:
    if not (0.0 <= pol.start_percent <= 1.0 and 0.0 <= pol.end_percent <= 1.0):
        raise ValueError("window outside [0, 1]")
    if pol.min_tokens < 0 or n_tokens < 1 or not (0.0 <= progress <= 1.0):
        raise ValueError("bad argument")
    if pol.hybrid and (pol.hybrid_guard_steps < 0 or n_steps < 1 or not (0 <= step < n_steps)):
        raise ValueError("hybrid needs the sampling step")
    ranges = listed_blocks(pol.dense_blocks or "")
    if n_tokens < pol.min_tokens:
        return SHORT
    if block_index >= 0 and any(lo <= block_index <= hi for lo, hi in ranges):
        return BLOCK
    if pol.hybrid and (step < pol.hybrid_guard_steps or step >= n_steps - pol.hybrid_guard_steps):
        return HYBRID
    if progress < pol.start_percent or progress > pol.end_percent:
        return WINDOW
    return SPARSE
