"""Greedy integer bit allocation by marginal gain, and the group layout.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract (integer widths handed out greedily by
marginal gain, so that blocks with more energy get more bits) and the
blockgtq README (bits move toward high-energy blocks while the average per
dim stays fixed).  Readings used here (the pages give no formula):

* budget: every block has two dims, so an average of A bits per dim over D
  dims is sum_j b_j = A * D / 2;
* start every block at b_min; while budget is left, give one more bit to
  the block with the largest gain s_j * (Dist(b_j) - Dist(b_j + 1)) among
  blocks below b_max; on an exact tie of the float64 gains the lower block
  index wins;
* Dist(b) is the N(0,1) Lloyd-Max distortion, the fixed constants
  ``lloyd_max.DISTORTION``.

Group layout (one TQ-MSE rotation per bit-width group, read as follows):
the dims of all blocks with the same width form one group; groups are
ordered by width, largest first; inside a group the dims are in ascending
order.  Width-0 groups (possible only with b_min = 0) store nothing.
"""
import numpy as np

from .energy import block_dims
from .lloyd_max import DISTORTION


def greedy_allocate(scores, avg_bits, b_min=1, b_max=4):
    """Integer widths [D/2] for one (layer, KV head) from float64 scores [D/2]."""
    scores = [float(s) for s in scores]
    nblk = len(scores)
    budget = avg_bits * nblk
    if not (b_min * nblk <= budget <= b_max * nblk):
        raise ValueError("average bits outside [b_min, b_max]")
    widths = [b_min] * nblk
    spent = b_min * nblk
    while spent < budget:
        best = -1
        best_gain = None
        for j in range(nblk):
            if widths[j] >= b_max:
                continue
            gain = scores[j] * (DISTORTION[widths[j]] - DISTORTION[widths[j] + 1])
            if best < 0 or gain > best_gain:
                best, best_gain = j, gain
        widths[best] += 1
        spent += 1
    return np.array(widths, dtype=np.int64)


def dim_widths(block_widths, head_dim, pairing=0):
    """Per-dim widths [D] from per-block widths [D/2]."""
    w = np.zeros(head_dim, dtype=np.int64)
    for j, (a, b) in enumerate(block_dims(head_dim, pairing)):
        w[a] = block_widths[j]
        w[b] = block_widths[j]
    return w


def group_layout(block_widths, head_dim, pairing=0):
    """Groups as a list of (width, dims ndarray), width-descending, dims ascending.

    Width-0 groups are left out (they have no codes and no norm).
    """
    w = dim_widths(block_widths, head_dim, pairing)
    groups = []
    for b in sorted(set(int(x) for x in w), reverse=True):
        if b == 0:
            continue
        groups.append((b, np.nonzero(w == b)[0]))
    return groups
