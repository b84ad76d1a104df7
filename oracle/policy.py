"""Context policy phi(j, r) -- oracle side.

Source: design-space paper (thelatestinai.com summary of arXiv 2609.22283),
Table 1 rows and Figure 1: a denoising update at level j that looks r chunks
back reads that history chunk at level phi(j, r); level 0 is fully denoised.

    clean        phi(j, r) = 0
    same-level   phi(j, r) = j
    progressive  phi(j, r) = max(j - r, 0)

phi is only used for history (r >= 1); a node always reads its own chunk at
its own level.
"""

CLEAN, SAME, PROGRESSIVE = "clean", "same", "progressive"
POLICY_CODES = {CLEAN: 0, SAME: 1, PROGRESSIVE: 2}


def phi(policy: str, j: int, r: int) -> int:
    if r < 1:
        raise ValueError("phi is defined for history chunks only (r >= 1)")
    if j < 0:
        raise ValueError("levels are non-negative")
    if policy == CLEAN:
        return 0
    if policy == SAME:
        return j
    if policy == PROGRESSIVE:
        return max(j - r, 0)
    raise ValueError(f"unknown policy {policy!r}")
