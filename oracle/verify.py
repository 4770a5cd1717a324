"""Greedy verify: per-row argmax, accept length and committed tokens (oracle; test infrastructure only).

Sources:

* "TandemLLM", introduction. Small drafters guess the next tokens and the big
  model checks every guess in one pass. A guess the model agrees with is a free
  token. At the first wrong guess the model puts in its own token. The output is
  the model's own greedy text, except where the two best tokens are within one
  ulp.
* "TandemLLM", "How it works" flowchart: the target verifies in one pass, then
  the longest path the model agrees with is kept.
* "Qwen3.8 on DGX Spark (GB10)", introduction: the target verifies every drafted
  token over the whole 248,320-row vocabulary.

Row layout: ``M = B * (D + 1)``. Row ``b * (D + 1) + i`` holds the target's logits
after the committed context plus drafts ``d[b, 0..i-1]``, so its argmax is the
target's greedy token for slot i of sequence b. Slot D (the last row) gives the
bonus token when every draft is accepted.

Readings where the pages are silent:

* Ties in argmax go to the lowest index.
* The accept length is ``L = min{i in [0, D) : d[b, i] != t[b(D+1) + i]}``, or D if
  there is no mismatch. The committed tokens are ``t[b(D+1) .. b(D+1) + L]``:
  the L accepted drafts followed by the target's own token at position L.
* Tree verify ("How it works": the drafters propose a tree, the target verifies the
  whole tree in one pass, and the longest path it agrees with is kept). A sequence
  has nodes 0..D: node 0 is the committed context, node k >= 1 holds draft token
  ``d[b, k-1]`` and has parent ``p[b, k-1]`` in ``[0, k-1]``. Row ``b(D+1) + k`` is
  the target's prediction after the root-to-k path. Node k is accepted when its
  parent is accepted and ``d[b, k-1] == t[b(D+1) + p[b, k-1]]`` (the root always is).
  The kept path ends at the accepted node of greatest depth, the lowest node index
  among equals; the accept length is its depth, and the committed tokens are the
  drafts on the path followed by the target's token at its end node. With
  ``p[b, k-1] = k-1`` (a chain) this is the accept rule above.
* Near ties. A row whose two largest logits differ by less than ``1e-3`` (in
  logit units) is excluded from exact argmax comparison. That is the pages'
  one-ulp caveat. A sequence is excluded from the exact accept-length comparison
  when an excluded row lies at a slot <= its oracle accept length.
"""

from __future__ import annotations

import numpy as np

NEAR_TIE = 1e-3


def argmax_ref(y: np.ndarray) -> np.ndarray:
    """t[m] = argmax_n y[m, n]; the lowest index wins among equal maxima."""
    y = np.asarray(y)
    if y.ndim != 2 or y.shape[1] == 0:
        raise ValueError("y must be [M, N] with N >= 1")
    if np.isnan(y).any():
        raise ValueError("argmax of NaN is undefined")
    best = np.full(y.shape[0], -1, dtype=np.int64)
    best_val = np.full(y.shape[0], -np.inf)
    for n in range(y.shape[1]):                 # scan left to right; strict > keeps the first maximum
        col = y[:, n]
        better = col > best_val
        best = np.where(better, n, best)
        best_val = np.where(better, col, best_val)
    # a row of all -inf: its first index
    best = np.where(best < 0, 0, best)
    return best


def argmax_fast(y: np.ndarray) -> np.ndarray:
    """Same definition as :func:`argmax_ref` through numpy's first-occurrence argmax.

    Used for the large sizes where the column loop is slow.
    """
    y = np.asarray(y)
    if np.isnan(y).any():
        raise ValueError("argmax of NaN is undefined")
    return np.argmax(y, axis=1).astype(np.int64)


def top2_gap(y: np.ndarray) -> np.ndarray:
    """Per row: largest value minus second largest (0 when the maximum is shared)."""
    y = np.asarray(y, dtype=np.float64)
    if y.shape[1] < 2:
        return np.full(y.shape[0], np.inf)
    part = -np.partition(-y, 1, axis=1)
    return part[:, 0] - part[:, 1]


def accept_ref(t: np.ndarray, drafts: np.ndarray, D: int) -> np.ndarray:
    """L[b] = first slot i < D where the draft differs from the target token, else D."""
    drafts = np.asarray(drafts, dtype=np.int64)
    B = drafts.shape[0] if drafts.ndim == 2 else 0
    if D < 0:
        raise ValueError("D must be >= 0")
    t = np.asarray(t, dtype=np.int64)
    if t.shape[0] != B * (D + 1):
        raise ValueError("t must have B*(D+1) rows")
    L = np.empty(B, dtype=np.int64)
    for b in range(B):
        length = D
        for i in range(D):
            if drafts[b, i] != t[b * (D + 1) + i]:
                length = i
                break
        L[b] = length
    return L


def committed_ref(t: np.ndarray, L: np.ndarray, D: int):
    """Tokens committed for each sequence: the L accepted drafts and then the target's token."""
    t = np.asarray(t, dtype=np.int64)
    return [t[b * (D + 1): b * (D + 1) + int(L[b]) + 1].copy() for b in range(len(L))]


def verify_ref(y: np.ndarray, drafts: np.ndarray, D: int, fast: bool = True):
    """Full greedy verify from logits: returns ``(t [M], L [B], gap [M])``."""
    t = argmax_fast(y) if fast else argmax_ref(y)
    L = accept_ref(t, drafts, D)
    return t, L, top2_gap(y)


def comparable_rows(gap: np.ndarray, tol: float = NEAR_TIE) -> np.ndarray:
    """Rows whose argmax must match exactly: top-2 gap at least ``tol``."""
    return np.asarray(gap) >= tol


def comparable_sequences(gap: np.ndarray, L: np.ndarray, D: int, tol: float = NEAR_TIE) -> np.ndarray:
    """Sequences whose accept length must match exactly. A sequence is excluded
    when a near-tie row sits at a slot <= its oracle accept length."""
    ok = comparable_rows(gap, tol)
    out = np.ones(len(L), dtype=bool)
    for b in range(len(L)):
        rows = ok[b * (D + 1): b * (D + 1) + int(L[b]) + 1]
        out[b] = bool(rows.all())
    return out


def accept_tree_ref(t: np.ndarray, drafts: np.ndarray, parents: np.ndarray, D: int):
    """Tree verify: returns ``(L [B], node [B])``, the depth and index of the kept path's end.

    Nodes are visited in index order; a parent always precedes its child, so one pass
    settles every node. A parent index outside ``[0, k-1]`` raises.
    """
    drafts = np.asarray(drafts, dtype=np.int64)
    parents = np.asarray(parents, dtype=np.int64)
    t = np.asarray(t, dtype=np.int64)
    B = drafts.shape[0] if drafts.ndim == 2 else 0
    if t.shape[0] != B * (D + 1) or (D > 0 and parents.shape != (B, D)):
        raise ValueError("t must have B*(D+1) rows and parents must be [B, D]")
    L = np.zeros(B, dtype=np.int64)
    node = np.zeros(B, dtype=np.int64)
    for b in range(B):
        base = b * (D + 1)
        accepted = [True] + [False] * D
        depth = [0] * (D + 1)
        for k in range(1, D + 1):
            p = int(parents[b, k - 1])
            if not 0 <= p < k:
                raise ValueError(f"parent of node {k} must be in [0, {k - 1}], got {p}")
            depth[k] = depth[p] + 1
            accepted[k] = accepted[p] and drafts[b, k - 1] == t[base + p]
            if accepted[k] and depth[k] > L[b]:
                L[b], node[b] = depth[k], k
    return L, node


def tree_path(parents: np.ndarray, b: int, node: int):
    """Nodes on the root-to-``node`` path of sequence b, root excluded, in path order."""
    path = []
    while node != 0:
        path.append(node)
        node = int(parents[b, node - 1])
    return path[::-1]


def committed_tree_ref(t: np.ndarray, drafts: np.ndarray, parents: np.ndarray, node: np.ndarray, D: int):
    """Committed tokens per sequence: the drafts on the kept path, then the target's token at its end."""
    t = np.asarray(t, dtype=np.int64)
    out = []
    for b in range(len(node)):
        path = tree_path(parents, b, int(node[b]))
        toks = [int(drafts[b, k - 1]) for k in path] + [int(t[b * (D + 1) + int(node[b])])]
        out.append(np.asarray(toks, dtype=np.int64))
    return out


def comparable_tree_sequences(gap: np.ndarray, parents: np.ndarray, D: int, tol: float = NEAR_TIE) -> np.ndarray:
    """Sequences whose tree verify must match exactly: every row of the sequence has a
    top-2 gap of at least ``tol`` (any row can decide a node's acceptance in a tree)."""
    ok = comparable_rows(gap, tol)
    B = len(ok) // (D + 1)
    return np.array([bool(ok[b * (D + 1): (b + 1) * (D + 1)].all()) for b in range(B)], dtype=bool)
