"""Routing-margin screen for synthetic layer inputs.

TEST INFRASTRUCTURE (same import rule as ``moe_oracle``): it decides, with the
oracle's fp64 router logits, which token rows of x must be drawn again so that the
routing decision is far from a tie, and asks the caller's ``redraw`` function for
the next attempt of those rows. It never draws numbers itself.

A token passes when, among its k+1 largest logits (k when E = k), every pair of
neighbours is at least ``margin`` apart: the gap between 1st and 2nd keeps the slot
order unambiguous, the gap between k-th and (k+1)-th keeps the expert set
unambiguous. Rows still failing after ``max_attempts`` draws are kept and reported
as near-ties.
"""
from __future__ import annotations

import numpy as np
import torch

from .moe_oracle import router_logits


def min_gap(logits: np.ndarray, k: int) -> np.ndarray:
    """Per token, the smallest gap between neighbours among its k+1 largest logits."""
    srt = -np.sort(-logits, axis=1)
    m = min(k + 1, logits.shape[1])
    if m < 2:
        return np.full(logits.shape[0], np.inf)
    return (srt[:, :m - 1] - srt[:, 1:m]).min(axis=1)


def screen_margin(x: torch.Tensor, w_router, logit_bias, k: int, redraw,
                  margin: float = 1e-2, max_attempts: int = 64, prep=None):
    """Return (x, attempts [T] int64, near_tie_rows [n] int64).

    ``redraw(rows, attempt)`` returns bf16 rows [len(rows), H] for attempt number
    ``attempt`` of the given row indices. ``prep``, if given, maps rows of x to what the
    router actually sees (for instance the normed activations).
    """
    prep = prep or (lambda rows: rows)
    x = x.clone()
    attempts = torch.zeros(x.shape[0], dtype=torch.int64)
    bad = np.nonzero(min_gap(router_logits(prep(x), w_router, logit_bias), k) < margin)[0]
    attempt = 0
    while bad.size and attempt < max_attempts:
        attempt += 1
        rows = torch.from_numpy(bad.astype(np.int64))
        x[rows] = redraw(rows, attempt).to(x.dtype)
        attempts[rows] = attempt
        gaps = min_gap(router_logits(prep(x[rows]), w_router, logit_bias), k)
        bad = bad[gaps < margin]
    return x, attempts, torch.from_numpy(bad.astype(np.int64))
