"""The tensor-core prefill's segment rule, restated for the tests (host-side scheduling only:
no method arithmetic). It must agree with `tc_plan` in csrc/kda_prefill_tc.cu, which
tests/test_segment_plan.py checks through the library's workspace size."""
from __future__ import annotations

SMS = 148
CHUNK = 64


def streamed(n_seqs: int, H: int, max_len: int, T_total: int) -> bool:
    """Whether the library walks each (sequence, head) in one CTA beside the intra-chunk
    kernel (its model of the two schedules, restated)."""
    pairs = n_seqs * H
    lc = -(-max_len // CHUNK)
    m = SMS // pairs
    tiles_us = 12.6 * ((-(-T_total // CHUNK) + n_seqs) * H)
    walk_seg = 5.1 * lc / (m + 1.26) if (m >= 2 and lc >= 16) else 1.9 * lc
    t_seg = tiles_us / 296.0 + walk_seg
    if not 1 <= pairs <= 100:
        return False
    t_str = max(1.9 * lc, tiles_us / (2.0 * (SMS - pairs))) + 10.0
    return t_str < 0.97 * t_seg


def segment_plan(n_seqs: int, H: int, max_len: int, T_total: int | None = None):
    """(first, seg, dec) in tokens, or None for one segment per sequence: segment 0 holds
    `first` tokens, segment j >= 1 holds `seg - (j - 1) dec`. T_total defaults to
    n_seqs * max_len."""
    pairs = n_seqs * H
    lc = -(-max_len // CHUNK)
    m = SMS // pairs
    if streamed(n_seqs, H, max_len, n_seqs * max_len if T_total is None else T_total):
        return None
    if m < 2 or lc < 16:
        return None
    for d in (2, 1, 0):
        n = max(4, -(-(5 * (lc + d * (m * (m - 1) // 2))) // (5 * m + 6)))
        lo = (n + 1) // 2 if n // 2 > 4 else 4
        if n - (m - 1) * d >= lo:
            break
    return CHUNK * (-(-(6 * n) // 5)), CHUNK * n, CHUNK * d


def segment_count(length: int, plan, max_segs: int | None = None) -> int:
    """Segments that hold `length` tokens under `plan` (1 when plan is None)."""
    if plan is None:
        return 1
    first, seg, dec = plan
    k, off = 1, first
    while off < length and (max_segs is None or k <= max_segs):
        off += seg - (k - 1) * dec
        k += 1
    return k
