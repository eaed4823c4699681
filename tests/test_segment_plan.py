"""Host-side checks of the tensor-core prefill's schedule and segment plan (CPU: no kernel runs).

The walk kernel runs, per (sequence, head), one CTA per later segment, and its CTAs wait for
one another's state hand-offs, so the plan must never ask for more CTAs than there are SMs:
max_segs - 1 <= 148 // pairs. The library's workspace size shows how many segments it
planned (the start states and flags take 128 * 128 * 4 + 4 bytes per (sequence, head,
segment) when there are three or more), and the restated rule in tests/plan.py must agree
with it."""
from __future__ import annotations

import pytest
import torch

from tests.plan import CHUNK, SMS, segment_count, segment_plan

TILE_BYTES = 4 * 128 * 64 * 2 + 64 * 64 * 2 + 128 * 4  # per (chunk slot, head)
UNIT_BYTES = 128 * 128 * 4 + 4                          # per (sequence, head, segment)
HEADER = 256


@pytest.fixture(scope="module")
def kda():
    from kimi_delta_attention_19_b200 import kda as k
    return k


def planned_max_segs(kda, n_seqs, H, max_len, T_total):
    """Segments the library planned for the longest sequence (0 when it is 1 or 2: the
    workspace then has no start states)."""
    shape = kda.make_shape(T_total, H, 128, 128, torch.bfloat16, n_seqs=n_seqs,
                           max_seqlen=max_len)
    ws = kda.workspace_size(shape)
    assert ws > 0
    n_slots = -(-T_total // CHUNK) + n_seqs
    tiles_off = ws - TILE_BYTES * n_slots * H
    ready = -(-(4 * n_slots * H) // 256) * 256  # per-tile ready flags
    if tiles_off == -(-(HEADER + ready) // 1024) * 1024:
        return 0
    segs = (tiles_off - HEADER - ready) // (UNIT_BYTES * n_seqs * H)
    assert -(-(HEADER + ready + UNIT_BYTES * n_seqs * H * segs) // 1024) * 1024 == tiles_off
    return segs


CASES = [(1, 32, 8192), (1, 16, 1 << 20), (8, 32, 32768), (6, 2, 3000), (3, 13, 1792),
         (1, 1, 1 << 16), (2, 3, 50000), (1, 74, 4096), (1, 49, 9000), (4, 9, 20000),
         (1, 37, 2048), (1, 2, 1024), (5, 7, 777)]


@pytest.mark.parametrize("n_seqs,H,max_len", CASES)
def test_plan_matches_library_and_fits_the_sms(kda, n_seqs, H, max_len):
    pairs = n_seqs * H
    plan = segment_plan(n_seqs, H, max_len)  # T_total = n_seqs * max_len, as below
    want = segment_count(max_len, plan)
    got = planned_max_segs(kda, n_seqs, H, max_len, T_total=max_len * n_seqs)
    assert got == (want if want > 2 else 0), (got, want, plan)
    if plan is None:
        return
    first, seg, dec = plan
    m = SMS // pairs
    # the walk kernel's grid: (segments - 1) CTAs per (sequence, head), all resident at once
    assert want - 1 <= m, (want, m)
    # every planned later segment holds at least four chunks, and m of them cover the longest
    # sequence after segment 0
    lengths = [seg - j * dec for j in range(m)]
    assert min(lengths) >= 4 * CHUNK, lengths
    assert first + sum(lengths) >= max_len
    assert first % CHUNK == 0 and seg % CHUNK == 0 and dec % CHUNK == 0


def test_shrinking_plan_offsets():
    """Segment 0 of 11 chunks, then 9, 7, 5 chunks: a sequence ending inside each segment."""
    plan = segment_plan(3, 13, 1792, T_total=1792 + 1000 + 1)
    assert plan == (11 * 64, 9 * 64, 2 * 64)
    assert [segment_count(n, plan) for n in (1, 704, 705, 1280, 1281, 1728, 1729, 1792)] == \
        [1, 1, 2, 2, 3, 3, 4, 4]


def test_streamed_schedule_choice():
    """The 8K x 32-head workload walks each (sequence, head) in one CTA beside the intra-chunk
    kernel; a million tokens of 16 heads, and varlen batches of 256 (sequence, head) pairs,
    keep the segmented schedule."""
    from tests.plan import streamed
    assert streamed(1, 32, 8192, 8192)
    assert not streamed(1, 16, 1 << 20, 1 << 20)
    assert not streamed(8, 32, 32768, 147651)
