"""The kernels' per-frame mask against the oracle's token rule, on the CPU.

gca_visible_prefix evaluates the same inline function the attention kernels
use (one prefix length per (query frame, walk-list entry)).  For every entry of
the walk lists a host-only cache produces — single frames and multi-frame
blocks, the anchor block, the three trajectory-memory variants, pages that
hold parts of several frames' summary tokens — the tokens the oracle's rule
lets each query frame see must be exactly the first `prefix` slots.
"""
import pytest

from oracle import gca as ogca
from windowed_memory_attention_b200 import gca, inputs

S = 6


def _slots(entry, keep):
    """(frame, tau) of every slot of a walk-list entry."""
    page, kind, frame, first, n_valid = entry
    if kind == gca.GCA_PAGE_IMAGE:
        return [(frame, keep + first + s) for s in range(n_valid)]
    return [((first + s) // keep, (first + s) % keep) for s in range(n_valid)]


@pytest.mark.parametrize("M,P,n,k,keep,anchor_block,fmax", [
    (150, 64, 2, 3, None, False, 1),     # multi-page frames, summary pages shared by frames
    (150, 64, 2, 3, 1, False, 1),        # camera token only
    (150, 64, 0, 3, 0, False, 1),        # sliding window
    (40, 64, 3, 2, None, True, 3),       # anchor block, blocks of up to 3 frames
    (40, 64, 2, 4, None, False, 3),      # multi-frame blocks
    (40, 64, 2, 4, 1, False, 2),
])
def test_visible_prefix_equals_the_token_rule(M, P, n, k, keep, anchor_block, fmax):
    T = 25
    kp = S if keep is None else keep
    mode = {None: gca.GCA_MEMORY_SUMMARY, 1: gca.GCA_MEMORY_CAMERA, 0: gca.GCA_MEMORY_NONE}[keep]
    w = inputs.TINY.with_(M=M, n=n, k=k, T=T, page_size=P)
    cache = gca.Cache.for_workload(w, device=gca.GCA_HOST_ONLY, trajectory_memory=mode,
                                   anchor_block=anchor_block, max_query_frames=fmax)
    checked = 0
    for t in range(T):
        cache.append(None, None)
        for F in range(1, min(fmax, t + 1) + 1):
            try:
                walk = cache.layout(F)
            except gca.GCAError as e:
                assert e.name == "GCA_ERR_STATE"            # a needed frame was evicted
                continue
            for i in range(t + 1 - F, t + 1):
                for entry in walk:
                    prefix = cache.visible_prefix(entry, i)
                    vis = [ogca.visible(i, j, tau, n=n, k=k, S=S, anchor_block=anchor_block, keep=kp)
                           for j, tau in _slots(entry, kp)]
                    assert vis == [True] * prefix + [False] * (len(vis) - prefix), (t, F, i, entry)
                    checked += 1
        cache.evict()
    assert checked > 100
    cache.close()


def test_a_page_of_summary_tokens_from_several_frames_is_cut_at_the_query_frame():
    # P = 64 holds the 6 summary tokens of frames 0..9 and 4 of frame 10
    w = inputs.TINY.with_(M=40, n=1, k=1, T=30, page_size=64)
    cache = gca.Cache.for_workload(w, device=gca.GCA_HOST_ONLY)
    for _ in range(12):
        cache.append(None, None)
        cache.evict()
    entry = next(e for e in cache.layout() if e[1] == gca.GCA_PAGE_SUMMARY)
    assert entry[3] == 0 and entry[4] == 64
    assert cache.visible_prefix(entry, 9) == 60           # frames 0..9
    assert cache.visible_prefix(entry, 10) == 64          # and the 4 tokens of frame 10 on it
    assert cache.visible_prefix(entry, 3) == 24
    cache.close()
