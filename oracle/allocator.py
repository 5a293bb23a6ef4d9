"""Page-table simulator for the paged GCA KV store.

TEST INFRASTRUCTURE (see oracle/gca.py's header for who may import it).  An
independent Python restatement of the page-table rules, used to check the
library's page tables bit for bit.

The pages say the cache is paged so that frames can be appended and evicted
without re-allocating a contiguous buffer, and that it is sized per layer with
room for scale (anchor) frames + window + slack (code walkthrough §3.4; news
article, inference paragraph).  The page layout itself is not printed, so the
rules below are this project's own definition, stated once and implemented
twice (here and in the C++ host code):

  * one pool of ``num_pages`` page ids, shared by every layer;
  * a frame keeps ``keep`` of its S special tokens as trajectory memory (S by
    default; 1 = the camera token only; 0 = none, the sliding-window cache):
    they go to one append-only summary stream, token s < keep of frame t at
    stream index keep*t+s, summary page (keep*t+s) // P, slot (keep*t+s) % P;
  * frame t owns ceil(M'/P) image pages, M' = M + S - keep, holding its other
    special tokens and then its M image tokens in token order (slot tau-keep);
  * pages are taken smallest free id first, in token order within a frame:
    a new summary page (when the frame's summary tokens cross a page
    boundary) before the frame's image pages;
  * capacity: (n + k + max_query_frames + frame_slack) * ceil(M'/P) image pages
    plus ceil(keep*max_frames/P) summary pages;
  * evict (after frame t): every non-anchor frame f <= t-k still holding image
    pages returns them to the free set; its summary tokens stay where they are,
    so eviction moves no bytes;
  * reset: the creation state (all pages free, no frames);
  * walk list for a query block of the F latest frames: the image pages of every
    full frame that some query frame of the block may see, in ascending frame
    order and page order, then every summary page in stream order.  Each entry
    is (page_id, kind, frame, first, n_valid): kind 0 = image, 1 = summary;
    for an image page ``frame`` is its frame and ``first`` the index of its
    slot 0 among the frame's M' image-page tokens; for a summary page ``first``
    is the stream index of slot 0 and ``frame`` = first // keep.
"""
from __future__ import annotations

import heapq
import math

IMAGE, SUMMARY = 0, 1


class CapacityError(RuntimeError):
    pass


class StateError(RuntimeError):
    pass


class PageTableSim:
    def __init__(self, *, M: int, S: int, P: int, n: int, k: int, max_frames: int,
                 max_query_frames: int = 1, frame_slack: int = 0,
                 anchor_block: bool = False, keep: int = None):
        self.M, self.S, self.P, self.n, self.k = M, S, P, n, k
        self.keep = S if keep is None else keep     # special tokens kept per frame
        self.Mi = M + S - self.keep                  # tokens of a full frame's image pages
        self.max_frames = max_frames
        self.anchor_block = anchor_block
        self.ipf = math.ceil(self.Mi / P)
        self.image_capacity = (n + k + max_query_frames + frame_slack) * self.ipf
        self.summary_capacity = math.ceil(self.keep * max_frames / P)
        self.num_pages = self.image_capacity + self.summary_capacity
        self.reset()

    def reset(self):
        self.free = list(range(self.num_pages))
        heapq.heapify(self.free)
        self.T = 0
        self.image_pages = {}          # frame -> [page ids] while the frame is full
        self.summary_pages = []

    def _take(self) -> int:
        return heapq.heappop(self.free)

    def append(self) -> int:
        """Open frame T; returns its index."""
        t = self.T
        if t >= self.max_frames:
            raise CapacityError("max_frames reached")
        kp = self.keep
        new_summary = sum(1 for s in range(kp) if (kp * t + s) % self.P == 0)
        if len(self.free) < self.ipf + new_summary:
            raise CapacityError("page pool exhausted")
        for s in range(kp):
            if (kp * t + s) % self.P == 0:
                self.summary_pages.append(self._take())
        self.image_pages[t] = [self._take() for _ in range(self.ipf)]
        self.T += 1
        return t

    def evict(self) -> int:
        t = self.T - 1
        count = 0
        for f in sorted(self.image_pages):
            if f >= self.n and f <= t - self.k:
                for p in self.image_pages.pop(f):
                    heapq.heappush(self.free, p)
                count += 1
        return count

    def _frame_seen(self, i: int, j: int) -> bool:
        if self.anchor_block and i < self.n and j < self.n:
            return True
        return j <= i and (j < self.n or j >= i - self.k + 1)

    def walk(self, F: int = 1):
        if F < 1 or F > self.T:
            raise StateError("query block larger than the stream")
        queries = range(self.T - F, self.T)
        for i in queries:
            for j in range(self.T):
                if self._frame_seen(i, j) and j not in self.image_pages:
                    raise StateError(f"frame {j} needed by query frame {i} was evicted")
        out = []
        for f in sorted(self.image_pages):
            if any(self._frame_seen(i, f) for i in queries):
                for seq, pid in enumerate(self.image_pages[f]):
                    first = seq * self.P
                    out.append((pid, IMAGE, f, first, min(self.P, self.Mi - first)))
        total = self.keep * self.T
        for seq, pid in enumerate(self.summary_pages):
            first = seq * self.P
            out.append((pid, SUMMARY, first // self.keep, first, min(self.P, total - first)))
        return out

    def resident_tokens(self) -> int:
        """Tokens held: image-page tokens of full frames plus every kept token."""
        return self.Mi * len(self.image_pages) + self.keep * self.T

    def slot_of(self, frame: int, tau: int):
        """(page id, slot) of token slot tau of a frame (tau < keep: summary stream)."""
        if tau < self.keep:
            idx = self.keep * frame + tau
            return self.summary_pages[idx // self.P], idx % self.P
        m = tau - self.keep
        return self.image_pages[frame][m // self.P], m % self.P
