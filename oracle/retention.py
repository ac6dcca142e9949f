"""Dual-stream paged KV retention: page table, free list, deferred eviction, rollback.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  Pure integer bookkeeping.

What the pages fix
------------------
* [3DRoPE-KV] "Dual-Stream Memory Layout": the patch stream holds one page of
  ``patches_per_frame`` tokens per frame; the first ``scale_frames`` pages stay for good,
  the next ``sliding_window`` pages are recycled, and when the window is full its oldest
  page goes back to a free list.  The special stream is append-only, holds the 6 special
  tokens of every frame and is never evicted.
* [3DRoPE-KV] "Attention Computation with Cached RoPE": the visible page table is ordered
  scale patch pages, then live window patch pages, then all special pages, and the last
  special page may be partly filled (its valid length is passed along).
* [KVBenefits] "Reduced KV Growth via Keyframe Streaming" and "Dynamic Keyframe Selection":
  non-keyframes are processed but not cached; a kept frame triggers the deferred eviction,
  a dropped frame's temporary entry is rolled back.

Readings where the pages leave a step open:

* A frame is appended tentatively, attends (its own tokens visible), then is committed
  (keyframe) or rolled back (non-keyframe).  Eviction happens at commit, i.e. after the
  attention of the frame that overflows the window ("deferred").
* Scale pages are the first ``scale_frames`` committed keyframes; later keyframes enter the
  window; a window longer than ``sliding_window`` returns its oldest page to the free list.
* The free list is a LIFO stack; a fresh cache pops pages 0, 1, ..., P-1 in order, where
  P = scale_frames + sliding_window + 1.  Evicted and rolled-back pages are pushed on top.
* The special stream is paged in pages of ``SPECIAL_PAGE`` = 128 tokens; the visible
  special tokens are the committed ones plus the current frame's.
* The keep / drop decision may also be taken after the frame's attention ([KVBenefits]
  "Dynamic Keyframe Selection" decides from what the frame shows): the frame is appended
  undecided (``is_keyframe=None``) and ``finish(keep)`` commits or rolls it back.  Keeping
  it then needs room in the special stream; otherwise the frame stays pending.  The result
  is the state an up-front decision ``is_keyframe=keep`` would have given.
"""

from __future__ import annotations

from dataclasses import dataclass, field

SPECIAL_PAGE = 128


class SequenceError(Exception):
    """A call out of order: append twice, attend with nothing appended, frame not increasing."""


class CapacityError(Exception):
    """The special stream is full: max_frames keyframes were already committed."""


@dataclass
class Visible:
    """The key set one frame's attention sees, in visible-page-table order."""

    scale_pages: list
    window_pages: list
    current_page: int
    n_special: int              # visible special tokens: committed + the current frame's
    special_pages: int          # ceil(n_special / SPECIAL_PAGE)
    last_page_len: int          # valid tokens in the last special page

    @property
    def patch_pages(self) -> list:
        return list(self.scale_pages) + list(self.window_pages) + [self.current_page]


@dataclass
class PagedRetention:
    """The retention state machine of one cache (one layer)."""

    scale_frames: int
    sliding_window: int
    max_frames: int
    specials_per_frame: int = 6
    scale: list = field(default_factory=list)     # [(page, frame)] in commit order
    window: list = field(default_factory=list)    # [(page, frame)] oldest first
    free: list = field(default_factory=list)      # stack, top = end
    n_special: int = 0                            # committed special tokens
    committed: list = field(default_factory=list)  # committed keyframe ids, in order
    pending: tuple | None = None                  # (page, frame, is_keyframe)
    last_frame: int = -1

    def __post_init__(self):
        if self.scale_frames < 0 or self.sliding_window < 0 or self.max_frames < 1:
            raise ValueError("bad retention sizes")
        self.reset()

    @property
    def num_pages(self) -> int:
        return self.scale_frames + self.sliding_window + 1

    def reset(self) -> None:
        """A fresh cache ([KVBenefits] "Cross-Window Alignment": clean_kv_cache)."""
        self.scale = []
        self.window = []
        self.free = list(range(self.num_pages - 1, -1, -1))
        self.n_special = 0
        self.committed = []
        self.pending = None
        self.last_frame = -1

    def append(self, frame_idx: int, is_keyframe: bool | None) -> tuple[int, int]:
        """Tentatively place frame_idx: pop a patch page, reserve 6 special slots.

        ``is_keyframe=None`` leaves the keep / drop decision to ``finish(keep)``.
        Returns (patch page id, first special slot).
        """
        if self.pending is not None:
            raise SequenceError("append while a frame is pending")
        if frame_idx <= self.last_frame:
            raise SequenceError("frame_idx must increase")
        if is_keyframe and len(self.committed) >= self.max_frames:
            raise CapacityError("special stream full")
        page = self.free.pop()
        self.pending = (page, int(frame_idx), None if is_keyframe is None else bool(is_keyframe))
        self.last_frame = int(frame_idx)
        return page, self.n_special

    def visible(self) -> Visible:
        """The pending frame's key set: scale -> window (old to new) -> own page -> specials."""
        if self.pending is None:
            raise SequenceError("attend without append")
        n_sp = self.n_special + self.specials_per_frame
        pages = -(-n_sp // SPECIAL_PAGE)
        return Visible(
            scale_pages=[p for p, _ in self.scale],
            window_pages=[p for p, _ in self.window],
            current_page=self.pending[0],
            n_special=n_sp,
            special_pages=pages,
            last_page_len=n_sp - SPECIAL_PAGE * (pages - 1),
        )

    def finish(self, keep: bool | None = None) -> int | None:
        """After the pending frame's attention: commit a keyframe or roll back.

        Commit fills scale first, then the window; a window longer than sliding_window
        returns its oldest page to the free stack (deferred eviction).  Returns the evicted
        page, or None.  Roll-back returns the frame's page and drops its specials.  A frame
        appended undecided needs ``keep``; one decided at append must not get it.
        """
        if self.pending is None:
            raise SequenceError("finish without append")
        page, frame, key = self.pending
        if (key is None) == (keep is None):
            raise SequenceError("decide a frame exactly once: at append or at finish")
        if key is None:
            if keep and len(self.committed) >= self.max_frames:
                raise CapacityError("special stream full")
            key = bool(keep)
        self.pending = None
        evicted = None
        if key:
            if len(self.scale) < self.scale_frames:
                self.scale.append((page, frame))
            else:
                self.window.append((page, frame))
                if len(self.window) > self.sliding_window:
                    evicted, _ = self.window.pop(0)
                    self.free.append(evicted)
            self.n_special += self.specials_per_frame
            self.committed.append(frame)
        else:
            self.free.append(page)
        return evicted

    def retained_frames(self) -> list:
        """Frames whose patch pages are held, in scale -> window order."""
        return [f for _, f in self.scale] + [f for _, f in self.window]

    def snapshot(self) -> dict:
        return {
            "scale_pages": [p for p, _ in self.scale],
            "scale_frames": [f for _, f in self.scale],
            "window_pages": [p for p, _ in self.window],
            "window_frames": [f for _, f in self.window],
            "free": list(self.free),
            "n_special": self.n_special,
            "pending": self.pending,
            "last_frame": self.last_frame,
        }


def retained_closed_form(committed: list, scale_frames: int, sliding_window: int) -> list:
    """Retained keyframes after committing ``committed`` (in order), without replaying.

    All of them while there are at most scale_frames + sliding_window; afterwards the first
    scale_frames and the last sliding_window ones.
    """
    m = len(committed)
    if m <= scale_frames + sliding_window:
        return list(committed)
    tail = list(committed[m - sliding_window:]) if sliding_window > 0 else []
    return list(committed[:scale_frames]) + tail


def keyframe_schedule(n_frames: int, interval: int) -> list:
    """is_keyframe per frame for a fixed interval: frame f is a keyframe iff f % interval == 0.

    [KVBenefits] "Working with the KV Cache API" streams with keyframe_interval=5.
    """
    return [(f % interval) == 0 for f in range(n_frames)]
