"""Page pool and prefix index, modelled the plain way -- TEST INFRASTRUCTURE ONLY.

The rules restated here (page titles behind the tags: see the package docstring):

* Physical blocks form a pool; a sequence gets blocks on demand and returns
  them when it finishes ([HB-07] Q028; [CN-06] 6.5 allocation flow; [KV-03]
  "一个请求的 KV Cache 怎样产生和消失").
* A block shared by several sequences carries a reference count and is not
  reclaimed while any user remains ([KV-04] "深入：引擎怎样找状态"; [HB-07]
  Q028 shared-prefix paragraph).
* Readings where the pages are silent: the free list is FIFO, initialised
  from a given order; alloc pops from the head and is all-or-nothing; a block
  whose count reaches 0 is pushed to the tail.
* Prefix reuse: a full block can be reused by a new request only when the
  whole token prefix up to and including that block is identical (same
  identity salt); the first difference stops the match even if later tokens
  agree again ([KV-04] prefix demo; [CN-06] 6.4). Partial blocks are never
  matched. Here that rule is modelled by brute force: a dict keyed by the
  full prefix tuple -- no hashing at all.
* A registered block whose count drops to 0 stays matchable while it sits in
  the free list; incref revives it. When alloc hands it out again it is
  unregistered, together with every longer prefix registered through it.
* Registering a prefix that is already registered keeps the first block.
"""
from __future__ import annotations

from collections import deque
from typing import Dict, List, Optional, Sequence, Tuple

# Error names shared in meaning (not in code) with the C ABI's status codes.
OOM = "OOM"
BAD_ID = "BAD_ID"
DOUBLE_FREE = "DOUBLE_FREE"
ARG = "ARG"
SHARED_TAIL = "SHARED_TAIL"


class PoolError(Exception):
    def __init__(self, kind: str):
        super().__init__(kind)
        self.kind = kind


class PoolModel:
    def __init__(self, num_pages: int, page_size: int, init_order: Optional[Sequence[int]] = None):
        if num_pages <= 0 or page_size <= 0:
            raise PoolError(ARG)
        order = list(range(num_pages)) if init_order is None else [int(x) for x in init_order]
        if sorted(order) != list(range(num_pages)):
            raise PoolError(ARG)
        self.num_pages = num_pages
        self.page_size = page_size
        self.free = deque(order)
        self.ref = [0] * num_pages
        self.indexes: List["PrefixModel"] = []

    # -- pool --------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def alloc(self, n: int) -> List[int]:
        if n < 0:
            raise PoolError(ARG)
        if n > len(self.free):
            raise PoolError(OOM)
        ids = [self.free.popleft() for _ in range(n)]
        for p in ids:
            self.ref[p] = 1
            for ix in self.indexes:
                ix.evict(p)
        return ids

    def _check_ids(self, ids: Sequence[int]) -> None:
        for p in ids:
            if not (0 <= int(p) < self.num_pages):
                raise PoolError(BAD_ID)

    def free_pages(self, ids: Sequence[int]) -> None:
        self._check_ids(ids)
        need: Dict[int, int] = {}
        for p in ids:
            need[int(p)] = need.get(int(p), 0) + 1
        for p, c in need.items():
            if c > self.ref[p]:
                raise PoolError(DOUBLE_FREE)
        for p in ids:
            p = int(p)
            self.ref[p] -= 1
            if self.ref[p] == 0:
                self.free.append(p)

    def incref(self, ids: Sequence[int]) -> None:
        self._check_ids(ids)
        for p in ids:
            if self.ref[int(p)] == 0 and not any(ix.is_registered(int(p)) for ix in self.indexes):
                raise PoolError(BAD_ID)
        for p in ids:
            p = int(p)
            if self.ref[p] == 0:
                self.free.remove(p)
            self.ref[p] += 1

    def refcount(self, p: int) -> int:
        self._check_ids([p])
        return self.ref[p]

    # -- per-step slot computation ([HB-07] Q028 block-size-4 example) -----
    def append_slots(self, tables: List[List[int]], max_blocks: int, lens: List[int]) -> List[int]:
        """For each sequence, the slot of the token appended at position lens[b].

        A new block is allocated first when lens[b] % P == 0 (all blocks of the
        step together, all-or-nothing, in sequence order). Appending into a
        block that another sequence also holds needs copy-on-write first
        ([HB-07] Q028, step 6 of the table) -> SHARED_TAIL. Updates the table
        rows and lens in place.
        """
        P = self.page_size
        need = [b for b, L in enumerate(lens) if L % P == 0]
        for b, L in enumerate(lens):
            if L // P >= max_blocks:
                raise PoolError(ARG)
            if L % P != 0 and self.ref[int(tables[b][L // P])] > 1:
                raise PoolError(SHARED_TAIL)
        new = self.alloc(len(need))
        for b, p in zip(need, new):
            tables[b][lens[b] // P] = p
        slots = []
        for b in range(len(lens)):
            L = lens[b]
            slots.append(int(tables[b][L // P]) * P + L % P)
            lens[b] = L + 1
        return slots


    # -- copy-on-write of shared partial tails ([HB-07] Q028 step 6; [CN-06] 6.5) ----
    def cow_tails(self, tables: List[List[int]], max_blocks: int, lens: List[int]) -> List[Tuple[int, int]]:
        """Give a sequence whose next append lands in a partial page that is
        still shared a private copy of that page.

        Sequences are taken in order; sequence b gets a copy when its tail
        page (lens[b] % P != 0) has refcount > 1 at that moment: a fresh page
        replaces the tail in its table row, one reference to the old page is
        dropped, and (old, new) is reported -- the caller copies the contents.
        The last holder keeps the original. All fresh pages are allocated
        together, all-or-nothing (a first pass counts them).
        """
        P = self.page_size
        sim = {}
        marked = []
        for b, L in enumerate(lens):
            if L < 0 or L // P >= max_blocks:
                raise PoolError(ARG)
            if L % P != 0:
                t = int(tables[b][L // P])
                if not (0 <= t < self.num_pages):
                    raise PoolError(BAD_ID)
                r = sim.get(t, self.ref[t])
                if r > 1:
                    marked.append(b)
                    sim[t] = r - 1
        fresh = self.alloc(len(marked))
        pairs = []
        for b, new in zip(marked, fresh):
            L = lens[b]
            old = int(tables[b][L // P])
            tables[b][L // P] = new
            self.free_pages([old])
            pairs.append((old, new))
        return pairs


class PrefixModel:
    """Brute-force prefix index: full token prefix (with salt) -> block id."""

    def __init__(self, page_size: int, salt: int = 0):
        self.P = page_size
        self.salt = int(salt)
        self.entries: Dict[Tuple[int, ...], int] = {}
        self.key_of_page: Dict[int, Tuple[int, ...]] = {}
        self.pool: Optional[PoolModel] = None

    def _key(self, tokens: Sequence[int], nblocks: int) -> Tuple[int, ...]:
        return (self.salt,) + tuple(int(t) for t in tokens[: nblocks * self.P])

    def is_registered(self, p: int) -> bool:
        return p in self.key_of_page

    def register(self, pool: PoolModel, tokens: Sequence[int], page_ids: Sequence[int]) -> None:
        if pool.page_size != self.P:
            raise PoolError(ARG)
        if self.pool is not None and self.pool is not pool:
            raise PoolError(ARG)
        nfull = len(tokens) // self.P
        if len(page_ids) < nfull:
            raise PoolError(ARG)
        pool._check_ids(page_ids[:nfull])
        for i in range(nfull):
            p = int(page_ids[i])
            if pool.ref[p] == 0:
                raise PoolError(BAD_ID)
            k = self._key(tokens, i + 1)
            if p in self.key_of_page and self.key_of_page[p] != k:
                raise PoolError(ARG)
        if self.pool is None:
            self.pool = pool
            pool.indexes.append(self)
        for i in range(nfull):
            k = self._key(tokens, i + 1)
            if k in self.entries:
                continue
            p = int(page_ids[i])
            self.entries[k] = p
            self.key_of_page[p] = k

    def match(self, tokens: Sequence[int]) -> List[int]:
        out = []
        for i in range(len(tokens) // self.P):
            p = self.entries.get(self._key(tokens, i + 1))
            if p is None:
                break
            out.append(p)
        return out

    def evict(self, p: int) -> None:
        k = self.key_of_page.pop(p, None)
        if k is None:
            return
        for key in [key for key in self.entries if len(key) >= len(k) and key[: len(k)] == k]:
            q = self.entries.pop(key)
            self.key_of_page.pop(q, None)

    def detach(self) -> None:
        if self.pool is not None:
            self.pool.indexes.remove(self)
            self.pool = None
