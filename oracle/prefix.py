"""Reference prefix cache by hash chain, in plain Python (test infrastructure;
see oracle/__init__.py for who may import it).

"vLLM KV Cache 实现机制", section 4.2: a full block is keyed by a hash of
(parent block hash, the exact tokens of the block, an extra hash); a request
reuses the longest cached prefix of whole blocks.  Section 3.2: reference
counts protect shared blocks; eviction is least-recently-used among the
unreferenced.  The hash is FNV-1a 64 over little-endian bytes of (parent
hash as u64, each token as u32, extra hash as u64), first parent 0 -- the
choice this library documents.  Hits compare the stored tokens, parent and
extra hash, so colliding hashes never share a block.
"""
from __future__ import annotations

FNV_OFFSET = 14695981039346656037
FNV_PRIME = 1099511628211
MASK = (1 << 64) - 1


def fnv1a(data: bytes, h: int = FNV_OFFSET) -> int:
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & MASK
    return h


def block_hash(parent: int, tokens, extra: int) -> int:
    data = parent.to_bytes(8, "little")
    data += b"".join((int(t) & 0xFFFFFFFF).to_bytes(4, "little") for t in tokens)
    data += extra.to_bytes(8, "little")
    return fnv1a(data)


def block_hashes(tokens, block_size: int, parent: int = 0, extra: int = 0) -> list[int]:
    out = []
    h = parent
    for i in range(len(tokens) // block_size):
        h = block_hash(h, tokens[i * block_size:(i + 1) * block_size], extra)
        out.append(h)
    return out


class RefPrefixCache:
    def __init__(self, block_size: int, capacity: int):
        self.bs, self.capacity = block_size, capacity
        self.entries = {}      # hash -> [parent, extra, tokens tuple, block_id, refs]
        self.order = []        # hashes, least recently used first

    def _touch(self, h):
        self.order.remove(h)
        self.order.append(h)

    def _find(self, h, parent, toks, extra):
        e = self.entries.get(h)
        if e is None or e[0] != parent or e[1] != extra or e[2] != tuple(toks):
            return None
        return e

    def match(self, tokens, extra=0, max_blocks=None):
        n = len(tokens) // self.bs if max_blocks is None else min(max_blocks, len(tokens) // self.bs)
        ids, parent = [], 0
        for i in range(n):
            t = [int(x) for x in tokens[i * self.bs:(i + 1) * self.bs]]
            h = block_hash(parent, t, extra)
            e = self._find(h, parent, t, extra)
            if e is None:
                break
            e[4] += 1
            self._touch(h)
            ids.append(e[3])
            parent = h
        return ids

    def insert(self, tokens, block_ids, extra=0):
        hs = block_hashes(tokens, self.bs, 0, extra)[:len(block_ids)]
        fresh = sum(1 for h in hs if h not in self.entries)
        if len(self.entries) + fresh > self.capacity:
            return None  # full: nothing inserted
        parent, added = 0, 0
        for i, h in enumerate(hs):
            t = [int(x) for x in tokens[i * self.bs:(i + 1) * self.bs]]
            if h not in self.entries:
                self.entries[h] = [parent, extra, tuple(t), int(block_ids[i]), 1]
                self.order.append(h)
                added += 1
            else:
                e = self._find(h, parent, t, extra)
                if e is not None:
                    e[4] += 1
                    self._touch(h)
            parent = h
        return added

    def release(self, tokens, num_blocks, extra=0):
        parent, released = 0, 0
        for i in range(num_blocks):
            t = [int(x) for x in tokens[i * self.bs:(i + 1) * self.bs]]
            h = block_hash(parent, t, extra)
            e = self._find(h, parent, t, extra)
            if e is not None and e[4] > 0:
                e[4] -= 1
                released += 1
            parent = h
        return released

    def evict(self, max_evict):
        out = []
        for h in list(self.order):
            if len(out) >= max_evict:
                break
            if self.entries[h][4] == 0:
                out.append(self.entries[h][3])
                del self.entries[h]
                self.order.remove(h)
        return out

    def __len__(self):
        return len(self.entries)
