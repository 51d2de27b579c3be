"""Plain model of the paged KV block manager (oracle; test infrastructure only).

What the pages fix:

* Physical blocks come from a free list; taking a block sets its reference count
  to 1, and a freed block goes back to the free list ("vLLM PagedAttention and
  continuous batching", section 4: the block allocator hands out the first free
  block and returns freed blocks to the end of the list).
* Blocks are taken on demand: a sequence holds ceil(tokens / B) blocks, and a new
  block is taken only when the current last block is full ("LLM Inference 8 -
  PagedAttention", section "PagedAttention의 동작 방식"; the blog's section 4,
  needed = ceil(total / block_size)).
* Sequences forked from one prompt (parallel samples, beams) share its physical
  blocks through reference counts; when one of them writes into a shared block,
  only that block is copied (copy-on-write, P3 -> P9 in the digest's framework
  flowchart; the blog's section 2).
* A preempted sequence's blocks can be moved to host memory and back ("PagedAttention
  - Efficient Memory Management for LLM Serving with vLLM", section "Method",
  scheduling: swapping to host RAM).

Readings where the pages are silent:

* Writes happen at a sequence's next position only (decode appends), so a
  copy-on-write can only hit the last block.
* A batch of appends either succeeds as a whole or changes nothing (not enough
  free blocks: error, no change).
* Swapping out copies every block of the sequence (shared ones included) to a
  host buffer in logical order and releases the device references; swapping in
  takes fresh blocks for them, in logical order.
"""

from collections import OrderedDict


class BlockManagerError(Exception):
    pass


class BlockManager:
    def __init__(self, num_blocks, block_size, free_order=None):
        self.B = int(block_size)
        self.free = list(range(num_blocks)) if free_order is None else list(free_order)
        self.ref = [0] * num_blocks
        self.seqs = OrderedDict()      # seq id -> {"tokens": n, "table": [blocks]}
        self.swapped = {}              # seq id -> {"tokens": n, "blocks": count}

    # -- allocator ----------------------------------------------------------
    def _take(self):
        if not self.free:
            raise BlockManagerError("no free block")
        b = self.free.pop(0)
        self.ref[b] = 1
        return b

    def _release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def num_free(self):
        return len(self.free)

    # -- sequences ------------------------------------------------------------
    def add_sequence(self, seq, num_tokens):
        if seq in self.seqs or seq in self.swapped:
            raise BlockManagerError("sequence exists")
        need = -(-num_tokens // self.B)
        if need > len(self.free):
            raise BlockManagerError("no free block")
        self.seqs[seq] = {"tokens": num_tokens, "table": [self._take() for _ in range(need)]}

    def fork(self, parent, child):
        if parent not in self.seqs or child in self.seqs or child in self.swapped:
            raise BlockManagerError("bad fork")
        p = self.seqs[parent]
        for b in p["table"]:
            self.ref[b] += 1
        self.seqs[child] = {"tokens": p["tokens"], "table": list(p["table"])}

    def _batch_needs(self, seqs):
        """Free blocks a batch of appends takes, counted by playing the batch out on
        reference counts alone: a sequence whose last block is full takes a new one;
        a write into a last block that still has another holder copies it and drops
        one holder, so the last of several writers of one block writes in place."""
        ref = list(self.ref)
        need = 0
        for q in seqs:
            s = self.seqs[q]
            j = s["tokens"] // self.B
            if j == len(s["table"]):
                need += 1
            elif ref[s["table"][j]] > 1:
                ref[s["table"][j]] -= 1
                need += 1
        return need

    def append_tokens(self, seqs):
        """One new token for each listed sequence: returns (slots, cow_pairs)."""
        for q in seqs:
            if q not in self.seqs:
                raise BlockManagerError("unknown sequence")
        if len(set(seqs)) != len(seqs):
            raise BlockManagerError("repeated sequence")
        if self._batch_needs(seqs) > len(self.free):
            raise BlockManagerError("no free block")
        slots, pairs = [], []
        for q in seqs:
            s = self.seqs[q]
            pos = s["tokens"]
            j = pos // self.B
            if j == len(s["table"]):
                s["table"].append(self._take())
            elif self.ref[s["table"][j]] > 1:
                old = s["table"][j]
                new = self._take()
                self._release(old)
                s["table"][j] = new
                pairs.append((old, new))
            slots.append(s["table"][j] * self.B + pos % self.B)
            s["tokens"] = pos + 1
        return slots, pairs

    def free_sequence(self, seq):
        if seq in self.swapped:
            del self.swapped[seq]
            return
        if seq not in self.seqs:
            raise BlockManagerError("unknown sequence")
        for b in self.seqs.pop(seq)["table"]:
            self._release(b)

    def block_table(self, seq):
        s = self.seqs[seq]
        return list(s["table"]), s["tokens"]

    # -- swapping ------------------------------------------------------------
    def swap_out(self, seq):
        """Returns the device blocks to copy to host slots 0..n-1, then releases them."""
        if seq not in self.seqs:
            raise BlockManagerError("unknown sequence")
        s = self.seqs.pop(seq)
        blocks = list(s["table"])
        for b in blocks:
            self._release(b)
        self.swapped[seq] = {"tokens": s["tokens"], "blocks": len(blocks)}
        return blocks

    def swap_in(self, seq):
        """Takes fresh blocks for a swapped sequence: host slot i goes to returned block i."""
        if seq not in self.swapped:
            raise BlockManagerError("unknown sequence")
        n = self.swapped[seq]["blocks"]
        if n > len(self.free):
            raise BlockManagerError("no free block")
        info = self.swapped.pop(seq)
        blocks = [self._take() for _ in range(n)]
        self.seqs[seq] = {"tokens": info["tokens"], "table": blocks}
        return blocks
