"""Block pool bookkeeping, plain Python (oracle; test infrastructure only).

Follows the page "Nano-vLLM-Ascend: lightweight LLM inference framework for
Ascend NPU", section 2.1 (PageAttention memory management):

* the KV cache is cut into blocks of ``block_size`` tokens (16 by default);
  a sequence of n tokens holds ceil(n / block_size) blocks, so its slots number
  ceil(n / block_size) * block_size (1000 tokens -> 63 blocks -> 1008 slots);
* a BlockTable maps each logical block of a sequence to a physical block;
* every block carries a reference count (shared prefix blocks count once per
  sequence that maps them; the same page's section 4.2 checks these counts to
  find leaks).

and the allocator role of BlockAllocator on the page "Ascend NPU LLM inference
optimisation: the vLLM-Ascend approach", section 2.1: one pool, handed out a
block at a time.  Block sharing across sequences is that page's section 4
("block sharing").

Policy (the pages do not state one; this reading is shared with the C++ pool):
the free list starts in ``free_order``; allocation pops from its head; a block
whose count drops to zero is appended to its tail; appending into a shared,
partly filled last block first copies it (copy-on-write) into a fresh block.
A token at logical position p sits in physical block table[p // bs], row
p % bs, whose slot number is table[p // bs] * bs + p % bs.
"""

from __future__ import annotations

from collections import deque


class PoolError(Exception):
    pass


class OutOfBlocks(PoolError):
    pass


def blocks_for(n_tokens: int, block_size: int) -> int:
    """ceil(n / block_size): the number of blocks a sequence of n tokens holds."""
    return -(-n_tokens // block_size)


class OraclePool:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise PoolError("bad pool size")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if free_order is None else [int(x) for x in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise PoolError("free_order must be a permutation of the block ids")
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.seqs: dict[int, dict] = {}   # seq_id -> {"blocks": [...], "len": n}

    # -- allocation ---------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        assert self.ref[b] == 0
        self.ref[b] = 1
        return b

    def alloc(self, seq_id: int, n_tokens: int) -> None:
        if seq_id in self.seqs or n_tokens < 0:
            raise PoolError("alloc: sequence exists or negative length")
        need = blocks_for(n_tokens, self.block_size)
        if need > len(self.free):
            raise OutOfBlocks("alloc")
        self.seqs[seq_id] = {"blocks": [self._take() for _ in range(need)], "len": n_tokens}

    def fork(self, parent: int, child: int, n_prefix: int) -> None:
        """The child maps the parent's first ceil(n_prefix/bs) blocks; each count goes up by one."""
        if parent not in self.seqs or child in self.seqs:
            raise PoolError("fork: unknown parent or existing child")
        p = self.seqs[parent]
        if n_prefix < 0 or n_prefix > p["len"]:
            raise PoolError("fork: prefix longer than parent")
        shared = p["blocks"][: blocks_for(n_prefix, self.block_size)]
        for b in shared:
            self.ref[b] += 1
        self.seqs[child] = {"blocks": list(shared), "len": n_prefix}

    def append(self, seq_id: int, n_tokens: int):
        """Extend a sequence by n tokens; returns (slots of the new tokens, copy-on-write (src, dst) pairs)."""
        if seq_id not in self.seqs or n_tokens < 0:
            raise PoolError("append: unknown sequence")
        s = self.seqs[seq_id]
        bs = self.block_size
        n0 = s["len"]
        cow = n_tokens > 0 and n0 % bs != 0 and self.ref[s["blocks"][-1]] > 1
        need = blocks_for(n0 + n_tokens, bs) - len(s["blocks"]) + (1 if cow else 0)
        if need > len(self.free):
            raise OutOfBlocks("append")
        pairs = []
        if cow:
            old = s["blocks"][-1]
            new = self._take()
            self.ref[old] -= 1
            s["blocks"][-1] = new
            pairs.append((old, new))
        slots = []
        for p in range(n0, n0 + n_tokens):
            if p % bs == 0:
                s["blocks"].append(self._take())
            slots.append(s["blocks"][p // bs] * bs + p % bs)
        s["len"] = n0 + n_tokens
        return slots, pairs

    def free_seq(self, seq_id: int) -> None:
        if seq_id not in self.seqs:
            raise PoolError("free: unknown sequence")
        for b in self.seqs.pop(seq_id)["blocks"]:
            self.ref[b] -= 1
            assert self.ref[b] >= 0
            if self.ref[b] == 0:
                self.free.append(b)

    # -- export ---------------------------------------------------------------
    def block_table(self, seq_ids, max_blocks: int):
        """Rows of physical block ids (padded with -1) and the context length of each sequence."""
        rows, lens = [], []
        for sid in seq_ids:
            s = self.seqs[sid]
            if len(s["blocks"]) > max_blocks:
                raise PoolError("block table row too short")
            rows.append(s["blocks"] + [-1] * (max_blocks - len(s["blocks"])))
            lens.append(s["len"])
        return rows, lens

    def stats(self) -> dict:
        used = sum(1 for r in self.ref if r > 0)
        tokens = sum(s["len"] for s in self.seqs.values())
        held = sum(len(s["blocks"]) for s in self.seqs.values())
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": len(self.free),
            "used_blocks": used,
            "shared_blocks": sum(1 for r in self.ref if r > 1),
            "num_seqs": len(self.seqs),
            "tokens": tokens,
            "table_refs": held,
            "ref_sum": sum(self.ref),
            # tokens stored / slots the sequences hold (per sequence, shared blocks counted per holder)
            "utilisation": (tokens / (held * self.block_size)) if held else 1.0,
        }


def replay(wl_ops, num_blocks: int, block_size: int, free_order, batch: int):
    """Run a workload's pool script on an oracle pool.

    Returns (pool, block_tables [batch][max_blocks] with -1 padding, context_lens,
    slot_mapping of the tokens written this step in script order, copy-on-write pairs).
    """
    pool = OraclePool(num_blocks, block_size, free_order)
    slot_mapping, cow_pairs = [], []
    for op in wl_ops:
        if op[0] == "alloc":
            pool.alloc(op[1], op[2])
        elif op[0] == "fork":
            pool.fork(op[1], op[2], op[3])
        elif op[0] in ("append", "append_new"):
            slots, pairs = pool.append(op[1], op[2])
            cow_pairs += pairs
            if op[0] == "append_new":
                slot_mapping += slots
        else:
            raise PoolError(op[0])
    ids = list(range(batch))
    max_blocks = max([len(pool.seqs[i]["blocks"]) for i in ids] + [1])
    rows, lens = pool.block_table(ids, max_blocks)
    return pool, rows, lens, slot_mapping, cow_pairs
