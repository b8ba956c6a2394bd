"""A model checker for the asynchronous pipelines inside one CTA of the tensor-core kernels (CPU only).

compute-sanitizer is not available, so the producer/consumer protocols of the tcgen05 kernels (mbarriers, TMA
copies, tensor-core ops and their commits, TMEM and shared-memory buffers) are checked here as models.  A
model lists, per warp role, the operations that role performs in program order:

    ("wait", bar, k)            wait for completion number k of mbarrier `bar` (parity k & 1)
    ("arrive", bar, n)          n arrivals
    ("arrive_tx", bar, n, tx)   n arrivals and tx expected transaction units
    ("tma", bar, tx, writes)    an asynchronous copy; on completion it writes `writes` and completes tx on bar
    ("mma", reads, writes, lbl) a tensor-core op; one role's ops run in its issue order, each at some later time
    ("commit", bar)             one arrival on bar once every earlier tensor-core op of the same role has run
    ("read", buf, tag)          a synchronous read (ld.shared, tcgen05.ld + wait) expecting content `tag`
    ("write", buf, tag)         a synchronous write (st.shared, tcgen05.st + wait)
    ("nbar", id, n)             a named barrier over n roles

`reads` / `writes` are lists of (buffer, tag); a tag names the data a buffer must hold (for example
("S", 3): the scores of pipeline step 3).  The scheduler interleaves the roles and the asynchronous
completions at random, with per-run skewed speeds so that some runs starve a role or the asynchronous units
for long stretches.  The tensor-core ops of different roles (two issuing threads) run in no fixed order
relative to each other.  It reports:

* a deadlock (no role can move and nothing asynchronous is pending);
* a wait that returns on another phase than the one it means (the barrier ran two phases ahead of the waiter,
  or the waiter is two phases ahead of the barrier);
* a buffer read while a write to it is pending, or read holding other data than the reader expects;
* a buffer overwritten while a tensor-core read or a copy into it is pending;
* the CTA ending (every role done: TMEM freed, shared memory released) while a tensor-core op, a commit or a
  copy is still in flight.
"""
from __future__ import annotations

import random


class ProtocolError(Exception):
    pass


class _Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.arrived = 0
        self.tx = 0
        self.completed = 0

    def maybe_complete(self):
        if self.arrived == self.count and self.tx == 0:
            self.completed += 1
            self.arrived = 0


class _Buf:
    def __init__(self):
        self.content = None
        self.pending_writes = 0  # tensor-core ops or copies that will write it
        self.pending_copies = 0  # the copies among them
        self.pending_reads = 0  # tensor-core ops that will read it


class PipelineModel:
    def __init__(self, seed: int):
        self.rng = random.Random(seed)
        self.bars: dict[str, _Bar] = {}
        self.bufs: dict[str, _Buf] = {}
        self.roles: dict[str, dict] = {}
        self.copies: list = []
        self.tc_queues: dict[str, list] = {}  # per issuing role, in its program order
        self.named: dict = {}
        self.released: dict = {}

    def bar(self, name: str, count: int) -> None:
        self.bars[name] = _Bar(name, count)

    def role(self, name: str, ops) -> None:
        self.roles[name] = {"gen": iter(ops), "op": None, "done": False}

    def _buf(self, name):
        if name not in self.bufs:
            self.bufs[name] = _Buf()
        return self.bufs[name]

    # ---- synchronous operations of a role ----
    def _ready(self, who, op):
        if op[0] != "wait":
            return True
        b = self.bars[op[1]]
        k = op[2]
        ready = (b.completed & 1) != (k & 1)
        if ready and b.completed != k + 1:
            raise ProtocolError(f"{who}: wait on {b.name} for phase {k} returned with {b.completed} phases done")
        return ready

    def _do(self, who, op):
        kind = op[0]
        if kind == "wait":
            return
        if kind in ("arrive", "arrive_tx"):
            b = self.bars[op[1]]
            if kind == "arrive_tx":
                b.tx += op[3]
            b.arrived += op[2]
            if b.arrived > b.count:
                raise ProtocolError(f"{who}: more arrivals on {b.name} than its count")
            b.maybe_complete()
        elif kind == "tma":
            for name, _ in op[3]:
                buf = self._buf(name)
                if buf.pending_reads:
                    raise ProtocolError(f"{who}: copy into {name} while a tensor-core read of it is pending")
                buf.pending_writes += 1
                buf.pending_copies += 1
            self.copies.append((op[1], op[2], op[3]))
        elif kind == "mma":
            for name, _ in op[1]:
                self._buf(name).pending_reads += 1
            for name, _ in op[2]:
                self._buf(name).pending_writes += 1
            self.tc_queues.setdefault(who, []).append(op)
        elif kind == "commit":
            self.tc_queues.setdefault(who, []).append(op)
        elif kind == "read":
            buf = self._buf(op[1])
            if buf.pending_writes:
                raise ProtocolError(f"{who}: read of {op[1]} while a write to it is pending")
            if buf.content != op[2]:
                raise ProtocolError(f"{who}: read of {op[1]} expected {op[2]}, found {buf.content}")
        elif kind == "write":
            buf = self._buf(op[1])
            if buf.pending_writes or buf.pending_reads:
                raise ProtocolError(f"{who}: write of {op[1]} ({op[2]}) while {buf.pending_writes} writes and "
                                    f"{buf.pending_reads} tensor-core reads are pending")
            buf.content = op[2]
        else:
            raise ProtocolError(f"{who}: unknown operation {op}")

    # ---- asynchronous completions ----
    def _complete_one(self):
        busy = [q for q in self.tc_queues.values() if q]
        kinds = (["copy"] if self.copies else []) + (["tc"] if busy else [])
        kind = self.rng.choice(kinds)
        if len(kinds) == 2 and self.rng.random() < 0.5:
            kind = self.prefer
        if kind == "copy":
            bar, tx, writes = self.copies.pop(self.rng.randrange(len(self.copies)))
            for name, tag in writes:
                buf = self._buf(name)
                buf.pending_writes -= 1
                buf.pending_copies -= 1
                buf.content = tag
            b = self.bars[bar]
            b.tx -= tx
            if b.tx < 0:
                raise ProtocolError(f"more transaction units completed on {bar} than expected")
            b.maybe_complete()
            return
        op = self.rng.choice(busy).pop(0)
        if op[0] == "commit":
            b = self.bars[op[1]]
            b.arrived += 1
            if b.arrived > b.count:
                raise ProtocolError(f"more commit arrivals on {b.name} than its count")
            b.maybe_complete()
            return
        for name, tag in op[1]:
            buf = self._buf(name)
            if buf.pending_copies:
                raise ProtocolError(f"tensor-core op {op[3]} reads {name} while a copy into it is pending")
            if tag is not None and buf.content != tag:
                raise ProtocolError(f"tensor-core op {op[3]} reads {name}: expected {tag}, found {buf.content}")
            buf.pending_reads -= 1
        for name, tag in op[2]:
            buf = self._buf(name)
            buf.pending_writes -= 1
            buf.content = tag

    def run(self, max_steps: int = 5_000_000) -> None:
        speed = {n: self.rng.choice([0.01, 0.1, 1.0, 1.0, 4.0]) for n in self.roles}
        p_async = self.rng.choice([0.01, 0.05, 0.3, 0.8])
        self.prefer = self.rng.choice(["copy", "tc"])
        for st in self.roles.values():
            st["op"] = next(st["gen"], None)
            st["done"] = st["op"] is None
        for _ in range(max_steps):
            if all(st["done"] for st in self.roles.values()) and (self.copies or any(self.tc_queues.values())):
                inflight = {n: len(q) for n, q in self.tc_queues.items() if q}
                raise ProtocolError(f"the CTA ends with tensor-core ops {inflight} and {len(self.copies)} copies in "
                                    "flight")
            runnable = []
            for name, st in self.roles.items():
                if st["done"]:
                    continue
                op = st["op"]
                if op[0] == "nbar":
                    rel = self.released.setdefault(op[1], set())
                    if name not in rel:
                        waiting = self.named.setdefault(op[1], set())
                        waiting.add(name)
                        if len(waiting) >= op[2]:
                            rel.update(waiting)
                            waiting.clear()
                    if name in rel:
                        runnable.append(name)
                elif self._ready(name, op):
                    runnable.append(name)
            pending = bool(self.copies) or any(self.tc_queues.values())
            if not runnable and not pending:
                if all(st["done"] for st in self.roles.values()):
                    return
                blocked = {n: st["op"] for n, st in self.roles.items() if not st["done"]}
                raise ProtocolError(f"deadlock: {blocked}")
            if pending and (not runnable or self.rng.random() < p_async):
                self._complete_one()
                continue
            name = self.rng.choices(runnable, weights=[speed[n] for n in runnable])[0]
            st = self.roles[name]
            op = st["op"]
            if op[0] == "nbar":
                self.released[op[1]].discard(name)
            else:
                self._do(name, op)
            st["op"] = next(st["gen"], None)
            st["done"] = st["op"] is None
        raise ProtocolError("step limit")
