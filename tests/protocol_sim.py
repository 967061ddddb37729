"""A small scheduler for CPU models of the kernels' mbarrier protocols.

A model lists its roles as generators of operations in a kernel's program
order:

  ("wait", barrier, n)          block until the barrier's n-th phase has
                                completed (the hardware's parity test; passing
                                on any other phase is reported as aliasing)
  ("arrive", barrier, k, phase) k arrivals, which must belong to `phase`
  ("tma", barrier, phase, bufs) arrive.expect_tx + one copy per (buffer,
                                version); copies land later, in any order
  ("pipe", op)                  issue a tensor-pipe operation (an MMA, a
                                tcgen05.cp, or ("commit", barrier)); the pipe
                                executes them later, in issue order
  anything else                 a local action, handed to `local_op`

and the scheduler runs them under a seeded random schedule.  Shared-memory
buffers are versioned: a copy may only land once every issued reader of the
buffer's previous version has run (`pipe_readers` names the buffers a pipe
operation reads; `tensor_op` checks them with `read_smem`).
"""
import random


class Hazard(AssertionError):
    pass


class Bar:
    """mbarrier: `count` arrivals and all expected copies complete a phase."""

    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.done = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self, n, tag):
        if tag != self.done:
            raise Hazard(f"{self.name}: arrival for phase {tag} while phase {self.done} is open")
        if n > self.pending:
            raise Hazard(f"{self.name}: {n} arrivals with {self.pending} pending")
        self.pending -= n
        self._maybe_complete()

    def expect_tx(self, copies, tag):
        self.tx += copies
        self.arrive(1, tag)

    def land(self):
        self.tx -= 1
        self._maybe_complete()

    def passes(self, target):
        # the hardware's parity test for "completion number `target` has happened"
        return (self.done & 1) == (target & 1)


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.B = {}
        self.pipe, self.copies = [], []
        self.smem, self.readers = {}, {}

    def bar(self, name, count=1):
        self.B[name] = Bar(name, count)

    def read_smem(self, buf, version):
        self.readers[buf] -= 1
        if self.smem.get(buf) != version:
            raise Hazard(f"read of {buf} expected {version}, holds {self.smem.get(buf)}")

    # to be provided by a model
    def roles(self):
        raise NotImplementedError

    def pipe_readers(self, op):
        return ()

    def tensor_op(self, op):
        raise NotImplementedError

    def local_op(self, role, op):
        raise NotImplementedError

    def _commit(self, name):
        b = self.B[name]
        b.arrive(1, b.done)

    def run(self, max_steps=5_000_000):
        roles = self.roles()
        cur = {k: next(g, None) for k, g in roles.items()}
        for _ in range(max_steps):
            runnable = [k for k, op in cur.items()
                        if op is not None and (op[0] != "wait" or self.B[op[1]].passes(op[2]))]
            if self.pipe:
                runnable.append("pipe")
            if self.copies:
                runnable.append("tma")
            if not runnable:
                blocked = {k: v for k, v in cur.items() if v is not None}
                if blocked:
                    raise Hazard(f"deadlock: {blocked}")
                return
            k = self.rng.choice(runnable)
            if k == "pipe":
                op = self.pipe.pop(0)
                if op[0] == "commit":
                    self._commit(op[1])
                else:
                    self.tensor_op(op)
                continue
            if k == "tma":  # copies land in any order
                buf, version, name = self.copies.pop(self.rng.randrange(len(self.copies)))
                if self.readers.get(buf, 0):
                    raise Hazard(f"copy into {buf} lands while {self.readers[buf]} issued readers have not run")
                self.smem[buf] = version
                self.B[name].land()
                continue
            op = cur[k]
            if op[0] == "wait":
                if self.B[op[1]].done != op[2]:
                    raise Hazard(f"{k}: wait for completion {op[2]} of {op[1]} passed at {self.B[op[1]].done}")
            elif op[0] == "arrive":
                self.B[op[1]].arrive(op[2], op[3])
            elif op[0] == "tma":
                _, name, tag, bufs = op
                self.B[name].expect_tx(len(bufs), tag)
                self.copies.extend((buf, version, name) for buf, version in bufs)
            elif op[0] == "pipe":
                for buf in self.pipe_readers(op[1]):
                    self.readers[buf] = self.readers.get(buf, 0) + 1
                self.pipe.append(op[1])
            else:
                self.local_op(k, op)
            cur[k] = next(roles[k], None)
        raise AssertionError("model did not finish")
