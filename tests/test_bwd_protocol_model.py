"""CPU models of the backward kernels' synchronisation protocols.

`attn_bwd_dkdv_kernel` and `attn_bwd_dq_kernel` (csrc/attn_bwd.cu) each run a
TMA producer warp, a single MMA-issuing thread, the in-order tensor pipe and
two elementwise warpgroups that split the columns of a tile.  These models
replay each role's waits, arrivals, copies and tensor-pipe operations in the
kernels' program order under random schedules (see tests/protocol_sim.py) and
check for deadlock, mbarrier phase aliasing and tensor/shared-memory hazards:

  dkdv  S^T and dP^T in two TMEM buffers (64 columns each); P^T and dS^T are
        written back over their first 32 columns, each warpgroup 16 of them,
        after both warpgroups have read their halves (named barrier); dV and
        dK accumulate; the next-but-one tile's products reuse the buffer.
  dq    S and dP (128 columns) are overwritten by the next tile's products as
        soon as both warpgroups have loaded them (s_free); dS is stored by the
        warpgroups once the previous dQ product has read it (ds_free).

Planted mistakes must be caught.
"""
import pytest

from tests.protocol_sim import Hazard, Sim

KV_STAGES = 4


class DkDv(Sim):
    """One CTA: a resident K/V key tile, nq 64-row query tiles streaming."""

    def __init__(self, nq, seed, plant=None):
        super().__init__(seed)
        self.nq, self.plant = nq, plant
        self.bar("a_full"), self.bar("done")
        for s in range(KV_STAGES):
            self.bar(("full", s)), self.bar(("empty", s))
        for b in range(2):
            self.bar(("sbuf", b))
        self.bar("ds_full", 256)
        self.bar("pair", 8)  # the named barrier between the two warpgroups (8 warps)
        # chunk c = columns [16c, 16c + 16) of buffer b: ("S", u) / ("P", u) for S^T, ("dP", u) / ("dS", u) for dP^T
        self.st = [[None] * 4 for _ in range(2)]
        self.dpt = [[None] * 4 for _ in range(2)]
        self.loaded = {}         # (buffer, u) -> warpgroups that loaded their half
        self.consumed = set()    # (buffer, u) whose P^T / dS^T the dV / dK products read
        self.acc = None          # last query tile accumulated into dV and dK

    def roles(self):
        r = {"producer": self.producer(), "mma": self.mma()}
        for wg in range(2):
            for w in range(4):
                r[("ew", wg, w)] = self.elementwise(wg, w)
        return r

    def producer(self):
        yield ("tma", "a_full", 0, [(("kv",), 0)])
        for u in range(self.nq):
            s = u % KV_STAGES
            yield ("wait", ("empty", s), u // KV_STAGES)
            yield ("tma", ("full", s), u // KV_STAGES, [(("st", s, c), u) for c in ("q", "do", "l")])

    def mma(self):
        yield ("wait", "a_full", 1)
        for u in range(min(2, self.nq)):
            yield ("wait", ("full", u), 1)
            yield ("pipe", ("sdp", u))
            yield ("pipe", ("commit", ("sbuf", u & 1)))
        for u in range(self.nq):
            s = u % KV_STAGES
            nxt = u + 2 < self.nq
            if nxt and self.plant == "early_sdp":
                yield ("wait", ("full", (u + 2) % KV_STAGES), (u + 2) // KV_STAGES + 1)
                yield ("pipe", ("sdp", u + 2))
                yield ("pipe", ("commit", ("sbuf", u & 1)))
            yield ("wait", "ds_full", u + 1)
            yield ("pipe", ("dvdk", u))
            yield ("pipe", ("commit", ("empty", s)))
            if nxt and self.plant != "early_sdp":
                yield ("wait", ("full", (u + 2) % KV_STAGES), (u + 2) // KV_STAGES + 1)
                yield ("pipe", ("sdp", u + 2))
                yield ("pipe", ("commit", ("sbuf", u & 1)))
        yield ("pipe", ("commit", "done"))

    def elementwise(self, wg, w):
        for u in range(self.nq):
            s, b = u % KV_STAGES, u & 1
            yield ("wait", ("full", s), u // KV_STAGES + 1)
            yield ("read_l", s, u)  # -lse, -delta and the validity words of the stage
            yield ("wait", ("sbuf", b), (u >> 1) + 1)
            yield ("load", wg, w, u)
            if self.plant != "no_pair_sync":
                yield ("arrive", "pair", 1, u)
                yield ("wait", "pair", u + 1)
            yield ("store", wg, w, u)
            yield ("arrive", "ds_full", 32, u)
        yield ("wait", "done", 1)
        yield ("epilogue", wg)

    def pipe_readers(self, op):
        if op[0] not in ("sdp", "dvdk"):
            return ()
        s = op[1] % KV_STAGES
        if op[0] == "sdp":
            return [("kv",), ("st", s, "q"), ("st", s, "do")]
        if op[0] == "dvdk":
            return [("st", s, "q"), ("st", s, "do")]
        return ()

    def tensor_op(self, op):
        kind, u = op
        s, b = u % KV_STAGES, u & 1
        if kind == "sdp":
            self.read_smem(("kv",), 0)
            self.read_smem(("st", s, "q"), u)
            self.read_smem(("st", s, "do"), u)
            for buf, cols in ((self.st, "S"), (self.dpt, "dP")):
                for c in range(4):
                    old = buf[b][c]
                    if old is None:
                        continue
                    v = old[1]
                    if old[0] in ("S", "dP") and len(self.loaded.get((b, v), ())) < 8:
                        raise Hazard(f"S^T/dP^T of tile {u} overwrite tile {v} before it was loaded")
                    if old[0] in ("P", "dS") and (b, v) not in self.consumed:
                        raise Hazard(f"S^T/dP^T of tile {u} overwrite P^T/dS^T of tile {v} before dV/dK read them")
                    buf[b][c] = None
                buf[b][:] = [(cols, u)] * 4
        elif kind == "dvdk":
            self.read_smem(("st", s, "q"), u)
            self.read_smem(("st", s, "do"), u)
            if self.st[b][:2] != [("P", u)] * 2 or self.dpt[b][:2] != [("dS", u)] * 2:
                raise Hazard(f"dV/dK of tile {u} read {self.st[b][:2]} / {self.dpt[b][:2]}")
            if self.acc != (None if u == 0 else u - 1):
                raise Hazard(f"dV/dK of tile {u} accumulate onto tile {self.acc}")
            self.consumed.add((b, u))
            self.acc = u
        else:
            raise AssertionError(op)

    def local_op(self, role, op):
        kind = op[0]
        if kind == "read_l":
            _, s, u = op
            if self.smem.get(("st", s, "l")) != u:
                raise Hazard(f"stage {s} holds {self.smem.get(('st', s, 'l'))} when tile {u} reads it")
        elif kind == "load":  # warpgroup wg reads chunks 2wg, 2wg + 1 of both buffers
            _, wg, w, u = op
            b = u & 1
            for buf, want in ((self.st, "S"), (self.dpt, "dP")):
                for c in (2 * wg, 2 * wg + 1):
                    if buf[b][c] != (want, u):
                        raise Hazard(f"warpgroup {wg} loads {want} of tile {u}, chunk {c} holds {buf[b][c]}")
            self.loaded.setdefault((b, u), set()).add((wg, w))
        elif kind == "store":  # warpgroup wg writes chunk wg of both buffers (P^T, dS^T)
            _, wg, w, u = op
            b = u & 1
            owner = wg // 2  # chunk wg is read by warpgroup wg // 2 (= 0)
            if sum(1 for x in self.loaded.get((b, u), ()) if x[0] == owner) < 4:
                raise Hazard(f"warpgroup {wg} stores P^T/dS^T of tile {u} over columns not yet loaded")
            for buf, new in ((self.st, "P"), (self.dpt, "dS")):
                if buf[b][wg] not in ((new, u), (("S" if new == "P" else "dP"), u)):
                    raise Hazard(f"warpgroup {wg} stores {new} of tile {u} over {buf[b][wg]}")
                buf[b][wg] = (new, u)
        elif kind == "epilogue":
            if self.acc != self.nq - 1:
                raise Hazard(f"epilogue reads dV/dK at tile {self.acc}")
        else:
            raise AssertionError(op)


class Dq(Sim):
    """One CTA: resident Q/dO rows, n 128-key tiles streaming (K ring 3, V ring 2)."""

    def __init__(self, n, seed, plant=None):
        super().__init__(seed)
        self.n, self.plant = n, plant
        for name in ("a_full", "s_full", "ds_free", "done"):
            self.bar(name)
        for s in range(3):
            self.bar(("kfull", s)), self.bar(("kempty", s))
        for s in range(2):
            self.bar(("full", s)), self.bar(("empty", s))
        self.bar("s_free", 256), self.bar("ds_full", 256)
        self.s = None                # tile whose S and dP the TMEM holds
        self.loaded = {}             # tile -> warps that loaded their columns
        self.ds = [None, None]       # dS halves: tile stored
        self.ds_warps = {}           # (tile, half) -> warps that stored
        self.ds_read = set()         # tiles whose dS the dQ product read
        self.acc = None

    def roles(self):
        r = {"producer": self.producer(), "mma": self.mma()}
        for wg in range(2):
            for w in range(4):
                r[("ew", wg, w)] = self.elementwise(wg, w)
        return r

    def producer(self):
        yield ("tma", "a_full", 0, [(("q",), 0), (("do",), 0)])
        for t in range(self.n):
            ks, vs = t % 3, t & 1
            yield ("wait", ("kempty", ks), t // 3)
            yield ("tma", ("kfull", ks), t // 3, [(("k", ks), t)])
            yield ("wait", ("empty", vs), t >> 1)
            yield ("tma", ("full", vs), t >> 1, [(("v", vs), t)])

    def mma(self):
        def sdp(t):
            yield ("wait", ("kfull", t % 3), t // 3 + 1)
            yield ("wait", ("full", t & 1), (t >> 1) + 1)
            yield ("pipe", ("sdp", t))
            yield ("pipe", ("commit", "s_full"))
            yield ("pipe", ("commit", ("empty", t & 1)))

        yield ("wait", "a_full", 1)
        if self.n:
            yield from sdp(0)
        for t in range(self.n):
            if self.plant != "no_s_free_wait":
                yield ("wait", "s_free", t + 1)
            if t + 1 < self.n:
                yield from sdp(t + 1)
            yield ("wait", "ds_full", t + 1)
            yield ("pipe", ("dq", t))
            yield ("pipe", ("commit", ("kempty", t % 3)))
            yield ("pipe", ("commit", "ds_free"))
        yield ("pipe", ("commit", "done"))

    def elementwise(self, wg, w):
        for t in range(self.n):
            yield ("wait", "s_full", t + 1)
            yield ("wait", ("kfull", t % 3), t // 3 + 1)
            yield ("read_mask", t)  # the key tile's validity words, published with the copy
            yield ("load", wg, w, t)
            yield ("arrive", "s_free", 32, t)
            if t > 0 and self.plant != "no_ds_free_wait":
                yield ("wait", "ds_free", t)
            yield ("store", wg, w, t)
            yield ("arrive", "ds_full", 32, t)
        yield ("wait", "done", 1)
        yield ("epilogue",)

    def pipe_readers(self, op):
        t = op[1]
        if op[0] == "sdp":
            return [("q",), ("do",), ("k", t % 3), ("v", t & 1)]
        if op[0] == "dq":
            return [("k", t % 3)]
        return ()

    def tensor_op(self, op):
        kind, t = op
        if kind == "sdp":
            for buf, ver in ((("q",), 0), (("do",), 0), (("k", t % 3), t), (("v", t & 1), t)):
                self.read_smem(buf, ver)
            if self.s is not None and len(self.loaded.get(self.s, ())) < 8:
                raise Hazard(f"S/dP of tile {t} overwrite tile {self.s} before it was loaded")
            self.s = t
        elif kind == "dq":
            self.read_smem(("k", t % 3), t)
            if self.ds != [t, t] or any(len(self.ds_warps.get((t, h), ())) < 4 for h in range(2)):
                raise Hazard(f"dQ of tile {t} reads dS {self.ds}")
            if self.acc != (None if t == 0 else t - 1):
                raise Hazard(f"dQ of tile {t} accumulates onto tile {self.acc}")
            self.ds_read.add(t)
            self.acc = t
        else:
            raise AssertionError(op)

    def local_op(self, role, op):
        kind = op[0]
        if kind == "read_mask":
            t = op[1]
            if self.smem.get(("k", t % 3)) != t:
                raise Hazard(f"K stage {t % 3} holds {self.smem.get(('k', t % 3))} when tile {t} reads its mask")
        elif kind == "load":
            _, wg, w, t = op
            if self.s != t:
                raise Hazard(f"warpgroup {wg} loads S/dP of tile {t}, TMEM holds {self.s}")
            self.loaded.setdefault(t, set()).add((wg, w))
        elif kind == "store":
            _, wg, w, t = op
            old = self.ds[wg]
            if old is not None and old != t and old not in self.ds_read:
                raise Hazard(f"warpgroup {wg} stores dS of tile {t} over dS of tile {old} before dQ read it")
            self.ds[wg] = t
            self.ds_warps.setdefault((t, wg), set()).add(w)
        elif kind == "epilogue":
            if self.acc != self.n - 1:
                raise Hazard(f"epilogue reads dQ at tile {self.acc}")
        else:
            raise AssertionError(op)


@pytest.mark.parametrize("nq", [1, 2, 3, 5, 9])
def test_dkdv_protocol(nq):
    for seed in range(15):
        DkDv(nq, seed=100 * nq + seed).run()


@pytest.mark.parametrize("n", [1, 2, 3, 4, 7])
def test_dq_protocol(n):
    for seed in range(15):
        Dq(n, seed=100 * n + seed).run()


@pytest.mark.parametrize("model,plant", [
    (DkDv, "no_pair_sync"),   # a warpgroup writes P^T over columns the other has not read
    (DkDv, "early_sdp"),      # the next-but-one S^T issued before dV/dK read P^T
    (Dq, "no_s_free_wait"),   # the next S issued before the warps loaded this one
    (Dq, "no_ds_free_wait"),  # dS stored before the previous dQ product read it
])
def test_planted_mistakes_are_caught(model, plant):
    caught = 0
    for seed in range(40):
        try:
            model(5, seed=seed, plant=plant).run()
        except Hazard:
            caught += 1
    assert caught > 0, plant
