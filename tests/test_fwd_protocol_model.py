"""A CPU model of the fine-stage forward kernels' synchronisation protocol.

The two forward kernels (`attn_fwd_kernel` in csrc/attn_fwd.cu and
`attn_fwd_fp4_kernel` in csrc/fp4.cu) coordinate a TMA producer warp, a
single MMA-issuing thread, the in-order tensor pipe and the softmax warps
through mbarriers, and they reuse tensor memory: P is written over the first
half of its S region, and in the NVFP4 kernel the scale factors of S_i are
parked in the second half of the other tile's S region.  This model replays
each role's waits, arrivals, copies and tensor-pipe operations in the
kernels' program order (per key tile: PV0(t), S0(t+1), PV1(t), S1(t+1)) under
random schedules: TMA copies land and tensor-pipe operations execute at random
later times, the tensor pipe in issue order, and `tcgen05.commit` arrives once
everything issued before it has executed.  It checks

  * no deadlock;
  * no mbarrier phase aliasing: a wait passes only on the phase its parity
    stands for, and every arrival belongs to the barrier's open phase (a warp
    running a phase ahead would otherwise complete a phase early);
  * no tensor- or shared-memory hazard: every reader of S, P, O, a scale
    region or a shared-memory stage sees the value it expects, and nothing is
    overwritten before its last reader has run.

Planted mistakes (a wait taken out, an arrival moved early, a product issued
out of order) must be caught; a harmless change (a later arrival) must not.
The model is test infrastructure for the protocol's design; the GPU parity
tests cover the kernels themselves.
"""
import pytest

from tests.protocol_sim import Hazard, Sim


class Model(Sim):
    def __init__(self, nbs, fp4, bs, seed, plant=None):
        super().__init__(seed)
        self.nbs, self.fp4, self.bs, self.plant = nbs, fp4, bs, plant
        self.QT = 2 if bs == 256 else 1          # 128-row query tiles per item
        self.KS, self.VS = (4, 3) if fp4 else (3, 2)  # K and V ring stages
        for n in ("q_full", "q_empty"):
            self.bar(n)
        for s in range(self.KS):
            self.bar(("k_full", s)), self.bar(("k_empty", s))
        for s in range(self.VS):
            self.bar(("v_full", s)), self.bar(("v_empty", s))
        for i in range(2):
            self.bar(("s_full", i)), self.bar(("o_full", i))
            for n in ("s_read", "p_full", "o_empty"):
                self.bar((n, i), 128)
        self.s_val = [None, None]         # product index held by S_i
        self.s_loaded = [set(), set()]    # softmax warps that loaded it
        self.hi = [None, None]            # S_i's second half: ("S", u) or ("sf", owner, u)
        self.sf_used = set()              # scale sets read by their product
        self.p = [None, None]             # P_i: [state, item, tile, warps]
        self.o = [None, None]             # O_i: (item, last tile accumulated)
        self.o_read = [set(), set()]      # epilogue warps that read the final O_i

    def items(self):
        return [(it, nb) for it, nb in enumerate(self.nbs) if nb > 0]

    def tiles(self, nb):
        return 2 * nb if self.bs == 256 else (nb + 1) // 2

    # ---------------------------------------------------------------- roles
    def producer(self):
        kit = vit = qit = 0
        for it, nb in self.items():
            yield ("wait", "q_empty", qit)
            yield ("tma", "q_full", qit, [(("q", c), it) for c in range(2 * self.QT)])
            qit += 1
            for t in range(self.tiles(nb)):
                s = kit % self.KS
                yield ("wait", ("k_empty", s), kit // self.KS)
                yield ("tma", ("k_full", s), kit // self.KS, [(("k", s, c), (it, t)) for c in range(2)])
                kit += 1
                s = vit % self.VS
                yield ("wait", ("v_empty", s), vit // self.VS)
                yield ("tma", ("v_full", s), vit // self.VS, [(("v", s, c), (it, t)) for c in range(2)])
                vit += 1

    def mma(self):
        kit = vit = qit = tiles = items = 0
        sn = [0, 0]
        for it, nb in self.items():
            n = self.tiles(nb)
            yield ("wait", "q_full", qit + 1)
            qit += 1

            def issue_s(i, sk, t):
                if self.fp4:
                    j = 1 - i
                    if sn[j] > 0 and self.plant != "no_s_read_wait":
                        yield ("wait", ("s_read", j), sn[j])
                    yield ("pipe", ("cp", i, sn[i]))
                yield ("pipe", ("S", i, sn[i], sk, (it, t), it))
                yield ("pipe", ("commit", ("s_full", i)))
                sn[i] += 1

            def issue_pv(i, sv, t):
                yield ("wait", ("p_full", i), tiles + 1)
                if t == 0:
                    yield ("wait", ("o_empty", i), items)
                if t == n - 1 and self.plant == "o_full_early":
                    yield ("pipe", ("commit", ("o_full", i)))
                yield ("pipe", ("PV", i, sv, (it, t)))
                if t == n - 1 and self.plant != "o_full_early":
                    yield ("pipe", ("commit", ("o_full", i)))

            sk = kit % self.KS
            yield ("wait", ("k_full", sk), kit // self.KS + 1)
            for i in range(self.QT):
                yield from issue_s(i, sk, 0)
            yield ("pipe", ("commit", ("k_empty", sk)))
            kit += 1
            for t in range(n):
                sv = vit % self.VS
                yield ("wait", ("v_full", sv), vit // self.VS + 1)
                more = t + 1 < n
                sk = kit % self.KS
                if self.plant == "s_before_pv" and more:
                    yield ("wait", ("k_full", sk), kit // self.KS + 1)
                    yield from issue_s(0, sk, t + 1)
                    yield from issue_pv(0, sv, t)
                else:
                    yield from issue_pv(0, sv, t)
                    if more:
                        yield ("wait", ("k_full", sk), kit // self.KS + 1)
                        yield from issue_s(0, sk, t + 1)
                if self.QT == 2:
                    yield from issue_pv(1, sv, t)
                yield ("pipe", ("commit", ("v_empty", sv)))
                vit += 1
                if more:
                    if self.QT == 2:
                        yield from issue_s(1, sk, t + 1)
                    yield ("pipe", ("commit", ("k_empty", sk)))
                    kit += 1
                tiles += 1
            yield ("pipe", ("commit", "q_empty"))
            items += 1

    def softmax_warp(self, i, w):
        tiles = items = 0
        for it, nb in self.items():
            n = self.tiles(nb)
            for t in range(n):
                yield ("wait", ("s_full", i), tiles + 1)
                yield ("ld_S", i, w, tiles)
                if self.fp4 and self.plant != "s_read_late":
                    yield ("arrive", ("s_read", i), 32, tiles)
                if self.plant == "p_full_early":
                    yield ("arrive", ("p_full", i), 32, tiles)
                yield ("st_P", i, w, it, t)
                if self.fp4 and self.plant == "s_read_late":
                    yield ("arrive", ("s_read", i), 32, tiles)
                if t > 0:
                    yield ("rescale_O", i, it, t)
                if self.plant != "p_full_early":
                    yield ("arrive", ("p_full", i), 32, tiles)
                tiles += 1
            yield ("wait", ("o_full", i), items + 1)
            yield ("epilogue", i, w, it, n)
            yield ("arrive", ("o_empty", i), 32, items)
            items += 1

    # ---------------------------------------------------------------- effects
    def tensor_op(self, op):
        kind = op[0]
        if kind == "cp":  # scales of S_i product u into the second half of S_j
            _, i, u = op
            j = 1 - i
            if self.s_val[j] is not None and len(self.s_loaded[j]) < 4:
                raise Hazard(f"scales of S{i}#{u} copied over S{j}#{self.s_val[j]} before it was loaded")
            if self.hi[j] is not None and self.hi[j][0] == "sf" and self.hi[j] not in self.sf_used:
                raise Hazard(f"scales of S{i}#{u} copied over unread scales {self.hi[j]}")
            self.hi[j] = ("sf", i, u)
        elif kind == "S":
            _, i, u, sk, kver, it = op
            for c in range(2 * self.QT):
                self.read_smem(("q", c), it)
            for c in range(2):
                self.read_smem(("k", sk, c), kver)
            if self.fp4:
                if self.hi[1 - i] != ("sf", i, u):
                    raise Hazard(f"S{i}#{u} reads scales {self.hi[1 - i]}")
                self.sf_used.add(("sf", i, u))
            if self.s_val[i] is not None and len(self.s_loaded[i]) < 4:
                raise Hazard(f"S{i}#{u} overwrites S{i}#{self.s_val[i]} before it was loaded")
            if self.p[i] is not None and self.p[i][0] != "read":
                raise Hazard(f"S{i}#{u} overwrites P{i} {self.p[i][:3]} before P V read it")
            if self.hi[i] is not None and self.hi[i][0] == "sf" and self.hi[i] not in self.sf_used:
                raise Hazard(f"S{i}#{u} overwrites unread scales {self.hi[i]}")
            self.s_val[i], self.s_loaded[i], self.hi[i], self.p[i] = u, set(), ("S", u), None
        elif kind == "PV":
            _, i, sv, (it, t) = op
            for c in range(2):
                self.read_smem(("v", sv, c), (it, t))
            if self.p[i] is None or self.p[i][:3] != ["stored", it, t]:
                raise Hazard(f"P V{i} of {(it, t)} reads P {self.p[i] and self.p[i][:3]}")
            self.p[i][0] = "read"
            if t == 0:
                if self.o[i] is not None and len(self.o_read[i]) < 4:
                    raise Hazard(f"P V{i} of item {it} restarts O{i} before the epilogue of {self.o[i]} read it")
                self.o_read[i] = set()
            elif self.o[i] != (it, t - 1):
                raise Hazard(f"P V{i} of {(it, t)} accumulates onto O{i} at {self.o[i]}")
            self.o[i] = (it, t)
        else:
            raise AssertionError(op)

    def local_op(self, role, op):
        kind = op[0]
        if kind == "ld_S":
            _, i, w, g = op
            if self.s_val[i] != g or self.hi[i] != ("S", g):
                raise Hazard(f"softmax {i} loads S#{g}: S holds {self.s_val[i]}, second half {self.hi[i]}")
            self.s_loaded[i].add(w)
        elif kind == "st_P":
            _, i, w, it, t = op
            if self.p[i] is None:
                self.p[i] = ["partial", it, t, set()]
            if self.p[i][1:3] != [it, t] or self.p[i][0] == "read":
                raise Hazard(f"softmax {i} stores P of {(it, t)} over {self.p[i][:3]}")
            self.p[i][3].add(w)
            if len(self.p[i][3]) == 4:
                self.p[i][0] = "stored"
        elif kind == "rescale_O":  # any warp may rescale its rows of O
            _, i, it, t = op
            if self.o[i] != (it, t - 1):
                raise Hazard(f"softmax {i} rescales O{i} at {self.o[i]}, expected {(it, t - 1)}")
        elif kind == "epilogue":
            _, i, w, it, n = op
            if self.o[i] != (it, n - 1):
                raise Hazard(f"epilogue {i} reads O{i} at {self.o[i]}, expected {(it, n - 1)}")
            self.o_read[i].add(w)
        else:
            raise AssertionError(op)

    # ---------------------------------------------------------------- scheduler hooks
    def roles(self):
        roles = {"producer": self.producer(), "mma": self.mma()}
        for i in range(self.QT):
            for w in range(4):
                roles[("softmax", i, w)] = self.softmax_warp(i, w)
        return roles

    def pipe_readers(self, op):
        if op[0] == "S":
            return [("q", c) for c in range(2 * self.QT)] + [("k", op[3], c) for c in range(2)]
        if op[0] == "PV":
            return [("v", op[2], c) for c in range(2)]
        return ()


ITEM_SETS = [
    [1, 2, 3],
    [4, 0, 1, 0, 0, 2, 5],
    [3] * 6,
    [0, 0, 1],
    [7, 1, 1, 6],
]


@pytest.mark.parametrize("fp4", [False, True], ids=["bf16", "nvfp4"])
@pytest.mark.parametrize("bs", [256, 64])
@pytest.mark.parametrize("items", range(len(ITEM_SETS)))
def test_protocol_has_no_deadlock_alias_or_hazard(fp4, bs, items):
    for seed in range(10):
        Model(ITEM_SETS[items], fp4, bs, seed=1000 * items + seed).run()


@pytest.mark.parametrize("plant,fp4,bs", [
    ("no_s_read_wait", True, 256),  # scales copied over an S its softmax has not loaded
    ("p_full_early", False, 256),   # a warp signals P before storing it
    ("p_full_early", True, 64),
    ("o_full_early", False, 256),   # O signalled complete before the item's last P V
    ("s_before_pv", False, 256),      # S(t+1) issued before the P V that reads P(t)
    ("s_before_pv", True, 64),
])
def test_planted_mistakes_are_caught(plant, fp4, bs):
    caught = 0
    for seed in range(30):
        try:
            Model([3, 2, 4, 1], fp4, bs, seed=seed, plant=plant).run()
        except Hazard:
            caught += 1
    assert caught > 0, plant


def test_later_s_read_arrival_is_still_safe():
    for seed in range(20):
        Model([3, 2, 4, 1], True, 256, seed=seed, plant="s_read_late").run()
