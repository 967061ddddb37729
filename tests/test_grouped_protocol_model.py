"""A CPU model of the grouped 64-token forward kernel's synchronisation protocol
(`attn_fwd_grouped64_kernel` in csrc/attn_fwd_grouped.cu).

On top of the forward kernels' protocol (modelled in
tests/test_fwd_protocol_model.py) this kernel adds a group builder warp that
writes each group's selection bitmaps into one of two shared-memory buffers
and hands it over on grp_full; eleven warps read it (two producers -- Q and
K tiles, V tiles -- while they walk the key streams, the MMA warp once, the
eight softmax warps while they walk them) and each releases it on grp_free.
(The producers could release early without harm: they walk each tile before
any softmax warp can reach it.  The softmax warps cannot.)  Each query tile of a group walks its own
key stream: a group carries the number of leading steps whose tile is the
same for both query tiles (one K and one V stage, released by the second
query tile's product) and each query tile's number of tiles (zero
included); later steps load one stage per query tile, and a step past one
query tile's end runs the other alone.  So the MMA warp keeps per-query-tile
counters for the p_full and o_empty phases, and a softmax warpgroup sits
out the groups that have no tile for it.  In the NVFP4 variant the scales of
S_i are copied into the other query tile's S columns (free once that tile's
softmax has loaded its latest S, signalled on s_read) before S_i is issued.  With a shared
queue (a caller workspace) the builder takes group tickets and, past the last
group, publishes an end marker the consumers stop on.  Q is released
(q_empty) once the group's last S product has been issued, so the next
group's Q load overlaps the last P V products.  A softmax
warp whose query block selected nothing in a tile does not load S at all.

The model replays every role in program order under random schedules and
checks, besides the hazards of the base model, that every read of a group
buffer sees the group it expects (the builder must not overwrite a buffer a
consumer is still walking).  Planted mistakes must be caught.
"""
import pytest

from tests.protocol_sim import Hazard
from tests.test_fwd_protocol_model import Model as FwdModel


class GroupedModel(FwdModel):
    def __init__(self, groups, seed, plant=None, skip_every=3, sentinel=False, fp4=False):
        super().__init__([], False, 256, seed, plant)
        self.fp4 = fp4
        self.KS, self.VS = (4, 4) if fp4 else (2, 3)  # the grouped kernel's K and V ring stages
        for st in range(self.KS):
            self.bar(("k_full", st)), self.bar(("k_empty", st))
        for st in range(self.VS):
            self.bar(("v_full", st)), self.bar(("v_empty", st))
        # [(shared steps, key tiles of query tile 0, of query tile 1, query tiles)]
        self.groups = groups
        self.skip_every = skip_every    # which (warp, tile) pairs select nothing
        # sentinel: the groups come from a shared queue; after the last one the
        # builder publishes an end marker the consumers stop on
        self.sentinel = sentinel
        for b in range(2):
            self.bar(("grp_full", b), 1)
            self.bar(("grp_free", b), 11)
        self.grp = [None, None]

    def consumer_groups(self):
        """Group slots a consumer walks: the groups, then (queue) the end marker."""
        n = len(self.groups) + (1 if self.sentinel else 0)
        for gl in range(n):
            yield gl, (self.groups[gl] if gl < len(self.groups) else None)

    # ---------------------------------------------------------------- roles
    def builder(self):
        for gl in range(len(self.groups) + (1 if self.sentinel else 0)):
            b = gl & 1
            if gl >= 2 and self.plant != "builder_no_free_wait":
                yield ("wait", ("grp_free", b), gl >> 1)
            yield ("write_grp", b, gl if gl < len(self.groups) else "end")
            yield ("arrive", ("grp_full", b), 1, gl >> 1)

    def producer(self, side):
        """side "k": Q and the K tiles; side "v": the V tiles (a warp of its own)."""
        kit = vit = qit = 0
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            ns, lens, nq = grp[0], grp[1:3], grp[3]
            yield ("read_grp", b, gl)
            n = max(lens)
            if n > 0:
                if side == "k":
                    yield ("wait", "q_empty", qit)
                    yield ("tma", "q_full", qit, [(("q", c), gl) for c in range(2 * nq)])
                    qit += 1
                for t in range(n):
                    yield ("read_grp", b, gl)
                    # one stage per distinct tile of the step, query tile 0's first
                    tags = ["sh"] if t < ns else [j for j in range(2) if t < lens[j]]
                    for tag in tags:
                        if side == "k":
                            s = kit % self.KS
                            yield ("wait", ("k_empty", s), kit // self.KS)
                            yield ("tma", ("k_full", s), kit // self.KS,
                                   [(("k", s, c), (gl, t, tag)) for c in range(2)])
                            kit += 1
                        else:
                            s = vit % self.VS
                            yield ("wait", ("v_empty", s), vit // self.VS)
                            yield ("tma", ("v_full", s), vit // self.VS,
                                   [(("v", s, c), (gl, t, tag)) for c in range(2)])
                            vit += 1
            yield ("arrive", ("grp_free", b), 1, gl >> 1)

    def mma(self):
        st = dict(kit=0, vit=0, sk=0, sv=0)
        qit = 0
        tiles, items = [0, 0], [0, 0]
        sn = [0, 0]
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            ns, lens, nq = grp[0], grp[1:3], grp[3]
            n = max(lens)
            yield ("read_grp", b, gl)
            yield ("arrive", ("grp_free", b), 1, gl >> 1)
            if n == 0:
                continue
            yield ("wait", "q_full", qit + 1)
            qit += 1
            if self.plant == "split_as_shared":  # a split step read from one stage, as a shared one
                ns = n

            def s_of(j, u):
                shared = u < ns
                if j == 0 or not shared:
                    st["sk"] = st["kit"] % self.KS
                    yield ("wait", ("k_full", st["sk"]), st["kit"] // self.KS + 1)
                tag = "sh" if shared else j
                if self.fp4:  # scales into the other tile's S columns, once its latest S is loaded
                    if sn[1 - j] > 0 and self.plant != "no_s_read_wait":
                        yield ("wait", ("s_read", 1 - j), sn[1 - j])
                    yield ("pipe", ("cp", j, sn[j]))
                yield ("pipe", ("S", j, sn[j], st["sk"], (gl, u, tag), gl))
                yield ("pipe", ("commit", ("s_full", j)))
                sn[j] += 1
                if j == 1 or not shared:
                    yield ("pipe", ("commit", ("k_empty", st["sk"])))
                    st["kit"] += 1

            def pv_of(j, u):
                shared = u < ns
                if j == 0 or not shared:
                    st["sv"] = st["vit"] % self.VS
                    yield ("wait", ("v_full", st["sv"]), st["vit"] // self.VS + 1)
                yield ("wait", ("p_full", j), tiles[j] + 1)
                if u == 0:
                    yield ("wait", ("o_empty", j), items[j])
                tag = "sh" if shared else j
                yield ("pipe", ("PV", j, st["sv"], (gl, u, tag)))
                if u == lens[j] - 1:
                    yield ("pipe", ("commit", ("o_full", j)))
                tiles[j] += 1
                if self.plant == "shared_counters" and j == 0:
                    tiles[1] = tiles[0]
                release = j == 1 or not shared or self.plant == "v_free_first_pv"
                if release:
                    yield ("pipe", ("commit", ("v_empty", st["sv"])))
                    st["vit"] += 1

            for j in range(2):
                if lens[j] > 0:
                    yield from s_of(j, 0)
            if n == 1 or self.plant == "q_free_first_s":
                yield ("pipe", ("commit", "q_empty"))  # Q is read by S products only
            for t in range(n):
                if t < lens[0]:
                    yield from pv_of(0, t)
                if t + 1 < lens[0]:
                    yield from s_of(0, t + 1)
                if t < lens[1]:
                    if self.plant == "v_free_first_pv" and t < ns:
                        st["vit"] -= 1  # the stage PV0 already released, read again
                    yield from pv_of(1, t)
                if t + 1 < lens[1]:
                    yield from s_of(1, t + 1)
                if t + 2 == n and self.plant != "q_free_first_s":
                    yield ("pipe", ("commit", "q_empty"))  # after the group's last S
            for j in range(2):
                if lens[j] > 0 or (self.plant == "shared_counters" and lens[0] > 0):
                    items[j] += 1

    def softmax_warp(self, i, w):
        tiles = items = 0
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            ns, lens, nq = grp[0], grp[1:3], grp[3]
            n = lens[i] if i < nq else 0
            yield ("read_grp", b, gl)
            if n == 0:
                yield ("arrive", ("grp_free", b), 1, gl >> 1)
                if i < nq:
                    yield ("write_empty_rows", i, w, gl)
                continue
            if self.plant == "softmax_frees_early":
                yield ("arrive", ("grp_free", b), 1, gl >> 1)
            for t in range(n):
                yield ("read_grp", b, gl)
                yield ("wait", ("s_full", i), tiles + 1)
                if (gl + t + w) % self.skip_every == 0:
                    yield ("skip_S", i, w, tiles)  # nothing selected: S is not loaded
                else:
                    yield ("ld_S", i, w, tiles)
                if self.fp4:
                    yield ("arrive", ("s_read", i), 32, tiles)
                yield ("st_P", i, w, gl, t)
                if t > 0:
                    yield ("rescale_O", i, gl, t)
                yield ("arrive", ("p_full", i), 32, tiles)
                tiles += 1
            if self.plant != "softmax_frees_early":
                yield ("arrive", ("grp_free", b), 1, gl >> 1)
            yield ("wait", ("o_full", i), items + 1)
            yield ("epilogue", i, w, gl, n)
            yield ("arrive", ("o_empty", i), 32, items)
            items += 1

    # ---------------------------------------------------------------- effects
    def tensor_op(self, op):
        if op[0] == "S":  # Q tile i only: the group may load one query tile
            _, i, u, sk, kver, gl = op
            for c in (2 * i, 2 * i + 1):
                self.read_smem(("q", c), gl)
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
            return
        if op[0] == "PV":  # the V stage carries its query tile's tag; P and O as in the base model
            _, i, sv, (gl, t, tag) = op
            for c in range(2):
                self.read_smem(("v", sv, c), (gl, t, tag))
            op = ("PV_checked", i, sv, (gl, t))
        if op[0] == "PV_checked":
            _, i, sv, (it, t) = op
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
            return
        super().tensor_op(op)

    def local_op(self, role, op):
        kind = op[0]
        if kind == "write_grp":
            self.grp[op[1]] = op[2]
        elif kind == "read_grp":
            if self.grp[op[1]] != op[2]:
                raise Hazard(f"{role} reads group buffer {op[1]} for group {op[2]}; it holds {self.grp[op[1]]}")
        elif kind == "skip_S":
            _, i, w, g = op
            if self.s_val[i] != g:
                raise Hazard(f"softmax {i} passes S#{g} while S holds {self.s_val[i]}")
            self.s_loaded[i].add(w)
        elif kind == "write_empty_rows":
            pass
        else:
            super().local_op(role, op)

    # ---------------------------------------------------------------- scheduler hooks
    def roles(self):
        roles = {"builder": self.builder(), "producer_k": self.producer("k"), "producer_v": self.producer("v"),
                 "mma": self.mma()}
        for i in range(2):
            for w in range(4):
                roles[("softmax", i, w)] = self.softmax_warp(i, w)
        return roles

    def pipe_readers(self, op):
        if op[0] == "S":
            return [("q", c) for c in (2 * op[1], 2 * op[1] + 1)] + [("k", op[3], c) for c in range(2)]
        if op[0] == "PV":
            return [("v", op[2], c) for c in range(2)]
        return super().pipe_readers(op)


# (shared steps, key tiles of query tile 0, of query tile 1, query tiles)
GROUP_SETS = [
    [(3, 3, 3, 2), (0, 2, 2, 2), (1, 4, 2, 2)],                           # shared, split, a tail of tile 0
    [(2, 5, 2, 2), (0, 0, 0, 2), (0, 1, 0, 1), (0, 0, 0, 1), (0, 3, 0, 1), (1, 1, 2, 2)],
    [(0, 1, 0, 1), (0, 2, 0, 1), (0, 1, 3, 2), (2, 2, 6, 2), (0, 0, 0, 2), (0, 0, 3, 2), (0, 2, 0, 1)],
    [(0, 2, 2, 2)] * 7,                                                    # split steps only
    [(0, 0, 0, 2), (0, 0, 0, 2), (0, 0, 0, 1)],
    [(0, 4, 1, 2), (0, 1, 4, 2), (0, 3, 0, 2), (4, 4, 4, 2)],              # one query tile empty, tails
]


@pytest.mark.parametrize("fp4", [False, True], ids=["16bit", "nvfp4"])
@pytest.mark.parametrize("sentinel", [False, True], ids=["static", "queue"])
@pytest.mark.parametrize("groups", range(len(GROUP_SETS)))
@pytest.mark.parametrize("skip_every", [2, 3, 5])
def test_grouped_protocol_has_no_deadlock_alias_or_hazard(groups, skip_every, sentinel, fp4):
    for seed in range(8):
        GroupedModel(GROUP_SETS[groups], seed=100 * groups + seed, skip_every=skip_every, sentinel=sentinel,
                     fp4=fp4).run()


def test_queue_with_no_group_for_this_cta_ends_cleanly():
    """A CTA whose first ticket is already past the end: only the end marker."""
    for seed in range(10):
        GroupedModel([], seed=seed, sentinel=True).run()


@pytest.mark.parametrize("plant", [
    "builder_no_free_wait",   # the builder overwrites a buffer consumers still walk
    "softmax_frees_early",    # softmax warps release a group before walking its key stream
    "shared_counters",        # one p_full / o_empty counter for both query tiles
    "q_free_first_s",         # Q released after the group's first S instead of its last
    "split_as_shared",        # a step with one tile per query tile read from one stage
    "v_free_first_pv",        # a shared V stage released by the first query tile's P V
    "no_s_read_wait",         # NVFP4: scales copied before the other tile's softmax loaded its S
])
def test_grouped_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(40):
        try:
            GroupedModel([(1, 3, 2, 2), (0, 2, 0, 1), (2, 4, 3, 2), (0, 1, 0, 1), (0, 2, 3, 2), (0, 3, 0, 1)],
                         seed=seed, plant=plant, fp4=plant == "no_s_read_wait").run()
        except Hazard:
            caught += 1
    assert caught > 0, plant
