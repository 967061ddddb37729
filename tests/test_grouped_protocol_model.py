"""A CPU model of the grouped 64-token forward kernel's synchronisation protocol
(`attn_fwd_grouped64_kernel` in csrc/attn_fwd.cu).

On top of the forward kernels' protocol (modelled in
tests/test_fwd_protocol_model.py) this kernel adds a group builder warp that
writes each group's selection bitmaps into one of two shared-memory buffers
and hands it over on grp_full; ten warps read it (the producer while it
walks the key stream, the MMA warp once, the eight softmax warps while they
walk it) and each releases it on grp_free.  (The producer could release
early without harm: it walks each tile before any softmax warp can reach
it.  The softmax warps cannot.)  Groups carry their own number of
key tiles (zero included) and of query tiles (one or two), so the MMA warp
keeps per-tile counters for the p_full and o_empty phases, and a softmax
warpgroup sits out the groups that have no second query tile.  With a shared
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
    def __init__(self, groups, seed, plant=None, skip_every=3, sentinel=False):
        super().__init__([], False, 256, seed, plant)
        self.groups = groups            # [(key tiles, query tiles)]
        self.skip_every = skip_every    # which (warp, tile) pairs select nothing
        # sentinel: the groups come from a shared queue; after the last one the
        # builder publishes an end marker the consumers stop on
        self.sentinel = sentinel
        for b in range(2):
            self.bar(("grp_full", b), 1)
            self.bar(("grp_free", b), 10)
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

    def producer(self):
        kit = vit = qit = 0
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            n, nq = grp
            yield ("read_grp", b, gl)
            if n > 0:
                yield ("wait", "q_empty", qit)
                yield ("tma", "q_full", qit, [(("q", c), gl) for c in range(2 * nq)])
                qit += 1
                for t in range(n):
                    yield ("read_grp", b, gl)
                    s = kit % self.KS
                    yield ("wait", ("k_empty", s), kit // self.KS)
                    yield ("tma", ("k_full", s), kit // self.KS, [(("k", s, c), (gl, t)) for c in range(2)])
                    kit += 1
                    s = vit % self.VS
                    yield ("wait", ("v_empty", s), vit // self.VS)
                    yield ("tma", ("v_full", s), vit // self.VS, [(("v", s, c), (gl, t)) for c in range(2)])
                    vit += 1
            yield ("arrive", ("grp_free", b), 1, gl >> 1)

    def mma(self):
        kit = vit = qit = 0
        tiles, items = [0, 0], [0, 0]
        if self.plant == "shared_counters":  # one counter for both query tiles, as the ungrouped kernel
            tiles, items = [0, 0], [0, 0]
        sn = [0, 0]
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            n, nq = grp
            yield ("read_grp", b, gl)
            yield ("arrive", ("grp_free", b), 1, gl >> 1)
            if n == 0:
                continue
            yield ("wait", "q_full", qit + 1)
            qit += 1

            def issue_s(i, sk, t):
                yield ("pipe", ("S", i, sn[i], sk, (gl, t), gl))
                yield ("pipe", ("commit", ("s_full", i)))
                sn[i] += 1

            def issue_pv(i, sv, t):
                yield ("wait", ("p_full", i), tiles[i] + 1)
                if t == 0:
                    yield ("wait", ("o_empty", i), items[i])
                yield ("pipe", ("PV", i, sv, (gl, t)))
                if t == n - 1:
                    yield ("pipe", ("commit", ("o_full", i)))
                tiles[i] += 1
                if self.plant == "shared_counters" and i == 0:
                    tiles[1] = tiles[0]

            sk = kit % self.KS
            yield ("wait", ("k_full", sk), kit // self.KS + 1)
            for i in range(nq):
                yield from issue_s(i, sk, 0)
            yield ("pipe", ("commit", ("k_empty", sk)))
            if n == 1 or self.plant == "q_free_first_s":
                yield ("pipe", ("commit", "q_empty"))  # Q is read by S products only
            kit += 1
            for t in range(n):
                sv = vit % self.VS
                yield ("wait", ("v_full", sv), vit // self.VS + 1)
                more = t + 1 < n
                sk = kit % self.KS
                yield from issue_pv(0, sv, t)
                if more:
                    yield ("wait", ("k_full", sk), kit // self.KS + 1)
                    yield from issue_s(0, sk, t + 1)
                if nq == 2:
                    yield from issue_pv(1, sv, t)
                yield ("pipe", ("commit", ("v_empty", sv)))
                vit += 1
                if more:
                    if nq == 2:
                        yield from issue_s(1, sk, t + 1)
                    yield ("pipe", ("commit", ("k_empty", sk)))
                    if t + 2 == n and self.plant != "q_free_first_s":
                        yield ("pipe", ("commit", "q_empty"))  # after the group's last S
                    kit += 1
            items[0] += 1
            if nq == 2 or self.plant == "shared_counters":
                items[1] += 1

    def softmax_warp(self, i, w):
        tiles = items = 0
        for gl, grp in self.consumer_groups():
            b = gl & 1
            yield ("wait", ("grp_full", b), (gl >> 1) + 1)
            if grp is None:
                yield ("read_grp", b, "end")
                break
            n, nq = grp
            yield ("read_grp", b, gl)
            if i >= nq or n == 0:
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
            if self.s_val[i] is not None and len(self.s_loaded[i]) < 4:
                raise Hazard(f"S{i}#{u} overwrites S{i}#{self.s_val[i]} before it was loaded")
            if self.p[i] is not None and self.p[i][0] != "read":
                raise Hazard(f"S{i}#{u} overwrites P{i} {self.p[i][:3]} before P V read it")
            self.s_val[i], self.s_loaded[i], self.hi[i], self.p[i] = u, set(), ("S", u), None
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
        roles = {"builder": self.builder(), "producer": self.producer(), "mma": self.mma()}
        for i in range(2):
            for w in range(4):
                roles[("softmax", i, w)] = self.softmax_warp(i, w)
        return roles

    def pipe_readers(self, op):
        if op[0] == "S":
            return [("q", c) for c in (2 * op[1], 2 * op[1] + 1)] + [("k", op[3], c) for c in range(2)]
        return super().pipe_readers(op)


GROUP_SETS = [
    [(3, 2), (2, 2), (4, 2)],
    [(5, 2), (0, 2), (1, 2), (0, 1), (3, 1), (2, 2)],   # empty groups, a last group of two blocks
    [(1, 1), (2, 1), (1, 2), (6, 2), (0, 2), (0, 2), (2, 1)],
    [(2, 2)] * 7,
    [(0, 2), (0, 2), (0, 1)],
]


@pytest.mark.parametrize("sentinel", [False, True], ids=["static", "queue"])
@pytest.mark.parametrize("groups", range(len(GROUP_SETS)))
@pytest.mark.parametrize("skip_every", [2, 3, 5])
def test_grouped_protocol_has_no_deadlock_alias_or_hazard(groups, skip_every, sentinel):
    for seed in range(8):
        GroupedModel(GROUP_SETS[groups], seed=100 * groups + seed, skip_every=skip_every, sentinel=sentinel).run()


def test_queue_with_no_group_for_this_cta_ends_cleanly():
    """A CTA whose first ticket is already past the end: only the end marker."""
    for seed in range(10):
        GroupedModel([], seed=seed, sentinel=True).run()


@pytest.mark.parametrize("plant", [
    "builder_no_free_wait",   # the builder overwrites a buffer consumers still walk
    "softmax_frees_early",    # softmax warps release a group before walking its key stream
    "shared_counters",        # one p_full / o_empty counter for both query tiles
    "q_free_first_s",         # Q released after the group's first S instead of its last
])
def test_grouped_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(40):
        try:
            GroupedModel([(3, 2), (2, 1), (4, 2), (1, 1), (2, 2), (3, 1)], seed=seed, plant=plant).run()
        except Hazard:
            caught += 1
    assert caught > 0, plant
