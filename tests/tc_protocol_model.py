"""Discrete-event model of the mbarrier protocol of the fused tensor-core kernel (one CTA).

The model follows ``block_sparse_attention_41_b200/csrc/fwd_tc.cu`` role by role. It has the TMA
producer, the QK^T issuer, the two PV issuers and the two softmax groups, each split into its
waits, arrivals and commits, over a sequence of work units of T tiles each. Copies and MMAs
complete after random delays. A run fails on:
- a deadlock: no role can move and nothing is in flight;
- a stale wait: a role waits for phase k of a barrier that has already completed phase k+1,
  so its parity test would block or pass wrongly;
- a hazard: a QK^T writing an S buffer whose P has not been consumed, a PV reading the wrong
  tile's P or V, a copy overwriting a K/V stage still being read, an O rescale or read with a PV
  in flight.

Barrier semantics: a barrier of count c completes a phase after c arrivals; a wait for phase k
(parity k & 1) passes once k + 1 phases have completed.

Three schedules are modelled. "split" (the kernel's): both softmax groups work on every tile,
each on half of its key columns, one thread issues every QK^T and one PV issuer per group
consumes every tile. "alternate": softmax group g takes the tiles t of each unit with
t & 1 == g (so the split does not depend on what the CTA ran before), owns S buffer g and its
own PV issuer, and rescales its accumulator without waiting, because its previous PV completed
before the QK^T that filled its S buffer was issued. "group_issuers": as "alternate", with one
thread per group issuing both the group's QK^T and its PV. The last two were measured slower
than "split" on the GPU; the model keeps their protocols checked.
"""
from __future__ import annotations

import random


class Bar:
    def __init__(self, name: str, count: int):
        self.name, self.count, self.pending, self.n = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.n += 1


class Protocol:
    """One CTA running `plan` (tiles per unit) with the kernel's K and V ring depths."""

    def __init__(self, plan, seed, nk=3, nv=2, mutation=None, route_in_kernel=False, schedule="split"):
        self.plan, self.nk, self.nv, self.mut = plan, nk, nv, mutation
        self.route_in_kernel = route_in_kernel  # no keep bits given: the softmax warps route from the Q tile
        self.alt = schedule in ("alternate", "group_issuers", "smem_p")
        self.group_issuers = schedule == "group_issuers"
        self.smem_p = schedule == "smem_p"
        self.dephase = schedule == "split_dephase"
        self.single = schedule == "split_single_issuer"
        self.rng = random.Random(seed)
        self.now, self.seq, self.events = 0, 0, []
        if schedule == "split_single_issuer":
            pv_count, v_count = 1, 1
        elif self.alt:  # one PV per tile: the owning group's
            pv_count = 2 if mutation == "alt_pvdone_count_2" else 1
            v_count = 1
        else:
            pv_count = 1 if mutation == "pvdone_count_1" else 2
            v_count = 2
        self.B = {"q": Bar("q", 1), "ofinal": Bar("ofinal", 1 if schedule == "split_single_issuer" else 2),
                  "list": Bar("list", 1)}
        for s in range(nk):
            self.B[f"kfull{s}"], self.B[f"kempty{s}"] = Bar(f"kfull{s}", 1), Bar(f"kempty{s}", 1)
        for s in range(nv):
            self.B[f"vfull{s}"], self.B[f"vempty{s}"] = Bar(f"vfull{s}", 1), Bar(f"vempty{s}", v_count)
        for b in range(2):
            self.B[f"sfull{b}"] = Bar(f"sfull{b}", 1)
            self.B[f"sfree{b}"] = Bar(f"sfree{b}", 2 if schedule == "split_dephase" else 1)
            self.B[f"pvg{b}"] = Bar(f"pvg{b}", 1)
            self.B[f"pvdone{b}"] = Bar(f"pvdone{b}", pv_count)
            for grp in range(2):
                self.B[f"pfull{b}{grp}"] = Bar(f"pfull{b}{grp}", 1)
        self.S = [None, None]          # (kind, tile, consumed): ("S", g) after QK(g), ("P", g) after softmax
        self.S_busy = [set(), set()]   # MMAs in flight on each S buffer
        self.halves = {}               # (buffer, tile) -> groups whose PV has completed
        self.K = [None] * nk
        self.V = [None] * nv
        self.O_busy = [0, 0]           # PVs in flight per accumulator
        self.P = [None, None]          # smem_p: tile whose P a group's shared-memory buffer holds
        self.P_busy = [0, 0]           # smem_p: PVs in flight reading each P buffer
        self.S_read = [None, None]     # smem_p: last tile whose S the group has read out of TMEM

    def buffer_of(self, g, t, bb):
        """S buffer and its use index for global tile g = t-th tile of the unit. "split": buffer
        g & 1, use g >> 1. "alternate": buffer t & 1 (the group), use bb[b] + (t >> 1), where bb
        counts each buffer's uses in earlier units."""
        if self.alt:
            b = t & 1
            return b, bb[b] + (t >> 1)
        return g & 1, g >> 1

    @staticmethod
    def advance(bb, T):
        bb[0] += (T + 1) >> 1
        bb[1] += T >> 1

    # ---- event machinery
    def later(self, fn):
        self.seq += 1
        self.events.append((self.now + self.rng.choice([1, 2, 5, 20, 60]), self.seq, fn))

    def run(self):
        if self.single:
            roles = {"producer": self.producer(), "mma": self.single_issuer(),
                     "sm0": self.softmax(0), "sm1": self.softmax(1)}
        elif self.dephase:
            roles = {"producer": self.producer(), "qk": self.dephase_qk(), "pv0": self.dephase_pv(0),
                     "pv1": self.dephase_pv(1), "sm0": self.dephase_softmax(0), "sm1": self.dephase_softmax(1)}
        elif self.smem_p:
            roles = {"producer": self.producer(), "is0": self.smem_issuer(0), "is1": self.smem_issuer(1),
                     "sm0": self.smem_softmax(0), "sm1": self.smem_softmax(1)}
        elif self.group_issuers:
            roles = {"producer": self.producer(), "is0": self.group_issuer(0), "is1": self.group_issuer(1),
                     "sm0": self.softmax(0), "sm1": self.softmax(1)}
        else:
            roles = {"producer": self.producer(), "qk": self.qk_issuer(), "pv0": self.pv_issuer(0),
                     "pv1": self.pv_issuer(1), "sm0": self.softmax(0), "sm1": self.softmax(1)}
        waiting = dict.fromkeys(roles)
        done, at_sync = set(), set()
        while True:
            moved = True
            while moved:
                moved = False
                for name, gen in roles.items():
                    if name in done or name in at_sync:
                        continue
                    if waiting[name] is not None:
                        bar, k = waiting[name]
                        if bar.n > k + 1:
                            raise AssertionError(f"stale wait: {name} waits phase {k} of {bar.name}, at {bar.n}")
                        if bar.n != k + 1:
                            continue
                        waiting[name] = None
                    try:
                        cmd = next(gen)
                    except StopIteration:
                        done.add(name)
                        moved = True
                        continue
                    moved = True
                    if cmd[0] == "wait":
                        waiting[name] = (self.B[cmd[1]], cmd[2])
                    else:  # "sync": the CTA-wide barrier at the end of a unit
                        at_sync.add(name)
                if at_sync and len(at_sync) == len(roles):
                    at_sync.clear()
                    moved = True
            if len(done) == len(roles):
                return
            if not self.events:
                raise AssertionError("deadlock: " + ", ".join(
                    f"{n} waits {w[0].name}[{w[1]}]" for n, w in waiting.items() if w))
            self.events.sort()
            self.now, _, fn = self.events.pop(0)
            fn()

    # ---- roles
    def producer(self):
        base = 0
        for u, T in enumerate(self.plan):
            self.later(self.B["q"].arrive)
            yield ("wait", "list", u)
            for t in range(T + 1):
                if t < T:
                    g = base + t
                    s = g % self.nk
                    if g >= self.nk:
                        yield ("wait", f"kempty{s}", g // self.nk - 1)

                    def load_k(s=s, g=g):
                        self.K[s] = g
                        self.B[f"kfull{s}"].arrive()
                    self.later(load_k)
                if t >= 1:
                    g = base + t - 1
                    s = g % self.nv
                    if g >= self.nv:
                        yield ("wait", f"vempty{s}", g // self.nv - (2 if self.mut == "vempty_one_back" else 1))

                    def load_v(s=s, g=g):
                        self.V[s] = g
                        self.B[f"vfull{s}"].arrive()
                    self.later(load_v)
            yield ("sync",)
            base += T

    def qk_issuer(self):
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            yield ("wait", "q", u)
            for t in range(T):
                g = base + t
                s = g % self.nk
                b, use = self.buffer_of(g, t, bb)
                # the kernel's order: the data-ready barrier first, the one that frees S[b] last
                yield ("wait", f"kfull{s}", g // self.nk)
                if t >= 2 and self.mut != "qk_skips_pvdone":
                    yield ("wait", f"pvdone{b}", use - 1)
                if self.S_busy[b]:
                    raise AssertionError(f"hazard: QK({g}) writes S{b} while {sorted(self.S_busy[b])} run")
                if self.S[b] is not None and self.S[b][0] == "P" and not self.S[b][2]:
                    raise AssertionError(f"hazard: QK({g}) overwrites P({self.S[b][1]}) before its PVs completed")
                if self.K[s] != g:
                    raise AssertionError(f"hazard: QK({g}) reads K stage {s} holding tile {self.K[s]}")
                self.S_busy[b].add(("QK", g))

                def qk_done(b=b, s=s, g=g):
                    self.S_busy[b].discard(("QK", g))
                    self.S[b] = ("S", g, False)
                    self.B[f"sfull{b}"].arrive()
                    self.B[f"kempty{s}"].arrive()
                self.later(qk_done)
            yield ("sync",)
            base += T
            self.advance(bb, T)

    def pv_issuer(self, grp):
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            for t in range(T):
                g = base + t
                s = g % self.nv
                b, use = self.buffer_of(g, t, bb)
                if self.alt and b != grp:
                    continue  # the other group's tile
                yield ("wait", f"vfull{s}", g // self.nv)  # V lands first; P is the last wait
                yield ("wait", f"pfull{b}{grp}", use)
                if self.S[b] is None or self.S[b][:2] != ("P", g):
                    raise AssertionError(f"hazard: PV{grp}({g}) finds {self.S[b]} in S{b}")
                if self.V[s] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) reads V stage {s} holding tile {self.V[s]}")
                self.S_busy[b].add(("PV", g, grp))
                self.O_busy[grp] += 1

                def pv_done(b=b, s=s, g=g):
                    self.S_busy[b].discard(("PV", g, grp))
                    self.O_busy[grp] -= 1
                    if self.V[s] != g:
                        raise AssertionError(f"hazard: V stage {s} overwritten during PV({g})")
                    self.halves.setdefault((b, g), set()).add(grp)
                    if self.halves[(b, g)] == ({grp} if self.alt else {0, 1}):
                        self.S[b] = ("P", g, True)
                    self.B[f"vempty{s}"].arrive()
                    self.B[f"pvdone{b}"].arrive()
                self.later(pv_done)

            def final_commit():
                if self.O_busy[grp]:  # a commit arrives once this thread's MMAs have completed
                    self.later(final_commit)
                else:
                    self.B["ofinal"].arrive()
            self.later(final_commit)
            yield ("sync",)
            base += T
            self.advance(bb, T)

    def group_issuer(self, grp):
        """One thread issues both products of group grp: for each of the group's tiles, QK^T into
        S[grp], then (once P is written) PV into O_grp; the next QK^T waits for that PV."""
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            yield ("wait", "q", u)
            for t in range(grp, T, 2):
                g = base + t
                b, use = self.buffer_of(g, t, bb)
                sk, sv = g % self.nk, g % self.nv
                if t >= 2 and self.mut != "qk_skips_pvdone":
                    yield ("wait", f"pvdone{b}", use - 1)
                yield ("wait", f"kfull{sk}", g // self.nk)
                if self.S_busy[b]:
                    raise AssertionError(f"hazard: QK({g}) writes S{b} while {sorted(self.S_busy[b])} run")
                if self.S[b] is not None and self.S[b][0] == "P" and not self.S[b][2]:
                    raise AssertionError(f"hazard: QK({g}) overwrites P({self.S[b][1]}) before its PV completed")
                if self.K[sk] != g:
                    raise AssertionError(f"hazard: QK({g}) reads K stage {sk} holding tile {self.K[sk]}")
                self.S_busy[b].add(("QK", g))

                def qk_done(b=b, s=sk, g=g):
                    self.S_busy[b].discard(("QK", g))
                    self.S[b] = ("S", g, False)
                    self.B[f"sfull{b}"].arrive()
                    self.B[f"kempty{s}"].arrive()
                self.later(qk_done)
                yield ("wait", f"pfull{b}{grp}", use)
                yield ("wait", f"vfull{sv}", g // self.nv)
                if self.S[b] is None or self.S[b][:2] != ("P", g):
                    raise AssertionError(f"hazard: PV{grp}({g}) finds {self.S[b]} in S{b}")
                if self.V[sv] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) reads V stage {sv} holding tile {self.V[sv]}")
                self.S_busy[b].add(("PV", g, grp))
                self.O_busy[grp] += 1

                def pv_done(b=b, s=sv, g=g):
                    self.S_busy[b].discard(("PV", g, grp))
                    self.O_busy[grp] -= 1
                    if self.V[s] != g:
                        raise AssertionError(f"hazard: V stage {s} overwritten during PV({g})")
                    self.S[b] = ("P", g, True)
                    self.B[f"vempty{s}"].arrive()
                    self.B[f"pvdone{b}"].arrive()
                self.later(pv_done)

            def final_commit():
                if self.O_busy[grp]:
                    self.later(final_commit)
                else:
                    self.B["ofinal"].arrive()
            self.later(final_commit)
            yield ("sync",)
            base += T
            self.advance(bb, T)

    # ---- split columns, one thread issuing every product; its MMAs complete in issue order
    def in_order(self, fn):
        """Schedule an MMA completion no earlier than the previous MMA of the same thread."""
        self.seq += 1
        when = max(self.now + self.rng.choice([1, 2, 5, 20, 60]), getattr(self, "last_mma", 0))
        self.last_mma = when
        self.events.append((when, self.seq, fn))

    def single_issuer(self):
        base = 0
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            yield ("wait", "q", u)

            def qk(t):
                g = base + t
                b, s = g & 1, g % self.nk
                yield ("wait", f"kfull{s}", g // self.nk)
                if self.K[s] != g:
                    raise AssertionError(f"hazard: QK({g}) reads K stage {s} holding tile {self.K[s]}")
                self.S_busy[b].add(("QK", g))

                def qk_done(b=b, s=s, g=g):
                    # in issue order, every PV that read the previous P of S[b] has completed
                    if any(x[0] == "PV" for x in self.S_busy[b]):
                        raise AssertionError(f"hazard: QK({g}) wrote S{b} while a PV still read it")
                    self.S_busy[b].discard(("QK", g))
                    self.S[b] = ("S", g, False)
                    self.B[f"sfull{b}"].arrive()
                    self.B[f"kempty{s}"].arrive()
                self.in_order(qk_done)
            for t in range(min(T, 2)):
                yield from qk(t)
            for t in range(T):
                g = base + t
                b, s = g & 1, g % self.nv
                yield ("wait", f"vfull{s}", g // self.nv)
                for grp in range(2):
                    yield ("wait", f"pfull{b}{grp}", g >> 1)
                    if self.S[b] is None or self.S[b][:2] != ("P", g):
                        raise AssertionError(f"hazard: PV{grp}({g}) finds {self.S[b]} in S{b}")
                    self.S_busy[b].add(("PV", g, grp))
                    self.O_busy[grp] += 1

                    def pv_done(b=b, g=g, grp=grp):
                        self.S_busy[b].discard(("PV", g, grp))
                        self.O_busy[grp] -= 1
                    self.in_order(pv_done)
                if self.V[s] != g:
                    raise AssertionError(f"hazard: PV({g}) reads V stage {s} holding tile {self.V[s]}")

                def commit(b=b, s=s, g=g):
                    if self.V[s] != g:
                        raise AssertionError(f"hazard: V stage {s} overwritten during PV({g})")
                    self.S[b] = ("P", g, True)
                    self.B[f"vempty{s}"].arrive()
                    self.B[f"pvdone{b}"].arrive()
                self.in_order(commit)
                if t + 2 < T:
                    yield from qk(t + 2)
            self.in_order(lambda: self.B["ofinal"].arrive())
            yield ("sync",)
            base += T

    # ---- split columns, P in shared memory, group 1 a phase behind
    def dephase_qk(self):
        base = 0
        self.reads = {}  # tile -> groups that have read their half of its S
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            yield ("wait", "q", u)
            for t in range(T):
                g = base + t
                b, s = g & 1, g % self.nk
                if t >= 2 and self.mut != "qk_skips_sfree":
                    yield ("wait", f"sfree{b}", (g - 2) >> 1)
                yield ("wait", f"kfull{s}", g // self.nk)
                if self.S_busy[b]:
                    raise AssertionError(f"hazard: QK({g}) writes S{b} while {sorted(self.S_busy[b])} run")
                if self.S[b] is not None and self.reads.get(self.S[b][1], set()) != {0, 1}:
                    raise AssertionError(f"hazard: QK({g}) overwrites S({self.S[b][1]}) before both halves were read")
                if self.K[s] != g:
                    raise AssertionError(f"hazard: QK({g}) reads K stage {s} holding tile {self.K[s]}")
                self.S_busy[b].add(("QK", g))

                def qk_done(b=b, s=s, g=g):
                    self.S_busy[b].discard(("QK", g))
                    self.S[b] = ("S", g, False)
                    self.B[f"sfull{b}"].arrive()
                    self.B[f"kempty{s}"].arrive()
                self.later(qk_done)
            yield ("sync",)
            base += T

    def dephase_pv(self, grp):
        base = 0
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            for t in range(T):
                g = base + t
                b, s = g & 1, g % self.nv
                yield ("wait", f"pfull{b}{grp}", g >> 1)
                yield ("wait", f"vfull{s}", g // self.nv)
                if self.P[grp] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) finds P of {self.P[grp]}")
                if self.V[s] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) reads V stage {s} holding tile {self.V[s]}")
                self.P_busy[grp] += 1
                self.O_busy[grp] += 1

                def pv_done(s=s, g=g):
                    self.P_busy[grp] -= 1
                    self.O_busy[grp] -= 1
                    if self.V[s] != g:
                        raise AssertionError(f"hazard: V stage {s} overwritten during PV({g})")
                    self.B[f"vempty{s}"].arrive()
                    self.B[f"pvg{grp}"].arrive()
                self.later(pv_done)

            def final_commit():
                if self.O_busy[grp]:
                    self.later(final_commit)
                else:
                    self.B["ofinal"].arrive()
            self.later(final_commit)
            yield ("sync",)
            base += T

    def dephase_softmax(self, grp):
        base = 0
        for u, T in enumerate(self.plan):
            if self.route_in_kernel:
                yield ("wait", "q", u)
            if grp == 0:
                self.B["list"].arrive()
            else:
                yield ("wait", "list", u)

            def read(g, release):
                b = g & 1
                if self.S[b] is None or self.S[b][:2] != ("S", g):
                    raise AssertionError(f"hazard: softmax{grp}({g}) finds {self.S[b]} in S{b}")
                if release:
                    self.reads.setdefault(g, set()).add(grp)
                    self.B[f"sfree{b}"].arrive()

            def weights(t):
                g = base + t
                if grp == 1:
                    read(g, True)  # the scores are read again, then released
                if t >= 1 and self.mut != "p_skips_pvdone":
                    yield ("wait", f"pvg{grp}", g - 1)
                if self.P_busy[grp]:
                    raise AssertionError(f"hazard: softmax{grp}({g}) overwrites P while a PV reads it")
                if self.O_busy[grp]:
                    raise AssertionError(f"hazard: rescale of O{grp} at tile {g} with a PV in flight")
                self.P[grp] = g
                self.B[f"pfull{g & 1}{grp}"].arrive()

            def maxes(t):
                g = base + t
                yield ("wait", f"sfull{g & 1}", g >> 1)
                read(g, grp == 0)

            for it in range(T + grp):
                if grp == 1 and it >= 1:
                    yield from weights(it - 1)
                if it < T:
                    yield from maxes(it)
                if grp == 0:
                    yield from weights(it)
            if T > 0:
                yield ("wait", "ofinal", u)
                if any(self.O_busy):
                    raise AssertionError("hazard: the epilogue reads O with a PV in flight")
            yield ("sync",)
            base += T

    def smem_issuer(self, grp):
        """Group grp's issuer with P in shared memory: the next QK^T into S[grp] waits only for the
        softmax to have read S out of TMEM; the PV reads P from the group's shared buffer."""
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            yield ("wait", "list", u)
            yield ("wait", "q", u)

            def qk(t):
                g = base + t
                sk = g % self.nk
                yield ("wait", f"kfull{sk}", g // self.nk)
                if self.S_busy[grp]:
                    raise AssertionError(f"hazard: QK({g}) writes S{grp} while {sorted(self.S_busy[grp])} run")
                if self.S[grp] is not None and self.S[grp][0] == "S" and self.S_read[grp] != self.S[grp][1]:
                    raise AssertionError(f"hazard: QK({g}) overwrites S({self.S[grp][1]}) before it was read")
                if self.K[sk] != g:
                    raise AssertionError(f"hazard: QK({g}) reads K stage {sk} holding tile {self.K[sk]}")
                self.S_busy[grp].add(("QK", g))

                def qk_done(s=sk, g=g):
                    self.S_busy[grp].discard(("QK", g))
                    self.S[grp] = ("S", g, False)
                    self.B[f"sfull{grp}"].arrive()
                    self.B[f"kempty{s}"].arrive()
                self.later(qk_done)
            if grp < T:
                yield from qk(grp)
            for t in range(grp, T, 2):
                g = base + t
                _, use = self.buffer_of(g, t, bb)
                if t + 2 < T:
                    if self.mut != "qk_skips_sfree":
                        yield ("wait", f"sfree{grp}", use)
                    yield from qk(t + 2)
                sv = g % self.nv
                yield ("wait", f"pfull{grp}{grp}", use)
                yield ("wait", f"vfull{sv}", g // self.nv)
                if self.P[grp] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) finds P of {self.P[grp]}")
                if self.V[sv] != g:
                    raise AssertionError(f"hazard: PV{grp}({g}) reads V stage {sv} holding tile {self.V[sv]}")
                self.P_busy[grp] += 1
                self.O_busy[grp] += 1

                def pv_done(s=sv, g=g):
                    self.P_busy[grp] -= 1
                    self.O_busy[grp] -= 1
                    if self.V[s] != g:
                        raise AssertionError(f"hazard: V stage {s} overwritten during PV({g})")
                    self.B[f"vempty{s}"].arrive()
                    self.B[f"pvdone{grp}"].arrive()
                self.later(pv_done)

            def final_commit():
                if self.O_busy[grp]:
                    self.later(final_commit)
                else:
                    self.B["ofinal"].arrive()
            self.later(final_commit)
            yield ("sync",)
            base += T
            self.advance(bb, T)

    def smem_softmax(self, grp):
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            if self.route_in_kernel:
                yield ("wait", "q", u)
            if grp == 0:
                self.B["list"].arrive()
            else:
                yield ("wait", "list", u)
            for t in range(grp, T, 2):
                g = base + t
                _, use = self.buffer_of(g, t, bb)
                yield ("wait", f"sfull{grp}", use)
                if self.S[grp] is None or self.S[grp][:2] != ("S", g):
                    raise AssertionError(f"hazard: softmax{grp}({g}) finds {self.S[grp]} in S{grp}")
                if t >= 2 and self.mut != "p_skips_pvdone":
                    yield ("wait", f"pvdone{grp}", use - 1)
                self.S_read[grp] = g
                self.B[f"sfree{grp}"].arrive()
                # writes P and may rescale O: both must be at rest
                if self.P_busy[grp]:
                    raise AssertionError(f"hazard: softmax{grp}({g}) overwrites P while a PV reads it")
                if self.O_busy[grp]:
                    raise AssertionError(f"hazard: rescale of O{grp} at tile {g} with a PV in flight")
                self.P[grp] = g
                self.B[f"pfull{grp}{grp}"].arrive()
            if T > 0:
                yield ("wait", "ofinal", u)
                if any(self.O_busy):
                    raise AssertionError("hazard: the epilogue reads O with a PV in flight")
            yield ("sync",)
            base += T
            self.advance(bb, T)

    def softmax(self, grp):
        base, bb = 0, [0, 0]
        for u, T in enumerate(self.plan):
            if self.route_in_kernel:
                yield ("wait", "q", u)  # q_bar comes from the Q tile in shared memory
            if grp == 0:
                self.B["list"].arrive()  # thread 0 of the softmax warps publishes the tile lists
            else:
                yield ("wait", "list", u)
            started = False
            for t in range(T):
                g = base + t
                b, use = self.buffer_of(g, t, bb)
                if self.alt and b != grp:
                    continue  # the other group's tile
                yield ("wait", f"sfull{b}", use)
                if self.S[b] is None or self.S[b][:2] not in (("S", g), ("P", g)):
                    raise AssertionError(f"hazard: softmax{grp}({g}) finds {self.S[b]} in S{b}")
                if self.alt:
                    # a lazy rescale may come at any tile after the group's first: O_grp must be at rest
                    if started and self.rng.random() < 0.5 and self.O_busy[grp]:
                        raise AssertionError(f"hazard: rescale of O{grp} at tile {g} with a PV in flight")
                    started = True
                    self.S[b] = ("P", g, False)
                    self.B[f"pfull{b}{grp}"].arrive()
                    continue
                if t > 0 and self.rng.random() < 0.3:
                    # a lazy rescale of O_grp: wait for the previous tile's PVs, then O_grp must be at rest
                    yield ("wait", f"pvdone{(g - 1) & 1}", (g - 1) >> 1)
                    if self.O_busy[grp]:
                        raise AssertionError(f"hazard: rescale of O{grp} at tile {g} with a PV in flight")
                self.S[b] = ("P", g, False)
                self.B[f"pfull{b}{grp}"].arrive()
            if T > 0:
                yield ("wait", "ofinal", u)
                if any(self.O_busy):
                    raise AssertionError("hazard: the epilogue reads O with a PV in flight")
            yield ("sync",)
            base += T
            self.advance(bb, T)


def random_plan(rng):
    return [rng.choice([1, 1, 2, 3, 4, 5, 7, 8, 13]) for _ in range(rng.randint(1, 6))]
