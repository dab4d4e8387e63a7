"""Host models of the mbarrier protocols of the two tcgen05 kernels that hand work
between warps: the sequence-parallel GDN kernel (gdn_seq.cu) and the softmax
attention kernel (gdn_attn.cu).

Each warp role is a coroutine that takes the kernel's waits and arrivals in the
kernel's order; copies and MMAs are asynchronous events that complete in any order
(a commit only after every earlier MMA of its warp).  A random scheduler interleaves
them, with one role slowed in some runs.  Every run must end, every parity wait must
find its barrier exactly one phase on (two phases on and the parity wait could never
succeed), and every buffer written must have been released by its readers.  Planted
protocol mistakes must be caught, so that the models are known to have teeth.

These are models written from the kernels' sources, not the kernels: they check the
protocol's design on the CPU (no GPU needed).
"""

import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class _World:
    """Barriers, in-flight asynchronous events and the set of completed events."""

    def __init__(self, counts, rnd):
        self.counts, self.rnd = counts, rnd
        self.bars, self.inflight, self.done, self.issued = {}, [], set(), {}

    def bar(self, name):
        if name not in self.bars:
            self.bars[name] = _Bar(self.counts(name))
        return self.bars[name]

    def wait(self, name, phase):
        b = self.bar(name)
        while b.done < phase + 1:
            yield
        assert b.done == phase + 1, f"parity alias: {name} waited for phase {phase}, found {b.done} done"

    def arrive(self, name):
        self.bar(name).arrive()

    def async_op(self, warp, ev, arrivals):
        prior = list(self.issued.setdefault(warp, []))
        self.issued[warp].append(ev)
        self.inflight.append((ev, prior, arrivals))

    def need(self, *evs):
        for e in evs:
            assert e in self.done, f"hazard: needs {e} done"

    def run(self, procs, max_steps=400000):
        alive = list(procs)
        slow = self.rnd.choice([None] + list(range(len(procs))))
        steps = 0
        while alive or self.inflight:
            steps += 1
            assert steps < max_steps, "deadlock"
            ready = [x for x in self.inflight if all(p in self.done for p in x[1])]
            if ready and (not alive or self.rnd.random() < 0.25):
                x = self.rnd.choice(ready)
                self.inflight.remove(x)
                self.done.add(x[0])
                for a in x[2]:
                    self.arrive(a)
                continue
            assert alive, "deadlock (nothing can complete)"
            weights = [0.03 if (slow is not None and p is procs[slow]) else 1.0 for p in alive]
            p = self.rnd.choices(alive, weights)[0]
            try:
                next(p)
            except StopIteration:
                alive.remove(p)


# ---------------------------------------------------------------- sequence-parallel kernel

_SEQ_COUNTS = dict(SREADY=8, PEGO=8, EREADY=4, OREADY=4, WREADY=4, FULL0=2, FULL1=2, GFREE=2)


def _seq_run(N, seed, mutation=None, early_release=False, pieces=None):
    """One stretch of N chunks (bf16 path): loader, Gram, W/U, chain-MMA, prep (as one
    role: its eight warps meet at named barriers) and the eight chain/output warps.
    The kernel releases a stage (K, Q, -W, scalars and its P tile) once P E has run.
    early_release models the alternative measured slower on the GPU: the stage
    released once MMA2 has read it, the P tile separately after P E (PFREE), and
    e^G/|q| read by the output warps as soon as READY arrives.
    pieces: lengths of the chains' pieces the CTA runs one after another (default one
    piece of N chunks); a piece's last chunk writes the state out instead of handing
    it on, and the next piece starts from its own initial state (chain_init)."""
    pieces = pieces or [N]
    assert sum(pieces) == N
    starts = {sum(pieces[:i]) for i in range(len(pieces))}
    ends = {sum(pieces[:i + 1]) - 1 for i in range(len(pieces))}
    w = _World(lambda name: _SEQ_COUNTS.get(name, 1), random.Random(seed))
    ready = (lambda s: "READY") if mutation == "one READY barrier" else (lambda s: f"READY{s}")
    ready_ph = (lambda n: n) if mutation == "one READY barrier" else (lambda n: n >> 1)
    for _ in range(8):                       # the chain warps' initial state: S of chunk 0 ready
        w.arrive("SREADY")
    w.done.add(("sread", 0))

    def loader():
        for n in range(N):
            s = n & 1
            if n >= 2:
                if mutation != "no SFREE wait":
                    yield from w.wait(f"SFREE{s}", (n - 2) >> 1)
                # the stage's K, Q, W and gate scalars are rewritten
                w.need(("gram", n - 2), ("wu", n - 2), ("m1", n - 2), ("m2", n - 2))
            w.async_op("loader", ("kq", n), [f"FULL{s}"])    # expect_tx arrival + the copy
            yield
            w.arrive(f"FULL{s}")                             # the gate scan written

    def gram():
        for n in range(N):
            s = n & 1
            yield from w.wait(f"FULL{s}", n >> 1)
            if n > 0 and mutation != "no GFREE wait":
                yield from w.wait("GFREE", n - 1)
            w.async_op("gram", ("gram", n), ["G1"])

    def wu():
        w.async_op("wu", ("v", 0), ["VFULL"])
        for n in range(N):
            s = n & 1
            if mutation != "no TREADY wait":
                yield from w.wait("TREADY", n)
            yield from w.wait("VFULL", n)
            if n >= 2:
                yield from w.wait(f"EQFREE{s}", (n - 2) >> 1)
                w.need(("store", n - 2))             # EQS[s] read out by the output of n - 2
            w.need(("tw", n), ("v", n))              # T, T' and the v tile of this chunk
            w.async_op("wu", ("wu", n), [f"WU{s}", "VFREE"])
            if n + 1 < N:
                if mutation != "no VFREE wait":
                    yield from w.wait("VFREE", n)
                w.need(("wu", n))                    # the v tile rewritten after the U MMA read it
                w.async_op("wu", ("v", n + 1), ["VFULL"])

    def chain_mma():
        for n in range(N):
            s = n & 1
            yield from w.wait(ready(s), ready_ph(n))
            yield from w.wait("WREADY", n)
            yield from w.wait("SREADY", n)
            w.need(("sread", n))
            w.async_op("cm", ("m1", n), ["M1"])
            yield from w.wait("EREADY", n)
            if n > 0:
                w.need(*(("rb", n - 1, q) for q in range(8)))   # SACC read back and decayed
            w.async_op("cm", ("m2", n), ["M2"] + ([f"SFREE{s}"] if early_release else []))
            yield from w.wait("PEGO", n)
            w.async_op("cm", ("pe", n), ["PEDONE"] + ([f"PFREE{s}"] if early_release else [f"SFREE{s}"]))

    def prep():
        for n in range(N):
            s = n & 1
            yield from w.wait(f"FULL{s}", n >> 1)
            yield from w.wait("G1", n)
            yield
            if n >= 2:
                # the chunk's per-row scalars (1/|k| e^{G_L-G}, e^G/|q|) into the stage
                w.need(*(("dl", n - 2, q) for q in range(4, 8)), *(("gq", n - 2, q) for q in range(4)))
            w.done.add(("cs", n))
            if n >= 2 and early_release and mutation != "no PFREE wait":
                yield from w.wait(f"PFREE{s}", (n - 2) >> 1)
            yield
            if n >= 2:
                w.need(("pe", n - 2))                # P[s] rewritten
            w.arrive("GFREE")
            w.arrive("GFREE")
            yield
            if n > 0:
                yield from w.wait(f"WU{(n - 1) & 1}", (n - 1) >> 1)
                w.need(("wu", n - 1))                # T, T' rewritten
            yield
            w.done.add(("tw", n))
            w.arrive("TREADY")
            w.arrive(ready(s))

    def chain_warp(q):
        A = q < 4                                    # TMEM lanes 0-63; q == 0 stores the output
        for n in range(N):
            s = n & 1
            last = n in ends
            if n in starts and n > 0:
                # chain_init: the S tile and SACC from the new piece's initial state
                w.need(("m1", n - 1), ("m2", n - 1))
                yield
                w.done.add(("rb", n - 1, q))
                w.done.add(("sread", n))
                w.arrive("SREADY")
            yield from w.wait(ready(s), ready_ph(n))
            if A and early_release and mutation != "late GQ read":
                w.need(("cs", n))
                w.done.add(("gq", n, q))             # e^G/|q| of the rows read at once
            if A:
                yield from w.wait(f"WU{s}", n >> 1)
                yield
                w.arrive("WREADY")
            yield from w.wait("M1", n)
            if not A:
                if n > 0:
                    w.need(("m2", n - 1))            # E' tile rewritten
                w.need(("cs", n))
                w.done.add(("dl", n, q))             # 1/|k| e^{G_L-G} read for E'
                yield
                w.arrive("EREADY")
                if n > 0:
                    yield from w.wait("OFREE", n - 1)
                    w.need(("pe", n - 1), ("store", n - 1))   # E tile rewritten
                yield
            else:
                yield
                if not (early_release and mutation != "late GQ read"):
                    w.need(("cs", n))
                    w.done.add(("gq", n, q))         # e^G/|q| read for the Q S scaling
            w.arrive("PEGO")
            if not last:
                yield from w.wait(f"FULL{(n + 1) & 1}", (n + 1) >> 1)
            yield from w.wait("M2", n)
            w.need(("m1", n))                        # S tile rewritten after MMA1 read it
            if not last:
                yield
                w.done.add(("rb", n, q))
                w.done.add(("sread", n + 1))
                w.arrive("SREADY")
            if A:
                yield from w.wait("PEDONE", n)
                w.need(("pe", n))                    # output rows into the E tile
                yield
                w.arrive("OREADY")
                if q == 0:
                    yield from w.wait("OREADY", n)
                    w.done.add(("store", n))
                    w.arrive("OFREE")
                    w.arrive(f"EQFREE{s}")

    w.run([loader(), gram(), wu(), chain_mma(), prep()] + [chain_warp(q) for q in range(8)])


@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("early_release", [False, True], ids=["stage_after_pe", "stage_after_mma2"])
def test_seq_kernel_protocol(N, early_release):
    for seed in range(60):
        _seq_run(N, seed, early_release=early_release)


@pytest.mark.parametrize("pieces", [[1, 1], [2, 3], [1, 4, 1], [3, 1, 2, 2]])
def test_seq_kernel_protocol_across_pieces(pieces):
    """A CTA's stretch spans the tail of one chain, whole chains and the head of another."""
    for seed in range(60):
        _seq_run(sum(pieces), seed, pieces=pieces)


@pytest.mark.parametrize("mutation", ["no SFREE wait", "one READY barrier", "no GFREE wait", "no VFREE wait",
                                      "no TREADY wait", "no PFREE wait", "late GQ read"])
def test_seq_kernel_protocol_model_catches_planted_mistakes(mutation):
    early = mutation in ("no PFREE wait", "late GQ read")     # mistakes of the early-release form
    caught = 0
    for seed in range(60):
        try:
            _seq_run(5, seed, mutation, early_release=early)
        except AssertionError:
            caught += 1
    assert caught > 0, f"the model missed: {mutation}"


# ---------------------------------------------------------------- softmax attention kernel

def _attn_run(n, seed, warps=16, mutation=None, KS=3, VS=2):
    """One CTA over n key tiles: the issuing warp and `warps` softmax warps.  Score
    buffers S[2], P buffers [2] with their P-written and P V-done barriers."""
    w = _World(lambda name: warps if name.startswith(("SFree", "PFull")) else 1, random.Random(seed))
    rnd = random.Random(seed + 7)
    one_pfull = mutation == "one PFull barrier"
    pf = (lambda j: "PFull") if one_pfull else (lambda j: f"PFull{j & 1}")
    pf_ph = (lambda j: j) if one_pfull else (lambda j: j >> 1)

    def producer():
        def load_k(j):
            if j >= KS:
                w.need(("S", j - KS))                # the K slot's previous tile read by its S
            w.async_op("dma", ("K", j), [f"K{j % KS}"])

        def load_v(j):
            if j >= VS:
                w.need(("PV", j - VS))               # the V slot's previous tile read by its P V
            w.async_op("dma", ("V", j), [f"V{j % VS}"])

        def start_s(j):
            yield from w.wait(f"K{j % KS}", j // KS)
            if j >= 2:
                w.need(*(("Sread", j - 2, q) for q in range(warps)))   # score buffer rewritten
            w.async_op("mma", ("S", j), [f"S{j & 1}"])

        for j in range(min(n, KS)):
            load_k(j)
        for j in range(min(n, VS)):
            load_v(j)
        yield from start_s(0)
        for j in range(n):
            if j + 1 < n:
                if j >= 1:
                    yield from w.wait(f"SFree{(j + 1) & 1}", (j - 1) >> 1)
                yield from start_s(j + 1)
            if j + KS < n:
                yield from w.wait(f"S{j & 1}", j >> 1)
                load_k(j + KS)
            if j >= 1 and j + 1 < n:
                yield from w.wait(f"PV{(j - 1) & 1}", (j - 1) >> 1)
                load_v(j + 1)
            yield from w.wait(pf(j), pf_ph(j))
            yield from w.wait(f"V{j % VS}", j // VS)
            w.need(*(("P", j, q) for q in range(warps)), ("V", j))
            w.async_op("mma", ("PV", j), [f"PV{j & 1}"])

    def softmax(q):
        for j in range(n):
            yield from w.wait(f"S{j & 1}", j >> 1)
            w.need(("S", j))
            w.done.add(("Sread", j, q))
            w.arrive(f"SFree{j & 1}")
            yield
            move = j > 0 and rnd.random() < 0.3      # the reference maximum moved: O is rescaled
            wait_for = j - 1 if move else j - 2
            if wait_for >= 0 and mutation != "no P V wait before P":
                yield from w.wait(f"PV{wait_for & 1}", wait_for >> 1)
            if j >= 2:
                w.need(("PV", j - 2))                # P buffer rewritten
            if move:
                w.need(("PV", j - 1))                # O rescaled after the last P V into it
            yield
            w.done.add(("P", j, q))
            w.arrive(pf(j))
        yield from w.wait(f"PV{(n - 1) & 1}", (n - 1) >> 1)

    w.run([producer()] + [softmax(q) for q in range(warps)])


@pytest.mark.parametrize("n", [1, 2, 3, 5, 9])
def test_attention_kernel_protocol(n):
    for seed in range(60):
        _attn_run(n, seed, warps=4)


@pytest.mark.parametrize("mutation", ["one PFull barrier", "no P V wait before P"])
def test_attention_protocol_model_catches_planted_mistakes(mutation):
    """A single P-written barrier for both P buffers is the form the kernel had before:
    the softmax can finish tile j + 1 before the issuing warp looks for tile j."""
    caught = 0
    for seed in range(100):
        try:
            _attn_run(6, seed, warps=4, mutation=mutation)
        except AssertionError:
            caught += 1
    assert caught > 0, f"the model missed: {mutation}"
