"""Model check of the chain kernel's mbarrier protocol (chain_fwd.cu), on the CPU.

The chain kernel hands work between three roles through mbarriers: a loader
thread (record tensor loads into double buffers), an issuer thread (the UMMA
products and their commits) and sixteen compute warps, grouped here by TMEM
lane quarter (lanes 0..63 form Vnew, lanes 64..127 read the output block,
all update the state).  This file restates that protocol as four kinds of
sequential programs and runs them under random interleavings, with tensor
loads completing in any order and products completing in issue order.

Checked on every run:
- every wait names the phase index it expects, and the hardware's parity test
  answers it unambiguously at every poll (the barrier has completed exactly
  that phase or the one before it; two phases ahead would alias);
- no barrier has more completions in flight than the protocol allows;
- no buffer (record slots, Vnew, S0, V^T, the output accumulators) is
  overwritten while a pending product or a compute warp may still read it;
- every run terminates (no deadlock).

The mutation tests remove one wait or arrival each and require the checker to
notice, so the checks above are not vacuous.
"""
import random

import pytest


class Barrier:
    """An mbarrier: `count` arrivals complete a phase; async completions arm it first."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done_phases, self.armed = name, count, count, 0, 0

    def arm(self):
        self.armed += 1
        assert self.armed <= 2, f"{self.name}: more than two completions in flight"

    def complete(self):
        assert self.armed > 0, f"{self.name}: completion without an armed operation"
        self.armed -= 1
        self.arrive()

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        if self.pending == 0:
            self.done_phases += 1
            self.pending = self.count

    def test(self, phase):
        """try_wait.parity for phase index `phase` (only its parity reaches the hardware)."""
        assert self.done_phases in (phase, phase + 1), (
            f"{self.name}: wait for phase {phase} with {self.done_phases} completed (parity alias)")
        return self.done_phases == phase + 1


class Protocol:
    """The barriers, buffers and the three kinds of programs for N chunks."""

    def __init__(self, nchunks, wq_buffers, mutation=None):
        self.N, self.WS, self.mut = nchunks, wq_buffers, mutation
        self.bars = {}
        for name in ("w0", "w1", "p0", "p1", "k0", "k1", "t0", "t1", "m1", "mb", "m3",
                     "we0", "we1", "te0", "te1", "pe0", "pe1"):
            self.bars[name] = Barrier(name)
        # compute-warp barriers; counts are lane-quarter groups (4 warps each in the kernel)
        for name, count in (("s0", 4), ("vt", 4), ("ke0", 4), ("ke1", 4),
                            ("vn0", 2), ("vn1", 2), ("out0", 2), ("out1", 2)):
            self.bars[name] = Barrier(name, count)
        self.buf = {}  # buffer -> what it holds: a chunk index, or (product, chunk) for D1

    def wait(self, bar, phase):
        while not self.bars[bar].test(phase):
            yield "blocked"

    def skip(self, what):
        return self.mut == what

    # ------------------------------------------------------------------ loader
    def loader(self):
        N, WS = self.N, self.WS

        def load(bar, slot, j):
            self.bars[bar].arm()
            yield ("async", (bar,), ("load", slot, j))

        for j in range(N):
            s, ph = j & 1, (j - 2) >> 1
            if j >= 2 and not self.skip("loader T' empty"):
                yield from self.wait(f"te{s}", ph)
            yield from load(f"t{s}", f"T{s}", j)
            if j >= 2:
                yield from self.wait(f"ke{s}", ph)
            yield from load(f"k{s}", f"K{s}", j)
            if j >= WS:
                yield from self.wait(f"we{j % WS}", (j - WS) // WS)
            yield from load(f"w{j % WS}", f"W{j % WS}", j)
            if j >= 2 and not self.skip("loader P empty"):
                yield from self.wait(f"pe{s}", ph)
            yield from load(f"p{s}", f"P{s}", j)

    # ------------------------------------------------------------------ issuer
    def issuer(self):
        N, WS = self.N, self.WS

        def product(bars, reads, name, writes=()):
            for b in bars:
                self.bars[b].arm()
            yield ("async", tuple(bars), ("mma", name, tuple(reads), tuple(writes)))

        def product_u(n):  # U = T'(n) V(n)
            yield from self.wait("vt", n)
            yield from self.wait(f"t{n & 1}", n >> 1)
            yield from product([f"te{n & 1}"] if n + 2 < N else [], [(f"T{n & 1}", n), ("VT", n)], f"U{n}")

        def product_3b(n):  # output rows += P(n) Vnew(n)
            yield from product(["mb"] + ([f"pe{n & 1}"] if n + 2 < N else []),
                               [(f"P{n & 1}", n), (f"VN{n & 1}", n), (f"D1_{n & 1}", ("1", n))], f"3b{n}",
                               writes=[(f"D1_{n & 1}", ("3b", n))])

        yield from product_u(0)
        for n in range(N):
            yield from self.wait("s0", n)
            yield from self.wait(f"w{n % WS}", n // WS)
            if n >= 2 and not self.skip("issuer output read"):
                yield from self.wait(f"out{n & 1}", (n - 2) >> 1)
            yield from product(["m1"] + ([f"we{n % WS}"] if n + WS < N else []),
                               [(f"W{n % WS}", n), ("S0", n)], f"1_{n}", writes=[(f"D1_{n & 1}", ("1", n))])
            if n >= 1:
                yield from self.wait(f"p{(n - 1) & 1}", (n - 1) >> 1)
                yield from product_3b(n - 1)
            if not self.skip("issuer Vnew"):
                yield from self.wait(f"vn{n & 1}", n >> 1)
            yield from self.wait(f"k{n & 1}", n >> 1)
            yield from product(["m3"], [(f"K{n & 1}", n), (f"VN{n & 1}", n)], f"3a{n}")
            if n + 1 < N:
                yield from product_u(n + 1)
        if N >= 2:
            yield from self.wait(f"out{N & 1}", (N - 2) >> 1)
        yield from self.wait(f"p{(N - 1) & 1}", (N - 1) >> 1)
        yield from product_3b(N - 1)

    # --------------------------------------------------------- compute warps
    def quarter(self, lq):
        """The four compute warps of TMEM lane quarter lq."""
        N, buf = self.N, self.buf

        def write(slot, j):
            buf[slot] = j
            yield "step"

        yield from write("S0", 0)
        self.bars["s0"].arrive()
        yield from write("VT", 0)
        self.bars["vt"].arrive()
        for n in range(N):
            yield from self.wait("m1", n)
            if lq < 2:  # Vnew(n) = U - W S0 (tokens of this quarter)
                yield from write(f"VN{n & 1}", n)
                self.bars[f"vn{n & 1}"].arrive()
            elif n >= 1:  # output block of chunk n-1
                if not self.skip("output waits 3b"):
                    yield from self.wait("mb", n - 1)
                assert buf.get(f"D1_{(n - 1) & 1}") == ("3b", n - 1), "output block read before 3b or after reuse"
                self.bars[f"out{(n - 1) & 1}"].arrive()
            if n + 1 < N:  # V^T(n+1): U(n) completed before product 1(n)
                yield from write("VT", n + 1)
                self.bars["vt"].arrive()
            yield from self.wait("m3", n)
            yield from self.wait(f"k{n & 1}", n >> 1)
            assert buf.get(f"K{n & 1}") == n, "e^{Gamma_C} read from a refilled buffer"
            if n + 2 < N and not self.skip("compute K-hat release"):
                self.bars[f"ke{n & 1}"].arrive()
            yield from write("S0", n + 1)
            self.bars["s0"].arrive()
        if lq >= 2:
            yield from self.wait("mb", N - 1)
            assert buf.get(f"D1_{(N - 1) & 1}") == ("3b", N - 1)

    # -------------------------------------------------------------- scheduler
    def run(self, seed):
        rnd = random.Random(seed)
        progs = {"loader": self.loader(), "issuer": self.issuer()}
        for lq in range(4):
            progs[f"q{lq}"] = self.quarter(lq)
        inflight = []  # (barriers, op)
        steps = 0
        while progs or inflight:
            steps += 1
            assert steps < 200000, "deadlock"
            who = rnd.choice(list(progs) + (["async"] * 2 if inflight else []))
            if who == "async":
                mmas = [x for x in inflight if x[1][0] == "mma"]
                loads = [x for x in inflight if x[1][0] == "load"]
                pool = rnd.choice([p for p in (mmas, loads) if p])
                op = pool[0] if pool is mmas else rnd.choice(pool)  # products in order, loads in any order
                inflight.remove(op)
                bars, what = op
                if what[0] == "mma":
                    for slot, j in what[2]:
                        assert self.buf.get(slot) == j, f"product {what[1]} read {slot} holding {self.buf.get(slot)}"
                    for slot, j in what[3]:
                        self.buf[slot] = j
                else:
                    self.buf[what[1]] = what[2]
                for b in bars:
                    self.bars[b].complete()
                continue
            try:
                ev = next(progs[who])
            except StopIteration:
                del progs[who]
                continue
            if isinstance(ev, tuple) and ev[0] == "async":
                bars, what = ev[1], ev[2]
                if what[0] == "load":
                    for _, other in inflight:
                        if other[0] == "mma":
                            assert all(slot != what[1] for slot, _ in other[2]), (
                                f"load into {what[1]} while product {other[1]} may read it")
                inflight.append((bars, what))
        for b in self.bars.values():
            assert b.armed == 0, f"{b.name}: completion still in flight at exit"


@pytest.mark.parametrize("wq_buffers", [1, 2])
def test_chain_protocol_random_interleavings(wq_buffers):
    for n in range(1, 8):
        for seed in range(60):
            Protocol(n, wq_buffers).run(seed)


@pytest.mark.parametrize("mutation", [
    "loader T' empty", "loader P empty", "issuer Vnew", "output waits 3b", "compute K-hat release",
])
def test_chain_protocol_mutations_are_caught(mutation):
    """Each planted protocol mistake must trip an assertion in some interleaving."""
    with pytest.raises(AssertionError):
        for n in range(2, 8):
            for seed in range(200):
                Protocol(n, 2, mutation).run(seed)
