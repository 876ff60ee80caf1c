"""Model check of the fused kernels' mbarrier protocol, on the CPU: csrc/attn_fwd.cu (BF16, a 3-stage K / V
ring) and csrc/attn_fwd_fp8.cu (E4M3, the same protocol with 4 stages), both with 8 tile descriptors.

Each role of a CTA (K loader, V loader, S = Q K^T issuer, O += P V issuer, the two softmax
warpgroups, the tensor pipe and the TMA engine) is written as the sequence of barrier operations it
performs in the kernel, for a CTA with T tiles.  Random interleavings are explored and three
properties checked for every wait on phase k of a barrier with c completed phases:

* no premature wait: c >= k when the wait starts (with c = k - 1 a parity wait would pass at once);
* no aliasing: the barrier never completes phase k + 1 before the waiter has seen phase k
  (two phases ahead, the parity would repeat and the wait would hang);
* no deadlock: some role can always make progress until every role is done.

The kernel's bounded waits turn a violation into a timeout status; this check keeps the protocol
free of them by construction.
"""
import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


def _roles(T, S, D):
    last = T - 1
    W = lambda name, k: ("wait", name, k)        # wait for phase k of a barrier
    A = lambda name: ("arrive", name)            # a thread's arrive
    TMA = lambda name: ("tma", name)             # bulk copy completing on a barrier later
    MMA = lambda *names: ("mma", list(names))    # products, then commits, through the tensor pipe

    def kprod():
        yield TMA("qfull")
        for t in range(T):
            if t >= S:
                yield W(f"kempty{t % S}", t // S - 1)
            yield A(f"dfull{t % D}")
            yield TMA(f"kfull{t % S}")
        for u in range(max(0, T - S), T):          # drain: no copy left in flight
            yield W(f"kfull{u % S}", u // S)
        yield W("qfull", 0)

    def vprod():
        for u in range(T):
            yield W(f"dfull{u % D}", u // D)
            if u >= S:
                yield W(f"vempty{u % S}", u // S - 1)
            yield TMA(f"vfull{u % S}")
        for u in range(max(0, T - S), T):
            yield W(f"vfull{u % S}", u // S)

    def qk():
        yield W("qfull", 0)
        for t in range(T):
            yield W(f"kfull{t % S}", t // S)
            if t >= 1:
                yield W("sread", t - 1)
            yield MMA("sfull", f"kempty{t % S}")
        yield MMA("mmadone")
        yield W("mmadone", 0)

    def pv():
        for u in range(T):
            yield W(f"dfull{u % D}", u // D)
            yield W(f"vfull{u % S}", u // S)
            for w in range(2):
                yield W(f"pready{w}", u)
                yield MMA(f"pvdone{w}")
            yield MMA(f"vempty{u % S}")
        yield MMA("mmadone2")
        yield W("mmadone2", 0)

    def softmax(w):
        for t in range(T):
            yield W(f"dfull{t % D}", t // D)
            yield W("sfull", t)
            yield A("sread")                          # S is in registers
            if t > 0:
                yield W(f"pvdone{w}", t - 1)          # O rescale / P buffer reuse
            yield A(f"pready{w}")
        yield W(f"pvdone{w}", last)                   # the last P V before the epilogue
        yield A("lbar")
        yield W("lbar", 0)

    return {"kprod": kprod(), "vprod": vprod(), "qk": qk(), "pv": pv(), "wg0": softmax(0), "wg1": softmax(1)}


def _explore(T, seed, S=3, D=8):
    rng = random.Random(seed)
    bars = {}

    def bar(name):
        if name not in bars:
            count = {"sread": 2, "pready0": 1, "pready1": 1, "lbar": 2}.get(name, 1)   # one model thread per warpgroup
            bars[name] = _Bar(count)
        return bars[name]

    roles = _roles(T, S, D)
    cur = {n: None for n in roles}
    copies, pipe = [], []
    for _ in range(200000):
        for n in list(roles):
            if cur[n] is None:
                try:
                    cur[n] = next(roles[n])
                except StopIteration:
                    del roles[n]
                    continue
                op = cur[n]
                if op[0] == "wait":
                    b = bar(op[1])
                    assert b.done >= op[2], f"premature wait: {n} on {op[1]} phase {op[2]} (done {b.done}, T={T})"
                    assert b.done <= op[2] + 1, f"aliased wait: {n} on {op[1]} phase {op[2]} (done {b.done}, T={T})"
        if not roles and not copies and not pipe:
            return
        ready = [n for n in roles if cur[n][0] != "wait" or bar(cur[n][1]).done >= cur[n][2] + 1]
        choices = ready + (["copy"] if copies else []) + (["pipe"] if pipe else [])
        assert choices, f"deadlock (T={T}): " + ", ".join(f"{n}: {cur[n]}" for n in roles)
        pick = rng.choice(choices)
        if pick == "copy":
            bar(copies.pop(rng.randrange(len(copies)))).arrive()
            continue
        if pick == "pipe":
            for name in pipe.pop(0):
                bar(name).arrive()
            continue
        op, cur[pick] = cur[pick], None
        if op[0] == "arrive":
            bar(op[1]).arrive()
        elif op[0] == "tma":
            copies.append(op[1])
        elif op[0] == "mma":
            pipe.append(op[1])
        for n in roles:                                  # a waiter must never fall two phases behind
            c = cur[n]
            if c is not None and c[0] == "wait":
                assert bar(c[1]).done <= c[2] + 1, f"aliased wait: {n} on {c[1]} phase {c[2]} (T={T})"
    raise AssertionError("step limit")


@pytest.mark.parametrize("stages", [3, 4], ids=["bf16", "fp8"])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 7, 8, 9, 17, 40])
def test_fused_kernel_barrier_protocol(T, stages):
    for seed in range(60):
        _explore(T, seed, S=stages)


def test_model_catches_a_descriptor_ring_too_small_for_the_stages():
    # with as many descriptors as stages the producer can overwrite a descriptor the V loader or
    # the P V issuer has not read yet: the model must report the resulting aliased wait
    with pytest.raises(AssertionError):
        for seed in range(200):
            _explore(40, seed, S=4, D=2)
