"""CPU model of the dequant GEMM's shared-memory pipeline protocol (csrc/qlora_gemm.cu).

The kernel's roles hand ring slots to one another through mbarriers whose waits test only the
parity of a phase, and its TMA copies land in any order.  This discrete-event model runs the
same roles as generators under a random scheduler: X producer, Q producer, the MMA thread,
four epilogue warps and two dequant groups of eight warps.  TMA copies complete in random
order and tensor-core work completes in issue order.

Each run checks three things:
* the model never deadlocks;
* every consumer sees the data of the step it expects;
* no slot is overwritten while reads of its previous contents are pending.

The protocol modelled:
* per step, the MMA thread waits for W-full and X-full and commits W-empty; with two token
  halves two MMA threads share the work (each waits for W-full and its own half's X-full and
  commits W-empty and the accumulator's full barrier, which then count two commits);
* X slots are refilled after the W-empty of the step DX earlier;
* Q and W slots are owned per dequant group;
* on a LoRA extension step every warp of the owning group waits for the slot's release,
  the group syncs, and the lead warp issues the TMA.
Both whole-tile and stream-K ranges of steps are covered.
"""

import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0
        self._maybe()

    def complete_tx(self, b):
        self.tx -= b
        self._maybe()

    def _maybe(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):  # try_wait.parity: the phase with this parity has completed
        return (self.phase & 1) != parity


def w_slot(it):
    return 2 * (it & 1) + ((it >> 1) & 1)


def w_par(it):
    return (it >> 2) & 1


class Fail(Exception):
    pass


def simulate(kt, n_ext, nh, qper, nacc, g0, n_steps, seed, all_warps_on_ext=True, dual=True):
    total = kt + n_ext
    DX = 2 if nh == 2 else 4
    SX, SW, NG, NW = DX * nh, 4, 2, 8
    issuers = [(0, 1), (1, 2)] if (dual and nh == 2) else [(0, nh)]
    ni = len(issuers)
    xf = [Bar(1) for _ in range(SX)]
    wf, we = [Bar(1) for _ in range(SW)], [Bar(ni) for _ in range(SW)]
    qf, qe = [Bar(1) for _ in range(NG * qper)], [Bar(NW) for _ in range(NG * qper)]
    af, ae = [Bar(ni) for _ in range(2)], [Bar(4) for _ in range(2)]
    xtag, wtag, qtag = [None] * SX, [None] * SW, [None] * (NG * qper)
    xreads, wreads = [0] * SX, [0] * SW
    tma, tensor = [], []

    def at(it):
        g = g0 + it
        return g // total, g % total

    segs, it = [], 0
    while it < n_steps:
        _, k0 = at(it)
        ln = min(total - k0, n_steps - it)
        segs.append((k0, ln))
        it += ln

    def wait(bar, parity):
        while not bar.done(parity):
            yield

    def x_producer():
        for j in range(n_steps):
            if j >= DX:
                yield from wait(we[w_slot(j - DX)], w_par(j - DX))
            for h in range(nh):
                s = (j % DX) * nh + h
                if xreads[s]:
                    raise Fail(f"X slot {s} refilled with reads pending (step {j})")
                xf[s].arrive(100)

                def land(s=s, j=j, h=h):
                    xtag[s] = (j, h)
                    xf[s].complete_tx(100)
                tma.append(land)

    def q_producer():
        vq = [0, 0]
        for j in range(n_steps):
            if at(j)[1] >= kt:
                continue
            g = j & 1
            v = vq[g]
            vq[g] += 1
            s = g * qper + v % qper
            yield from wait(qe[s], ((v // qper) & 1) ^ 1)
            qf[s].arrive(10)

            def land(s=s, j=j):
                qtag[s] = j
                qf[s].complete_tx(10)
            tma.append(land)

    def mma(h_lo, h_hi):
        it = 0
        for si, (k0, ln) in enumerate(segs):
            ab, use = (si & 1, si >> 1) if nacc == 2 else (0, si)
            yield from wait(ae[ab], (use & 1) ^ 1)
            for _ in range(ln):
                ws = w_slot(it)
                xs = [(it % DX) * nh + h for h in range(h_lo, h_hi)]
                yield from wait(wf[ws], w_par(it))
                for s in xs:
                    yield from wait(xf[s], (it // DX) & 1)
                if wtag[ws] != it:
                    raise Fail(f"MMA step {it}: W slot {ws} holds {wtag[ws]}")
                for h, s in zip(range(h_lo, h_hi), xs):
                    if xtag[s] != (it, h):
                        raise Fail(f"MMA step {it}: X slot {s} holds {xtag[s]}")
                wreads[ws] += 1
                for s in xs:
                    xreads[s] += 1

                def done(ws=ws, xs=xs):
                    wreads[ws] -= 1
                    for s in xs:
                        xreads[s] -= 1
                    we[ws].arrive()
                tensor.append(done)
                it += 1
            tensor.append(lambda ab=ab: af[ab].arrive())

    def epilogue():
        for si in range(len(segs)):
            ab, use = (si & 1, si >> 1) if nacc == 2 else (0, si)
            yield from wait(af[ab], use & 1)
            ae[ab].arrive()

    group_bar = {g: [0] * NW for g in range(NG)}

    def dequant(g, w):
        vq = n = 0
        for it in range(g, n_steps, NG):
            k = at(it)[1]
            ws = w_slot(it)
            if k < kt:
                s = g * qper + vq % qper
                u = vq // qper
                vq += 1
                yield from wait(qf[s], u & 1)
                if qtag[s] != it:
                    raise Fail(f"dequant step {it}: Q slot {s} holds {qtag[s]}")
                qe[s].arrive()
                yield from wait(we[ws], w_par(it) ^ 1)
                if wreads[ws]:
                    raise Fail(f"W slot {ws} written with reads pending (step {it})")
                n += 1
                group_bar[g][w] = n
                while min(group_bar[g]) < n:
                    yield
                if w == 0:
                    wtag[ws] = it
                    wf[ws].arrive()
            elif all_warps_on_ext or w == 0:
                yield from wait(we[ws], w_par(it) ^ 1)
                if all_warps_on_ext:
                    n += 1
                    group_bar[g][w] = n
                    while min(group_bar[g]) < n:
                        yield
                if w != 0:
                    continue
                if wreads[ws]:
                    raise Fail(f"W slot {ws} loaded with reads pending (step {it})")
                wf[ws].arrive(7)

                def land(ws=ws, it=it):
                    wtag[ws] = it
                    wf[ws].complete_tx(7)
                tma.append(land)

    roles = [x_producer(), q_producer()] + [mma(lo, hi) for lo, hi in issuers]
    roles += [epilogue() for _ in range(4)]
    roles += [dequant(g, w) for g in range(NG) for w in range(NW)]
    rng = random.Random(seed)
    idle = 0
    while roles or tma or tensor:
        if (tma or tensor) and rng.random() < 0.3:
            if tensor and (not tma or rng.random() < 0.5):
                tensor.pop(0)()
            else:
                tma.pop(rng.randrange(len(tma)))()
            idle = 0
            continue
        if not roles:
            continue
        r = rng.choice(roles)
        try:
            next(r)
        except StopIteration:
            roles.remove(r)
        idle += 1
        if idle > 200000:
            return "deadlock"
    return "ok"


def _cases(n, seed=7):
    rng = random.Random(seed)
    for i in range(n):
        kt = rng.choice([1, 2, 3, 4, 5, 7, 9, 16, 33])
        n_ext = rng.choice([1, 2])
        total = kt + n_ext
        nh, qper, nacc = rng.choice([1, 2]), rng.choice([4, 8, 16]), rng.choice([1, 2])
        if rng.random() < 0.5:
            g0, n_steps = rng.randrange(0, 3 * total), rng.randint(1, 4 * total)  # stream-K
        else:
            g0, n_steps = 0, total * rng.randint(1, 4)                           # whole tiles
        yield kt, n_ext, nh, qper, nacc, g0, n_steps, i


@pytest.mark.parametrize("case", list(_cases(150)))
def test_protocol_randomised(case):
    kt, n_ext, nh, qper, nacc, g0, n_steps, seed = case
    assert simulate(kt, n_ext, nh, qper, nacc, g0, n_steps, seed) == "ok"


@pytest.mark.parametrize("case", list(_cases(40, seed=11)))
def test_protocol_one_mma_thread(case):
    """The single-issuer protocol (fused launches, one token half) passes the same checks
    with two token halves too."""
    kt, n_ext, nh, qper, nacc, g0, n_steps, seed = case
    assert simulate(kt, n_ext, nh, qper, nacc, g0, n_steps, seed, dual=False) == "ok"


def test_model_catches_extension_step_aliasing():
    """With only the lead warp waiting on an extension step's W slot, the other warps can meet
    the slot's barrier two phases on and write it while the tensor core still reads it: one
    reduction step per tile plus two extension steps (K = 64, r > 64) shows it."""
    outcomes = set()
    for seed in range(200, 330):
        try:
            outcomes.add(simulate(1, 2, 2, 8, 1, 0, 12, seed, all_warps_on_ext=False))
        except Fail:
            outcomes.add("fail")
    assert "fail" in outcomes
    for seed in range(200, 330):
        assert simulate(1, 2, 2, 8, 1, 0, 12, seed) == "ok"
