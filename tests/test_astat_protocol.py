"""The resident-A kernel's barrier protocol, modelled on the CPU.

pe_astat_kernel runs five roles per CTA pair that hand work to one another
through mbarriers with parity waits: weight TMA issuers (both CTAs), the MMA
thread (leader CTA), A producers (both CTAs) and epilogue warps (both CTAs).
A parity wait passes while the barrier's completed-phase count has the other
parity, so a waiter that falls two phases behind would pass on the wrong phase
and one that runs ahead would wait for ever.  This model replays the roles'
loops with the kernel's pass ranges, ring indices, parities, chunk waits and
chunk releases, as cooperative actors, and checks for many shapes that

  - every wait passes on exactly the phase the waiter means: the barrier has
    completed that phase and not the next one (no lapping), and the parity
    the kernel passes is that phase's parity;
  - every actor finishes (no deadlock) and every pass reaches the epilogue.

Three planted protocol mistakes (a producer that skips its release wait, an
MMA thread that never releases the last chunk, an issuer parity off by one)
must each be caught.  The model covers the protocol only; the kernel's
arithmetic is checked against the oracle on the GPU.
"""
from __future__ import annotations

import pytest

# k-steps per resident-A chunk: 8 image-row segments of p columns = p/2
# k-steps (7 for p = 14); parametrised below


class Bar:
    def __init__(self, name, count, log):
        self.name, self.count, self.pending, self.done, self.log = name, count, count, 0, log

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: more arrivals than the count"
        self.log[0] += 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class Lapped(AssertionError):
    pass


class Deadlock(AssertionError):
    pass


def parity_wait(bar: Bar, parity: int, phase: int):
    """Wait for completed phase `phase` (0-based; -1 = the phase before the
    first, complete from the start) with the kernel's parity argument."""
    if parity != (phase & 1) and phase >= 0:
        raise AssertionError(f"{bar.name}: parity {parity} passed for phase {phase}")
    if phase < 0:
        if parity != 1:
            raise AssertionError(f"{bar.name}: a fresh barrier is passed only with parity 1")
        return
    while True:
        if bar.done == phase + 1:
            return
        if bar.done > phase + 1:
            raise Lapped(f"{bar.name}: waiting for phase {phase}, {bar.done} completed")
        yield


def simulate(num_passes, ntn, npairs_cap, nb, n_iss, nks, bug=None, cks=7):
    npairs = min(num_passes, npairs_cap)
    nst = (nks + 3) // 4          # weight stages of 4 k-steps
    nch = (nks + cks - 1) // cks
    for pair in range(npairs):
        q0 = num_passes * pair // npairs
        q1 = num_passes * (pair + 1) // npairs
        assert q1 > q0
        log = [0]
        full_w = [Bar(f"full_w{s}", 1, log) for s in range(nb)]     # leader: expect_tx + both CTAs' bytes
        empty_w = [Bar(f"empty_w{s}", 1, log) for s in range(nb)]   # multicast commit (one per CTA, alike)
        full_a = [Bar(f"full_a{h}", 2, log) for h in range(nch)]    # producers of both CTAs
        empty_a = [Bar(f"empty_a{h}", 1, log) for h in range(nch)]
        tfull = [Bar(f"tfull{a}", 1, log) for a in range(2)]
        tempty = [Bar(f"tempty{a}", 2, log) for a in range(2)]      # epilogues of both CTAs
        landed = {}
        done = {"mma": 0, "epi": [0, 0], "stores": [0, 0]}

        def issuer(rank, iss):
            g = 0
            for _q in range(q0, q1):
                for _j in range(nst):
                    if g % n_iss == iss:
                        s = g % nb
                        par = ((g // nb) & 1) ^ 1
                        if bug == "issuer_parity":
                            par ^= 1 if g // nb else 0
                        yield from parity_wait(empty_w[s], par, g // nb - 1)
                        key = (s, g // nb)
                        landed[key] = landed.get(key, 0) + 1
                        if landed[key] == 2:    # both halves of the stage have landed
                            full_w[s].arrive()
                    g += 1

        def mma():
            ws = acc = 0
            wph = accph = aph = 0
            wuse = [0] * nb
            ause = [0, 0]
            gathers = 0
            for q in range(q0, q1):
                n = q % ntn
                new_a = q == q0 or n == 0
                last_a = q == q1 - 1 or n == ntn - 1
                yield from parity_wait(tempty[acc], accph ^ 1, ause[acc] - 1)
                hw = 0 if new_a else nch          # next A chunk to await (first pass over a block)
                hr = 0 if last_a else nch         # next A chunk to release (last pass over a block)
                for j in range(nst):
                    s0 = 4 * j
                    slast = min(s0 + 3, nks - 1)
                    while hw < nch and hw * cks <= slast:   # the chunks this stage reads
                        yield from parity_wait(full_a[hw], aph, gathers)
                        hw += 1
                    yield from parity_wait(full_w[ws], wph, wuse[ws])
                    wuse[ws] += 1
                    empty_w[ws].arrive()
                    # chunks whose last k-step is issued go back to the producers
                    while hr < nch and min((hr + 1) * cks, nks) - 1 <= slast:
                        if not (bug == "no_last_release" and hr == nch - 1):
                            empty_a[hr].arrive()
                        hr += 1
                    ws += 1
                    if ws == nb:
                        ws, wph = 0, wph ^ 1
                assert not new_a or hw == nch, "a block's first pass awaits every chunk"
                assert not last_a or hr == nch, "a block's last pass releases every chunk"
                tfull[acc].arrive()
                ause[acc] += 1
                acc += 1
                if acc == 2:
                    acc, accph = 0, accph ^ 1
                if last_a:
                    aph ^= 1
                    gathers += 1
                done["mma"] += 1

        def producer(rank):
            mfirst, mlast = q0 // ntn, (q1 - 1) // ntn
            for idx in range((mlast - mfirst + 1) * nch):
                G, h = divmod(idx, nch)
                if bug != "producer_skips_wait":
                    yield from parity_wait(empty_a[h], (G & 1) ^ 1, G - 1)
                full_a[h].arrive()
                done["stores"][rank] += 1
            return
            yield

        def epilogue(rank):
            acc = accph = 0
            seen = [0, 0]
            for _q in range(q0, q1):
                yield from parity_wait(tfull[acc], accph, seen[acc])
                seen[acc] += 1
                tempty[acc].arrive()
                done["epi"][rank] += 1
                acc += 1
                if acc == 2:
                    acc, accph = 0, accph ^ 1

        live = [issuer(r, i) for r in range(2) for i in range(n_iss)]
        live += [mma(), producer(0), producer(1), epilogue(0), epilogue(1)]
        while live:
            before = (log[0], len(live))
            for a in list(live):
                try:
                    next(a)
                except StopIteration:
                    live.remove(a)
            if live and (log[0], len(live)) == before:
                raise Deadlock(f"pair {pair} passes [{q0}, {q1}) ntn {ntn} nb {nb} n_iss {n_iss} nks {nks}")
        assert done["mma"] == q1 - q0
        assert done["epi"] == [q1 - q0, q1 - q0]
        nblocks = (q1 - 1) // ntn - q0 // ntn + 1
        assert done["stores"] == [nblocks * nch, nblocks * nch]


SHAPES = [(232, 5, 74), (4, 10, 74), (4, 5, 74), (1, 1, 74), (3, 5, 2), (7, 3, 4), (2, 20, 5), (9, 1, 3),
          (5, 5, 1)]


@pytest.mark.parametrize("mt,ntn,npairs", SHAPES)
@pytest.mark.parametrize("nb,n_iss", [(2, 2), (3, 3), (4, 3), (8, 3), (5, 2)])
@pytest.mark.parametrize("nks,cks", [(37, 7), (12, 3), (1, 1), (48, 8), (27, 6)])
def test_protocol_completes_on_the_intended_phases(mt, ntn, npairs, nb, n_iss, nks, cks):
    if mt * ntn > 400 and (nb, n_iss) != (4, 3):
        pytest.skip("the full-size grouped case runs with the default ring only")
    simulate(mt * ntn, ntn, npairs, nb, n_iss, nks, cks=cks)


@pytest.mark.parametrize("bug,exc", [("producer_skips_wait", Lapped), ("no_last_release", Deadlock),
                                     ("issuer_parity", AssertionError)])
def test_planted_protocol_mistakes_are_caught(bug, exc):
    with pytest.raises(exc):
        simulate(3 * 5, 5, 1, 3, 3, 37, bug=bug)
