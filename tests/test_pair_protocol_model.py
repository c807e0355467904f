"""A randomised model of the CTA-pair GEMM's barrier protocol (gemm_pair.cuh).

The kernel's roles are modelled as cooperating threads with random latencies:
per CTA (two per pair) an activation producer, a code producer and 4 dequant
groups of 4 warps; in the leader CTA the MMA issuer.  Barriers follow mbarrier
semantics: a phase completes when its arrivals and expected transaction bytes
are in, and a parity wait passes once the phase of that parity has completed.
The model checks what the protocol must guarantee:

- every MMA reads the activation tile and the dequantised W tile of its own
  step, from both CTAs (no stale slot);
- no slot is refilled while an MMA or a dequant warp still reads it;
- nothing deadlocks, for any number of main and adapter steps.

The ring sizes are the kernel's (4 activation/W slots, 8 code slots, 4 dequant
groups).  A planted fault — a dequant warp that does not wait for the slot's
MMAs before writing — must be caught, which shows the checks can fail.
"""
import heapq
import random

import pytest

STAGES, CSTAGES, GROUPS, WARPS = 4, 8, 4, 4


class _Bar:
    """mbarrier: arrival count, transaction bytes, completed-phase counter."""

    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        self._done()

    def arrive_expect_tx(self, units):
        self.tx += units
        self.arrive()

    def complete_tx(self, units):
        self.tx -= units
        self._done()

    def _done(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):  # try_wait.parity
        return (self.phase & 1) != parity


def simulate(n_main, n_lora, seed, skip_slot_wait=False):
    rng = random.Random(seed)
    n_total = n_main + n_lora
    clock, queue, seq, waiting, errors = [0.0], [], [0], [], []

    def later(dt, fn):
        seq[0] += 1
        heapq.heappush(queue, (clock[0] + dt, seq[0], fn))

    def resume(gen):
        while True:
            try:
                op = next(gen)
            except StopIteration:
                return
            if op[0] == "wait":
                if op[1].passed(op[2]):
                    continue
                waiting.append((gen, op[1], op[2]))
                return
            later(op[1], lambda g=gen: resume(g))
            return

    def wake():
        moved = True
        while moved:
            moved = False
            for w in list(waiting):
                if w in waiting and w[1].passed(w[2]):
                    waiting.remove(w)
                    resume(w[0])
                    moved = True

    cta = [{"afull": [_Bar(1) for _ in range(STAGES)], "empty": [_Bar(1) for _ in range(STAGES)],
            "cfull": [_Bar(1) for _ in range(CSTAGES)], "cempty": [_Bar(WARPS) for _ in range(CSTAGES)],
            "A": [None] * STAGES, "B": {}, "Blora": [None] * STAGES, "C": [None] * CSTAGES,
            "mma_reading": [0] * STAGES, "c_reading": [0] * CSTAGES} for _ in range(2)]
    ready = [_Bar(2 * WARPS) for _ in range(STAGES)]  # the leader's: 4 warps of each CTA

    def act_producer(c):
        d = cta[c]
        for it in range(n_total):
            s, ph = it % STAGES, (it // STAGES) & 1
            yield ("wait", d["empty"][s], ph ^ 1)
            if d["mma_reading"][s]:
                errors.append(f"activation slot {s} refilled under an MMA (cta {c}, step {it})")
            lora = it >= n_main
            d["afull"][s].arrive_expect_tx(2 if lora else 1)

            def land_a(s=s, it=it):
                d["A"][s] = it
                d["afull"][s].complete_tx(1)
            later(rng.uniform(0.5, 5.0), land_a)
            if lora:  # the adapter tile goes into the W slot
                def land_b(s=s, it=it):
                    if d["mma_reading"][s]:
                        errors.append(f"W slot {s} refilled under an MMA (cta {c}, step {it})")
                    d["Blora"][s] = it
                    d["afull"][s].complete_tx(1)
                later(rng.uniform(0.5, 5.0), land_b)
            yield ("delay", rng.uniform(0.0, 0.3))

    def code_producer(c):
        d = cta[c]
        for it in range(n_main):
            cs, ph = it % CSTAGES, (it // CSTAGES) & 1
            yield ("wait", d["cempty"][cs], ph ^ 1)
            if d["c_reading"][cs]:
                errors.append(f"code slot {cs} refilled while read (cta {c}, step {it})")
            d["cfull"][cs].arrive_expect_tx(1)

            def land(cs=cs, it=it):
                d["C"][cs] = it
                d["cfull"][cs].complete_tx(1)
            later(rng.uniform(0.5, 5.0), land)
            yield ("delay", rng.uniform(0.0, 0.3))

    def dequant_warp(c, g, w):
        d = cta[c]
        for it in range(g, n_total, GROUPS):
            s, ph = it % STAGES, (it // STAGES) & 1
            if it < n_main:
                cs, cph = it % CSTAGES, (it // CSTAGES) & 1
                yield ("wait", d["cfull"][cs], cph)
                if d["C"][cs] != it:
                    errors.append(f"stale codes (cta {c}, step {it})")
                d["c_reading"][cs] += 1
                yield ("delay", rng.uniform(0.01, 0.2))  # codes into registers
                d["c_reading"][cs] -= 1
                d["cempty"][cs].arrive()
                if not skip_slot_wait:
                    yield ("wait", d["empty"][s], ph ^ 1)  # the slot's previous MMAs are done
                if d["mma_reading"][s]:
                    errors.append(f"W slot {s} written under an MMA (cta {c}, step {it})")
                yield ("delay", rng.uniform(0.1, 1.5))  # decode and store
                if d["mma_reading"][s]:
                    errors.append(f"W slot {s} written under an MMA (cta {c}, step {it})")
                d["B"][(s, w)] = it
            yield ("wait", d["afull"][s], ph)
            ready[s].arrive()

    def issuer():
        for it in range(n_total):
            s, ph = it % STAGES, (it // STAGES) & 1
            yield ("wait", ready[s], ph)
            for c in range(2):
                d = cta[c]
                if d["A"][s] != it:
                    errors.append(f"MMA {it} read activation step {d['A'][s]} (cta {c})")
                if it < n_main:
                    got = [d["B"].get((s, w)) for w in range(WARPS)]
                    if got != [it] * WARPS:
                        errors.append(f"MMA {it} read W steps {got} (cta {c})")
                elif d["Blora"][s] != it:
                    errors.append(f"MMA {it} read adapter step {d['Blora'][s]} (cta {c})")
                d["mma_reading"][s] += 1

            def complete(s=s):  # the multicast commit arrives on both CTAs' empty barrier
                for c in range(2):
                    cta[c]["mma_reading"][s] -= 1
                    cta[c]["empty"][s].arrive()
            later(rng.uniform(0.2, 3.0), complete)
            yield ("delay", rng.uniform(0.05, 0.5))

    for c in range(2):
        resume(act_producer(c))
        resume(code_producer(c))
        for g in range(GROUPS):
            for w in range(WARPS):
                resume(dequant_warp(c, g, w))
    resume(issuer())
    wake()
    while queue:
        clock[0], _, fn = heapq.heappop(queue)
        fn()
        wake()
    if waiting:
        errors.append(f"deadlock: {len(waiting)} roles waiting")
    return errors


STEP_COUNTS = [(1, 0), (1, 1), (2, 1), (3, 0), (5, 2), (8, 1), (17, 1), (64, 1), (128, 1), (128, 0)]


@pytest.mark.parametrize("n_main,n_lora", STEP_COUNTS)
def test_protocol_orders_every_slot(n_main, n_lora):
    for seed in range(30):
        errors = simulate(n_main, n_lora, seed)
        assert not errors, (seed, errors[:3])


def test_model_catches_a_missing_slot_wait():
    caught = sum(bool(simulate(17, 1, seed, skip_slot_wait=True)) for seed in range(30))
    assert caught >= 10
