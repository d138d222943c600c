"""Host model of the block-scaled (UE8M0) GEMM's barrier protocol.

Roles of gemm_mx_kernel (fp8q_gemm_mx.cuh), meeting only through mbarriers:
  * producer: per slab, wait empty[s] (the slab STAGES back released the
    stage), then the copies (A, B tiles and both scale atoms) land on full[s];
  * MMA thread: per tile, wait tempty[b] (the epilogue has read the tile two
    back out of accumulator b); per slab, wait full[s], copy the atoms to the
    scale-factor columns and issue the MMAs; one commit per slab arrives on
    empty[s] once they complete, and one per tile on tfull[b];
  * epilogue warps: per tile, wait tfull[b], read the accumulator, each warp
    arrives on tempty[b].
Waits are parity waits.  The model replays random interleavings with
asynchronous copy and MMA completion and checks that every schedule finishes,
no parity wait passes on an earlier phase, no stage is refilled before its
MMAs read it, no accumulator is overwritten before all eight warps read it,
and the scale-factor columns are never rewritten while an MMA still reads them
(the copy and the MMAs of one thread execute in order).
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, phase_index):
        ok = (self.done % 2) != (phase_index % 2)
        if ok:
            assert self.done >= phase_index + 1, "parity wait passed on an earlier phase"
        return ok


def simulate(tiles, nkb, stages=6, warps=8, seed=0, max_steps=1_000_000):
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(stages)]
    empty = [Bar(1) for _ in range(stages)]
    tfull = [Bar(1) for _ in range(2)]
    tempty = [Bar(warps) for _ in range(2)]
    J = tiles * nkb
    stage_slab, stage_busy = [None] * stages, [False] * stages
    acc_tile, acc_readers = [None] * 2, [0] * 2
    prod_j = 0
    mma_t, mma_kb = 0, 0          # next tile / slab of the MMA thread
    epi_t = [0] * warps
    tma, pipe = [], []            # in-flight copies; tensor-pipe queue (in order): ("mma", j, s, b) / ("tile", t, b)
    sf_owner = None               # slab whose scale factors sit in the TMEM columns
    finished = 0

    def acts():
        a = []
        if prod_j < J:
            s = prod_j % stages
            if prod_j < stages or empty[s].passes(prod_j // stages - 1):
                a.append("prod")
        if mma_t < tiles:
            b = mma_t % 2
            j = mma_t * nkb + mma_kb
            if mma_kb == 0 and not tempty[b].passes(mma_t // 2 - 1) and mma_t >= 2:
                pass
            elif full[j % stages].passes(j // stages):
                a.append("mma")
        for w in range(warps):
            t = epi_t[w]
            if t < tiles and tfull[t % 2].passes(t // 2):
                a.append(("epi", w))
        if tma:
            a.append("land")
        if pipe:
            a.append("pipe")
        return a

    steps = 0
    while finished < tiles * warps:
        a = acts()
        assert a, "deadlock"
        act = rng.choice(a)
        steps += 1
        assert steps < max_steps
        if act == "prod":
            s = prod_j % stages
            assert not stage_busy[s], "stage refilled before its MMAs read it"
            tma.append((prod_j, s))
            prod_j += 1
        elif act == "land":
            j, s = tma.pop(rng.randrange(len(tma)))
            stage_slab[s], stage_busy[s] = j, True
            full[s].arrive()
        elif act == "mma":
            b = mma_t % 2
            j = mma_t * nkb + mma_kb
            s = j % stages
            assert stage_slab[s] == j
            if mma_kb == 0:
                assert acc_readers[b] == 0, "accumulator overwritten before the epilogue read it"
            # scale-factor copy and the MMAs go to the tensor pipe in issue order
            pipe.append(("cp", j, s, b))
            pipe.append(("mma", j, s, b))
            mma_kb += 1
            if mma_kb == nkb:
                pipe.append(("tile", mma_t, b))
                mma_t, mma_kb = mma_t + 1, 0
        elif act == "pipe":
            kind, x, *rest = pipe.pop(0)       # in order
            if kind == "cp":
                sf_owner = x
            elif kind == "mma":
                j, (s, b) = x, rest
                assert sf_owner == j, "scale-factor columns hold another slab's atoms"
                stage_busy[s] = False
                empty[s].arrive()
            else:
                t, b = x, rest[0]
                acc_tile[b], acc_readers[b] = t, warps
                tfull[b].arrive()
        else:
            w = act[1]
            t = epi_t[w]
            b = t % 2
            assert acc_tile[b] == t, "epilogue read an accumulator holding another tile"
            acc_readers[b] -= 1
            tempty[b].arrive()
            epi_t[w] += 1
            finished += 1
    return steps


@pytest.mark.parametrize("seed", range(10))
def test_mx_protocol_random_schedules(seed):
    simulate(tiles=5, nkb=6, seed=seed)


@pytest.mark.parametrize("nkb", [1, 2, 7])
def test_mx_protocol_tile_lengths(nkb):
    for seed in range(5):
        simulate(tiles=4, nkb=nkb, seed=50 + seed)
