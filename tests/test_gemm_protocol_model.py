"""The CTA-local GEMM's barrier protocol, modelled on the CPU.

A model (not the kernel itself) of the mbarrier protocol between the A/B and
scale producers, the MMA issuer, the tensor pipe's in-order commits and the
eight (2-SM form: sixteen) scale-staging / fold warps of the CTA-local NVFP4
GEMM, with the parities the kernel waits on.  Random interleavings check
that the protocol always completes (no deadlock), that the fold reads the
chunk the MMAs wrote into each partial buffer, and that the MMAs never
overwrite a partial before every fold warp has read it.  A change to the
kernel's protocol belongs here first."""
import random

import pytest


class Bar:
    """mbarrier: `count` arrivals complete a phase; try_wait.parity(P) succeeds
    once the phase of parity P has completed (a fresh barrier: P = 1)."""

    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


def run(actors, rnd):
    state = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive:
        runnable = [i for i in alive
                    if state[i] is None or state[i][0] != "wait" or state[i][1].done(state[i][2])]
        if not runnable:
            raise RuntimeError("deadlock")
        i = rnd.choice(runnable)
        try:
            op = next(actors[i])
        except StopIteration:
            alive.remove(i)
            continue
        if op[0] == "arrive":
            for b in op[1]:
                b.arrive()
            state[i] = None
        elif op[0] == "noop":
            state[i] = None
        else:
            state[i] = op


def simulate(ncta, num_tiles, KT, NPART, NBUF_ST, ABS, SFS, seed, fold_parity_flip=0):
    """ncta = 1 (1-SM) or 2 (pair: the MMA waits on the leader's barriers and
    commits to both CTAs; the peer's warps arrive on the leader's)."""
    rnd = random.Random(seed)
    total = num_tiles * KT
    nfold = 8 * ncta
    ab_full = [Bar(ncta) for _ in range(ABS)]  # leader: every CTA's copies
    ab_empty = [[Bar(1) for _ in range(ABS)] for _ in range(ncta)]
    sfs_full = [[Bar(1) for _ in range(SFS)] for _ in range(ncta)]
    sfs_empty = [[Bar(4) for _ in range(SFS)] for _ in range(ncta)]
    sft_full = [Bar(4 * ncta) for _ in range(NBUF_ST)]  # leader
    sft_empty = [[Bar(1) for _ in range(NBUF_ST)] for _ in range(ncta)]
    part_full = [[Bar(1) for _ in range(NPART)] for _ in range(ncta)]
    part_empty = [Bar(nfold) for _ in range(NPART)]  # leader
    content = [[None] * NPART for _ in range(ncta)]
    readers = [set() for _ in range(NPART)]
    staged = [[None] * NBUF_ST for _ in range(ncta)]
    commits = []

    def ab_producer(r):
        for g in range(total):
            s = g % ABS
            yield ("wait", ab_empty[r][s], ((g // ABS) & 1) ^ 1)
            yield ("arrive", [ab_full[s]])

    def sf_producer(r):
        for g in range(total):
            s = g % SFS
            yield ("wait", sfs_empty[r][s], ((g // SFS) & 1) ^ 1)
            yield ("arrive", [sfs_full[r][s]])

    def mma():
        for g in range(total):
            s, b = g % ABS, g % NBUF_ST
            yield ("wait", sft_full[b], (g // NBUF_ST) & 1)
            yield ("wait", ab_full[s], (g // ABS) & 1)
            assert all(staged[r][b] == g for r in range(ncta))
            for c in range(2):
                q = 2 * g + c
                pb = q % NPART
                yield ("wait", part_empty[pb], ((q // NPART) & 1) ^ 1)
                if content[0][pb] is not None:
                    assert len(readers[pb]) == nfold, "partial overwritten before it was read"

                def write(pb=pb, q=q):
                    for r in range(ncta):
                        content[r][pb] = q
                    readers[pb].clear()
                commits.append(([part_full[r][pb] for r in range(ncta)], write))
            commits.append(([ab_empty[r][s] for r in range(ncta)], None))
            commits.append(([sft_empty[r][b] for r in range(ncta)], None))
            yield ("noop",)

    def tensor_pipe():  # completes committed work in order, at random times
        left = total * 4
        while left:
            if commits:
                bars, act = commits.pop(0)
                if act:
                    act()
                yield ("arrive", bars)
                left -= 1
            else:
                yield ("noop",)

    def fold_warp(r, qd, h):
        g_st, g = h, 0
        for _ in range(num_tiles):
            for _ in range(KT):
                while g_st < total and g_st < g + NBUF_ST:
                    s, b = g_st % SFS, g_st % NBUF_ST
                    yield ("wait", sfs_full[r][s], (g_st // SFS) & 1)
                    if g_st >= NBUF_ST:
                        yield ("wait", sft_empty[r][b], ((g_st // NBUF_ST) & 1) ^ 1)
                    staged[r][b] = g_st
                    yield ("arrive", [sfs_empty[r][s], sft_full[b]])
                    g_st += 2
                for c in range(2):
                    q = 2 * g + c
                    pb = q % NPART
                    yield ("wait", part_full[r][pb], ((q // NPART) & 1) ^ fold_parity_flip)
                    assert content[r][pb] == q, "fold read the wrong chunk"
                    readers[pb].add((r, qd, h))
                    yield ("arrive", [part_empty[pb]])
                g += 1

    actors = [ab_producer(r) for r in range(ncta)] + [sf_producer(r) for r in range(ncta)] + \
             [mma(), tensor_pipe()] + \
             [fold_warp(r, qd, h) for r in range(ncta) for h in range(2) for qd in range(4)]
    run(actors, rnd)


@pytest.mark.parametrize("npart,nbuf", [(2, 5), (3, 4)], ids=["two-partials", "three-partials"])
def test_one_cta_protocol(npart, nbuf):
    for seed in range(60):
        simulate(1, num_tiles=2, KT=5, NPART=npart, NBUF_ST=nbuf, ABS=4, SFS=8, seed=seed)


def test_pair_protocol():
    for seed in range(40):
        simulate(2, num_tiles=2, KT=5, NPART=3, NBUF_ST=4, ABS=4, SFS=8, seed=seed)


def test_the_model_catches_a_wrong_wait_parity():
    with pytest.raises((AssertionError, RuntimeError)):
        for seed in range(40):
            simulate(1, num_tiles=2, KT=5, NPART=3, NBUF_ST=4, ABS=4, SFS=8, seed=seed,
                     fold_parity_flip=1)
