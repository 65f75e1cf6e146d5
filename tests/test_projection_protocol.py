"""A model of the output projection kernel's mbarrier protocol (csrc/msda_proj.cu),
run on the CPU under random interleavings of its roles.

The kernel's chunks g = 0, 1, ... flow through a ring of 4 shared-memory
stages; a stage's "full" barrier completes when its TMA bytes land and its
"empty" barrier when the MMAs that read it are done.  Row tiles alternate
between two tensor-memory accumulators, handed over with "acc_full" (MMA
commit) and "acc_empty" (4 epilogue warps arrive).  The model uses the same
parity arithmetic as the kernel:

  producer     chunk g waits empty[g % S] for parity (g / S - 1) & 1 when g >= S
  MMA issuer   tile t waits acc_empty[t & 1] for parity (t / 2 - 1) & 1 when t >= 2,
               chunk g waits full[g % S] for parity (g / S) & 1
  epilogue     tile t waits acc_full[t & 1] for parity (t / 2) & 1
  tail         the producer waits full and empty of the last S chunks

and checks that every role finishes, that no stage is refilled while its MMAs
may still read it, and that no accumulator is overwritten before the epilogue
has read it.

The precise (3 x TF32) variant runs 2 stages and adds a splitter role between
the copies and the MMAs:

  splitter     chunk g waits full[g % S] for parity (g / S) & 1, splits the
               stage into TF32 heads and remainders, then arrives on split[g % S]
  MMA issuer   chunk g waits split[g % S] (instead of full) for parity (g / S) & 1  An mbarrier phase with parity P counts as complete while the
barrier's current phase parity differs from P, as mbarrier.try_wait.parity
defines it."""
import random

import pytest

STAGES = 4
EPILOGUE_WARPS = 4


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def complete(self, parity):
        return (self.phase & 1) != parity


def run_protocol(tiles, chunks_per_tile, seed, precise=False):
    rng = random.Random(seed)
    S = 2 if precise else STAGES
    full = [Barrier(1) for _ in range(S)]
    split = [Barrier(1) for _ in range(S)]
    empty = [Barrier(1) for _ in range(S)]
    acc_full = [Barrier(1), Barrier(1)]
    acc_empty = [Barrier(EPILOGUE_WARPS), Barrier(EPILOGUE_WARPS)]
    total = tiles * chunks_per_tile
    stage_state = [None] * S          # None | ("loading", g) | ("landed", g) | ("used", g)
    acc_state = [None, None]          # None | "busy" | "full" | "read"
    copies, mma_work = [], []
    st = {"pg": 0, "mg": 0, "mt": 0, "mc": 0, "sg": 0}
    epi = [0] * EPILOGUE_WARPS
    read_count = [0, 0]

    def producer():
        g = st["pg"]
        if g >= total:
            return False
        s = g % S
        if g >= S and not empty[s].complete((g // S - 1) & 1):
            return False
        assert stage_state[s] is None or stage_state[s][0] == "used", (g, stage_state[s])
        stage_state[s] = ("loading", g)
        copies.append(g)
        st["pg"] += 1
        return True

    def mma_issuer():
        t = st["mt"]
        if t >= tiles:
            return False
        acc = t & 1
        if st["mc"] == 0 and t >= 2 and not acc_empty[acc].complete((t // 2 - 1) & 1):
            return False
        g = st["mg"]
        s = g % S
        ready = split[s] if precise else full[s]
        if not ready.complete((g // S) & 1):
            return False
        assert stage_state[s] == (("split" if precise else "landed"), g), (g, stage_state[s])
        if st["mc"] == 0:
            assert acc_state[acc] in (None, "read"), (t, acc_state[acc])
            acc_state[acc] = "busy"
        mma_work.append(("chunk", g, s))
        st["mg"] += 1
        st["mc"] += 1
        if st["mc"] == chunks_per_tile:
            mma_work.append(("tile", t, acc))
            st["mc"] = 0
            st["mt"] += 1
        return True

    def splitter():
        g = st["sg"]
        if not precise or g >= total:
            return False
        s = g % S
        if not full[s].complete((g // S) & 1):
            return False
        assert stage_state[s] == ("landed", g), (g, stage_state[s])
        stage_state[s] = ("split", g)
        split[s].arrive()
        st["sg"] += 1
        return True

    def epilogue(w):
        t = epi[w]
        if t >= tiles:
            return False
        acc = t & 1
        if not acc_full[acc].complete((t // 2) & 1):
            return False
        assert acc_state[acc] == "full", (t, acc_state[acc])
        acc_empty[acc].arrive()
        read_count[acc] += 1
        if read_count[acc] == EPILOGUE_WARPS:
            acc_state[acc] = "read"
            read_count[acc] = 0
        epi[w] += 1
        return True

    def tma_engine():
        if not copies:
            return False
        g = copies.pop(rng.randrange(len(copies)))  # copies may land out of order
        s = g % S
        assert stage_state[s] == ("loading", g)
        stage_state[s] = ("landed", g)
        full[s].arrive()
        return True

    def tensor_core():
        if not mma_work:
            return False
        item = mma_work.pop(0)  # MMAs and their commits complete in issue order
        if item[0] == "chunk":
            _, g, s = item
            stage_state[s] = ("used", g)
            empty[s].arrive()
        else:
            _, t, acc = item
            acc_state[acc] = "full"
            acc_full[acc].arrive()
        return True

    actors = [producer, mma_issuer, tma_engine, tensor_core, splitter] + \
             [lambda w=w: epilogue(w) for w in range(EPILOGUE_WARPS)]
    while True:
        order = actors[:]
        rng.shuffle(order)
        if not any(a() for a in order):
            break
    assert st["pg"] == total and st["mg"] == total and st["mt"] == tiles, st
    assert all(e == tiles for e in epi), epi
    for g in range(max(0, total - S), total):  # the producer's tail waits succeed
        assert full[g % S].complete((g // S) & 1)
        assert empty[g % S].complete((g // S) & 1)


@pytest.mark.parametrize("precise", [False, True])
@pytest.mark.parametrize("seed", range(60))
def test_protocol_random_interleavings(seed, precise):
    r = random.Random(1000 + seed)
    run_protocol(tiles=r.randint(0, 7), chunks_per_tile=r.randint(1, 9), seed=seed,
                 precise=precise)


def test_protocol_catches_a_wrong_parity():
    """The model is sharp: waiting for the wrong empty parity lets the producer
    refill a stage whose MMAs have not finished, which the model rejects (or
    the roles stall)."""
    S = STAGES
    empty = Barrier(1)
    # After one completion (chunk 0's MMAs), chunk S may refill: parity 0 is done.
    empty.arrive()
    assert empty.complete((S // S - 1) & 1)
    # The wrong parity (g / S) & 1 = 1 would not be complete yet: the kernel would stall.
    assert not empty.complete((S // S) & 1)
