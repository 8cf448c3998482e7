"""Model check of the backward kernel's buffer discipline (CPU, no GPU).

The gradient kernel has no producer warps: every thread loads rows with
cp.async groups, and the staged dK/dV slices leave through TMA bulk groups.
Its correctness rests on the order of those asynchronous operations against
the tensor-core products, which a parity test only exercises for the
timings the GPU happens to produce.  This model replays, for random list
lengths, the order the kernel issues them in:

  prologue    Q | dO, K(0) | V(0), K(1) (half 0 | half 1 of the warps),
              wait_group 1 | 0, barrier, scores(0)
  chunk c     wait scores(c); V(c+1) -> the V stage (half 1);
              softmax(c); drain of chunk c-1, slices NS/2..NS-1;
              wait_group 0 (when c+1 < nch); barrier;
              gradients(c), then scores(c+1); wait gradients(c);
              K(c+2) -> the K stage of c (half 0); drain of chunk c, slices 0..NS/2-1

with every copy completing as late as its waits allow and every tensor-core
product completing in issue order as late as its barrier waits allow.  It
checks that no product is issued before the rows it reads have landed, that
no copy overwrites a stage a product still reads, and that no staged slice
is rewritten while a bulk reduction still reads it (two staging slots; every
lane commits one bulk group per slice and waits until at most one of its
groups is unread).  Planted ordering mistakes must each be caught.
"""
from __future__ import annotations

import random

import pytest


class Bug(Exception):
    pass


class Lane:
    """One thread's cp.async groups: each group is a set of (buffer, chunk) loads."""

    def __init__(self):
        self.groups = []  # pending groups, oldest first

    def commit(self, loads):
        self.groups.append(list(loads))

    def wait_group(self, n, landed):
        while len(self.groups) > n:
            for ld in self.groups.pop(0):
                landed.add(ld)


def simulate_loads(nch, rng, mutant=None):
    """K stages (2), one V stage; products complete in issue order, as late as allowed."""
    landed = set()          # (buffer, chunk) whose copy has completed
    readers = []            # in-flight products: (name, chunk, {buffers it reads})
    h0, h1 = Lane(), Lane()

    def issue_load(lane, buf, c):
        # the stage must not be read by a product still in flight
        for name, cc, reads in readers:
            if (buf, cc) in reads and cc != c:
                raise Bug(f"{buf} of chunk {c} loaded while {name}({cc}) still reads it")
        lane.commit([(buf, c)])

    def kbuf(c):
        return f"K{c % 2}"

    def issue_product(name, c, reads):
        for r in reads:
            if r not in landed:
                raise Bug(f"{name}({c}) issued before {r} landed")
        readers.append((name, c, set(reads)))

    def complete_through(name, c):
        # products complete in issue order: pop up to and including (name, c)
        while readers:
            n, cc, _ = readers.pop(0)
            if (n, cc) == (name, c):
                return
        raise Bug(f"{name}({c}) completed but was never issued")

    # prologue
    h0.commit([("Q", 0)])
    h1.commit([("dO", 0)])
    issue_load(h0, kbuf(0), 0)
    issue_load(h1, "V", 0)
    if nch > 1:
        issue_load(h0, kbuf(1), 1)
        h0.wait_group(1, landed)
    else:
        h0.wait_group(0, landed)
    h1.wait_group(0, landed)
    # barrier, then scores(0)
    issue_product("scores", 0, [("Q", 0), ("dO", 0), (kbuf(0), 0), ("V", 0)])
    for c in range(nch):
        if c + 1 < nch and mutant == "v_before_scores_done":
            issue_load(h1, "V", c + 1)                      # planted: before scores(c) is done
        complete_through("scores", c)                      # wait scores(c)
        if c + 1 < nch and mutant != "v_before_scores_done":
            issue_load(h1, "V", c + 1)                      # V stage is free
        if c + 1 < nch:
            w = 1 if mutant == "wait_group_1" else 0
            h0.wait_group(w, landed)
            h1.wait_group(w, landed)
        # barrier; gradients(c) then scores(c+1)
        issue_product("grads", c, [("Q", 0), ("dO", 0), (kbuf(c), c)])
        if c + 1 < nch:
            issue_product("scores", c + 1, [(kbuf(c + 1), c + 1), ("V", c + 1)])
        if mutant == "k_before_grads_done" and c + 2 < nch:
            issue_load(h0, kbuf(c + 2), c + 2)
        complete_through("grads", c)                        # wait gradients(c)
        if mutant != "k_before_grads_done" and c + 2 < nch:
            issue_load(h0, kbuf(c + 2), c + 2)
        if rng.random() < 0.5:  # some copies land early: completion order is free
            for lane in (h0, h1):
                if lane.groups and rng.random() < 0.5:
                    for ld in lane.groups.pop(0):
                        landed.add(ld)


def simulate_staging(nslices, rng, mutant=None):
    """32 lanes, two slots; per slice each lane issues a bulk read of the slot or not
    (runs: lanes 0 and 16; single rows: lanes with a key); reads finish as late as the
    waits allow."""
    pending = [[] for _ in range(32)]   # per lane: groups, oldest first; a group = set of slots
    unread = {0: set(), 1: set()}       # slot -> lanes whose bulk read of it is unfinished
    pattern = None
    for n in range(nslices):
        slot = n & 1
        if n % rng.choice([1, 2, 3]) == 0:   # the chunk (and its run / row pattern) changes
            kind = rng.choice(["run", "rows", "none", "mixed"])
            if kind == "run":
                pattern = {0, 16}
            elif kind == "rows":
                pattern = {l for l in range(32) if rng.random() < 0.8}
            elif kind == "none":
                pattern = set()
            else:
                pattern = {0} | {l for l in range(16, 32) if rng.random() < 0.8}
        # every lane: wait until at most one of its groups is unread, then the warp syncs
        for lane in range(32):
            while len(pending[lane]) > 1:
                for s in pending[lane].pop(0):
                    unread[s].discard(lane)
        if unread[slot]:
            raise Bug(f"slice {n}: slot {slot} rewritten while lanes {sorted(unread[slot])} still read it")
        # stage, fence, sync, issue, commit
        for lane in range(32):
            issued = lane in pattern
            if issued:
                unread[slot].add(lane)
            if issued or mutant != "commit_only_when_issuing":
                pending[lane].append({slot} if issued else set())
        # reads may finish early
        for lane in range(32):
            if pending[lane] and rng.random() < 0.3:
                for s in pending[lane].pop(0):
                    unread[s].discard(lane)


@pytest.mark.parametrize("seed", range(6))
def test_loads_and_stages_are_ordered(seed):
    rng = random.Random(seed)
    for _ in range(200):
        simulate_loads(rng.choice([1, 2, 3, 4, 7]), rng)


@pytest.mark.parametrize("mutant", ["wait_group_1", "v_before_scores_done", "k_before_grads_done"])
def test_load_model_catches_planted_errors(mutant):
    rng = random.Random(1)
    with pytest.raises(Bug):
        for _ in range(200):
            simulate_loads(rng.choice([2, 3, 4, 7]), rng, mutant=mutant)


@pytest.mark.parametrize("seed", range(6))
def test_staging_slots_are_never_rewritten_while_read(seed):
    rng = random.Random(seed)
    for _ in range(100):
        simulate_staging(rng.randint(2, 40), rng)


def test_staging_model_catches_commit_only_when_issuing():
    rng = random.Random(3)
    with pytest.raises(Bug):
        for _ in range(200):
            simulate_staging(rng.randint(4, 40), rng, mutant="commit_only_when_issuing")
