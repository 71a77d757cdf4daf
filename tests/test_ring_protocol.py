"""A randomized model check, on the CPU, of the synchronisation protocol of the
L=16 VJP backward's shared-memory codeword ring (csrc/bcjr_l16.cuh): NS stages,
each filled by one bulk copy whose completion advances the stage's mbarrier
phase; 16 warps consume the 8 blocks of every backward step in order, each
waiting for the phase parity of the fill it needs, and the sixteenth warp to
release a stage issues the fill of the block NS positions later (none past the
sequence's last step); one thread primes blocks 0 .. NS-1 at the start of each
sequence's backward.

The model lets warps advance in random order and copies land after random
delays, and checks what the kernel relies on: every wait ends (no deadlock), a
warp reads the chunk of the block it is at, no fill lands in a stage that a
warp has yet to release, the phase a waiting warp sees never runs two fills
ahead (parity would alias), no copy is in flight when a CTA finishes, and the
stage and parity of block k are k mod NS and (k / NS) mod 2 in every step (as
the kernel's comments state for NS = 2, 8 blocks per step).
"""
import random

import pytest

WARPS, KB = 16, 8


class Stage:
    def __init__(self):
        self.completed = 0        # phases completed (fills landed)
        self.issued = 0           # fills issued
        self.chunk = None         # block k held once the last fill landed
        self.pending = None       # (chunk) of the fill in flight
        self.releases = 0         # release counter (all warps, all fills)


def run_cta(n_steps, n_seqs, NS, seed, step_barrier=True):
    rng = random.Random(seed)
    stages = [Stage() for _ in range(NS)]
    blocks_per_seq = n_steps * KB
    total = n_seqs * blocks_per_seq
    # per-warp position: index b of the next block (over all sequences of the CTA)
    pos = [0] * WARPS
    primed_seq = -1
    in_flight = []                 # stage indices with a fill in flight

    def fill(s, k):
        st = stages[s]
        assert st.pending is None, "a second fill issued while one is in flight"
        assert st.releases == 16 * st.issued, "fill issued before every warp released the stage"
        st.pending = k
        st.issued += 1
        in_flight.append(s)

    def land(s):
        st = stages[s]
        st.chunk, st.pending = st.pending, None
        st.completed += 1
        in_flight.remove(s)

    guard = 0
    while min(pos) < total or in_flight:
        guard += 1
        assert guard < 10_000_000, "no progress"
        # priming: one thread, after the barrier that closes the previous sequence
        seq_front = min(pos) // blocks_per_seq
        if seq_front > primed_seq and min(pos) < total and all(p == seq_front * blocks_per_seq for p in pos):
            for i in range(NS):
                fill((seq_front * blocks_per_seq + i) % NS, i)
            primed_seq = seq_front
        choices = []
        if in_flight:
            choices.append(("land", rng.choice(in_flight)))
        for w in range(WARPS):
            if pos[w] < total and (pos[w] // blocks_per_seq) <= primed_seq:
                choices.append(("warp", w))
        assert choices, "deadlock: nothing can move"
        kind, x = rng.choice(choices)
        if kind == "land":
            land(x)
            continue
        w = x
        b = pos[w]
        s = b % NS
        k = (b % blocks_per_seq) % KB
        t_rev = (b % blocks_per_seq) // KB          # backward step index: 0 is step n-1
        if step_barrier and k == 0 and t_rev > 0:
            # the step's __syncthreads: every warp has finished the previous step
            if any(pos[v] < b for v in range(WARPS)):
                continue
        fill_no = b // NS                            # fill of stage s that holds block b (per CTA)
        parity = fill_no & 1
        st = stages[s]
        # mbarrier.try_wait.parity: true once the phase of this parity has completed
        assert st.completed <= fill_no + 1, "the stage ran two fills ahead of a waiting warp"
        if st.completed < fill_no + 1:
            continue                                 # still waiting
        assert st.completed == fill_no + 1 and (st.completed - 1) & 1 == parity
        assert st.chunk == k, f"warp {w} at block {k} reads chunk {st.chunk}"
        # the kernel's loop constants for NS = 2, 8 blocks per step
        if NS == 2:
            assert s == k % NS and parity == (k // NS) & 1
        # release; the sixteenth warp refills the stage with block k + NS
        st.releases += 1
        if st.releases % 16 == 0:
            last_step = t_rev == n_steps - 1
            if not (last_step and k + NS >= KB):
                fill(s, (k + NS) % KB)
        pos[w] += 1
    # nothing in flight when the CTA ends, and every fill was consumed by all warps
    assert not in_flight
    for st in stages:
        assert st.releases == 16 * st.issued
    return True


@pytest.mark.parametrize("n_steps,n_seqs", [(1, 1), (2, 3), (5, 2), (37, 2)])
@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("step_barrier", [True, False])
def test_ring_protocol_two_stages(n_steps, n_seqs, seed, step_barrier):
    """Two stages as in the kernel, with and without the per-step barrier (the
    ring does not depend on it)."""
    assert run_cta(n_steps, n_seqs, NS=2, seed=seed, step_barrier=step_barrier)


@pytest.mark.parametrize("NS", [3, 4])
def test_ring_protocol_other_stage_counts(NS):
    """The protocol itself holds for any stage count (the kernel uses two)."""
    assert run_cta(9, 2, NS=NS, seed=NS)


def test_stage_and_parity_are_loop_constants():
    """With NS = 2 and 8 blocks per step, block k of every step of every
    sequence is stage k % 2 and fill parity (k // 2) % 2."""
    NS = 2
    for n_steps in (1, 3, 256):
        for seq in range(3):
            for t_rev in range(n_steps):
                for k in range(KB):
                    b = (seq * n_steps + t_rev) * KB + k
                    assert b % NS == k % NS
                    assert (b // NS) & 1 == (k // NS) & 1
