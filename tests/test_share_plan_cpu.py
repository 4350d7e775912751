"""The split-KV share plan the decode kernels and the combine agree on, checked as
arithmetic on the host (no GPU): the admitted blocks of all (row, KV head) pairs laid
end to end, cut into shares of max(ceil(total / P), 2) blocks, one per CTA; CTA p
writes one partial slot p + r for every pair r its share touches, and the combine
finds the slots of pair r as p0 = off_r // chunk, ns = (off_r + c_r - 1) // chunk -
p0 + 1.  These are the rules the CUDA plan (plan_kernel, plan_local) and merge
(combine_merge) implement; this test pins the invariants they rely on: every admitted
block is streamed by exactly one CTA, slots are distinct and below P + R (the
workspace holds P + R slots), and the combine's formula names exactly the CTAs that
wrote the pair."""
import numpy as np
import pytest

K_MIN_CHUNK = 2


def plan(counts, P):
    row_off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    total = int(row_off[-1])
    chunk = max(-(-total // P), K_MIN_CHUNK)
    return row_off, total, chunk


@pytest.mark.parametrize("seed", range(40))
def test_shares_cover_every_block_once_and_slots_are_distinct(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 300))
    P = int(rng.choice([1, 2, 7, 148, 296]))
    dens = rng.choice([0.0, 0.05, 0.5, 1.0])
    counts = rng.binomial(int(rng.integers(1, 4096)), dens, size=R)
    counts[rng.random(R) < 0.2] = 0                      # empty pairs
    row_off, total, chunk = plan(counts, P)
    seen = np.zeros(total, dtype=np.int64)
    writers = {r: [] for r in range(R)}
    slots = set()
    for p in range(P):
        a, e = p * chunk, min((p + 1) * chunk, total)
        if a >= e:
            continue
        seen[a:e] += 1
        r0 = int(np.searchsorted(row_off, a, side="right") - 1)
        r1 = int(np.searchsorted(row_off, e - 1, side="right") - 1)
        for r in range(r0, r1 + 1):
            if counts[r] == 0:
                continue
            slot = p + r
            assert slot not in slots
            assert slot < P + R
            slots.add(slot)
            writers[r].append(p)
    assert np.all(seen == 1)
    for r in range(R):
        c, off = int(counts[r]), int(row_off[r])
        if c == 0:
            assert writers[r] == []
            continue
        p0 = off // chunk
        ns = (off + c - 1) // chunk - p0 + 1
        assert writers[r] == list(range(p0, p0 + ns))
