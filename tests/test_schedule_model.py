"""The split schedule of the decode, restated on the host from its definition
(sequences laid out as units, `item_cost` page-less units before each
sequence, CTA groups of min(HT, ncta) members sharing a unit range, partial
results in slot (b + g) * HT + ht), and checked for the properties the merge
and the workspace rely on, over random problem shapes:
- every page of every segment (sequence, row tile) is worked on exactly once;
- no two items share a workspace slot, and every slot fits the workspace
  that qkn_decode_workspace_size sizes (the C-ABI host code);
- the merge's view of a segment (first group and split count, splits HT
  slots apart) names exactly the slots its items wrote.
CPU only."""
import ctypes
import random

import pytest

import qk_normed_latent_qkn_b200 as qkn

BLOCK = 64


def pages_of(L, s_q, max_blocks):
    return 0 if L < s_q or L > max_blocks * BLOCK else (L + BLOCK - 1) // BLOCK


def schedule(lens, s_q, max_blocks, ht_count, ncta, item_cost):
    """Items (b, ht, p0, p1, slot) of every CTA, by the definition above."""
    n = [pages_of(L, s_q, max_blocks) for L in lens]
    units = [x + item_cost if x > 0 else 0 for x in n]
    starts = [sum(units[:b]) for b in range(len(lens))]
    total = sum(units)
    hc = min(ht_count, ncta)
    ng = max(1, ncta // hc)
    q = max(1, -(-total // ng))
    items = []
    for cta in range(ncta):
        g, h0 = divmod(cta, hc)
        if g >= ng or h0 >= ht_count:
            continue
        lo, hi = g * q, min(g * q + q, total)
        for b in range(len(lens)):
            pg0 = starts[b] + item_cost
            a, e = max(lo, pg0), min(hi, starts[b] + units[b])
            if n[b] == 0 or a >= e:
                continue
            for ht in range(h0, ht_count, hc):
                items.append((b, ht, a - pg0, e - pg0, (b + g) * ht_count + ht))
    return items, n, starts, q


def merge_view(b, ht, n, starts, q, ht_count, item_cost):
    pg0 = starts[b] + item_cost
    g0 = pg0 // q
    nitems = (pg0 + n[b] - 1) // q - g0 + 1
    first = (b + g0) * ht_count + ht
    return [first + i * ht_count for i in range(nitems)]


def workspace_slots(batch, s_q, heads, rows, ncta):
    """Slots the workspace holds for row tile `rows`, read back from qkn_decode_workspace_size."""
    dims = qkn.Dims(num_heads=heads, num_groups=1, r_kv=512, d_h=128, d_rope=64, dtype=qkn.BF16)
    size = ctypes.c_size_t(0)
    lib = qkn.raw_library()
    assert lib.qkn_decode_workspace_size(ctypes.byref(dims.c()), batch, s_q, ncta, ctypes.byref(size)) == qkn.OK
    return size.value


@pytest.mark.parametrize("seed", range(40))
def test_schedule_covers_every_page_once_with_unique_slots(seed):
    rng = random.Random(seed)
    batch = rng.randint(1, 40)
    s_q = rng.choice([1, 2])
    max_blocks = rng.randint(1, 40)
    lens = [rng.choice([rng.randint(s_q, max_blocks * BLOCK), 0, max_blocks * BLOCK + 1])
            if rng.random() < 0.1 else rng.randint(s_q, max_blocks * BLOCK) for _ in range(batch)]
    ht_count = rng.choice([1, 2, 3, 4, 16])
    ncta = rng.choice([1, 2, 3, 5, 7, 64, 148])
    item_cost = rng.choice([0, 1, 2, 3])
    items, n, starts, q = schedule(lens, s_q, max_blocks, ht_count, ncta, item_cost)

    covered = {}
    for b, ht, p0, p1, slot in items:
        assert 0 <= p0 < p1 <= n[b]
        for p in range(p0, p1):
            assert (b, ht, p) not in covered, "page worked on twice"
            covered[(b, ht, p)] = slot
    expected = {(b, ht, p) for b in range(batch) for ht in range(ht_count) for p in range(n[b])}
    assert set(covered) == expected

    slots = [it[4] for it in items]
    assert len(slots) == len(set(slots)), "two items share a slot"
    assert max(slots, default=0) < batch * ht_count + ncta      # the workspace's slot count

    for b in range(batch):
        if n[b] == 0:
            continue
        for ht in range(ht_count):
            mine = sorted(it[4] for it in items if it[0] == b and it[1] == ht)
            assert mine == merge_view(b, ht, n, starts, q, ht_count, item_cost)


def test_workspace_holds_the_slots():
    # rows of partial results the workspace reserves cover (batch * HT + ncta) slots of every row tile
    for batch, s_q, heads, ncta in [(32, 1, 128, 148), (8, 2, 64, 148), (3, 1, 16, 5), (1, 1, 4, 1)]:
        ws = workspace_slots(batch, s_q, heads, 64, ncta)
        for rows in (8, 16, 32, 64):
            ht = -(-s_q * heads // rows)
            need = (batch * ht + ncta) * rows * (512 + 1) * 4        # partial O and lse, fp32
            assert ws >= need, (batch, s_q, heads, rows, ws, need)


@pytest.mark.parametrize("seed", range(40))
def test_cost_accounting_split_counts_match_the_schedule(seed):
    # the benchmark's merge byte count takes its split counts from roofline.split_counts: they must be
    # the number of items each segment gets under the schedule's definition
    from qk_normed_latent_qkn_b200.roofline import split_counts
    rng = random.Random(1000 + seed)
    batch, s_q, max_blocks = rng.randint(1, 40), rng.choice([1, 2]), rng.randint(1, 40)
    lens = [rng.randint(s_q, max_blocks * BLOCK) if rng.random() > 0.1 else rng.choice([0, max_blocks * BLOCK + 1])
            for _ in range(batch)]
    ht_count, ncta, item_cost = rng.choice([1, 2, 3, 4, 16]), rng.choice([1, 2, 3, 5, 7, 64, 148]), rng.choice([0, 3])
    items, _n, _starts, _q = schedule(lens, s_q, max_blocks, ht_count, ncta, item_cost)
    counts = split_counts(lens, s_q, max_blocks, ht_count, ncta, item_cost)
    for b in range(batch):
        for ht in range(ht_count):
            assert sum(1 for it in items if it[0] == b and it[1] == ht) == counts[b]
