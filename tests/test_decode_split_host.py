"""The decode kernel's balanced split, modelled on the host (no GPU).

With a split workspace csrc/gemv.cu gives CTA c of P an equal share of the
U = groups x k-tiles units (group-major; the first U mod P CTAs one more) and
works through them as "segments", one per group it touches.  Only a CTA's
first and last segments can cover part of a group.  Each output of a shared
group has one 64-bit workspace word holding the sum of the k-tile counts
added so far, the number of parts and the sum of the parts' partial sums, each
biased by 2^25, and every segment adds (k, 1, v + 2^25) to it with one atomic.
A CTA's last segment loads its words when it starts; at its end it writes the
outputs from them if they already hold every other part, else it adds its
part and writes them if its addition completed them.  A shared first segment
adds its part without looking at the result and re-loads its words when the
CTA's last segment starts; at the end it writes the outputs they show
complete.  This model restates the partition, the word and that protocol,
runs the parts of a word under random interleavings, and checks:
- every k-tile of every group belongs to exactly one segment; shares differ
  by at most one unit;
- each output is written at least once, always with the full sum (twice only
  with the same value);
- the words are zero afterwards, launch after launch;
- the fields never overflow, and the workspace indices stay inside
  bitlinear_decode_workspace_bytes.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ternary_weight_linear_bitlinear_b200", "csrc", "gemv.cu")
K_SHIFT, PARTS_SHIFT, BIAS = 45, 36, 1 << 25


def test_model_matches_kernel_source():
    """The partition, the word's fields and the completion tests the model
    restates are the kernel's (csrc/gemv.cu)."""
    src = open(SRC).read()
    assert "const int U = n_groups * KB, q = U / P, rem = U - q * P;" in src
    assert "u0 = q * c + (c < rem ? c : rem);" in src
    assert "u1 = u0 + q + (c < rem ? 1 : 0);" in src
    assert "constexpr int kSplitKShift = %d;" % K_SHIFT in src
    assert "constexpr int kSplitPartsShift = %d;" % PARTS_SHIFT in src
    assert "constexpr long long kSplitBias = 1ll << 25;" in src
    assert "if (split_k(wd) + my_k != KB)" in src
    assert "if (split_k(wd) + my_k == KB) {" in src
    assert "if (split_k(first_w[j]) == KB) {" in src
    # The tensor-core decode kernel uses the same word, partition and tests.
    tc = open(SRC.replace("gemv.cu", "gemv_tc.cu")).read()
    assert "constexpr int kSplitKShift = %d;" % K_SHIFT in tc
    assert "constexpr int kSplitPartsShift = %d;" % PARTS_SHIFT in tc
    assert "constexpr long long kSplitBias = 1ll << 25;" in tc
    assert "const int U = n_mb * KB, q = U / P, rem = U - q * P;" in tc
    assert "u0 = q * c + (c < rem ? c : rem);" in tc
    assert "if (split_k(wd) + my_k != KB) wd = atomicAdd(w, split_word(my_k, vt));" in tc
    assert "if (split_k(wd) + my_k == KB) {" in tc
    assert "if (split_k(first_w[t]) == KB) {" in tc


def segments(n_groups, KB, P, c):
    """CTA c's segments (group, kb0, kb1), as the kernel computes them."""
    U = n_groups * KB
    q, rem = divmod(U, P)
    u0 = q * c + min(c, rem)
    u1 = u0 + q + (1 if c < rem else 0)
    if u1 <= u0:
        return []
    g_first = u0 // KB
    out = []
    for g in range(g_first, (u1 - 1) // KB + 1):
        kb0 = max(u0 - g * KB, 0)
        kb1 = min(u1 - g * KB, KB)
        out.append((g, kb0, kb1))
    return out


@pytest.mark.parametrize("n_groups,KB,P", [(896, 32, 296), (896, 32, 148), (1, 1, 296),
                                           (17, 10, 444), (688, 16, 592), (256, 43, 296),
                                           (4, 1, 148), (3000, 3, 740)])
def test_partition_covers_every_k_tile_once(n_groups, KB, P):
    seen = [[0] * KB for _ in range(n_groups)]
    sizes = []
    for c in range(P):
        segs = segments(n_groups, KB, P, c)
        sizes.append(sum(kb1 - kb0 for _, kb0, kb1 in segs))
        for i, (g, kb0, kb1) in enumerate(segs):
            assert 0 <= kb0 < kb1 <= KB
            # only a CTA's first and last segments may be partial
            if 0 < i < len(segs) - 1:
                assert (kb0, kb1) == (0, KB)
            for k in range(kb0, kb1):
                seen[g][k] += 1
    assert all(v == 1 for row in seen for v in row)
    assert max(sizes) - min(sizes) <= 1


def word(k, v):
    return (k << K_SHIFT) + (1 << PARTS_SHIFT) + (v + BIAS)


def w_k(w):
    return w >> K_SHIFT


def w_sum(w):
    parts = (w >> PARTS_SHIFT) & 511
    return (w & ((1 << PARTS_SHIFT) - 1)) - parts * BIAS


class Word:
    def __init__(self):
        self.w = 0
        self.emitted = []


def last_agent(cell, KB, k, v):
    """The kernel's steps for a CTA's last segment on one output word."""
    pre = cell.w                           # loaded when the segment starts
    yield
    # ... the segment's MMAs ...
    yield
    wd = pre
    if w_k(wd) + k != KB:
        wd = cell.w                        # atomicAdd: returns the old word
        cell.w += word(k, v)
    if w_k(wd) + k == KB:
        cell.emitted.append(v + w_sum(wd))
        yield
        cell.w = 0


def first_agent(cell, KB, k, v, reload_after_add=True):
    """A CTA's shared first segment: add without a look, re-load the word
    when the CTA's last segment starts, write at the CTA's end if complete."""
    if not reload_after_add:               # a broken order: load first
        seen = cell.w
        yield
        cell.w += word(k, v)
    else:
        cell.w += word(k, v)               # red.global.add
        yield
        # ... the CTA's other segments ...
        seen = cell.w                      # the re-load
    yield
    if w_k(seen) == KB:
        cell.emitted.append(w_sum(seen))
        yield
        cell.w = 0


def run_word(parts, kinds, KB, rng, launches=3, reload_after_add=True):
    cell = Word()
    for _ in range(launches):
        cell.emitted = []
        values = [rng.randint(-(BIAS - 1), BIAS - 1) for _ in parts]
        agents = [last_agent(cell, KB, k, v) if kind == "last" else
                  first_agent(cell, KB, k, v, reload_after_add)
                  for k, v, kind in zip(parts, values, kinds)]
        live = list(range(len(agents)))
        while live:
            a = rng.choice(live)
            try:
                next(agents[a])
            except StopIteration:
                live.remove(a)
        assert cell.emitted, "no one wrote the output"
        assert all(e == sum(values) for e in cell.emitted), (cell.emitted, sum(values))
        assert cell.w == 0


@pytest.mark.parametrize("seed", range(300))
def test_split_protocol_random_interleavings(seed):
    rng = random.Random(900 + seed)
    KB = rng.randint(2, 40)
    n = rng.randint(2, min(KB, 5))
    cuts = sorted(rng.sample(range(1, KB), n - 1))
    parts = [b - a for a, b in zip([0] + cuts, cuts + [KB])]
    # Part 0 is a CTA's last segment (the group's head), the final part a
    # CTA's shared first segment (its tail), the ones between whole-range
    # segments, which are their CTA's last.
    kinds = ["last"] * (n - 1) + ["first"]
    run_word(parts, kinds, KB, rng)


def test_split_model_catches_a_load_before_the_add():
    """A first segment that looks at its word before adding its own part can
    leave an output unwritten: the model sees it."""
    with pytest.raises(AssertionError):
        for seed in range(300):
            rng = random.Random(seed)
            run_word([5, 7], ["last", "first"], 12, rng, reload_after_add=False)


def test_word_fields_hold_their_extremes():
    """Up to 410 parts (65536 / 160 base-3 k-tiles) of |v| < 2^25 and a
    k-tile total up to 410 stay inside their fields."""
    KB = 410
    for v in (-(BIAS - 1), 0, BIAS - 1):
        w = sum(word(1, v) for _ in range(KB))
        assert w_k(w) == KB and (w >> PARTS_SHIFT) & 511 == KB
        assert w_sum(w) == KB * v
    assert 2 * 128 * 65536 < BIAS


def ws_bytes(d_out, T):
    """bitlinear_decode_workspace_bytes, restated."""
    rows = (16 * (d_out // 16 + 1) + 127) // 128 * 128
    return (8 * rows * T + 255) // 256 * 256


@pytest.mark.parametrize("d_out", [16, 32, 272, 6912, 6928, 18960, 28672])
@pytest.mark.parametrize("T", [1, 8, 9, 16])
def test_workspace_indices_in_bounds(d_out, T):
    """Group g's words sit at [g T 16R, (g + 1) T 16R) (warp-MMA kernel), a
    128-row block b's at [128 b T, 128 (b + 1) T) (tensor-core kernel); every
    index either kernel can form is inside the workspace."""
    n_rt = d_out // 16
    for R in (1, 2):
        n_groups = (n_rt + R - 1) // R
        last = (n_groups - 1) * T * 16 * R + T * 16 * R - 1
        assert 8 * (last + 1) <= ws_bytes(d_out, T)
    n_mb = (d_out + 127) // 128
    last = ((n_mb - 1) * T + (T - 1)) * 128 + 127
    assert 8 * (last + 1) <= ws_bytes(d_out, T)
