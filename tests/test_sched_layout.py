"""The stable fill's count table, enumerated on the host: the per-full-block
offsets the plan kernel writes (blocks after the block in its sequence, and
their running sum) and the slot a scheduler CTA (block gb, 128-token slice y,
kv head g) takes for a bucket (full block f, g) give every (CTA, bucket) pair
its own slot, inside the size the workspace carves, each bucket's slots one
contiguous segment in token order (the order that makes a bucket's entries
ascending).  No GPU needed."""
import math

import pytest


def _layout(seqlens, B, Hkv):
    nyb = math.ceil(B / 128)
    blocks = []          # (gb, seq, j, len, fbase)
    full_nlater, full_cm = [], []
    pairs = 0
    fb_base = 0
    for s, L in enumerate(seqlens):
        nb, nf = math.ceil(L / B), L // B
        for i in range(nb):
            blocks.append((len(blocks), s, i, min(B, L - i * B), fb_base))
            if (i + 1) * B <= L:
                full_nlater.append(nb - 1 - i)
                full_cm.append(pairs + i * (nb - 1) - i * (i - 1) // 2)
        pairs += nf * (nb - 1) - nf * (nf - 1) // 2
        fb_base += nf
    slots = {}
    for gb, s, j, ln, fbase in blocks:
        for y in range(math.ceil(ln / 128)):
            for g in range(Hkv):
                for i in range(j):
                    fb = fbase + i
                    seg = (full_cm[fb] * Hkv + g * full_nlater[fb]) * nyb
                    slot = seg + (j - i - 1) * nyb + y
                    assert (fb, g, gb, y) not in slots
                    slots[(fb, g, gb, y)] = (slot, seg, full_nlater[fb] * nyb)
    N = sum(math.ceil(L / B) for L in seqlens)
    bound = N * (N - 1) // 2 * Hkv * nyb
    return slots, bound, sum(seqlens) // B + len(seqlens)


@pytest.mark.parametrize("seqlens,B,Hkv", [
    ([32768], 4096, 8),
    ([4096, 12288, 32768, 65536, 131072, 131072], 4096, 8),
    ([700, 1300], 128, 2),
    ([1000, 3000, 129, 2125], 128, 2),
    ([900], 64, 2),
    ([1024, 333], 256, 1),
    ([5000, 63, 64, 65, 4096], 192, 3),
])
def test_slots_distinct_bounded_contiguous_in_token_order(seqlens, B, Hkv):
    slots, bound, nblk_max = _layout(seqlens, B, Hkv)
    vals = [v[0] for v in slots.values()]
    assert len(set(vals)) == len(vals)                    # one slot per (CTA, bucket)
    N = nblk_max                                          # the carve's bound uses nblk_max
    cap = N * (N - 1) // 2 * Hkv * math.ceil(B / 128)
    assert bound <= cap and all(0 <= v < cap for v in vals)
    segs = {}
    for (fb, g, gb, y), (slot, seg, n) in slots.items():
        assert seg <= slot < seg + n                      # inside its bucket's segment
        segs.setdefault((fb, g), []).append(((gb, y), slot))
    spans = []
    for key, lst in segs.items():
        lst.sort()
        assert [s for _, s in lst] == sorted(s for _, s in lst)   # token order = slot order
        spans.append((lst[0][1], lst[-1][1]))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 < b0                                    # segments do not overlap
