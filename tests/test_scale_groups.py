"""The grouped scale words' slot rule, checked on the host over many tile
sequences.

The E4M3 kernel gives one set of UE8M0 scale words to a group of up to four
consecutive K blocks of a tile (four one-block stages, or one stage of two or
four blocks), and keeps group g's words in shared-memory and TMEM slot
g mod STAGES.  Rewriting a slot is safe only if the slot's previous group
ended at least STAGES stages before the new group's first stage: only then
have that group's copy and MMAs completed (the producer refilled the new
group's stage after the commit of the stage STAGES earlier).  This walks the
stage sequence the way the kernel's MMA and scale warps do (tiles of any K
range, split-K slices that start anywhere) and checks that rule and the byte
index of every K block.
"""
import numpy as np
import pytest


def sf_group(kps: int) -> int:
    """Stages sharing one set of scale words (the kernel's kSfGroup)."""
    return 4 if kps == 1 else 1


def walk(tiles, kps: int, stages: int):
    """tiles: (kb_begin, kb_end) per tile, in the CTA's order.  Returns the
    groups as [first stage, last stage, slot] and every (stage, K block, byte)."""
    it = gc = 0
    groups, blocks = [], []
    g = sf_group(kps)
    for b, e in tiles:
        for kb in range(b, e, kps):
            q = (kb - b) // kps
            if q % g == 0:
                groups.append([it, it, gc % stages])
                gc += 1
            else:
                groups[-1][1] = it
            for j in range(kps):
                if kb + j < e:
                    blocks.append((it, kb + j, (q % g) * kps + j, b))
            it += 1
    return groups, blocks


@pytest.mark.parametrize("kps", [1, 2, 4])
@pytest.mark.parametrize("stages", [2, 3, 4, 6, 8, 9])
def test_a_slot_is_rewritten_only_after_its_group_drained(kps, stages):
    rng = np.random.default_rng(kps * 100 + stages)
    for _ in range(200):
        tiles = []
        for _ in range(rng.integers(1, 12)):
            b = int(rng.integers(0, 60))
            tiles.append((b, b + int(rng.integers(1, 24))))
        groups, blocks = walk(tiles, kps, stages)
        last_of_slot = {}
        for first, last, slot in groups:
            if slot in last_of_slot:
                assert last_of_slot[slot] <= first - stages, (tiles, first, slot)
            last_of_slot[slot] = last
        for stage, kb, byte, b in blocks:
            # the byte is the K block's place in its group (four one-block
            # stages, or one stage of KPS blocks), counted from the tile's
            # first K block
            assert 0 <= byte < 4
            assert byte == (kb - b) % (sf_group(kps) * kps)


def test_one_block_stages_share_words_in_fours():
    groups, blocks = walk([(0, 10)], kps=1, stages=4)
    assert [(f, l) for f, l, _ in groups] == [(0, 3), (4, 7), (8, 9)]
    assert [s for _, _, s in groups] == [0, 1, 2]
    # a tile boundary starts a new group even mid-four
    groups, _ = walk([(5, 7), (0, 3)], kps=1, stages=4)
    assert [(f, l) for f, l, _ in groups] == [(0, 1), (2, 4)]
