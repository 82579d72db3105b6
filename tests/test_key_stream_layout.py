"""Host-side check of the key-stream layout the attention kernel relies on.

The kernel lays the kept chunks of a query chunk (ascending, the diagonal
chunk last) into 128-slot key tiles: each piece starts on an 8-slot
boundary, and a chunk that reaches a tile's end continues at slot 0 of the
next tile. Its scheduler hands each work item the diagonal chunk's first
stream slot D = sum of round8(length) over the other chunks, and the
softmax masks, in tile kt with dt = D - 128 kt < 128, every slot from
max(qt - c_start + dt + 1, 0) on for the query token qt.

This test walks the layout slot by slot, as the producer does, on random
chunk layouts and checks that the threshold rule masks exactly the kept
slots whose key token lies after the query token (brute force), and that
the tile count is ceil(sum of round8(length) / 128).
"""
import random

BN = 128


def round8(x):
    return (x + 7) & ~7


def walk(chunks):
    """Tiles of (slot -> key token) for the kept slots, cutting pieces as the
    producer does."""
    tiles, sq, seg_pos = [], 0, 0
    while sq < len(chunks):
        slot, kept = 0, {}
        while slot < BN and sq < len(chunks):
            s0, ln = chunks[sq]
            rows = min(ln - seg_pos, BN - slot)
            for x in range(rows):
                kept[slot + x] = s0 + seg_pos + x
            slot += round8(rows)
            seg_pos += rows
            if seg_pos == ln:
                seg_pos, sq = 0, sq + 1
        tiles.append(kept)
    return tiles


def random_item(rng):
    n = rng.randint(1, 40)
    lens = [rng.choice([rng.randint(1, 9), rng.randint(1, 300)]) for _ in range(n)]
    offs = [0]
    for ln in lens:
        offs.append(offs[-1] + ln)
    i = rng.randrange(n)
    c_start, c_end = offs[i], offs[i + 1]
    q0 = c_start + BN * rng.randrange((c_end - c_start + BN - 1) // BN)
    q_rows = min(BN, c_end - q0)
    sel = sorted(rng.sample(range(i), rng.randint(0, i))) if i else []
    chunks = [(offs[j], lens[j]) for j in sel] + [(c_start, q0 + q_rows - c_start)]
    return chunks, c_start, q0, q_rows


def test_threshold_rule_is_the_causal_mask():
    rng = random.Random(7)
    checked = 0
    for _ in range(1500):
        chunks, c_start, q0, q_rows = random_item(rng)
        total = sum(round8(ln) for _, ln in chunks)
        D = total - round8(chunks[-1][1])
        tiles = walk(chunks)
        assert len(tiles) == (total + BN - 1) // BN
        for kt, kept in enumerate(tiles):
            dt = D - BN * kt
            for r in range(q_rows):
                qt = q0 + r
                thr = max(qt - c_start + dt + 1, 0) if dt < BN else None
                for col, tok in kept.items():
                    masked = thr is not None and col >= thr
                    assert masked == (tok > qt), (kt, r, col, tok)
                    checked += 1
    assert checked > 1_000_000


def test_pieces_start_on_8_slot_boundaries_and_chunks_stay_contiguous():
    rng = random.Random(11)
    for _ in range(300):
        chunks, _, _, _ = random_item(rng)
        tiles = walk(chunks)
        # stream slot of every kept key, in walk order
        stream = []
        for kt, kept in enumerate(tiles):
            stream += [(BN * kt + col, tok) for col, tok in sorted(kept.items())]
        pos = 0
        for s0, ln in chunks:
            slots = [s for s, tok in stream if s0 <= tok < s0 + ln]
            assert slots == list(range(pos, pos + ln))
            pos += round8(ln)
