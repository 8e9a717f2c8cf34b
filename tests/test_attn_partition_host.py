"""The tensor-core attention's work partition, checked on the host (no GPU).

The persistent attention kernel cuts a line of work units into chunks: each (request,
row block, kv head) sequence takes kAttnSeqUnits units for its start, then one unit per
64-key tile (its context tiles, then the block's own keys).  The schedule kernel sums
the units, the producers walk each chunk as pieces (one per sequence whose tiles the
chunk holds) and write piece (sequence q, chunk k) to partial slot q + k, and the merge
kernel finds a sequence's pieces and halves from T, Z and the request's offset alone.

This test restates those three views in Python, with the start charge read from the
kernels' header, and checks on random batches that:
- the pieces cover every tile of every valid sequence exactly once,
- partial slots never collide and stay inside the workspace's slot count,
- the merge's view of each sequence (its pieces, their tile counts and which halves
  exist) is the producers' view,
- the number of chunks respects the workspace bound, and every chunk's work is within
  one unit of the others'.
"""
import math
import pathlib
import re

import numpy as np
import pytest

TT = 64            # keys per tile
ROWS = 128         # query rows per row block
HDR = pathlib.Path(__file__).resolve().parents[1] / "hybrid_mamba_attention_b200" / "csrc" / "kernels.cuh"


def seq_start_units():
    m = re.search(r"constexpr int kAttnSeqUnits = (\d+);", HDR.read_text())
    assert m, "kAttnSeqUnits not found in kernels.cuh"
    return int(m.group(1))


W = seq_start_units()


def schedule(ctx, K, Hkv, G, max_ctx, grid, z_req, max_chunks):
    """The schedule kernel: offsets on the line, T, Z and the number of chunks."""
    R = K * G
    n_rb = -(-R // ROWS)
    spr = Hkv * n_rb
    nbt = -(-K // TT)

    def units(c_len):
        return 0 if c_len < 0 or c_len > max_ctx else W + -(-c_len // TT) + nbt

    off = [0]
    for c_len in ctx:
        off.append(off[-1] + units(c_len) * spr)
    T = off[-1]
    Z = z_req if z_req > 0 else -(-T // grid)
    Z = max(Z, -(-T // max_chunks), 1)
    n_chunks = -(-T // Z)
    return off, T, Z, n_chunks, spr


def producer_pieces(off, T, Z, n_chunks, spr, C, grid):
    """Every CTA's walk over its chunks: pieces (c, r, first tile, tiles, chunk)."""
    pieces = []
    for b in range(grid):
        k = b
        if k >= n_chunks:
            continue
        pos, end = k * Z, min(T, k * Z + Z)
        c = max(i for i in range(C) if off[i] <= pos)  # the last request with off[c] <= pos
        while True:
            n_tiles = 0
            done = False
            while n_tiles == 0:
                if pos >= end:
                    k += grid
                    if k >= n_chunks:
                        done = True
                        break
                    pos, end = k * Z, min(T, k * Z + Z)
                    c = max(i for i in range(C) if off[i] <= pos)
                while off[c + 1] <= pos:
                    c += 1
                tw = (off[c + 1] - off[c]) // spr
                rel = pos - off[c]
                r = rel // tw
                u0 = rel - r * tw
                u1 = min(tw, u0 + (end - pos))
                pos += u1 - u0
                lt0 = max(u0 - W, 0)
                n_tiles = max(u1 - W - lt0, 0)
            if done:
                break
            pieces.append((c, r, lt0, n_tiles, k))
    return pieces


def merge_view(off, Z, spr, c, r):
    """The merge kernel's view of sequence (c, r): (slot, tiles in the piece, halves)."""
    tw = (off[c + 1] - off[c]) // spr
    t_seq = tw - W
    s0 = off[c] + r * tw + W
    k0 = s0 // Z
    ns = 2 * ((s0 + t_seq - 1) // Z - k0 + 1) if t_seq > 0 else 0
    out = []
    for p in range(ns // 2):
        lo, hi = max(s0, (k0 + p) * Z), min(s0 + t_seq, (k0 + p + 1) * Z)
        halves = [hh for hh in (0, 1) if hi - lo > hh]
        out.append((c * spr + r + k0 + p, hi - lo, halves))
    return out


CASES = [
    # C, K, Hkv, G, ctx range, grid, z_req (units; 0 = one chunk per SM)
    (1, 16, 8, 4, (2048, 2048), 148, 0),
    (3, 1, 1, 4, (0, 200), 148, 0),
    (8, 16, 8, 4, (512, 16384), 148, 0),
    (32, 16, 8, 4, (512, 8192), 148, 0),
    (128, 16, 8, 4, (512, 16384), 148, 0),
    (128, 16, 8, 5, (1024, 32768), 148, 0),
    (16, 33, 8, 4, (0, 3000), 148, 0),        # R = 132: two row blocks
    (64, 64, 2, 4, (0, 5000), 148, 0),        # R = 256
    (24, 16, 8, 4, (0, 9000), 148, 3),        # explicit short chunks: many pieces per sequence
    (24, 16, 8, 4, (0, 9000), 148, 40),
    (5, 8, 4, 4, (0, 700), 7, 0),             # a small grid
]


@pytest.mark.parametrize("C,K,Hkv,G,ctx_range,grid,z_req", CASES)
def test_partition_covers_every_tile_once_with_distinct_slots(C, K, Hkv, G, ctx_range, grid, z_req):
    rng = np.random.default_rng(C * 1000 + K)
    max_ctx = 40000
    ctx = rng.integers(ctx_range[0], ctx_range[1] + 1, size=C).tolist()
    if C >= 3:
        ctx[1] = -1              # invalid lengths: no units, no pieces (the merge writes zeros)
        ctx[-1] = max_ctx + 1
    max_chunks = 2048 if z_req > 0 else 256
    off, T, Z, n_chunks, spr = schedule(ctx, K, Hkv, G, max_ctx, grid, z_req, max_chunks)
    assert n_chunks <= max_chunks
    pieces = producer_pieces(off, T, Z, n_chunks, spr, C, grid)

    # every tile of every valid sequence exactly once; nothing for invalid ones
    nbt = -(-K // TT)
    covered = {}
    for c, r, lt0, n, k in pieces:
        assert n > 0
        for t in range(lt0, lt0 + n):
            key = (c, r, t)
            assert key not in covered, f"tile {key} in two pieces"
            covered[key] = k
    for c, c_len in enumerate(ctx):
        valid = 0 <= c_len <= max_ctx
        t_seq = -(-c_len // TT) + nbt if valid else 0
        for r in range(spr):
            for t in range(t_seq):
                assert (c, r, t) in covered, f"tile {(c, r, t)} missing"
    assert len(covered) == sum((-(-x // TT) + nbt) * spr for x in ctx if 0 <= x <= max_ctx)

    # slots: distinct, inside the workspace's C * spr + max_chunks slots
    slots = [c * spr + r + k for c, r, _, _, k in pieces]
    assert len(set(slots)) == len(slots)
    assert max(slots) < C * spr + max_chunks

    # the merge finds exactly the producers' pieces of each sequence, with their sizes
    by_seq = {}
    for c, r, lt0, n, k in pieces:
        by_seq.setdefault((c, r), []).append((c * spr + r + k, n))
    for c, c_len in enumerate(ctx):
        if not 0 <= c_len <= max_ctx:
            continue
        for r in range(spr):
            view = merge_view(off, Z, spr, c, r)
            assert [(s, n) for s, n, _ in view if n > 0] == sorted(by_seq[(c, r)])
            for s, n, halves in view:
                assert halves == [hh for hh in (0, 1) if n > hh]  # half h = the piece's tiles of parity h

    # every chunk holds Z units (the last one the rest)
    for k in range(n_chunks):
        assert min(T, (k + 1) * Z) - k * Z == (Z if k < n_chunks - 1 else T - k * Z)


def test_sequence_starts_are_charged_as_work():
    # With one chunk per SM, a CTA whose chunk crosses many short sequences gets fewer
    # tiles than one that holds part of a long sequence: the start units even out the
    # cost of the pieces (each a Q load, page lookups and partials).
    ctx = [100] * 64 + [60000]
    off, T, Z, n_chunks, spr = schedule(ctx, 16, 1, 4, 70000, 8, 0, 256)
    pieces = producer_pieces(off, T, Z, n_chunks, spr, len(ctx), 8)
    per_cta_tiles = {}
    per_cta_pieces = {}
    for c, r, lt0, n, k in pieces:
        per_cta_tiles[k] = per_cta_tiles.get(k, 0) + n
        per_cta_pieces[k] = per_cta_pieces.get(k, 0) + 1
    for k in per_cta_tiles:
        # units = tiles + W per piece that starts a sequence in the chunk: equal across
        # chunks up to one sequence start cut by a boundary
        assert abs(per_cta_tiles[k] + W * per_cta_pieces[k] - Z) <= W + 1 or k == n_chunks - 1
    assert per_cta_tiles[0] < per_cta_tiles[n_chunks - 2]
