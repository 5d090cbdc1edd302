"""CPU checks of the work partitions the GEMM kernels use (csrc/qlora_gemm.cu,
csrc/nf4_gemv.cu), written out from their definitions.

Stream-K (dequant GEMM):
* T = tiles × steps per tile is cut into G ranges [floor(b T / G), floor((b+1) T / G)).
* A tile cut between CTAs leaves a partial in CTA b's head slot (slot 0) when the tile starts
  b's range, and in its tail slot (slot 1) otherwise.
* The finalize finds the owners of a tile's first and last steps as
  b = ((g + 1) G - 1) // T.

Few-token forward:
* U = row tiles × 64-blocks units are cut the same way into G ranges.
* Each range is walked in stages of at most 4 blocks that never straddle a row tile.
* Segment s of CTA b writes slot (b, s).
* The finalize reads, for row tile rt, the CTAs from owner(first unit) to owner(last unit).
  The first of them holds the tile as segment rt - (its first unit // KB); the rest hold it
  as segment 0.

Both are checked on random shapes: every unit is covered exactly once, and the finalize
finds exactly the slots the kernel wrote, in step order.
"""

import random


def _sk_start(b, T, G):
    return b * T // G


def test_stream_k_partition():
    rng = random.Random(3)
    for _ in range(1500):
        n_tiles = rng.randint(1, 159)
        total = rng.randint(2, 300)
        G = min(rng.choice([132, 148, 160]), n_tiles * total)
        T = n_tiles * total
        covered = {}
        written = {}
        whole = set()
        for b in range(G):
            g0, n = _sk_start(b, T, G), _sk_start(b + 1, T, G) - _sk_start(b, T, G)
            assert n >= 1
            it = 0
            while it < n:
                t, k0 = divmod(g0 + it, total)
                ln = min(total - k0, n - it)
                for k in range(k0, k0 + ln):
                    assert (t, k) not in covered
                    covered[(t, k)] = b
                if k0 == 0 and ln == total:
                    whole.add(t)
                else:
                    slot = 0 if it == 0 else 1
                    assert (b, slot) not in written
                    written[(b, slot)] = (t, k0, ln)
                it += ln
        assert len(covered) == T
        owner = lambda g: ((g + 1) * G - 1) // T  # noqa: E731
        for t in range(n_tiles):
            gs = t * total
            bf, bl = owner(gs), owner(gs + total - 1)
            assert covered[(t, 0)] == bf and covered[(t, total - 1)] == bl
            if bf == bl:
                assert t in whole
                continue
            ks = 0
            for b in range(bf, bl + 1):
                slot = 0 if _sk_start(b, T, G) >= gs else 1
                tt, k0, ln = written[(b, slot)]
                assert (tt, k0) == (t, ks)
                ks += ln
            assert ks == total


def _gemv_stages(u0, u1, KB, blk=4):
    """The kernel's stage walk: (row tile, first block, blocks, segment, ends segment)."""
    out, u, seg = [], u0, 0
    while u < u1:
        rt = u // KB
        e = min((rt + 1) * KB, u1)
        kb = u - rt * KB
        while True:
            left = e - (rt * KB + kb)
            out.append((rt, kb, min(left, blk), seg, left <= blk))
            if left <= blk:
                break
            kb += blk
        u, seg = e, seg + 1
    return out


def test_few_token_partition():
    rng = random.Random(5)
    for _ in range(1500):
        N, K = 64 * rng.randint(1, 300), 64 * rng.randint(1, 120)
        KB = K // 64
        U = ((N + 127) // 128) * KB
        G = min(2 * rng.choice([132, 148, 160]), U)
        per = (U + G - 1) // G
        max_seg = (per + KB - 1) // KB + 1
        covered, written = {}, set()
        for b in range(G):
            u0, u1 = U * b // G, U * (b + 1) // G
            assert u1 > u0
            for rt, kb, nblk, seg, seg_end in _gemv_stages(u0, u1, KB):
                assert 1 <= nblk <= 4 and seg < max_seg
                for x in range(nblk):
                    u = rt * KB + kb + x
                    assert u0 <= u < u1 and u not in covered
                    covered[u] = b
                if seg_end:
                    written.add((b, seg, rt))
        assert len(covered) == U
        for rt in range((N + 127) // 128):
            us, ue = rt * KB, rt * KB + KB
            bf, bl = ((us + 1) * G - 1) // U, (ue * G - 1) // U
            assert covered[us] == bf and covered[ue - 1] == bl
            seg0 = rt - (U * bf // G) // KB
            for b in range(bf, bl + 1):
                assert (b, seg0 if b == bf else 0, rt) in written


def test_step_cursor_matches_division():
    """The dequant groups advance (tile, step) by two steps without dividing; every tile has
    at least two steps, so one advance wraps at most once."""
    rng = random.Random(11)
    for _ in range(3000):
        total, streamk = rng.randint(2, 70), rng.random() < 0.5
        G, g0 = rng.randint(1, 148), rng.randint(0, 500)
        bx = rng.randrange(G)

        def at(it):
            if streamk:
                return divmod(g0 + it, total)
            lt = it // total
            return bx + lt * G, it - lt * total
        for g in (0, 1):
            t, k = at(g)
            for it in range(g, g + 120, 2):
                assert (t, k) == at(it)
                k += 2
                if k >= total:
                    k -= total
                    t += 1 if streamk else G
