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


def test_swiglu_pair_schedule():
    """The SwiGLU epilogue's tile order (qlora_gemm_kernel's paired schedule): CTA b takes
    pairs q = b, b + G, ... of (gate row tile j, token tile tq), each as the gate tile
    tq * row_tiles + j and then the up tile tq * row_tiles + j + half.  Checked: every tile of
    every token tile is computed exactly once, each up tile right after its own gate tile by the
    same CTA, and the dequant cursor's division-free walk (two steps at a time, j advanced by G
    and wrapped into tq) lands where the division formula does."""
    rng = random.Random(23)
    for _ in range(400):
        half = rng.randint(1, 120)        # gate row tiles (I / 128)
        row_tiles = 2 * half
        token_tiles = rng.randint(1, 12)
        G = rng.choice([132, 148, 160])
        total = rng.randint(2, 70)
        pairs = half * token_tiles

        def at(b, it):
            lt, k = divmod(it, total)
            q = b + (lt >> 1) * G
            tq, j = divmod(q, half)
            return tq * row_tiles + j + (lt & 1) * half, k
        seen = {}
        for b in range(G):
            my_pairs = (pairs - 1 - b) // G + 1 if b < pairs else 0
            n = 2 * my_pairs * total
            order = []
            for it in range(0, n, total):
                t, k = at(b, it)
                assert k == 0
                assert t not in seen
                seen[t] = b
                order.append(t)
            for i in range(0, len(order), 2):
                gate, up = order[i], order[i + 1]
                assert up == gate + half and (gate % row_tiles) < half
            for g in (0, 1):  # the cursor: set once, then advanced without dividing
                if n <= g:
                    continue
                t, k = at(b, g)
                lt = g // total
                q = b + (lt >> 1) * G
                tq, j = divmod(q, half)
                for it in range(g, n, 2):
                    assert (t, k) == at(b, it)
                    k += 2
                    if k >= total:
                        k -= total
                        lt += 1
                        if lt % 2 == 0:
                            j += G
                            while j >= half:
                                j -= half
                                tq += 1
                        t = tq * row_tiles + j + (lt & 1) * half
        assert len(seen) == row_tiles * token_tiles


def test_gemm_plan_properties():
    """The dequant GEMM's launch plan (qlora_gemm_plan, host only) on random problems:
    * token tiles: one half of M rounded up to 16 for M <= 256, else two halves of a multiple
      of 16 in [128, 256];
    * stream-K exactly when 512-token tiles would leave SMs idle;
    * the grid and the partial-sum bytes that follow from the schedule;
    * qlora_workspace_bytes covers the partial sums of both GEMMs of a layer for every device
      of up to 160 SMs."""
    import os
    from nf4_base_lora_blockwise_b200 import abi
    if not os.path.exists(abi.LIB_PATH):
        from nf4_base_lora_blockwise_b200 import build
        build.build()
    rng = random.Random(17)
    for _ in range(400):
        M = rng.choice([1, 7, 16, 33, 128, 200, 256, 257, 300, 1024, 2048, 4096, 8192, 16384])
        N, K = 64 * rng.randint(1, 300), 64 * rng.randint(2, 300)
        r = rng.choice([8, 16, 64])
        sms = rng.choice([132, 148, 160])
        for trans in (False, True):
            rows, steps = (K, N // 64) if trans else (N, K // 64)
            steps += ((r + 15) // 16 * 16 + 63) // 64
            p = abi.qlora_gemm_plan(M, rows, steps, sms)
            if M <= 256:
                assert p["nh"] == 1 and p["bt"] == max(16, (M + 15) // 16 * 16)
            else:
                assert p["nh"] == 2 and p["bt"] % 16 == 0 and 128 <= p["bt"] <= 256
            G = min(sms, 160)
            tt = p["bt"] * p["nh"]
            tiles = ((rows + 127) // 128) * ((M + tt - 1) // tt)
            wide = ((rows + 127) // 128) * ((M + (512 if M > 256 else tt) - 1)
                                           // (512 if M > 256 else tt))
            assert p["streamk"] == (1 if wide < G else 0)
            if p["streamk"]:
                assert p["bt"] == (256 if M > 256 else p["bt"])
                assert p["grid"] == min(tiles * steps, G)
                assert p["partial_bytes"] == p["grid"] * 2 * tt * 128 * 4
            else:
                assert p["grid"] == G and tiles >= G and p["partial_bytes"] == 0
        if M > 32:  # the few-token forward has its own slots; larger M uses these GEMMs only
            need = abi.qlora_workspace_bytes(M, N, K, r)
            for trans in (False, True):
                rows, steps = (K, N // 64) if trans else (N, K // 64)
                steps += ((r + 15) // 16 * 16 + 63) // 64
                for s2 in (100, 132, 148, 160):
                    assert abi.qlora_gemm_plan(M, rows, steps, s2)["partial_bytes"] <= need


def test_gemm_plan_headline_tile():
    """q_proj 4096 -> 4096 at 4096 tokens on 148 SMs: 480-token tiles (288 tiles, two per CTA
    on 140 CTAs) instead of 512 (256 tiles, where 108 CTAs run two)."""
    from nf4_base_lora_blockwise_b200 import abi
    p = abi.qlora_gemm_plan(4096, 4096, 64 + 1, 148)
    assert (p["bt"], p["nh"], p["streamk"], p["grid"]) == (240, 2, 0, 148)


def _windows(M, tq, bt, nh):
    """The 128-token windows of token tile tq: per half with valid tokens, rows [0, 128) and,
    past 128 valid tokens, rows [bt - 128, bt) writing rows 128 .. bt - 1.  Each window as
    (half, first row, first row it writes)."""
    rest = M - tq * bt * nh
    out = []
    for h in range(nh):
        toks = min(bt, rest - h * bt)
        if toks > 0:
            out.append((h, 0, 0))
        if toks > 128:
            out.append((h, bt - 128, 256 - bt))
    return out


def _rank_ring_fits(bt, nh, slot):
    """The GEMM's shared-memory plan with the rank operand's ring (one slot per X ring step)
    after the W ring (4 x 16 KB), the code ring (2 << qlog tiles of 4 KB; shallower if needed),
    the X ring (2 or 4 steps of bt x 128 B per half) and 2 KB of alignment and barriers."""
    qlog = 4 if bt <= 64 else (3 if bt <= 128 else 2)
    dx = 2 if nh == 2 else 4
    while True:
        smem = 2048 + (2 << qlog) * 4096 + 4 * 16384 + dx * nh * bt * 128
        if smem + dx * slot <= 232448:
            return True
        if qlog <= 1:
            return False
        qlog -= 1


def test_rank_fusion_decision_and_coverage():
    """qlora_gemm_rank_fusable against a model of the fused down-projection's schedule.  When it
    fuses, the launch runs whole tiles of two halves of 144..240 tokens (the accumulator's 2 bt
    TMEM columns leave room for the window's), n r is a multiple of 8 up to 32 (dX: r = 16 or
    32), the rank operand's ring fits in shared memory, and every token tile's windows fall on
    its tiles in the first wave of tiles that reaches it, their written rows covering each valid
    token exactly once.  It never fuses what the kernels cannot: n r above 32 or not a multiple
    of 8, dX with r = 8 or 24, 256 tokens or fewer."""
    import os
    from nf4_base_lora_blockwise_b200 import abi
    if not os.path.exists(abi.LIB_PATH):
        from nf4_base_lora_blockwise_b200 import build
        build.build()
    rng = random.Random(23)
    fused = 0
    for _ in range(400):
        M = rng.choice([17, 33, 300, 1024, 1300, 2048, 4096, 6000, 8192, 16384])
        rows = 64 * rng.randint(2, 260)
        steps = rng.randint(2, 200)
        R = rng.choice([8, 16, 24, 32, 40, 64])
        r = rng.choice([x for x in (8, 16, 24, 32) if x <= R and R % x == 0])
        trans = rng.random() < 0.5
        sms = rng.choice([132, 148])
        bt = abi.qlora_gemm_rank_fusable(M, rows, steps, sms, R, r, trans)
        if R > 32 or M <= 256 or (trans and r not in (16, 32)):
            assert bt == 0, (M, rows, steps, R, r, trans)
        if not bt:
            continue
        fused += 1
        nh, G = 2, min(sms, 160)
        npad = (R + 15) // 16 * 16
        assert 144 <= bt <= 240 and bt % 16 == 0 and 2 * bt + npad <= 512
        assert _rank_ring_fits(bt, nh, 128 * r if trans else 128 * npad)
        row_tiles = (rows + 127) // 128
        token_tiles = (M + bt * nh - 1) // (bt * nh)
        assert row_tiles * token_tiles >= G  # whole tiles, one CTA per SM
        for tq in range(token_tiles):
            wins = _windows(M, tq, bt, nh)
            t0 = tq * row_tiles
            assert len(wins) <= min(row_tiles, (t0 // G + 1) * G - t0)
            valid = min(bt * nh, M - tq * bt * nh)
            cover = sorted(h * bt + w0 + row for h, w0, own0 in wins for row in range(own0, 128)
                           if h * bt + w0 + row < valid)
            assert cover == list(range(valid)), (M, tq, bt)
    assert fused > 20
    # The headline layer fuses in both directions: 4096 tokens, q_proj 4096 -> 4096, r = 16.
    assert abi.qlora_gemm_rank_fusable(4096, 4096, 64 + 1, 148, 16, 16, False) == 240
    assert abi.qlora_gemm_rank_fusable(4096, 4096, 64 + 1, 148, 16, 16, True) == 240


def test_backward_side_sms():
    """SMs the backward gives to dB / dA beside the dX GEMM (qlora_backward_side_sms, host
    only): an even count in [2, 32] or 0; 0 in mode 0, for stream-K shapes and M <= 256; mode 1
    gives either 0 or mode 2's split, and 0 for R > 32 or dY above 48 MiB; with s SMs given
    away the GEMM's plan on the rest is still whole tiles on every remaining SM; and the q_proj
    backward (4096 tokens, 4096 x 4096, r 16) gives 20 of 148 SMs, so the GEMM runs its 256
    tiles of 512 tokens two per CTA on 128 CTAs."""
    from nf4_base_lora_blockwise_b200 import abi
    assert abi.qlora_backward_side_sms(4096, 4096, 4096, 16, 148, 1) == 20
    p = abi.qlora_gemm_plan(4096, 4096, 64 + 1, 128)
    assert (p["bt"] * p["nh"], p["streamk"], p["grid"]) == (512, 0, 128)
    assert abi.qlora_backward_side_sms(4096, 4096, 4096, 16, 148, 0) == 0
    assert abi.qlora_backward_side_sms(4096, 4096, 4096, 64, 148, 1) == 0   # R > 32
    assert abi.qlora_backward_side_sms(4096, 4096, 4096, 64, 148, 2) > 0
    assert abi.qlora_backward_side_sms(8192, 4096, 14336, 16, 148, 1) == 0  # dY 64 MiB
    assert abi.qlora_backward_side_sms(256, 4096, 4096, 16, 148, 2) == 0
    assert abi.qlora_backward_side_sms(4096, 4096, 4096, 16, 32, 2) == 0    # too few SMs
    rng = random.Random(23)
    seen = 0
    for _ in range(300):
        M = rng.choice([128, 256, 300, 1024, 2048, 3000, 4096, 8192, 16384])
        N, K = 64 * rng.randint(1, 460), 128 * rng.randint(1, 230)
        R = rng.choice([8, 16, 32, 64])
        sms = rng.choice([132, 148, 160])
        s = abi.qlora_backward_side_sms(M, N, K, R, sms, 2)
        assert s == 0 or (s % 2 == 0 and 2 <= s <= 32)
        s1 = abi.qlora_backward_side_sms(M, N, K, R, sms, 1)
        assert s1 in (0, s)
        if R > 32 or 2 * M * N > 48 * 2**20:
            assert s1 == 0
        steps = N // 64 + ((R + 15) // 16 * 16 + 63) // 64
        full = abi.qlora_gemm_plan(M, K, steps, sms)
        if M <= 256 or full["streamk"]:
            assert s == 0
        if s == 0:
            continue
        seen += 1
        part = abi.qlora_gemm_plan(M, K, steps, sms - s)
        assert part["streamk"] == 0 and part["grid"] == sms - s
    assert seen > 20
