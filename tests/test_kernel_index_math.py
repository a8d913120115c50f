"""Host-side checks of the index arithmetic of the selector and covariance kernels,
restated from their sources: every row is copied exactly once and inside its buffer,
every byte count matches the copies it announces, the Jacobi rotation schedule is
a round-robin tournament, and the covariance kernel's shared-memory carve-up is
aligned and inside its allocation. No GPU is needed."""
from __future__ import annotations

import itertools

import pytest

SEL_THREADS = 256
SEL_NW = SEL_THREADS // 32
SEL_STAGES = 3


def pow2ceil(x):
    p = 1
    while p < x:
        p *= 2
    return p


def ring_rows_per_stage(G):
    """sel_ring_bytes: rows (512-byte slots) a warp holds per stage."""
    GP = pow2ceil(G)
    return 32 // GP if GP >= 4 else 8


# ------------------------------------------------------------ Jacobi schedule
def circle_pairs(m, rnd):
    """Pairs of one round of the covariance kernel's schedule (thread t < m/2)."""
    out = []
    for t in range(m // 2):
        a, b = t, m - 1 - t
        p = 0 if a == 0 else 1 + (a - 1 + rnd) % (m - 1)
        q = 1 + (b - 1 + rnd) % (m - 1)
        out.append((min(p, q), max(p, q)))
    return out


@pytest.mark.parametrize("m", [2, 4, 6, 16, 32, 64])
def test_jacobi_round_robin(m):
    seen = []
    for rnd in range(m - 1):
        pairs = circle_pairs(m, rnd)
        flat = [i for pq in pairs for i in pq]
        assert sorted(flat) == list(range(m)), f"round {rnd}: pairs not disjoint / not covering"
        assert all(p != q for p, q in pairs)
        seen += pairs
    assert sorted(seen) == sorted(itertools.combinations(range(m), 2)), "a pair missing or repeated in a sweep"


# ------------------------------------------------------------ scorer ring
def scorer_copies(D, G, nbv):
    """The first-order scorer's bulk copies: (warp, m, slot, first row, rows) and the
    bytes each (warp, m) announces."""
    LPR = D // 4
    RPW = 32 // LPR
    GP = pow2ceil(G)
    RS = min(8, max(1, LPR // GP))
    BATCH = RPW * RS
    nbt = (nbv + BATCH - 1) // BATCH
    copies, announced = [], {}
    for warp in range(SEL_NW):
        nmine = (nbt - warp + SEL_NW - 1) // SEL_NW if nbt > warp else 0
        for m in range(nmine):
            rb = (warp + m * SEL_NW) * BATCH
            nvalid = min(BATCH, nbv - rb)
            assert nvalid >= 1
            announced[(warp, m)] = nvalid * D * 4
            got = 0
            for lane in range(RS):
                r0 = rb + lane * RPW
                nr = min(RPW, nbv - r0)
                if nr > 0:
                    copies.append((warp, m, lane, r0, nr))
                    got += nr * D * 4
            assert got == announced[(warp, m)], "expect_tx differs from the bytes copied"
    return copies, RS


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 7, 8])
@pytest.mark.parametrize("nbv", [0, 1, 7, 8, 9, 63, 64, 65, 512, 1031])
def test_scorer_ring_covers_rows_once(D, G, nbv):
    copies, RS = scorer_copies(D, G, nbv)
    rows = sorted(r for (_, _, _, r0, nr) in copies for r in range(r0, r0 + nr))
    assert rows == list(range(nbv))
    assert RS <= ring_rows_per_stage(G), "stage rows exceed the ring's allocation"
    for (warp, m, slot, r0, nr) in copies:
        assert nr * D * 4 <= 512, "a copy larger than its 512-byte slot"
        f4 = ((m % SEL_STAGES) * RS + slot) * SEL_THREADS + warp * 32  # float4 index of the slot
        assert f4 + 32 <= SEL_STAGES * ring_rows_per_stage(G) * SEL_THREADS


# ------------------------------------------------------------ second-order ring
def cobs_copies(G, r, nbv):
    RSC = ring_rows_per_stage(G)
    assert r <= RSC
    bpb = RSC // r
    nbt = (nbv + bpb - 1) // bpb
    out = []
    for warp in range(SEL_NW):
        nmine = (nbt - warp + SEL_NW - 1) // SEL_NW if nbt > warp else 0
        for m in range(nmine):
            b0 = (warp + m * SEL_NW) * bpb
            nrows = min(bpb, nbv - b0) * r
            assert nrows >= r
            for lane in range(nrows):
                row = b0 * r + lane  # factor lane % r of block b0 + lane // r
                out.append((warp, m, lane, row))
            assert nrows <= RSC
    return out, RSC


@pytest.mark.parametrize("G", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("r", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("nbv", [1, 5, 64, 513])
def test_cobs_ring_covers_factor_rows_once(G, r, nbv):
    if r > ring_rows_per_stage(G):
        pytest.skip("this rank takes the direct-load path")
    copies, RSC = cobs_copies(G, r, nbv)
    rows = sorted(row for (_, _, _, row) in copies)
    assert rows == list(range(nbv * r))
    for (warp, m, lane, row) in copies:
        f4 = ((m % SEL_STAGES) * RSC + lane) * SEL_THREADS + warp * 32
        assert f4 + 32 <= SEL_STAGES * RSC * SEL_THREADS


def test_cobs_leaders_sum_whole_blocks():
    # after the transpose reduction lane c holds value c / SPAN = row * GP + head; a
    # leader (first row of a block) adds the values r - 1 ... shifts above it, which
    # must be the same head's later rows of the same block, inside the warp
    for G in (1, 2, 3, 4, 5, 7, 8):
        GP = pow2ceil(G)
        RSC = ring_rows_per_stage(G)
        NV = RSC * GP
        SPAN = 32 // NV
        for r in range(1, RSC + 1):
            bpb = RSC // r
            for lane in range(32):
                vi = lane // SPAN
                row, g = divmod(vi, GP)
                if lane % SPAN or g >= G or row % r or row >= bpb * r:
                    continue
                for t in range(1, r):
                    src = lane + t * GP * SPAN
                    assert src < 32
                    vs = src // SPAN
                    assert vs % GP == g and vs // GP == row + t and (row + t) // r == row // r


# ------------------------------------------------------------ covariance smem
def cov_layout(L, D):
    m = (L + 1) & ~1
    kx = L * (D + 1) * 4
    mean = (kx + 15) & ~15
    A = mean + D * 8
    V = A + m * (m + 1) * 8
    rot = V + m * (m + 1) * 8
    pr = rot + (m // 2) * 16
    red = pr + (m // 2) * 8
    sel = red + 32 * 8
    end = sel + 8 * 4
    total = ((L * (D + 1) * 4 + 15) & ~15) + D * 8 + 2 * m * (m + 1) * 8 + (m // 2) * 16 + (m // 2) * 8 + 64 * 8
    return dict(mean=mean, A=A, V=V, rot=rot, pr=pr, red=red, sel=sel, end=end, total=total)


@pytest.mark.parametrize("L", [16, 32, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_cov_smem_layout(L, D):
    o = cov_layout(L, D)
    for k in ("mean", "A", "V", "red"):
        assert o[k] % 8 == 0, k
    assert o["rot"] % 16 == 0, "double2 rotations need 16-byte alignment"
    assert o["end"] <= o["total"], "carve-up runs past the allocation"
    assert o["total"] <= 227 * 1024


# ------------------------------------------------------------ WildCat producer
def wc_fidx(j, i, m):
    """Tiled factor index: F[j][i] at (i / 32) * 32 m + 32 j + i % 32."""
    return (i >> 5) * (32 * m) + 32 * j + (i & 31)


@pytest.mark.parametrize("Ncap,m", [(1, 1), (31, 3), (32, 4), (33, 5), (100, 7), (1000, 64)])
def test_wildcat_factor_tiles_bijective(Ncap, m):
    # every (row j < m, token i < Ncap rounded up to 32) has its own slot inside the
    # m rows of the factor, ahead of the residual diagonal and the column sums
    n32 = (Ncap + 31) & ~31
    idx = {wc_fidx(j, i, m) for j in range(m) for i in range(n32)}
    assert len(idx) == m * n32 and min(idx) == 0 and max(idx) == m * n32 - 1
    # a batch's t rows are one contiguous run of 32 t floats
    for t in (1, m):
        run = sorted(wc_fidx(j, 32 + lane, m) for j in range(t) for lane in range(32)) if n32 > 32 else []
        if run:
            assert run == list(range(run[0], run[0] + 32 * t))
    # per-pair stride and the workspace bytes of the C entry
    per_pair = (m + 1) * n32 + 8 * m
    assert m * n32 + n32 + 8 * m == per_pair


def transpose_reduce(vals, N, MASK):
    """Restatement of transpose_reduce<N, MASK> over 32 lanes (vals[lane][k])."""
    v = [list(x) for x in vals]
    while MASK >= 1:
        if N > 1:
            nv = []
            for lane in range(32):
                up = (lane & MASK) != 0
                other = lane ^ MASK
                row = []
                for j in range(N // 2):
                    keep = v[lane][j + N // 2] if up else v[lane][j]
                    up_o = (other & MASK) != 0
                    send_o = v[other][j] if up_o else v[other][j + N // 2]
                    row.append(keep + send_o)
                nv.append(row)
            v, N = nv, N // 2
        else:
            v = [[v[lane][0] + v[lane ^ MASK][0]] for lane in range(32)]
        MASK //= 2
    return [x[0] for x in v]


@pytest.mark.parametrize("esize,D", [(2, 128), (2, 64), (4, 128), (4, 64)])
def test_wildcat_lane_layout_covers_rows(esize, D):
    che = 16 // esize
    cpl = D // che // 8
    assert cpl * che * 8 == D
    # the 8 lanes of a group read the 16-byte chunks c + 8 kk of a row: each once
    chunks = sorted(c + 8 * kk for c in range(8) for kk in range(cpl))
    assert chunks == list(range(D // che))
    # lane l's partial for row 8 (l / 8) + k is v[k]; after the 8-value transpose
    # reduction lane l holds the sum over its group of v[l % 8]: row l's dot product
    part = [[1000.0 * (8 * (lane >> 3) + k) + (lane & 7) for k in range(8)] for lane in range(32)]
    out = transpose_reduce(part, 8, 4)
    for lane in range(32):
        assert out[lane] == 8 * 1000.0 * lane + sum(range(8))


# ------------------------------------------------------------ QGC radix selection
def kth_largest_radix(keys, rc):
    """Restatement of qg_kth_largest: radix selection on 8-bit digits below the bits
    all keys share, then a direct ranking of at most 32 candidates."""
    M = (1 << 64) - 1
    a, o = M, 0
    for x in keys:
        a &= x
        o |= x
    hb = (a ^ o).bit_length() - 1
    assert hb >= 0
    pmask = 0 if hb == 63 else (~((2 << hb) - 1)) & M
    prefix = a & pmask
    need = rc
    top = hb
    while True:
        lo = top - 7
        dmask = (255 << lo) if lo >= 0 else (255 >> (-lo))
        hist = [0] * 256
        for x in keys:
            if x & pmask == prefix:
                hist[((x >> lo) if lo >= 0 else (x << (-lo))) & 255] += 1
        # lanes hold bins 255 - 8 L - j: a descending walk over the digits
        acc = 0
        for dig in range(255, -1, -1):
            if acc + hist[dig] >= need:
                above, cdig = acc, hist[dig]
                break
            acc += hist[dig]
        need -= above
        prefix |= (dig << lo) if lo >= 0 else (dig >> (-lo))
        pmask |= dmask
        if cdig <= 32:
            break
        top -= 8
    cand = [x for x in keys if x & pmask == prefix]
    assert len(cand) <= 32
    win = [x for x in cand if sum(y > x for y in cand) == need - 1]
    assert len(win) == 1
    return win[0]


@pytest.mark.parametrize("seed", range(6))
def test_qgc_radix_selection_matches_sort(seed):
    import random
    import struct
    rng = random.Random(seed)
    for trial in range(16):
        nc = rng.choice([2, 3, 17, 33, 100, 1000, 3000])
        kind = trial % 4
        m0 = rng.randrange(0, 1 << 20)
        keys = []
        for m in range(m0, m0 + nc):
            if kind == 0:
                t = rng.random() * 1e-3
            elif kind == 1:
                t = 0.0 if rng.random() < 0.7 else rng.random()  # many equal scores
            elif kind == 2:
                t = 10 ** rng.uniform(-30, 0)
            else:
                t = 0.25  # all equal: order by member position alone
            tb = struct.unpack("<I", struct.pack("<f", t))[0]
            keys.append((tb << 32) | (0xFFFFFFFF - m))
        for rc in {1, 2, nc // 2 or 1, nc - 1, min(28, nc - 1)}:
            if not 1 <= rc < nc:
                continue
            assert kth_largest_radix(keys, rc) == sorted(keys, reverse=True)[rc - 1]


def test_qgc_inverted_position_and_or_closed_form():
    # AND and OR of 2^32 - 1 - m over m0 <= m < m1, as the selection forms them
    import random
    rng = random.Random(5)
    M = 0xFFFFFFFF
    for _ in range(300):
        m0 = rng.randrange(0, 1 << 20)
        m1 = m0 + rng.choice([2, 3, 31, 32, 33, 1000, rng.randrange(2, 5000)])
        lo_v, hi_v = M - (m1 - 1), M - m0
        dv = lo_v ^ hi_v
        lmask = 0 if dv == 0 else (M >> (32 - dv.bit_length()))
        a = o = None
        for m in range(m0, m1):
            v = M - m
            a = v if a is None else a & v
            o = v if o is None else o | v
        assert (lo_v & ~lmask & M) == a and (lo_v | lmask) == o


def test_qgc_merge_transpose_lanes():
    # the proxy merge reduces sixteen proxies' partial dots with the 16-value transpose
    # starting at lane mask 16: lane l then holds proxy (l >> 1) % 16's whole dot
    part = [[1000.0 * k + lane for k in range(16)] for lane in range(32)]
    out = transpose_reduce(part, 16, 16)
    for lane in range(32):
        assert out[lane] == 32 * 1000.0 * ((lane >> 1) & 15) + sum(range(32))
