"""Layout invariants of the persistent decode kernel, checked on the CPU.

The kernel (expert_offload_b200/csrc/stack.cu) keeps activations, h vectors
and a ring of expert bytes in shared memory with padded rows and 16-byte
aligned bulk copies.  This test restates its index arithmetic and checks, for
every shape the workloads use, that each shared-memory access is aligned for
its width and in bounds and that every ring item's copy covers the rows the
consumers read.  (A misaligned float2 store once came from a wrong padding
formula; this pins the fixed one.)
"""
import pytest

K_STAGE, K_BB, K_HS_PAIRS, K_CW = 17408, 136, 16, 8


def xpad(c):
    return c + 2 * (c >> 6)


def span16(off, ln):
    a16 = off & ~15
    return a16, ((off + ln + 15) & ~15) - a16, off - a16


@pytest.mark.parametrize("T,H,I,k", [(1, 2048, 512, 8), (2, 2048, 512, 8), (5, 2048, 512, 8),
                                     (8, 2048, 512, 8), (8, 256, 128, 4), (1, 256, 128, 4)])
def test_shared_memory_accesses_are_aligned_and_in_bounds(T, H, I, k):
    nbH, nbI = -(-H // 256), -(-I // 256)
    Hp, Ip = nbH * 256, nbI * 256
    HxRow, HsRow = Hp + 2 * (Hp >> 6), Ip // 16 * 20
    # activations: float2 stores of column pairs, lane slices of 64 contiguous
    for c in range(0, Hp, 2):
        for t in range(T):
            off = t * HxRow + xpad(c)
            assert off % 2 == 0 and off + 2 <= T * HxRow
    for lane in range(32):
        pb, pq = lane >> 2, lane & 3
        if pb >= nbH:
            continue
        col0 = pb * 256 + pq * 64
        for i in range(32):
            assert xpad(col0) + 2 * i == xpad(col0 + 2 * i)       # slice stays contiguous
    # h staging: float4 stores, float2 reads of 16-value chunks
    for ps in range(K_HS_PAIRS):
        for c in range(0, Ip, 4):
            off = ps * HsRow + (c >> 4) * 20 + (c & 15)
            assert off % 4 == 0 and off + 4 <= K_HS_PAIRS * HsRow
    # padded layouts put the lanes of a warp on distinct bank pairs
    banks = {(xpad(((l >> 2) * 256 + (l & 3) * 64)) % 32) for l in range(16) if (l >> 2) < nbH}
    assert len(banks) == min(16, 4 * nbH)
    banks = {(c * 20) % 32 for c in range(8)}
    assert len(banks) == 8


@pytest.mark.parametrize("T,H,I,k,G", [(1, 2048, 512, 8, 148), (8, 2048, 512, 8, 148),
                                       (8, 256, 128, 4, 148), (1, 2048, 512, 8, 132)])
def test_ring_items_cover_what_consumers_read(T, H, I, k, G):
    nbH, nbI = -(-H // 256), -(-I // 256)
    rowB_gu, rowB_d = nbH * K_BB, nbI * K_BB
    mg = I * rowB_gu
    eb = 2 * mg + H * rowB_d
    assert eb % 16 == 0
    n_gu, n_d = (K_STAGE // 2 - 16) // rowB_gu, (K_STAGE - 16) // rowB_d
    U = min(T * k, 128)
    for c in range(G):
        fill = 0
        for q in range(2 * U):
            down = q >= U
            lo = c * (H if down else I) // G
            hi = (c + 1) * (H if down else I) // G
            nmax = n_d if down else n_gu
            r0 = lo
            while r0 < hi:
                n = min(nmax, hi - r0)
                rowB = rowB_d if down else rowB_gu
                bases = [2 * mg] if down else [0, mg]
                spans = [span16(b + r0 * rowB, n * rowB) for b in bases]
                need = sum(s[1] for s in spans)
                if fill + need > K_STAGE:
                    fill = 0
                off = fill
                for a16, ln, dl in spans:
                    assert off % 16 == 0 and ln % 16 == 0 and a16 % 16 == 0
                    assert a16 + ln <= eb and off + ln <= K_STAGE
                    assert dl in (0, 8)
                    # the last row's last byte read lies inside the copy
                    assert dl + n * rowB <= ln
                    off += ln
                fill += need
                r0 += n


# ----------------------------------------------------------------------------
# decode1.cu: the one-token persistent kernel.  Restates its shared-memory
# layout (launcher) and per-CTA spans (kernel) and checks every bulk copy and
# shared-memory read against them.
D1_W, D1_MAX_DROWS, D1_SMEM = 8, 16, 232448
D1_SHARED = 16 * 8 * 2 + 16 * 8 + 16 * 4 + 16      # D1Shared, upper bound


def up16(b):
    return (b + 15) // 16 * 16


def xp4(c):
    return c + 4 * (c >> 6)


def decode1_layout(H, I, E, k, G):
    nbH, nbI = -(-H // 256), -(-I // 256)
    Hp = nbH * 256
    rowB_gu, rowB_d = nbH * K_BB, nbI * K_BB
    gspan = up16(-(-I // G) * rowB_gu + 15)
    dspan = up16(-(-H // G) * rowB_d + 15)
    gu_part = max(2 * gspan, up16(nbI * 4 * 68 * 4))     # also stages h: pieces of 64 floats, 68 apart
    slot = (gu_part + dspan + 127) // 128 * 128
    off = k * slot
    lay = dict(slot=slot, up=gspan, down=gu_part, gspan=gspan, dspan=dspan, xs=off)
    off += up16((Hp + 4 * (Hp >> 6)) * 4)
    lay["ptab"] = off
    off += 2 * E * 8
    lay["ltab_stride"] = up16(E)
    lay["ltab"] = off
    off += 2 * lay["ltab_stride"]
    lay["ysh"] = off
    off += D1_W * D1_MAX_DROWS * 4
    lay["sh"] = up16(off)
    lay["total"] = lay["sh"] + D1_SHARED
    return lay


def decode1_accepts(H, I, E, k, G):
    return (1 <= k <= 16 and H <= 2048 and H % 8 == 0 and I <= 1024 and I % 16 == 0
            and -(-I // 256) in (1, 2, 4)
            and E <= 512 and E % 16 == 0 and -(-H // G) <= D1_MAX_DROWS)


@pytest.mark.parametrize("H,I,E,k,G", [(2048, 512, 256, 8, 148), (2048, 512, 512, 8, 148),
                                       (256, 128, 16, 4, 148), (2048, 1024, 128, 8, 148),
                                       (2048, 512, 256, 16, 148), (1024, 1024, 64, 6, 132)])
def test_decode1_copies_and_reads_stay_in_their_slot(H, I, E, k, G):
    assert decode1_accepts(H, I, E, k, G)
    lay = decode1_layout(H, I, E, k, G)
    assert lay["total"] <= D1_SMEM
    for key in ("slot", "up", "down", "xs", "ptab", "ltab", "ysh", "sh"):
        assert lay[key] % 16 == 0, key              # bulk-copy and cp.async destinations
    nbH, nbI = -(-H // 256), -(-I // 256)
    rowB_gu, rowB_d = nbH * K_BB, nbI * K_BB
    mg = I * rowB_gu
    eb = 2 * mg + H * rowB_d                # expert bytes; the kernels take multiples of 16
    assert eb % 16 == 0
    for c in range(G):
        gu_lo, gu_hi = c * I // G, (c + 1) * I // G
        d_lo, d_hi = c * H // G, (c + 1) * H // G
        assert d_hi - d_lo <= D1_MAX_DROWS
        for off, n, rowB, region, cap in ((gu_lo * rowB_gu, gu_hi - gu_lo, rowB_gu, "up", lay["gspan"]),
                                          (mg + gu_lo * rowB_gu, gu_hi - gu_lo, rowB_gu, "up", lay["gspan"]),
                                          (2 * mg + d_lo * rowB_d, d_hi - d_lo, rowB_d, "down", lay["dspan"])):
            src, ln, delta = span16(off, n * rowB)
            if n == 0:
                continue
            assert src % 16 == 0 and ln % 16 == 0 and ln <= cap
            assert src + ln <= eb                       # never past the expert's last byte
            assert delta % 8 == 0                       # float2 scale/zero and uint2 nibble reads
            # reads: rows r < n, blocks of 136 bytes, within the copied span
            last = delta + (n - 1) * rowB + rowB
            assert last <= ln
    # the next slot starts after the largest span set; h fits the gate/up part
    assert lay["down"] >= 2 * lay["gspan"] and lay["down"] + lay["dspan"] <= lay["slot"]
    assert nbI * 4 * 68 * 4 <= lay["down"]
    # staged h pieces: 16-byte aligned, quarter-warps on distinct bank quads
    for q0 in range(0, 32, 8):
        starts = {((lane % (nbI * 4)) * 68) % 32 for lane in range(q0, q0 + 8)}
        assert len(starts) == min(8, nbI * 4)
    assert lay["xs"] + up16((nbH * 256 + 4 * (nbH * 256 >> 6)) * 4) <= lay["ptab"]
    # x: f32 at column xp4(c); lanes read 64-wide slices with 16-byte loads
    Hp = nbH * 256
    for lane in range(32):
        pb, pq = lane >> 2, lane & 3
        if pb >= nbH:
            continue
        c0 = pb * 256 + pq * 64
        assert (lay["xs"] + 4 * xp4(c0)) % 16 == 0
        for i in range(64):
            assert xp4(c0 + i) == xp4(c0) + i                 # slice contiguous
        assert xp4(c0 + 63) < Hp + 4 * (Hp >> 6)
    # down phase: lane piece pc of row rs reads its block's scale/zero and 32
    # payload bytes; P lanes per row tile the warp
    P = nbI * 4
    assert 32 % P == 0
    for lane in range(32):
        pc = lane % P
        for ri in range(D1_MAX_DROWS):
            off = ri * rowB_d + (pc >> 2) * K_BB
            assert off + 8 + (pc & 3) * 32 + 32 <= D1_MAX_DROWS * rowB_d
    # quarter-warps of 16-byte loads hit distinct bank quads
    for q0 in range(0, 32, 8):
        starts = {xp4((l >> 2) * 256 + (l & 3) * 64) % 32 for l in range(q0, q0 + 8) if (l >> 2) < nbH}
        assert len(starts) == len([l for l in range(q0, q0 + 8) if (l >> 2) < nbH])


def test_decode1_declines_shapes_outside_its_registers():
    assert not decode1_accepts(4096, 512, 256, 8, 148)      # a lane covers 64 of at most 2048 columns
    assert not decode1_accepts(2048, 2048, 256, 8, 148)     # two 16-value h chunks per lane
    assert not decode1_accepts(2048, 512, 256, 17, 148)     # two slots per warp
    assert not decode1_accepts(2048, 512, 250, 8, 148)      # 16-byte table copies
    assert not decode1_accepts(2048, 768, 128, 8, 148)      # 12 lanes per down row do not tile a warp
