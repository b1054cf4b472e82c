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
