"""Host model check of the decode GEMM's scale staging (no GPU). The scale
warps copy, per stage, the absmax of the tile's 8 units x 2 row groups x 8
rows x 4 blocks into a [unit][row group][row][block] table of 4-byte words,
either one 16-byte copy per (unit, row group, row) (fp32, K % 256 == 0, 16-byte
aligned base) or one 4-byte copy per block; consumer lane (g, q) of the warp
for block blk reads words g * 4 + blk of each unit's two row groups. The index
arithmetic below restates csrc/decode_gemm.cu's (rows of unit i and row group
rgi: SwiGLU halves, interleaved gate/up or plain) and checks, over shapes with
partial tiles, rows past the stack and K tails, that every word a consumer
reads holds the scale of its (row, block), that each word is written once per
stage, that 16-byte copies start on 16-byte boundaries, and that no copy
reads past the scale tensor.
"""
import pytest


def wrow(epi, N, ebase, j0, i, rgi, rr):
    j = j0 + i
    if epi == 0:
        return ebase + 16 * j + 8 * rgi + rr
    if epi == 1:
        return ebase + 8 * j + rr + rgi * (N // 2)
    return ebase + 2 * (8 * j + rr) + rgi


def check_tile(N, K, E, epi, e, j0, S, base_mod16):
    KB = K // 64
    KC = (KB + 3) // 4
    upb = (N // 2 + 7) // 8 if epi else (N + 15) // 16
    nunits = min(8, upb - j0)
    wide = KB % 4 == 0 and base_mod16 == 0
    ebase = e * N
    total = E * N * KB
    for kc in range(KC):
        words = {}
        for sw in range(S):
            for lane in range(32):
                r = lane & 7 if wide else lane >> 2
                blk = 0 if wide else lane & 3
                wrg, wu = (lane >> 3) & 1, sw + S * (lane >> 4)
                vmask = 0
                for i in range(nunits):
                    for rgi in range(2):
                        if wrow(epi, N, ebase, j0, i, rgi, r) < ebase + N:
                            vmask |= 1 << (2 * i + rgi)
                e00 = wrow(epi, N, ebase, j0, 0, 0, r) * KB + blk
                du = (wrow(epi, N, ebase, j0, 1, 0, r) - wrow(epi, N, ebase, j0, 0, 0, r)) * KB
                dg = (wrow(epi, N, ebase, j0, 0, 1, r) - wrow(epi, N, ebase, j0, 0, 0, r)) * KB
                ek = e00 + kc * 4
                dst0 = r * 16 + blk * 4
                if wide:
                    for jj in range(4 // S):
                        i = wu + 2 * S * jj
                        valid = (vmask >> (2 * i + wrg)) & 1
                        dst = dst0 + i * 256 + wrg * 128
                        assert dst % 16 == 0 and dst + 16 <= 2048
                        el = ek + i * du + wrg * dg
                        if valid:
                            assert (el * 4 + base_mod16) % 16 == 0 and el + 4 <= total
                        for w in range(4):
                            assert dst + 4 * w not in words
                            words[dst + 4 * w] = el + w if valid else None
                else:
                    kok = kc * 4 + blk < KB
                    for i in range(sw, nunits, S):
                        for rgi in range(2):
                            valid = kok and (vmask >> (2 * i + rgi)) & 1
                            dst = dst0 + i * 256 + rgi * 128
                            assert dst + 4 <= 2048 and dst not in words
                            el = ek + i * du + rgi * dg
                            if valid:
                                assert el < total
                            words[dst] = el if valid else None
        for blk in range(4):
            kb = kc * 4 + blk
            for ui in range(nunits):
                for g in range(8):
                    for rg in range(2):
                        row = wrow(epi, N, ebase, j0, ui, rg, g)
                        if kb < KB and row < ebase + N:
                            assert words[g * 16 + blk * 4 + ui * 256 + rg * 128] == row * KB + kb


@pytest.mark.parametrize("N,K,E,epi", [
    (256, 2048, 3, 0), (1536, 2048, 3, 1), (2880, 2880, 2, 0), (5760, 2880, 2, 2),
    (5760, 2880, 2, 1), (1536, 768, 2, 1), (200, 1024, 2, 0), (104, 640, 2, 1), (136, 192, 2, 2),
])
def test_scale_staging(N, K, E, epi):
    upb = (N // 2 + 7) // 8 if epi else (N + 15) // 16
    for S in (1, 2):
        for base_mod16 in (0, 4):
            for e in range(E):
                for j0 in range(0, upb, 8):
                    check_tile(N, K, E, epi, e, j0, S, base_mod16)
