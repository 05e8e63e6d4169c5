"""Host logic of the decode K split (no GPU): the workspace size the library asks for.

With G CTAs sharing U = tiles * (K/128) (tile, K block) units, CTA c takes the units
[c*U/G, (c+1)*U/G).  These tests enumerate that partition directly, check that it
covers every unit once, and check the library's workspace size against the most
CTAs any tile is shared by.
"""
import pytest

import moe_grouped_gemm_quantize_b200 as lnq


def partition(tiles: int, nkb: int, G: int):
    U = tiles * nkb
    runs = [(c * U // G, (c + 1) * U // G) for c in range(G)]
    owners = [[] for _ in range(tiles)]
    for c, (u0, u1) in enumerate(runs):
        for u in range(u0, u1):
            owners[u // nkb].append(c)
    return runs, owners


def expected_bytes(M, N, K, sms):
    if M < 1 or M > 64 or K % 128 or K < 256:
        return 0
    bnq = 32 if M <= 32 else 64
    tiles = -(-N // 128) * -(-M // bnq)
    nkb = K // 128
    if tiles >= sms:
        return 0
    G = min(sms, tiles * nkb)
    _, owners = partition(tiles, nkb, G)
    slots = max(len(set(o)) for o in owners)
    r256 = lambda b: -(-b // 256) * 256
    # a fixed 4 KiB counter region, then the partial tiles
    return 4096 + r256(tiles * slots * 128 * bnq * 4)


@pytest.mark.parametrize("tiles,nkb,G", [(96, 32, 148), (3, 8, 24), (7, 9, 40), (96, 2, 148), (1, 64, 64), (1, 64, 40)])
def test_partition_covers_every_unit_once_in_contiguous_runs(tiles, nkb, G):
    runs, owners = partition(tiles, nkb, G)
    assert runs[0][0] == 0 and runs[-1][1] == tiles * nkb
    assert all(a[1] == b[0] for a, b in zip(runs, runs[1:]))
    assert all(u1 > u0 for u0, u1 in runs)
    # each CTA's run touches at most two tiles only partly
    for u0, u1 in runs:
        first, last = u0 // nkb, (u1 - 1) // nkb
        partial = [t for t in range(first, last + 1)
                   if not (u0 <= t * nkb and (t + 1) * nkb <= u1)]
        assert len(partial) <= 2
    # the CTAs sharing a tile are consecutive
    for o in owners:
        s = sorted(set(o))
        assert s == list(range(s[0], s[-1] + 1))


@pytest.mark.parametrize("M,N,K,sms", [
    (1, 12288, 4096, 148), (8, 12288, 4096, 148), (32, 12288, 4096, 148), (33, 12288, 4096, 148),
    (64, 12288, 4096, 148), (64, 12288, 4096, 132), (5, 384, 1024, 148), (64, 1152, 4096, 148),
    (17, 400, 2048, 148), (64, 256, 256, 148), (1, 16, 65536, 148), (64, 4096, 12288, 148),
])
def test_workspace_bytes_match_the_partition(M, N, K, sms):
    got = lnq.lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, sms)
    assert got == expected_bytes(M, N, K, sms)
    assert got % 256 == 0


@pytest.mark.parametrize("M,N,K", [(65, 12288, 4096), (2048, 4096, 4096), (64, 12288, 128),
                                   (64, 148 * 128, 4096), (64, 20000, 4096), (0, 256, 256), (64, 256, 100)])
def test_products_that_do_not_split_need_no_workspace(M, N, K):
    assert lnq.lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, 148) == 0


def test_default_decode_shape_needs_three_slots_per_tile():
    # N = 12288 -> 96 weight tiles over 148 SMs; 32 K blocks per tile, 20.76 per CTA
    b = lnq.lnq_fp8_block_gemm_nt_workspace_bytes(64, 12288, 4096, 148)
    assert b == 4096 + 96 * 3 * 128 * 64 * 4
