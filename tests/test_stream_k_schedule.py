"""The stream-K warp-MMA GEMV's schedule, checked on the CPU.

The kernel (UW_KERNEL_MMA_SK) gives warp w of W the units [w U / W, (w+1) U / W)
of the U = (n / 16) x (k / 128) units in tile-major order, finds the warp
owning unit u as ((u + 1) W - 1) / U, and has each warp store its first cut
piece in fragment set 2w and its last in 2w + 1; the warp that finishes a cut
tile reads the pieces of warps owner(first unit) .. owner(last unit), taking
set 2w + 1 from the first owner when that warp's run began in an earlier tile.
These formulas are restated here (the host sizes the grid with W = min(SMs x
warps per CTA, U), which makes every run non-empty) and walked for every
shape the kernel serves, the way each warp walks its run: every unit has one
owner, every cut tile's pieces come from exactly the warps the reader visits,
and every fragment set the reader takes was written once, by that warp, for
that tile.
"""
import pytest

SMS = 148


def unit0(w, units, warps):
    return w * units // warps


def owner(u, units, warps):
    return ((u + 1) * warps - 1) // units


def walk(n, k, warps_per_cta, sms=SMS):
    tiles, cpr = n // 16, k // 128
    units = tiles * cpr
    warps = min(sms * warps_per_cta, units)
    written = {}          # fragment set -> tile
    pieces = {}           # tile -> warps that stored a piece
    whole = {}            # tile -> the warp that wrote it without a fix-up
    for w in range(warps):
        ub, ue = unit0(w, units, warps), unit0(w + 1, units, warps)
        assert ue > ub, "empty run"
        t_first = ub // cpr
        ct, ci = t_first, ub - t_first * cpr
        piece0 = ci
        for j in range(ue - ub):
            assert owner(ub + j, units, warps) == w
            ci += 1
            if ci == cpr or j == ue - ub - 1:
                if piece0 == 0 and ci == cpr:
                    assert ct not in whole and ct not in pieces
                    whole[ct] = w
                else:
                    slot = 2 * w + (0 if ct == t_first else 1)
                    assert slot not in written
                    written[slot] = ct
                    pieces.setdefault(ct, []).append(w)
                if ci == cpr:
                    ci, ct = 0, ct + 1
                piece0 = ci
    assert sorted(list(whole) + list(pieces)) == list(range(tiles))
    for t, ws in pieces.items():
        wf, wl = owner(t * cpr, units, warps), owner(t * cpr + cpr - 1, units, warps)
        assert ws == list(range(wf, wl + 1)), (t, ws, wf, wl)
        for w in ws:
            slot = 2 * w + (1 if (w == wf and unit0(wf, units, warps) < t * cpr) else 0)
            assert written[slot] == t
    return warps, len(pieces)


@pytest.mark.parametrize("n,k", [(14336, 4096), (4096, 14336), (28672, 8192), (8192, 28672), (1024, 1024),
                                 (4096, 1024), (2048, 4096), (256, 14336), (64, 128), (320, 1408),
                                 (192, 1408), (448, 2432), (768, 2048)])
@pytest.mark.parametrize("warps_per_cta", [1, 4, 8, 11, 12, 16])
def test_every_unit_one_owner_and_every_piece_read_once(n, k, warps_per_cta):
    walk(n, k, warps_per_cta)


def test_fewer_units_than_warps_gives_one_unit_per_warp():
    warps, cut = walk(1024, 1024, 16)         # 512 units, fewer than 148 x 16 warps
    assert warps == 512 and cut == 64         # every tile in 8 pieces
    warps, cut = walk(64, 128, 16)            # 4 units: a single CTA with spare warps
    assert warps == 4 and cut == 0            # one chunk per row: every tile is whole
