"""Host logic of the W4A8 product's work units (CPU only): which output tiles
are split along K, and the workspace that follows.  Without a device the
library plans for 148 SMs (a B200).

The plan, restated: with T tiles of 128 x 128 and G = K / 256 groups, a cost
in group-times per CTA (a unit costs its groups plus 1.5) picks between
splitting every tile into S slices (waves of T * S units over the SMs) and
keeping the tiles of whole waves whole while only the R = T mod 148 tiles of
the last wave are split into min(148 / R, G / 2, 16) slices.  The workspace is
a 256-byte-rounded array of int32 arrival counters for the split tiles, then
their fp32 partial tiles [split tiles][slices][128][128].
"""

import pytest

SMS = 148
TILE_BYTES = 128 * 128 * 4


def _lib():
    from w4_quant_matmul_b200 import _lib as L
    try:
        return L.load()
    except Exception as e:  # noqa: BLE001 - the library is built by the suite
        pytest.skip(f"library not built: {e}")


def _plan(M, N, K):
    """The plan restated in Python (see the module docstring)."""
    tiles = -(-M // 128) * -(-N // 128)
    G = K // 256
    best, best_cost = (tiles, 1), float("inf")  # (full tiles, slices)
    for sp in range(1, 17):
        if sp > G or (sp > 1 and G // sp < 4):
            break
        waves = -(-(tiles * sp) // SMS)
        cost = waves * (G / sp + 1.5) + (0.25 * sp if sp > 1 else 0.0)
        if cost < best_cost - 1e-9:
            best, best_cost = ((0 if sp > 1 else tiles), sp), cost
    full = tiles // SMS * SMS
    rest = tiles - full
    if full and rest:
        s = min(SMS // rest, G // 2, 16)
        if s >= 2:
            cost = (full // SMS) * (G + 1.5) + (G / s + 1.5) + 0.25 * s
            if cost < best_cost - 1e-9:
                best = (full, s)
    full_tiles, slices = best
    split = tiles - full_tiles if slices > 1 else 0
    if split == 0:
        return 0
    return -(-(split * 4) // 256) * 256 + split * slices * TILE_BYTES


@pytest.fixture(scope="module")
def lib():
    L = _lib()
    if L.w4_check_device_error() == 0:
        import torch
        if torch.cuda.is_available():
            pytest.skip("the plan depends on the device's SM count; checked here for 148")
    return L


@pytest.mark.parametrize("M,N,K", [
    (1024, 18944, 2560),   # 1184 tiles: eight whole waves, nothing split
    (2048, 19456, 2560),   # 2432 tiles: 16 waves + 64 tiles split in two
    (256, 19456, 2560),    # 304 tiles: two waves + 8 tiles split in five
    (2048, 2560, 9728),    # 320 tiles: two waves + 24 tiles split in six
    (256, 2560, 9728),     # 40 tiles: every tile split in three
    (512, 2560, 9728),     # 80 tiles: every tile split in five
    (128, 128, 256),       # one tile, one group: nothing to split
    (4096, 151936, 2560),  # the lm_head as a prefill product
])
def test_workspace_follows_the_unit_plan(lib, M, N, K):
    assert lib.w4a8_mmq_workspace_size(M, N, K) == _plan(M, N, K)


def test_whole_waves_need_no_workspace(lib):
    for waves in (1, 2, 8):
        assert lib.w4a8_mmq_workspace_size(128 * waves, 128 * SMS, 2560) == 0
