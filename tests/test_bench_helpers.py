"""Host-side helpers of bench.py (no GPU): the reference arm's step sizing,
the byte model of the token-major comparator, and the argument surface the
driver relies on."""
import bench
from long_context_decode_bit_b200 import accounting


def test_reference_keys_bounds_the_run():
    n = 1 << 20
    # Few steps: whole groups.
    assert bench.reference_keys(n, 3, 1, 1) == n
    # The default 100 + 10 steps: a prefix of whole tiles, about 2 minutes.
    ns = bench.reference_keys(n, 100, 10, 1)
    assert ns < n and ns % 2048 == 0
    assert 100.0 <= 110 * ns / 0.6e6 <= 121.0
    # Never below 8 tiles (or n), whatever K is.
    assert bench.reference_keys(n, 10 ** 6, 0, 1) == 8 * 2048
    assert bench.reference_keys(5000, 10 ** 6, 0, 1) == 5000
    # More groups per step: fewer keys each.
    assert bench.reference_keys(n, 100, 10, 4) < ns


def test_token_major_bytes_move_whole_rows():
    n, D, G = 1 << 20, 128, 4
    for r in (16, 32, 128):
        b = accounting.token_major_scan_bytes(n, r, G, D)
        assert b == n * D // 2 + r * 2 * (n // 64) + G * D * 4
    # Against the channel-major read of the same 32 channels at 4 bits: 3.8x.
    cm = accounting.scan_bytes(n, 32 * 4, 32, G, D)
    tm = accounting.token_major_scan_bytes(n, 32, G, D)
    assert 3.7 < tm / cm < 3.9


def test_argument_surface():
    a = bench.parse_args([])
    assert (a.gpus, a.steps, a.warmup, a.impl, a.case) == (1, 100, 10, "fathom", None)
    assert a.warmup >= 3
    for case in bench.CASES:
        assert bench.parse_args(["--case", case]).case == case
    assert bench.parse_args(["--impl", "reference"]).impl == "reference"
