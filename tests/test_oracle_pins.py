"""The oracle against its pins (CPU only).  See oracle_checks.py for what each
check compares with and why that pins the oracle to something other than
itself."""
import pytest

import oracle_checks as oc


@pytest.mark.parametrize("check", oc.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_bf16_rounding(orc):
    # round to nearest, ties to even, on hand-picked bit patterns
    import struct
    def f(bits):
        return struct.unpack("<f", struct.pack("<I", bits))[0]
    assert orc.f32_to_bf16(f(0x3F808000)) == 0x3F80      # tie, even stays
    assert orc.f32_to_bf16(f(0x3F818000)) == 0x3F82      # tie, odd rounds up
    assert orc.f32_to_bf16(f(0x3F808001)) == 0x3F81      # above the tie
    assert orc.f32_to_bf16(f(0x7F7FFFFF)) == 0x7F80      # overflow to inf
    assert orc.f32_to_bf16(1.0) == 0x3F80 and orc.bf16_to_f32(0xC000) == -2.0
