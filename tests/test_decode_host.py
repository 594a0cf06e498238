"""Host-side logic of the decode loop's cache sizing (no GPU)."""
from medusa_head_speculative_02_b200.synthetic import CONFIGS


def test_headroom_extends_capacity_only():
    c = CONFIGS["7b_b1"]
    assert c.headroom == 0 and c.Lcap == c.L_hi + c.N
    d = c.scaled(headroom=10 * (c.K + 1))
    assert d.Lcap == c.Lcap + 60
    assert (d.B, d.d, d.V, d.N, d.L_lo, d.L_hi) == (c.B, c.d, c.V, c.N, c.L_lo, c.L_hi)
