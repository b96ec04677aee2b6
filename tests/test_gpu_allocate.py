"""GPU parity of brs_allocate_bits against the oracle's allocator on the
same FP64 costs.  Widths must be identical except where the FP64 logarithm
and exponential of the two math libraries can land on different sides of a
rounding point: b* within 1e-9 of a half-integer, or a budget move decided
by costs equal to 1e-12 (both counted; none expected here)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _costs(rng, kind, n):
    if kind == "lognormal":
        return np.exp(rng.normal(0, 3, n))
    if kind == "zeros":
        c = np.exp(rng.normal(0, 2, n))
        c[rng.random(n) < 0.3] = 0.0
        return c
    if kind == "allzero":
        return np.zeros(n)
    if kind == "equal":
        return np.full(n, 0.37)
    if kind == "gamma":   # decay-like persistence weights times squared ranges
        s = np.exp(rng.uniform(np.log(1e-3), 0, n))
        return (1 / np.expm1(2 * s)) * rng.uniform(0.1, 2, n) ** 2
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["lognormal", "zeros", "allzero", "equal", "gamma"])
@pytest.mark.parametrize("n,groups,avg,bmin,bmax", [(4096, 2, 4.0, 2, 8), (128, 5, 3.0, 2, 8),
                                                    (1000, 1, 2.5, 1, 8), (4096, 1, 4.0, 2, 6)])
def test_allocate_matches_oracle(kind, n, groups, avg, bmin, bmax):
    import torch
    from bit_recurrent_state_b200 import brs
    from oracle import oracle as O
    rng = np.random.default_rng(n + groups)
    c = np.concatenate([_costs(rng, kind, n) for _ in range(groups)])
    dev = torch.from_numpy(c).cuda()
    bits = torch.zeros(n * groups, dtype=torch.uint8, device="cuda")
    offs = torch.zeros(groups * (n + 1), dtype=torch.int32, device="cuda")
    brs.allocate_bits(dev, n, avg, bmin, bmax, bits, offs, offset_unit=16)
    torch.cuda.synchronize()
    gb = bits.cpu().numpy()
    go = offs.cpu().numpy().view(np.uint32).reshape(groups, n + 1)
    for g in range(groups):
        cg = c[g * n:(g + 1) * n]
        ob, fl = O.allocate_bits(cg, avg, bmin, bmax)
        assert fl == 0
        bg = gb[g * n:(g + 1) * n]
        assert int(bg.astype(int).sum()) == int(avg * n)
        diff = bg != ob
        if diff.any():
            pos = cg > 0
            gm = np.exp(np.mean(np.log(cg[pos])))
            bstar = avg + 0.5 * np.log2(cg[diff] / gm)
            assert np.all(np.abs(np.abs(bstar - np.floor(bstar)) - 0.5) < 1e-9), (g, np.nonzero(diff))
        np.testing.assert_array_equal(go[g], np.concatenate([[0], np.cumsum(bg.astype(np.int64))]) * 16)


def test_allocate_argument_errors():
    import torch
    from bit_recurrent_state_b200 import brs
    c = torch.ones(12, dtype=torch.float64, device="cuda")
    b = torch.zeros(12, dtype=torch.uint8, device="cuda")
    with pytest.raises(brs.BrsError):
        brs.allocate_bits(c, 5, 4.0, 2, 8, b)          # 12 not a multiple of 5
    brs.allocate_bits(c, 12, 4.5, 2, 8, b)             # 54 bits: fine
    with pytest.raises(brs.BrsError):
        brs.allocate_bits(c, 12, 9.0, 2, 8, b)         # infeasible
