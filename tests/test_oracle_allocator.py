"""Pins of the decay-aware allocator: the pages' worked examples, the
continuous solution's AM/GM gain, budget, monotonicity, brute force."""
import itertools
import math

import numpy as np
import pytest

from conftest import golden


def test_erasure_rate_worked_example(orc):
    g = golden("erasure_rate_example.txt")
    s, C, beta = float(g["s"]), int(g["C"]), float(g["beta"])
    k = np.array([1.0, 1.0]) / np.sqrt(2.0)
    # approximate rate: A = EMA(a^2) = e^{-2s}, K = EMA(beta (2-beta) k_0^2)
    A = math.exp(-2 * s)
    K = beta * (2 - beta) * k[0] ** 2
    approx = orc.gamma_hat(A, K, C)
    assert round(approx, 2) == float(g["gamma_approx"])
    # exact rate: diagonal of the observability Gramian, brute force over
    # lags, F = (I - k a^T) D with a = beta k, D = e^{-s} I
    F = (np.eye(2) - np.outer(k, beta * k)) * math.exp(-s)
    e0 = np.array([1.0, 0.0])
    tot, Fl = 0.0, np.eye(2)
    for _ in range(20000):
        Fl = F @ Fl
        tot += float(np.sum((Fl @ e0) ** 2))
    assert round(tot, 1) == float(g["gamma_exact"])
    # the closed form of the persistence sum (no erasure): 1/expm1(2s)
    assert abs(orc.gamma_hat(A, 0.0, 1) - sum(math.exp(-2 * s * l) for l in range(1, 20000))) < 1e-9


def test_allocation_worked_example(orc):
    g = golden("allocation_example.txt")
    wA = orc.gamma_hat(math.exp(-2 * float(g["s_A"])), 0.0, 1)
    wB = orc.gamma_hat(math.exp(-2 * float(g["s_B"])), 0.0, 1)
    assert round(wA, 1) == float(g["weight_A"])
    assert round(wB, 3) == float(g["weight_B"])
    assert round(wA / wB) == pytest.approx(float(g["ratio"]), abs=1)
    assert round(0.5 * math.log2(wA / wB), 2) == float(g["bits_apart"])
    bits, fl = orc.allocate_bits([wA, wB], float(g["avg_bits"]), 1, 8)
    assert fl == 0
    assert list(bits) == [int(g["bits_A"]), int(g["bits_B"])]
    uni = (wA + wB) * 2.0 ** (-2 * float(g["avg_bits"]))
    alloc = wA * 2.0 ** (-2 * int(bits[0])) + wB * 2.0 ** (-2 * int(bits[1]))
    assert round(uni, 3) == float(g["cost_uniform"])
    assert round(alloc, 3) == float(g["cost_allocated"])


def test_continuous_solution_am_gm(orc):
    """Costs built so that b* = avg + log2(c/GM)/2 lands on integers: the
    allocator must return exactly them, and the proxy-cost gain over uniform
    widths must be AM(c)/GM(c)."""
    rng = np.random.default_rng(5)
    for _ in range(20):
        N = 16
        target = rng.integers(1, 12, N).astype(float)
        avg = target.mean()                    # avg * N is an integer by construction
        gm = np.exp(rng.uniform(-3, 3))
        c = gm * 4.0 ** (target - avg)
        bits, fl = orc.allocate_bits(c, avg, 1, 16)
        assert fl == 0
        np.testing.assert_array_equal(bits, target)
        uni = np.sum(c) * 2.0 ** (-2 * avg)
        opt = np.sum(c * 2.0 ** (-2 * target))
        am = c.mean()
        gmv = np.exp(np.mean(np.log(c)))
        assert uni / opt == pytest.approx(am / gmv, rel=1e-9)


def test_budget_equal_costs_and_monotone(orc):
    rng = np.random.default_rng(6)
    for trial in range(50):
        N = int(rng.integers(4, 400))
        c = np.exp(rng.normal(0, 3, N))
        if trial % 5 == 0:
            c[rng.integers(N, size=N // 4)] = 0.0
        bits, fl = orc.allocate_bits(c, 4.0, 2, 8)
        assert fl == 0
        assert int(bits.astype(int).sum()) == 4 * N
        assert bits.min() >= 2 and bits.max() <= 8
        order = np.argsort(-c, kind="stable")
        assert np.all(np.diff(bits[order].astype(int)) <= 0)    # monotone in c
    bits, _ = orc.allocate_bits(np.full(64, 0.37), 4.0, 2, 8)
    assert np.all(bits == 4)
    bits, _ = orc.allocate_bits(np.zeros(64), 4.0, 2, 8)
    assert np.all(bits == 4)


def test_infeasible_budget_rejected(orc):
    _, fl = orc.allocate_bits(np.ones(3), 4.5, 2, 8)        # 13.5 bits: not an integer
    assert fl == orc.EINVAL
    _, fl = orc.allocate_bits(np.ones(3), 9.0, 2, 8)
    assert fl == orc.EINVAL


def test_brute_force_gap(orc):
    """Round-and-adjust against the true integer optimum of sum c 4^-b on
    tiny sets: the adjusted solution is always feasible and its proxy cost
    is reported relative to the optimum (the pages do not claim integer
    optimality; it must stay within a factor 2 here)."""
    rng = np.random.default_rng(7)
    worst = 1.0
    for _ in range(200):
        N = int(rng.integers(2, 6))
        c = np.exp(rng.normal(0, 2.5, N))
        bits, fl = orc.allocate_bits(c, 4.0, 2, 8)
        got = float(np.sum(c * 4.0 ** (-bits.astype(float))))
        best = min(float(np.sum(c * 4.0 ** (-np.array(b, float))))
                   for b in itertools.product(range(2, 9), repeat=N) if sum(b) == 4 * N)
        assert got >= best * (1 - 1e-12)
        worst = max(worst, got / best)
    assert worst < 2.0


def test_storage_accounting(orc):
    g = golden("storage_accounting.txt")
    kda32 = orc.Config(B=1, H=1, d=128, k_hi=16, block=32)
    kda128 = orc.Config(B=1, H=1, d=128, k_hi=16, block=128)
    tiny = orc.Config(B=1, H=2, d=32, k_hi=4, block=32)
    assert orc.bits_per_value(kda32) == float(g["damp_9875"])
    assert orc.bits_per_value(tiny) == float(g["damp_9875"])
    assert orc.bits_per_value(kda128) == 9.21875
    assert round(100 * (1 - orc.bits_per_value(kda32) / 32), 1) == float(g["damp_reduction_percent"])
    vb = orc.Config(B=1, H=32, d=128, storage=orc.STORE_VARBIT, hadamard=0, avg_bits=4.0)
    assert orc.bits_per_value(vb) == 4.0 + float(g["varbit_3bit_width_extra_bits"]) / 128
    assert round(4.0 + float(g["varbit_4bit_width_extra_bits"]) / 128, 3) == float(g["varbit_4156"])
    # physical bytes per head of the measured layouts
    assert orc.state_bytes(orc.Config(B=64, H=32, d=128, k_hi=16, block=128))[0] == 18880 * 2048
    assert orc.state_bytes(orc.Config(B=1, H=2, d=32, k_hi=4, block=32))[0] == 1264 * 2
    assert orc.state_bytes(orc.Config(B=256, H=32, Hk=16, d=128, k_hi=0, block=128,
                                      decay_per_key=0))[0] == 16896 * 256 * 32
    # the 4-bit low tier ([DAMP] b = 4): 16 FP16 rows, 112 rows of 4-bit codes
    # (64 bytes each) and the same FP16 scale/zero per block
    int4_32 = orc.Config(B=1, H=1, d=128, k_hi=16, block=32, low_bits=4)
    int4_128 = orc.Config(B=1, H=1, d=128, k_hi=16, block=128, low_bits=4)
    assert orc.state_bytes(int4_32)[0] == 16 * 128 * 2 + 112 * 64 + 112 * 4 * 4
    assert orc.state_bytes(int4_128)[0] == 16 * 128 * 2 + 112 * 64 + 112 * 4
    assert orc.bits_per_value(int4_32) == 6.375 and orc.bits_per_value(int4_128) == 5.71875
    for cfg in (int4_32, int4_128):
        assert orc.bits_per_value(cfg) == orc.state_bytes(cfg)[0] * 8 / (128 * 128)
