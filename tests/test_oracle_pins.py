"""Pins of the CPU oracle to facts the pages and the mathematics fix (no GPU needed).

The pages print no worked numbers for the encoding, so each pin here is derived from a
closed form, an invariant, an exact integer computation or a brute-force formulation that
is written differently from the oracle (see the docstring of each test); the configuration
values they do print (level table, table size, primes) are fixtures under tests/golden/. Together they are
chosen so that a dropped corner, a swapped axis, a wrong sign, a wrong prime, a wrong
resolution rounding or a deduplicated gradient each fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import Grid

PRIMES = (1, 2654435761, 805459861)   # NeRFace-HG section 2; Repro-HG section 2.2


def bigint_hash(c0, c1, c2, T=None):
    """The pages' form of the hash: exact integer products XORed, reduced mod 2^32 (and mod
    T). Python integers never wrap, so this is a different arithmetic from the oracle's
    uint32 wraparound; they agree because a power-of-two modulus keeps only low bits."""
    c0, c1, c2 = int(c0), int(c1), int(c2)
    h = ((c0 % 2**32) * PRIMES[0]) ^ ((c1 % 2**32) * PRIMES[1]) ^ ((c2 % 2**32) * PRIMES[2])
    h %= 2**32
    return h if T is None else h % T


# ---------------------------------------------------------------------------------------
# Hash
# ---------------------------------------------------------------------------------------

def test_hash_primes_and_hand_values():
    """h(1,0,0), h(0,1,0), h(0,0,1) are the three primes themselves; h(1,1,1) is their
    XOR, worked by hand: 0x9E3779B1 ^ 0x30025795 = 0xAE352E24, then ^ 1 = 0xAE352E25."""
    assert oracle.hash3(0, 0, 0) == 0
    assert oracle.hash3(1, 0, 0) == 1
    assert oracle.hash3(0, 1, 0) == 2654435761 == 0x9E3779B1
    assert oracle.hash3(0, 0, 1) == 805459861 == 0x30025795
    assert oracle.hash3(1, 1, 1) == 0xAE352E25
    # mod 2^19 and 2^10 of h(1,1,1): low bits of 0xAE352E25
    assert oracle.hash3(1, 1, 1) % 2**19 == 0x52E25 == 339493
    assert oracle.hash3(1, 1, 1) % 2**10 == 0x225 == 549


def test_hash_matches_bigint_form():
    """Random corners, including negative and > 2^31 ones: uint32 wraparound equals the
    exact-integer form of the pages reduced mod 2^32 and mod every power-of-two T."""
    rng = np.random.default_rng(1)
    cs = rng.integers(-2**33, 2**33, size=(2000, 3))
    cs[:500] = rng.integers(0, 4097, size=(500, 3))
    for c in cs:
        c0, c1, c2 = (int(v) for v in c)
        h = oracle.hash3(c0, c1, c2)
        assert h == bigint_hash(c0, c1, c2)
        for log2T in (4, 10, 19, 22, 24):
            assert h % (1 << log2T) == bigint_hash(c0, c1, c2, 1 << log2T)


def test_hash_invariants():
    """Algebraic facts of an XOR of per-axis products: x prime 1 (h(c0,0,0) = c0); XOR
    separability; scaling all coordinates by 2^s shifts h left by s; stepping an even c0
    by one flips bit 0 only."""
    rng = np.random.default_rng(2)
    for _ in range(500):
        c0, c1, c2 = (int(v) for v in rng.integers(0, 2**20, size=3))
        h = oracle.hash3(c0, c1, c2)
        assert oracle.hash3(c0, 0, 0) == c0
        assert h == oracle.hash3(c0, 0, 0) ^ oracle.hash3(0, c1, 0) ^ oracle.hash3(0, 0, c2)
        s = int(rng.integers(0, 8))
        assert oracle.hash3(c0 << s, c1 << s, c2 << s) == (h << s) % 2**32
        e = c0 & ~1
        assert oracle.hash3(e + 1, c1, c2) == oracle.hash3(e, c1, c2) ^ 1


# ---------------------------------------------------------------------------------------
# Resolutions
# ---------------------------------------------------------------------------------------

def exact_floor_resolution(L, N_min, N_max, l):
    """floor(N_min * (N_max/N_min)^(l/(L-1))) by exact integer search: n is below the
    exact value iff n^(L-1) * N_min^l <= N_min^(L-1) * N_max^l."""
    rhs = N_min ** (L - 1) * N_max ** l
    lo, hi = 1, N_max + 1
    while hi - lo > 1:          # largest n with n^(L-1) N_min^l <= rhs
        mid = (lo + hi) // 2
        if mid ** (L - 1) * N_min ** l <= rhs:
            lo = mid
        else:
            hi = mid
    return lo


def near_integer_from_below(L, N_min, N_max, l):
    """True when the exact value is not an integer but within 1e-9 relative of the next
    one (where the oracle's reading rounds up instead of flooring)."""
    n = exact_floor_resolution(L, N_min, N_max, l)
    if n ** (L - 1) * N_min ** l == N_min ** (L - 1) * N_max ** l:
        return False
    # value^(L-1) = rhs / N_min^l; compare (n+1)^(L-1) with (1+1e-9)^(L-1) * value^(L-1)
    v = Fraction(N_min ** (L - 1) * N_max ** l, N_min ** l)
    return Fraction(n + 1) ** (L - 1) <= v * Fraction(1 + Fraction(1, 10**9)) ** (L - 1)


def test_resolutions_workload_grids():
    """The workload grids. b = 2 for N 2->16 with L=4; b = 2^(1/3) for 16->512 (so levels
    0, 3, 6, ... are 16, 32, 64, ... exactly); b = 2^(8/15) for 16->4096. The coarsest and
    finest levels of the 16->512 grid are the 16^3 and 512^3 of Repro-HG section 2.1.
    Expected values are the exact-integer floors (no floating point)."""
    for L, a, b in [(4, 2, 16), (16, 16, 512), (16, 16, 4096)]:
        want = [exact_floor_resolution(L, a, b, l) for l in range(L)]
        assert oracle.resolutions(L, a, b) == want
    assert oracle.resolutions(4, 2, 16) == [2, 4, 8, 16]
    r = oracle.resolutions(16, 16, 512)
    assert r[0] == 16 and r[-1] == 512 and r[3] == 32 and r[6] == 64 and r[9] == 128
    # the finest level equals N_max (a literal double floor would give 4095 here)
    assert oracle.resolutions(16, 16, 4096)[-1] == 4096


def test_resolutions_random_grids():
    """Random (L, N_min, N_max): the oracle's rounding equals the exact-integer floor except
    where the exact value sits within 1e-9 below an integer (none expected)."""
    rng = np.random.default_rng(3)
    for _ in range(300):
        L = int(rng.integers(2, 33))
        a = int(rng.integers(1, 2**10))
        b = int(rng.integers(a, 2**20 + 1))
        got = oracle.resolutions(L, a, b)
        for l in (0, 1, L // 2, L - 2, L - 1):
            if near_integer_from_below(L, a, b, l):
                continue
            assert got[l] == exact_floor_resolution(L, a, b, l), (L, a, b, l)
        assert got[0] == a and got[-1] == b
        assert all(got[i] <= got[i + 1] for i in range(L - 1))


def test_resolutions_invalid():
    with pytest.raises(ValueError):
        oracle.resolutions(0, 16, 512)
    with pytest.raises(ValueError):
        oracle.resolutions(4, 16, 8)
    with pytest.raises(ValueError):
        oracle.resolutions(1, 16, 512)
    assert oracle.resolutions(1, 16, 16) == [16]


# ---------------------------------------------------------------------------------------
# Forward
# ---------------------------------------------------------------------------------------

def tiny_grid(F=2, log2T=10, dtype=oracle.F32):
    return Grid(4, F, log2T, 2, 16, dtype)


def test_forward_vertex_exact():
    """At a grid vertex the encoding is the table entry of that vertex, bit for bit. With
    x = k/2 (exact in fp32) every level of the 2->16 grid lands on a vertex (all N_l are
    multiples of 2), so out[p][l*F+f] == table[l][h(x*N_l) mod T][f]."""
    g = tiny_grid()
    rng = np.random.default_rng(4)
    table = (rng.random((g.L, g.T, g.F), dtype=np.float32) - 0.5).astype(np.float32)
    k = rng.integers(0, 3, size=(64, 3))
    x = (k / 2.0).astype(np.float32)
    out = g.forward(x, table)
    for p in range(x.shape[0]):
        for l, n in enumerate(g.res):
            v = [int(k[p, i]) * n // 2 for i in range(3)]
            h = bigint_hash(*v, T=g.T)
            for f in range(g.F):
                assert out[p, l * g.F + f] == np.float64(table[l, h, f])
    # finer vertices are exact only from their own level on: x = k/16 at level 3
    kf = rng.integers(0, 17, size=(64, 3))
    xf = (kf / 16.0).astype(np.float32)
    outf = g.forward(xf, table)
    for p in range(xf.shape[0]):
        h = bigint_hash(*(int(v) for v in kf[p]), T=g.T)
        assert list(outf[p, 3 * g.F:4 * g.F]) == [np.float64(t) for t in table[3, h]]


def test_forward_weights_sum_to_one():
    """With every table entry equal to 1 the encoding is the sum of the 8 trilinear
    weights, which is exactly 1; a dropped or doubled corner moves it by a whole weight."""
    for F in (1, 2, 4, 8):
        g = Grid(3, F, 6, 3, 27)
        rng = np.random.default_rng(5 + F)
        x = rng.random((500, 3), dtype=np.float32)
        out = g.forward(x, np.ones((g.L, g.T, g.F), dtype=np.float32))
        assert np.max(np.abs(out - 1.0)) <= 4 * np.finfo(np.float64).eps


def test_forward_linear_in_table():
    """Linearity in the table: integer-valued tables A, B and integer alpha, beta make
    alpha*A + beta*B exact in fp32, so enc(aA + bB) = a enc(A) + b enc(B) to fp64 rounding."""
    g = tiny_grid(F=4)
    rng = np.random.default_rng(6)
    A = rng.integers(-1000, 1000, size=(g.L, g.T, g.F)).astype(np.float32)
    B = rng.integers(-1000, 1000, size=(g.L, g.T, g.F)).astype(np.float32)
    x = rng.random((300, 3), dtype=np.float32)
    lhs = g.forward(x, (3 * A - 5 * B).astype(np.float32))
    rhs = 3 * g.forward(x, A) - 5 * g.forward(x, B)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def hat_basis_encode(x, table, res, T):
    """Brute force in a different formulation: the trilinear interpolant is the sum over
    ALL integer vertices v near the point of prod_i max(0, 1 - |x_i N_l - v_i|) times the
    vertex's hashed entry (tensor-product hat functions). Vertices are enumerated in a box
    around the point; x_i N_l is the same fp32 product the pages take."""
    N = x.shape[0]
    L, _, F = table.shape
    out = np.zeros((N, L * F))
    for p in range(N):
        for l, n in enumerate(res):
            xs = [float(np.float32(x[p, i]) * np.float32(n)) for i in range(3)]
            base = [int(np.floor(v)) for v in xs]
            acc = np.zeros(F)
            for a in range(base[0] - 2, base[0] + 3):
                for b in range(base[1] - 2, base[1] + 3):
                    for c in range(base[2] - 2, base[2] + 3):
                        w = (max(0.0, 1 - abs(xs[0] - a)) * max(0.0, 1 - abs(xs[1] - b)) *
                             max(0.0, 1 - abs(xs[2] - c)))
                        if w:
                            acc += w * table[l, bigint_hash(a, b, c, T)].astype(np.float64)
            out[p, l * F:(l + 1) * F] = acc
    return out


def test_forward_brute_force_hat_basis():
    """4 points, 2 levels (L=2, F=2, T=2^10, N 2->4) and 200 points on the 4-level tiny
    grid: the oracle equals the hat-basis sum. Pairing a fraction with the wrong axis, or
    a weight with the wrong sign, changes the result far beyond 1e-12."""
    rng = np.random.default_rng(7)
    g = Grid(2, 2, 10, 2, 4)
    table = rng.standard_normal((g.L, g.T, g.F)).astype(np.float32)
    x = rng.random((4, 3), dtype=np.float32)
    np.testing.assert_allclose(g.forward(x, table), hat_basis_encode(x, table, g.res, g.T),
                               rtol=0, atol=1e-12)
    g = tiny_grid()
    table = rng.standard_normal((g.L, g.T, g.F)).astype(np.float32)
    x = rng.random((200, 3), dtype=np.float32)
    x[:10] = np.float32(1.0)                               # x = 1.0: voxel N_l, corner N_l + 1
    x[10:20] = np.float32(1.0 - 2.0**-24)
    x[20:30] = np.float32(0.0)
    x[30:40] = -rng.random((10, 3), dtype=np.float32)      # outside the cube: no clamping
    np.testing.assert_allclose(g.forward(x, table), hat_basis_encode(x, table, g.res, g.T),
                               rtol=0, atol=1e-12)


def test_forward_fp16_table_decoding():
    """fp16 tables: the oracle's own binary16 decoder equals numpy's for every bit
    pattern, subnormals included, and an fp16 table encodes like its exact fp32 copy."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    g16 = tiny_grid(dtype=oracle.F16)
    g32 = tiny_grid()
    rng = np.random.default_rng(8)
    t16 = ((rng.random((4, 1024, 2), dtype=np.float32) * 2 - 1) * 1e-4).astype(np.float16)
    x = rng.random((300, 3), dtype=np.float32)
    np.testing.assert_array_equal(g16.forward(x, t16), g32.forward(x, t16.astype(np.float32)))


# ---------------------------------------------------------------------------------------
# Backward
# ---------------------------------------------------------------------------------------

def test_backward_adjoint_identity():
    """The forward pass is linear in the table t, so <g, fwd(t)> = <bwd(g), t> exactly in
    real arithmetic; in fp64 both sides agree to ~1e-13 relative."""
    for (L, F, log2T, a, b) in [(4, 2, 10, 2, 16), (3, 4, 8, 5, 40), (2, 1, 4, 2, 4)]:
        g = Grid(L, F, log2T, a, b)
        rng = np.random.default_rng(9 + F)
        x = rng.random((1000, 3), dtype=np.float32)
        t = rng.standard_normal((L, g.T, F)).astype(np.float32)
        up = rng.standard_normal((1000, L * F)).astype(np.float32)
        lhs = float(np.sum(up.astype(np.float64) * g.forward(x, t)))
        rhs = float(np.sum(g.backward(x, up) * t.astype(np.float64)))
        assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)


def test_backward_finite_differences():
    """Central differences of <g, fwd(t)> on integer-valued tables with step 1 (exact in
    fp32) equal the backward's entries: the function is linear, so the difference quotient
    is the derivative up to rounding. Touched and untouched entries are both probed."""
    grid = Grid(4, 2, 10, 2, 16)
    rng = np.random.default_rng(10)
    x = rng.random((8, 3), dtype=np.float32)
    t = rng.integers(-50, 50, size=(grid.L, grid.T, grid.F)).astype(np.float32)
    up = rng.standard_normal((8, grid.L * grid.F)).astype(np.float32)
    grad = grid.backward(x, up)
    touched = np.argwhere(grad != 0)
    probes = [tuple(v) for v in touched[rng.choice(len(touched), 24, replace=False)]]
    probes += [(0, 1, 0), (3, 1023, 1), (2, 500, 0)]
    upd = up.astype(np.float64)
    for j in probes:
        tp, tm = t.copy(), t.copy()
        tp[j] += 1
        tm[j] -= 1
        fd = (np.sum(upd * grid.forward(x, tp)) - np.sum(upd * grid.forward(x, tm))) / 2
        assert abs(fd - grad[j]) <= 1e-9 * max(1.0, abs(grad[j])), (j, fd, grad[j])


def test_backward_brute_force_unit_tables_with_collisions():
    """T = 2^4 (heavy collisions, corners of one point often share an entry). Sweeping
    unit tables e_j gives every gradient entry as <g, fwd(e_j)>; colliding corners must
    each add their own weight, so a backward that deduplicated would fail here."""
    grid = Grid(2, 2, 4, 2, 4)
    rng = np.random.default_rng(11)
    x = rng.random((50, 3), dtype=np.float32)
    up = rng.standard_normal((50, grid.L * grid.F)).astype(np.float32)
    grad = grid.backward(x, up)
    idx = grid.indices(x)
    assert any(len(set(idx[p, l])) < 8 for p in range(50) for l in range(2))
    for j in np.ndindex(grid.L, grid.T, grid.F):
        e = np.zeros((grid.L, grid.T, grid.F), dtype=np.float32)
        e[j] = 1
        want = np.sum(up.astype(np.float64) * grid.forward(x, e))
        assert abs(want - grad[j]) <= 1e-12 * max(1.0, abs(want))


def test_backward_accumulates_and_thread_count_invariant():
    """The gradient accumulates into the given array, and the per-level parallel run gives
    the same bits as the serial one (level slices are disjoint)."""
    grid = Grid(4, 2, 10, 2, 16)
    rng = np.random.default_rng(12)
    x = rng.random((500, 3), dtype=np.float32)
    up = rng.standard_normal((500, 8)).astype(np.float32)
    serial = grid.backward(x, up, nthreads=1)
    par = grid.backward(x, up, nthreads=4)
    np.testing.assert_array_equal(serial, par)
    twice = grid.backward(x, up, dtable=serial.copy())
    np.testing.assert_allclose(twice, 2 * serial, rtol=0, atol=1e-13 * np.max(np.abs(serial)))
    fwd1 = grid.forward(x, rng.random((4, 1024, 2), dtype=np.float32), nthreads=1)
    assert fwd1.shape == (500, 8)


def test_indices_match_bigint_hash():
    """Index export: idx[p][l][c] for corner offsets (c&1, c>>1&1, c>>2&1) equals the
    exact-integer hash of floor(fp32(x*N_l)) + offset, mod T."""
    grid = Grid(4, 2, 10, 2, 16)
    rng = np.random.default_rng(13)
    x = rng.random((100, 3), dtype=np.float32)
    x[:5] = np.float32(1.0)
    idx = grid.indices(x)
    for p in range(100):
        for l, n in enumerate(grid.res):
            v = [int(np.floor(np.float32(x[p, i]) * np.float32(n))) for i in range(3)]
            for c in range(8):
                cc = [v[i] + ((c >> i) & 1) for i in range(3)]
                assert idx[p, l, c] == bigint_hash(*cc, T=grid.T)


# ---------------------------------------------------------------------------------------
# Gradient with respect to the coordinates
# ---------------------------------------------------------------------------------------

def test_backward_x_finite_differences_exact():
    """Inside a voxel the encoding is linear along each axis (trilinear = multilinear), so
    a central difference is the derivative up to rounding. On the 2->16 grid (powers of
    two) with x = (k + 1/2)/32 and h = 2^-12, every x*N_l and (x +- h)*N_l is exact in fp32
    and x +- h stays inside the same voxel at every level."""
    g = Grid(4, 2, 10, 2, 16)
    rng = np.random.default_rng(21)
    table = rng.standard_normal((4, 1024, 2)).astype(np.float32)
    k = rng.integers(0, 32, size=(40, 3))
    x = ((k + 0.5) / 32.0).astype(np.float32)
    up = rng.standard_normal((40, 8)).astype(np.float32)
    dx = g.backward_x(x, table, up)
    h = np.float32(2.0 ** -12)
    for i in range(3):
        xp, xm = x.copy(), x.copy()
        xp[:, i] += h
        xm[:, i] -= h
        fd = np.sum(up.astype(np.float64) * (g.forward(xp, table) - g.forward(xm, table)), axis=1) / (2 * float(h))
        np.testing.assert_allclose(dx[:, i], fd, rtol=1e-9, atol=1e-9)


def test_backward_x_constant_table_is_zero():
    """A constant table gives a constant encoding: the weight derivatives of the 8 corners
    sum to zero along every axis."""
    g = Grid(4, 4, 10, 2, 16)
    rng = np.random.default_rng(22)
    x = rng.random((300, 3), dtype=np.float32)
    up = rng.standard_normal((300, 16)).astype(np.float32)
    dx = g.backward_x(x, np.full((4, 1024, 4), 0.75, dtype=np.float32), up)
    assert np.max(np.abs(dx)) <= 1e-12


def test_backward_x_affine_table_reproduced():
    """Trilinear interpolation reproduces affine functions: with table[l][h(v)] = A v
    (integer A, no hash collision among the grid's vertices at T = 2^20) the encoding at
    level l is A (x N_l), so dL/dx_i = sum_l sum_f g[l, f] A[f, i] N_l exactly."""
    g = Grid(3, 2, 20, 2, 8)
    rng = np.random.default_rng(23)
    A = rng.integers(-3, 4, size=(2, 3)).astype(np.float64)
    table = np.zeros((3, g.T, 2), dtype=np.float32)
    for l, n in enumerate(g.res):
        seen = set()
        for v in np.ndindex(n + 2, n + 2, n + 2):
            h = bigint_hash(*v, T=g.T)
            assert h not in seen, "hash collision among grid vertices"
            seen.add(h)
            table[l, h] = (A @ np.array(v, dtype=np.float64)).astype(np.float32)
    x = rng.random((200, 3), dtype=np.float32)
    up = rng.standard_normal((200, 6)).astype(np.float32)
    want = np.zeros((200, 3))
    for l, n in enumerate(g.res):
        want += float(n) * (up[:, 2 * l:2 * l + 2].astype(np.float64) @ A)
    np.testing.assert_allclose(g.backward_x(x, table, up), want, rtol=1e-12, atol=1e-9)


# ---------------------------------------------------------------------------------------
# Sparse Adam
# ---------------------------------------------------------------------------------------

def test_adam_untouched_elements_unchanged():
    """An element with zero gradient was not sampled: parameter, m and v stay as they are."""
    rng = np.random.default_rng(30)
    p, m, v = rng.standard_normal(100), rng.standard_normal(100), rng.random(100)
    g = np.zeros(100, dtype=np.float32)
    p2, m2, v2 = oracle.adam_step(p, m, v, g, step=7, lr=1e-2)
    np.testing.assert_array_equal(p2, p)
    np.testing.assert_array_equal(m2, m)
    np.testing.assert_array_equal(v2, v)


def test_adam_first_step_closed_form():
    """From m = v = 0 at t = 1 the bias corrections give m_hat = g and v_hat = g^2, so the
    step is lr * g / (|g| + eps)."""
    rng = np.random.default_rng(31)
    p = rng.standard_normal(1000)
    g = rng.standard_normal(1000).astype(np.float32)
    p2, m2, v2 = oracle.adam_step(p, np.zeros(1000), np.zeros(1000), g, step=1, lr=0.01, beta1=0.9,
                                  beta2=0.99, eps=1e-8)
    gd = g.astype(np.float64)
    np.testing.assert_allclose(p2, p - 0.01 * gd / (np.abs(gd) + 1e-8), rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(m2, 0.1 * gd, rtol=1e-15)
    np.testing.assert_allclose(v2, 0.01 * gd * gd, rtol=1e-13)


def test_adam_constant_gradient_closed_form():
    """With a constant gradient the bias-corrected moments stay exactly g and g^2, so after
    t steps theta = theta_0 - t * lr * g / (|g| + eps)."""
    rng = np.random.default_rng(32)
    p0 = rng.standard_normal(200)
    g = rng.standard_normal(200).astype(np.float32)
    p, m, v = p0.copy(), np.zeros(200), np.zeros(200)
    for t in range(1, 6):
        p, m, v = oracle.adam_step(p, m, v, g, step=t, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-12)
    gd = g.astype(np.float64)
    np.testing.assert_allclose(p, p0 - 5 * 1e-3 * gd / (np.abs(gd) + 1e-12), rtol=1e-12, atol=1e-14)


def test_adam_matches_torch_adam_where_touched():
    """Where every gradient is nonzero the sparse step is torch.optim.Adam without weight
    decay (a library implementation of the same textbook update), in fp64."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(33)
    p0 = rng.standard_normal(500)
    prm = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.Adam([prm], lr=5e-3, betas=(0.9, 0.99), eps=1e-10, weight_decay=0.0)
    p, m, v = p0.copy(), np.zeros(500), np.zeros(500)
    for t in range(1, 4):
        g = (rng.standard_normal(500).astype(np.float32) + 0.25).astype(np.float32)
        g[g == 0] = 1.0
        prm.grad = torch.tensor(g.astype(np.float64))
        opt.step()
        p, m, v = oracle.adam_step(p, m, v, g, step=t, lr=5e-3, beta1=0.9, beta2=0.99, eps=1e-10)
    np.testing.assert_allclose(p, prm.detach().numpy(), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------------------
# Encoding + MLP
# ---------------------------------------------------------------------------------------

def bf16_bits(a):
    """Round-to-nearest-even fp32 -> bf16 bit patterns (numpy)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u >> 16) & 1) + 0x7FFF
    return ((u + r) >> 16).astype(np.uint16)


def bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_bf16_decode():
    bits = np.arange(0, 65536, 97, dtype=np.uint32).astype(np.uint16)
    for b in bits:
        with np.errstate(invalid="ignore"):          # NaN patterns
            want = bf16_values(np.array([b]))[0]
        got = oracle.bf16_to_double(int(b))
        assert (got == want) or (np.isnan(got) and np.isnan(want))


# Pins of the MLP that the mathematics fixes exactly. The grid doubles its resolution at
# every level (N 4 -> 2^17, b = 2), so x = k/4 is a vertex at every level and the encoding is
# the table entry at the hashed vertex, exactly (P2); the entry is found here with Python big
# ints, not with the oracle. Tables hold small integers and the weights are 0, +-1 or small
# integers, all exact in bf16, so every layer is exact in fp64 and the pins compare exactly.
MLP_GRID = (16, 2, 10, 4, 2**17)     # L, F, log2T, N_min, N_max: in = L*F = 32


def mlp_vertex_inputs(seed):
    L, F, log2T, nmin, nmax = MLP_GRID
    rng = np.random.default_rng(seed)
    table = rng.integers(-4, 5, size=(L, 2**log2T, F)).astype(np.float32)
    k = np.stack(np.meshgrid(*[np.arange(5)] * 3, indexing="ij"), -1).reshape(-1, 3)
    x = (k / 4.0).astype(np.float32)
    e = np.zeros((len(k), L * F))
    for p, kp in enumerate(k):
        for l in range(L):
            v = [int(ki) * (nmin << l) // 4 for ki in kp]          # x * N_l, an integer
            e[p, l * F:(l + 1) * F] = table[l, bigint_hash(*v) % 2**log2T]
    return Grid(*MLP_GRID), x, table, e


def bf16_int(a):
    """bf16 bit patterns of small integers (exact)."""
    return bf16_bits(np.asarray(a, dtype=np.float32))


def test_mlp_split_weights_give_absolute_values():
    """W1 = [I; -I], b1 = 0 gives a1 = (relu(e), relu(-e)); W2 a permutation, b2 = 0 keeps
    them; W3's first row of ones sums them: y0 = sum_k |e_k| + b3_0. Its second row weights
    the permuted activations by 1..64, which fixes which activation each W2 row reads."""
    g, x, table, e = mlp_vertex_inputs(61)
    n = 32
    w1 = np.zeros((64, n))
    w1[:n, :n] = np.eye(n)
    w1[n:, :n] = -np.eye(n)
    perm = np.random.default_rng(62).permutation(64)
    w2 = np.eye(64)[perm]                         # a2_j = a1_perm[j]
    w3 = np.zeros((4, 64))
    w3[0] = 1.0
    w3[1] = np.arange(1, 65)
    b1, b2 = np.zeros(64, np.float32), np.zeros(64, np.float32)
    b3 = np.array([3.0, -5.0, 0.0, 7.0], np.float32)
    y = g.mlp_forward(x, table, bf16_int(w1), b1, bf16_int(w2), b2, bf16_int(w3), b3)
    np.testing.assert_array_equal(y[:, 0], np.abs(e).sum(1) + 3.0)
    a1 = np.concatenate([np.maximum(e, 0), np.maximum(-e, 0)], 1)
    np.testing.assert_array_equal(y[:, 1], (a1[:, perm] * np.arange(1, 65)).sum(1) - 5.0)
    np.testing.assert_array_equal(y[:, 2], 0.0)
    np.testing.assert_array_equal(y[:, 3], 7.0)
    assert np.any(e < 0) and np.any(e > 0)


def test_mlp_first_relu_zeroes_negative_preactivations():
    """W1 = I, b1 = -1: a1_k = max(e_k - 1, 0), so every entry below 1 is cut to zero;
    W2 = I, b2 = 100 keeps layer 2 linear (a2 = a1 + 100 > 0, so its own ReLU cannot redo
    the cut); y0 = sum_k max(e_k - 1, 0) + 32 * 100."""
    g, x, table, e = mlp_vertex_inputs(63)
    w1 = np.zeros((64, 32))
    w1[:32] = np.eye(32)
    w3 = np.zeros((4, 64))
    w3[0, :32] = 1.0
    b1 = np.full(64, -1.0, np.float32)
    b2 = np.full(64, 100.0, np.float32)
    y = g.mlp_forward(x, table, bf16_int(w1), b1, bf16_int(np.eye(64)), b2, bf16_int(w3), np.zeros(4, np.float32))
    np.testing.assert_array_equal(y[:, 0], np.maximum(e - 1.0, 0).sum(1) + 3200.0)
    assert np.any(e < 1) and np.any(e > 1)


def test_mlp_second_relu_zeroes_negative_preactivations():
    """W1 = I, b1 = 100 keeps layer 1 linear (a1 = e + 100 > 0); W2 = -I, b2 = 101 gives
    a2_k = max(1 - e_k, 0), cut to zero wherever e_k > 1; y0 = sum_k max(1 - e_k, 0), with
    rows of W3 = 2 and a bias added to the other outputs."""
    g, x, table, e = mlp_vertex_inputs(64)
    w1 = np.zeros((64, 32))
    w1[:32] = np.eye(32)
    w3 = np.zeros((4, 64))
    w3[0, :32] = 1.0
    w3[2, :32] = 2.0
    b1 = np.full(64, 100.0, np.float32)
    b2 = np.full(64, 101.0, np.float32)
    b2[32:] = -1.0                                # rows with no input: relu(-1) = 0
    b3 = np.array([0.0, 1.5, 0.25, -2.0], np.float32)
    y = g.mlp_forward(x, table, bf16_int(w1), b1, bf16_int(-np.eye(64)), b2, bf16_int(w3), b3)
    want = np.maximum(1.0 - e, 0).sum(1)
    np.testing.assert_array_equal(y[:, 0], want)
    np.testing.assert_array_equal(y[:, 1], 1.5)
    np.testing.assert_array_equal(y[:, 2], 2 * want + 0.25)
    np.testing.assert_array_equal(y[:, 3], -2.0)
    assert np.any(e > 1) and np.any(e < 1)


# ---------------------------------------------------------------------------------------
# D-dimensional inputs (2^D corners; primes of Repro-HG sections 2.2 and 3)
# ---------------------------------------------------------------------------------------

PRIMES7 = (1, 2654435761, 805459861, 3674653429, 2097192037, 1434869437, 2165219737)


def bigint_hash_nd(c, T=None):
    h = 0
    for ci, pi in zip(c, PRIMES7):
        h ^= (int(ci) % 2**32) * pi
    h %= 2**32
    return h if T is None else h % T


def test_hash_nd_bigint_and_primes():
    rng = np.random.default_rng(90)
    for D in range(1, 8):
        for c in rng.integers(-2**33, 2**33, size=(200, D)):
            assert oracle.hash_nd(c) == bigint_hash_nd(c)
        for i in range(D):        # unit vectors give the primes themselves
            e = np.zeros(D, dtype=np.int64)
            e[i] = 1
            assert oracle.hash_nd(e) == PRIMES7[i]
    assert oracle.hash_nd([1, 1, 1, 1]) == 1 ^ 2654435761 ^ 805459861 ^ 3674653429


@pytest.mark.parametrize("D", [2, 4])
def test_nd_indices_equal_bigint_hash_of_every_corner(D):
    """Every exported index of a D-dimensional point equals the big-int hash of
    floor(fp32(x_i * N_l)) + offset_i mod T, corner c having offset bit i = (c >> i) & 1,
    laid out [point][level][corner]; points inside, on and outside the unit cube."""
    L, log2T = 5, 12
    g = oracle.GridND(D, L, 2, log2T, 3, 300)
    rng = np.random.default_rng(96 + D)
    x = (rng.random((150, D)) * 2.0 - 0.5).astype(np.float32)
    x[0] = 0.0
    x[1] = 1.0
    x[2] = np.float32(1.0 - 2**-24)
    idx = g.indices(x)
    assert idx.shape == (150, L, 2**D)
    for p in range(150):
        for l, n in enumerate(g.res):
            v = [int(np.floor(np.float32(x[p, i]) * np.float32(n))) for i in range(D)]
            for c in range(2**D):
                corner = [v[i] + ((c >> i) & 1) for i in range(D)]
                assert idx[p, l, c] == bigint_hash_nd(corner, 2**log2T), (p, l, c)


def test_nd_at_three_dimensions_equals_3d_oracle():
    g3, gn = Grid(4, 2, 10, 2, 16), oracle.GridND(3, 4, 2, 10, 2, 16)
    rng = np.random.default_rng(91)
    x = rng.random((300, 3), dtype=np.float32)
    t = rng.standard_normal((4, 1024, 2)).astype(np.float32)
    up = rng.standard_normal((300, 8)).astype(np.float32)
    np.testing.assert_array_equal(gn.indices(x), g3.indices(x))
    np.testing.assert_array_equal(gn.forward(x, t), g3.forward(x, t))
    np.testing.assert_array_equal(gn.backward(x, up), g3.backward(x, up))
    np.testing.assert_array_equal(gn.backward_x(x, t, up), g3.backward_x(x, t, up))


def hat_basis_nd(x, table, res, T):
    N, D = x.shape
    L, _, F = table.shape
    out = np.zeros((N, L * F))
    for p in range(N):
        for l, n in enumerate(res):
            xs = [float(np.float32(x[p, i]) * np.float32(n)) for i in range(D)]
            base = [int(np.floor(v)) for v in xs]
            for off in np.ndindex(*([4] * D)):
                v = [base[i] - 1 + off[i] for i in range(D)]
                w = 1.0
                for i in range(D):
                    w *= max(0.0, 1 - abs(xs[i] - v[i]))
                if w:
                    out[p, l * F:(l + 1) * F] += w * table[l, bigint_hash_nd(v, T)].astype(np.float64)
    return out


@pytest.mark.parametrize("D", [2, 4])
def test_nd_forward_hat_basis_and_weight_sum(D):
    g = oracle.GridND(D, 3, 2, 10, 2, 8)
    rng = np.random.default_rng(92 + D)
    t = rng.standard_normal((3, 1024, 2)).astype(np.float32)
    x = rng.random((40, D), dtype=np.float32)
    x[0] = np.float32(1.0)
    x[1] = np.float32(0.0)
    np.testing.assert_allclose(g.forward(x, t), hat_basis_nd(x, t, g.res, g.T), rtol=0, atol=1e-12)
    ones = g.forward(x, np.ones((3, 1024, 2), dtype=np.float32))
    assert np.max(np.abs(ones - 1.0)) <= 8 * np.finfo(np.float64).eps


@pytest.mark.parametrize("D", [2, 4])
def test_nd_backward_adjoint_and_input_gradient(D):
    g = oracle.GridND(D, 4, 2, 10, 2, 16)
    rng = np.random.default_rng(95 + D)
    t = rng.standard_normal((4, 1024, 2)).astype(np.float32)
    up = rng.standard_normal((60, 8)).astype(np.float32)
    k = rng.integers(0, 32, size=(60, D))
    x = ((k + 0.5) / 32.0).astype(np.float32)
    lhs = float(np.sum(up.astype(np.float64) * g.forward(x, t)))
    rhs = float(np.sum(g.backward(x, up) * t.astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)
    dx = g.backward_x(x, t, up)
    h = np.float32(2.0 ** -12)
    for i in range(D):
        xp, xm = x.copy(), x.copy()
        xp[:, i] += h
        xm[:, i] -= h
        fd = np.sum(up.astype(np.float64) * (g.forward(xp, t) - g.forward(xm, t)), axis=1) / (2 * float(h))
        np.testing.assert_allclose(dx[:, i], fd, rtol=1e-9, atol=1e-9)

# ---------------------------------------------------------------------------------------
# Values the pages print (tests/golden/, each file citing its page and section)
# ---------------------------------------------------------------------------------------

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_level_table():
    t = golden("repro_hg_level_table.json")
    r = oracle.resolutions(t["levels"], t["coarsest_resolution"], t["finest_resolution"])
    assert r[0] == t["coarsest_resolution"] and r[-1] == t["finest_resolution"]
    g = Grid(t["levels"], t["features"], t["log2_table_size"], t["coarsest_resolution"], t["finest_resolution"])
    assert g.T == 2 ** 19 and g.L * g.F == 32
    # the printed level-2 row is the table's inconsistency: the schedule gives 20 there
    assert r[1] == 20 != t["printed_level_2_resolution"] and r[3] == t["printed_level_2_resolution"]


def test_golden_parameter_count():
    t = golden("nerface_hg_parameter_count.json")
    g = Grid(t["levels"], t["features"], 19, 16, 512)
    assert g.T == t["entries_per_level"]
    assert g.L * g.T * g.F == 16 * 524288 * 2 == 16777216


def test_golden_primes():
    t = golden("hash_primes.json")
    p3 = t["primes_3d"]
    assert [oracle.hash3(1, 0, 0), oracle.hash3(0, 1, 0), oracle.hash3(0, 0, 1)] == p3
    assert tuple(p3) == PRIMES
    for i, prime in enumerate(t["primes_nd"]):
        e = [0] * len(t["primes_nd"])
        e[i] = 1
        assert oracle.hash_nd(e) == prime
