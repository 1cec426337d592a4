"""Seeded random configurations against the oracle, for every entry point.

Encoding (indices, forward, fp32 and fp16 backward, dL/dx): per seed a random dimension D (2, 3 or
4), level count, feature width, table size, resolution range, table dtype, forward gather,
backward reduction mode and schedule, and a random point count (1 to 700, so most batches
end in a ragged tile) whose first rows sit on the cube's faces, just inside its upper face
or outside it. Every entry point is held to the bars of the fixed-shape parity tests:
indices bit-exact; forward within rtol * sum_c w_c |e_c|; fp32 gradients within 1e-5
relative L2 per level; fp16 gradients within the fp16 accumulation model; dL/dx within
1e-5 of its absolute-term bound (scaled by 2^(D-3) for D > 3: twice the corners per level).

Sparse Adam: random levels, widths, table sizes, dtypes, gradient sparsity, step counts and
the fused clear, each step against the oracle's step from the GPU's state (the bars of
run_adam_steps). Encoding + MLP: every input width the MLP takes (L * F = 16, 32, 48, 64)
with F from 1 to 8, random grids, dtypes and gathers, and point counts that leave ragged
128-point tiles, against the oracle within the propagated bf16 bound of check_mlp."""
import numpy as np
import pytest

import oracle
import workloads
from tests.test_parity import (FWD_RTOL, THREADS, check_gradient, check_half_gradient, check_mlp, dev, mlp_weights,
                               run_adam_steps)

torch = pytest.importorskip("torch")

GATHER = {"auto": 0, "corner": 1, "sector": 2, "pair": 3, "lanes": 4}
BACKWARD = {"auto": 0, "atomic": 1, "dedup": 2, "runs": 3, "dedup_adaptive": 4, "run_lanes": 5}
SCHEDULE = {"auto": 0, "point": 1, "level": 2}
EDGE = np.array([0.0, 1.0, 1.0 - 2**-24, 0.5, -0.25, 1.5], dtype=np.float32)


def config(seed):
    """The random configuration of one seed: options the library accepts for it (D != 3
    takes CORNER or LANES gathers and ATOMIC or RUN_LANES reductions; RUN_LANES, and the
    deduplicating and run-merging reductions, take F <= 4)."""
    rng = np.random.default_rng(1000 + seed)
    D = int(rng.choice([2, 3, 3, 3, 4]))
    L = int(rng.integers(1, 20))
    F = int(rng.choice([1, 2, 4, 8]))
    log2T = int(rng.integers(4, 15))
    n_min = int(rng.integers(1, 40))
    n_max = n_min if L == 1 else int(rng.integers(n_min, 3000))
    dtype = str(rng.choice(["f32", "f16"]))
    if D == 3:
        gather = str(rng.choice(list(GATHER)))
        backward = str(rng.choice(list(BACKWARD) if F <= 4 else ["auto", "atomic"]))
        schedule = str(rng.choice(list(SCHEDULE)))
    else:
        gather = str(rng.choice(["auto", "corner", "lanes"]))
        backward = str(rng.choice(["auto", "atomic"] + (["run_lanes"] if F <= 4 else [])))
        schedule = "auto"
    n = int(rng.integers(1, 700))
    return dict(D=D, L=L, F=F, log2T=log2T, N_min=n_min, N_max=n_max, dtype=dtype, gather=gather,
                backward=backward, schedule=schedule, n=n)


def inputs(c, seed):
    rng = np.random.default_rng(2000 + seed)
    table = workloads.table_values(rng, c["L"], 2 ** c["log2T"], c["F"], c["dtype"])
    x = rng.random((c["n"], c["D"]), dtype=np.float32)
    k = min(c["n"], 8)
    x[:k] = EDGE[rng.integers(0, len(EDGE), size=(k, c["D"]))]
    g = workloads.upstream_grads(rng, c["n"], c["L"] * c["F"])
    return x, table, g


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(48))
def test_random_configuration(seed):
    import multiresolution_hash_grid_b200 as hg
    c = config(seed)
    D, L, F, log2T, n = c["D"], c["L"], c["F"], c["log2T"], c["n"]
    f16 = c["dtype"] == "f16"
    grid = hg.HashGrid(L, F, log2T, c["N_min"], c["N_max"], hg.HASHGRID_F16 if f16 else hg.HASHGRID_F32,
                       forward_gather=GATHER[c["gather"]], backward_mode=BACKWARD[c["backward"]],
                       schedule=SCHEDULE[c["schedule"]], D=D)
    odt = oracle.F16 if f16 else oracle.F32
    og = (oracle.Grid(L, F, log2T, c["N_min"], c["N_max"], odt) if D == 3 else
          oracle.GridND(D, L, F, log2T, c["N_min"], c["N_max"], odt))
    x, table, g = inputs(c, seed)
    x_d, t_d, g_d = dev(x), dev(table), dev(g)

    np.testing.assert_array_equal(grid.indices(x_d).cpu().numpy().view(np.uint32), og.indices(x), err_msg=str(c))

    out = grid.forward(x_d, t_d).cpu().numpy().astype(np.float64)
    ref = og.forward(x, table, nthreads=THREADS)
    bound = og.forward(x, np.abs(table), nthreads=THREADS)
    rtol = FWD_RTOL[c["dtype"]] if D == 3 else 1e-6
    assert np.all(np.abs(out - ref) <= rtol * bound + 1e-30), c

    gref = og.backward(x, g, nthreads=THREADS)
    got = grid.backward(x_d, g_d).cpu().numpy()
    check_gradient(got, gref)
    np.testing.assert_array_equal(got == 0, gref == 0, err_msg=str(c))

    dh = torch.zeros((L, 2**log2T, F), dtype=torch.float16, device="cuda")
    hg.hashgrid_backward_half(grid.handle, x_d, g_d, n, dh)
    torch.cuda.synchronize()
    check_half_gradient(og, x, g, dh.cpu().numpy())

    dx = grid.backward_input(x_d, g_d, t_d).cpu().numpy().astype(np.float64)
    dxref = og.backward_x(x, table, g, nthreads=THREADS)
    tmax = float(np.max(np.abs(table.astype(np.float64))))
    B = np.zeros(n)
    for l, r in enumerate(og.res):
        B += float(r) * 2.0 * np.sum(np.abs(g[:, l * F:(l + 1) * F].astype(np.float64)), axis=1) * tmax
    assert np.all(np.abs(dx - dxref) <= 1e-5 * B[:, None] * 2.0 ** max(D - 3, 0) + 1e-30), c


def test_configurations_cover_every_option():
    """The 48 seeds reach every gather, reduction mode and schedule for D = 3, every
    N-d option, both dtypes and all four feature widths (checked on the host)."""
    cs = [config(s) for s in range(48)]
    three = [c for c in cs if c["D"] == 3]
    assert {c["gather"] for c in three} == set(GATHER)
    assert {c["backward"] for c in three} == set(BACKWARD)
    assert {c["schedule"] for c in three} == set(SCHEDULE)
    nd = [c for c in cs if c["D"] != 3]
    assert {c["D"] for c in nd} == {2, 4}
    assert {c["gather"] for c in nd} == {"auto", "corner", "lanes"}
    assert {c["backward"] for c in nd} == {"auto", "atomic", "run_lanes"}
    assert {c["dtype"] for c in cs} == {"f32", "f16"} and {c["F"] for c in cs} == {1, 2, 4, 8}


def adam_config(seed):
    rng = np.random.default_rng(3000 + seed)
    return dict(dtype=str(rng.choice(["f32", "f16"])), zero_grad=bool(rng.integers(0, 2)),
                L=int(rng.integers(2, 9)), F=int(rng.choice([1, 2, 4, 8])), log2T=int(rng.integers(4, 15)),
                steps=int(rng.integers(1, 5)), zero_frac=float(rng.choice([0.0, 0.5, 0.9, 0.99])))


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(16))
def test_random_adam(seed):
    c = adam_config(seed)
    run_adam_steps(c["dtype"], c["zero_grad"], c["L"], c["F"], c["log2T"], c["steps"], c["zero_frac"], 4000 + seed)


def mlp_config(seed):
    rng = np.random.default_rng(5000 + seed)
    K = int(rng.choice([16, 32, 48, 64]))
    F = int(rng.choice([f for f in (1, 2, 4, 8) if K % f == 0 and K // f <= 32]))
    L = K // F
    n_min = int(rng.integers(2, 40))
    n_max = n_min if L == 1 else int(rng.integers(n_min, 3000))
    return dict(L=L, F=F, log2T=int(rng.integers(4, 17)), N_min=n_min, N_max=n_max,
                dtype=str(rng.choice(["f32", "f16"])), gather=str(rng.choice(["auto", "corner"])),
                n=int(rng.integers(1, 700)))


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(16))
def test_random_mlp(seed):
    import multiresolution_hash_grid_b200 as hg
    c = mlp_config(seed)
    L, F, log2T, n = c["L"], c["F"], c["log2T"], c["n"]
    f16 = c["dtype"] == "f16"
    grid = hg.HashGrid(L, F, log2T, c["N_min"], c["N_max"], hg.HASHGRID_F16 if f16 else hg.HASHGRID_F32,
                       forward_gather=GATHER[c["gather"]])
    og = oracle.Grid(L, F, log2T, c["N_min"], c["N_max"], oracle.F16 if f16 else oracle.F32)
    rng = np.random.default_rng(6000 + seed)
    table = (rng.standard_normal((L, 2**log2T, F)) * 0.3).astype(np.float16 if f16 else np.float32)
    x = rng.random((n, 3), dtype=np.float32)
    k = min(n, 8)
    x[:k] = EDGE[rng.integers(0, len(EDGE), size=(k, 3))]
    wts = mlp_weights(rng, L * F)
    y = torch.full((n, 4), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hg.hashgrid_mlp_forward(grid.handle, dev(x), n, dev(table), *[dev(w) for w in wts], y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, c
    check_mlp(og, x, table, wts, y.cpu().numpy())


def test_adam_and_mlp_configurations_cover_the_options():
    """Host check: the Adam seeds reach both dtypes, both clear settings, every width and
    a dense and a nearly empty gradient; the MLP seeds every input width, F = 1..8, both
    dtypes and both producer forms."""
    a = [adam_config(s) for s in range(16)]
    assert {c["dtype"] for c in a} == {"f32", "f16"} and {c["zero_grad"] for c in a} == {True, False}
    assert {c["F"] for c in a} == {1, 2, 4, 8} and {0.0, 0.99} <= {c["zero_frac"] for c in a}
    m = [mlp_config(s) for s in range(16)]
    assert {c["L"] * c["F"] for c in m} == {16, 32, 48, 64} and {c["F"] for c in m} == {1, 2, 4, 8}
    assert {c["dtype"] for c in m} == {"f32", "f16"} and {c["gather"] for c in m} == {"auto", "corner"}


def level_config(seed):
    rng = np.random.default_rng(7000 + seed)
    L = int(rng.integers(8, 15))
    n_min = int(rng.integers(2, 40))
    return dict(L=L, F=int(rng.choice([2, 4])), log2T=int(rng.integers(19, 21)), N_min=n_min,
                N_max=int(rng.integers(400, 3000)), dtype=str(rng.choice(["f32", "f16"])),
                gather=str(rng.choice(["auto", "corner"])), backward=str(rng.choice(["auto", "atomic", "runs"])),
                n=int(rng.integers(1, 700)))


def level_groups(c):
    """The level-major schedule's grouping rule (consecutive levels while their reachable
    entries, min(T, (N_l + 2)^3) at 4F bytes, stay within 32 MB), restated to check that
    the seeds below reach several groups."""
    lo, acc = [0], 0.0
    for l, r in enumerate(oracle.resolutions(c["L"], c["N_min"], c["N_max"])):
        b = min(2.0 ** c["log2T"], (r + 2.0) ** 3) * c["F"] * 4
        if l > 0 and acc + b > 32 * 2**20:
            lo.append(l)
            acc = 0.0
        acc += b
    return lo + [c["L"]]


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(8))
def test_random_level_groups(seed):
    """The level-major schedule on tables of 2^19 and 2^20 entries, whose levels fall into
    several groups of different sizes: indices, forward, fp32 and fp16 gradients against
    the oracle."""
    import multiresolution_hash_grid_b200 as hg
    c = level_config(seed)
    L, F, log2T, n = c["L"], c["F"], c["log2T"], c["n"]
    f16 = c["dtype"] == "f16"
    grid = hg.HashGrid(L, F, log2T, c["N_min"], c["N_max"], hg.HASHGRID_F16 if f16 else hg.HASHGRID_F32,
                       forward_gather=GATHER[c["gather"]], backward_mode=BACKWARD[c["backward"]],
                       schedule=SCHEDULE["level"])
    og = oracle.Grid(L, F, log2T, c["N_min"], c["N_max"], oracle.F16 if f16 else oracle.F32)
    rng = np.random.default_rng(8000 + seed)
    table = workloads.table_values(rng, L, 2**log2T, F, c["dtype"])
    x = rng.random((n, 3), dtype=np.float32)
    k = min(n, 8)
    x[:k] = EDGE[rng.integers(0, len(EDGE), size=(k, 3))]
    g = workloads.upstream_grads(rng, n, L * F)
    x_d, t_d, g_d = dev(x), dev(table), dev(g)
    np.testing.assert_array_equal(grid.indices(x_d).cpu().numpy().view(np.uint32), og.indices(x), err_msg=str(c))
    out = grid.forward(x_d, t_d).cpu().numpy().astype(np.float64)
    ref = og.forward(x, table, nthreads=THREADS)
    bound = og.forward(x, np.abs(table), nthreads=THREADS)
    assert np.all(np.abs(out - ref) <= FWD_RTOL[c["dtype"]] * bound + 1e-30), c
    got = grid.backward(x_d, g_d).cpu().numpy()
    check_gradient(got, og.backward(x, g, nthreads=THREADS))
    dh = torch.zeros((L, 2**log2T, F), dtype=torch.float16, device="cuda")
    hg.hashgrid_backward_half(grid.handle, x_d, g_d, n, dh)
    torch.cuda.synchronize()
    check_half_gradient(og, x, g, dh.cpu().numpy())


def test_level_group_configurations_have_several_groups():
    """Host check: every level-major seed splits its levels into at least two groups, and
    the seeds include groups of more than one level."""
    gs = [level_groups(level_config(s)) for s in range(8)]
    assert all(len(g) >= 3 for g in gs), gs
    assert any(max(b - a for a, b in zip(g, g[1:])) > 1 for g in gs), gs
