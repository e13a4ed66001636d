"""Pins of the float64 oracle to facts that do not come from the oracle itself.

Each pin targets a plausible mistake: a dropped term, a wrong sign or index, a
transposed operand, the wrong KL direction, the wrong mask or scale.  The last
test plants such mistakes in (a copy of) the oracle, on the CPU, and checks
that some pin catches each one.

Sources of truth used here:
* closed forms derived by hand (the Bernoulli case N=2 and the uniform-vs-one-hot
  case in tests/golden/uniform_vs_onehot.json);
* torch's own fp64 ``log_softmax`` + ``kl_div`` and autograd on tiny inputs
  (a library routine, independent of the NumPy oracle);
* central finite differences of the oracle's own loss (pins the backward to
  the forward);
* invariants: KL >= 0, identical rows give zero, an orthogonal change of basis
  leaves the relation unchanged, RoPE depends only on relative position;
* the pages' exactness claim: the tiled linear-memory algorithms equal the
  dense definition to ~1e-12.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dense, tiled
import workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_pair(N, d, seed, noise=0.7):
    xt, xs = workload.gaussian_pair((N, d), seed, noise, torch.float64)
    return xt.numpy(), xs.numpy()


# ---------------------------------------------------------------- closed forms

def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


@pytest.mark.parametrize("causal", [True, False])
def test_n2_bernoulli_closed_form(causal):
    """N=2: every row is a two-point distribution, so KL is the Bernoulli KL."""
    d = 4
    s = 1.0 / math.sqrt(d)
    xt = np.array([[1.0, -0.5, 0.25, 2.0], [0.5, 1.5, -1.0, 0.0]])
    xs = np.array([[-0.75, 0.5, 1.0, 0.5], [1.25, -0.25, 0.5, 1.0]])
    a = np.array([0.3, -0.7])            # upstream dkl per row
    zt = lambda i, j: s * float(xt[i] @ xt[j])
    zs = lambda i, j: s * float(xs[i] @ xs[j])

    def bern_kl(p, q):
        return p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))

    # row 1: p = P(j=1)
    p1, q1 = _sigmoid(zt(1, 1) - zt(1, 0)), _sigmoid(zs(1, 1) - zs(1, 0))
    if causal:
        kl_ref = [0.0, bern_kl(p1, q1)]
        # G(1,0) = a1 ((1-q1) - (1-p1)) = a1 (p1 - q1); G(1,1) = a1 (q1 - p1); row 0 is zero.
        g10, g11 = a[1] * (p1 - q1), a[1] * (q1 - p1)
        dx0 = s * g10 * xs[1]
        dx1 = s * (g10 * xs[0] + 2.0 * g11 * xs[1])
    else:
        p0, q0 = _sigmoid(zt(0, 1) - zt(0, 0)), _sigmoid(zs(0, 1) - zs(0, 0))   # P(j=1) on row 0
        kl_ref = [bern_kl(p0, q0), bern_kl(p1, q1)]
        g00, g01 = a[0] * (p0 - q0), a[0] * (q0 - p0)
        g10, g11 = a[1] * (p1 - q1), a[1] * (q1 - p1)
        # (G + G^T) X_s
        dx0 = s * (2 * g00 * xs[0] + (g01 + g10) * xs[1])
        dx1 = s * ((g10 + g01) * xs[0] + 2 * g11 * xs[1])
    r = dense.fwd_unit(xt, xs, causal=causal)
    np.testing.assert_allclose(r["kl"], kl_ref, rtol=1e-13, atol=1e-15)
    dx = dense.bwd_unit(xt, xs, dkl=a, causal=causal)
    np.testing.assert_allclose(dx, np.stack([dx0, dx1]), rtol=1e-12, atol=1e-15)


def test_uniform_vs_onehot_golden():
    g = json.load(open(os.path.join(GOLDEN, "uniform_vs_onehot.json")))["inputs"]
    N, d, t, c = g["N"], g["d"], g["t"], g["c"]
    dkl = np.array(g["dkl"])
    s = 1.0 / math.sqrt(d)
    xt = np.full((N, d), t / math.sqrt(d))
    xs = c * np.eye(N, d)
    a = s * c * c
    kl_ref = np.array([-math.log(i + 1) + math.log(math.exp(a) + i) - a / (i + 1) for i in range(N)])
    r = dense.fwd_unit(xt, xs)
    assert r["kl"][0] == 0.0
    np.testing.assert_allclose(r["kl"], kl_ref, rtol=1e-13, atol=1e-15)
    # teacher LSE: log(i+1) + s t^2 ; student: log(e^a + i)
    np.testing.assert_allclose(r["lse_t"], [math.log(i + 1) + s * t * t for i in range(N)], rtol=1e-14)
    np.testing.assert_allclose(r["lse_s"], [math.log(math.exp(a) + i) for i in range(N)], rtol=1e-14)
    G = np.zeros((N, N))
    for i in range(N):
        for j in range(i + 1):
            rs = (math.exp(a) if j == i else 1.0) / (math.exp(a) + i)
            G[i, j] = dkl[i] * (rs - 1.0 / (i + 1))
    dx_ref = s * c * (G + G.T)
    np.testing.assert_allclose(dense.bwd_unit(xt, xs, dkl=dkl), dx_ref, rtol=1e-12, atol=1e-16)
    # the unit loss L = (1/n) sum_i kl_i of the same closed form
    L_ref = sum(kl_ref) / N
    assert abs(dense.unit_loss(r["kl"]) - L_ref) <= 1e-14 * abs(L_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_unit_loss_matches_default_backward(causal):
    """L = (1/n) sum_i kl_i is the loss whose gradient the default upstream
    gradient (1/n per row) produces: central differences of unit_loss with
    respect to X_s equal bwd_unit(dkl=None).  A wrong normaliser (sum, 1/(n-1))
    or a wrong row count fails this."""
    N, d = 9, 4
    xt, xs = _rand_pair(N, d, seed=77)
    g = dense.bwd_unit(xt, xs, None, causal)
    h = 1e-6
    fd = np.zeros_like(xs)
    for i in range(N):
        for k in range(d):
            xp, xm = xs.copy(), xs.copy()
            xp[i, k] += h
            xm[i, k] -= h
            lp = dense.unit_loss(dense.fwd_unit(xt, xp, causal)["kl"])
            lm = dense.unit_loss(dense.fwd_unit(xt, xm, causal)["kl"])
            fd[i, k] = (lp - lm) / (2 * h)
    np.testing.assert_allclose(fd, g, rtol=1e-6, atol=1e-10)


# ------------------------------------------------------- library cross-check

def _torch_reference(xt, xs, dkl, causal):
    """fp64 torch: log_softmax + kl_div + autograd (independent of the oracle)."""
    xt = torch.tensor(xt, dtype=torch.float64)
    xs = torch.tensor(xs, dtype=torch.float64, requires_grad=True)
    N, d = xt.shape
    s = d ** -0.5
    mask = torch.ones(N, N, dtype=torch.bool)
    if causal:
        mask = torch.tril(mask)
    lt = torch.log_softmax((xt @ xt.T * s).masked_fill(~mask, float("-inf")), dim=-1)
    ls = torch.log_softmax((xs @ xs.T * s).masked_fill(~mask, float("-inf")), dim=-1)
    pointwise = torch.nn.functional.kl_div(ls.masked_fill(~mask, 0.0), lt.masked_fill(~mask, 0.0),
                                           log_target=True, reduction="none")
    kl = torch.where(mask, pointwise, torch.zeros_like(pointwise)).sum(-1)
    (kl * torch.tensor(dkl)).sum().backward()
    return kl.detach().numpy(), xs.grad.numpy()


@pytest.mark.parametrize("N,d,causal", [(1, 4, True), (5, 4, True), (17, 8, True), (33, 8, False),
                                        (40, 16, True)])
def test_against_torch_kl_div_autograd(N, d, causal):
    xt, xs = _rand_pair(N, d, seed=N * 7 + d)
    dkl = np.linspace(-1.0, 2.0, N)
    kl_ref, dx_ref = _torch_reference(xt, xs, dkl, causal)
    r = dense.fwd_unit(xt, xs, causal=causal)
    np.testing.assert_allclose(r["kl"], kl_ref, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dense.bwd_unit(xt, xs, dkl=dkl, causal=causal), dx_ref,
                               rtol=1e-10, atol=1e-13)


# --------------------------------------------------------- finite differences

@pytest.mark.parametrize("N,d,causal", [(3, 4, True), (8, 4, True), (17, 8, True), (8, 8, False)])
def test_finite_differences(N, d, causal):
    xt, xs = _rand_pair(N, d, seed=100 + N)
    dkl = np.linspace(0.5, 1.5, N) / N

    def loss(x):
        return float((dense.fwd_unit(xt, x, causal=causal)["kl"] * dkl).sum())

    h = 1e-6
    num = np.zeros_like(xs)
    for i in range(N):
        for k in range(d):
            xp, xm = xs.copy(), xs.copy()
            xp[i, k] += h
            xm[i, k] -= h
            num[i, k] = (loss(xp) - loss(xm)) / (2 * h)
    ana = dense.bwd_unit(xt, xs, dkl=dkl, causal=causal)
    assert np.max(np.abs(num - ana)) <= 1e-6 * np.max(np.abs(ana)) + 1e-10


# ------------------------------------------------------------------ invariants

@pytest.mark.parametrize("causal", [True, False])
def test_kl_nonnegative_and_w_identity(causal):
    xt, xs = _rand_pair(96, 16, seed=5, noise=1.5)
    r = dense.fwd_unit(xt, xs, causal=causal)
    assert np.all(r["kl"] >= -1e-15)
    np.testing.assert_allclose(r["kl"], r["w"] + r["lse_s"] - r["lse_t"], atol=1e-12)


def test_identical_inputs_give_exact_zero():
    xt, _ = _rand_pair(50, 8, seed=9)
    r = dense.fwd_unit(xt, xt.copy())
    assert np.all(r["kl"] == 0.0)
    assert np.all(dense.bwd_unit(xt, xt.copy()) == 0.0)


def test_orthogonal_change_of_basis():
    """X_s = X_t Q with Q orthogonal leaves X X^T, hence the relation, unchanged."""
    xt, _ = _rand_pair(40, 8, seed=11)
    q, _ = np.linalg.qr(np.random.default_rng(3).standard_normal((8, 8)))
    r = dense.fwd_unit(xt, xt @ q)
    assert np.max(np.abs(r["kl"])) < 1e-12
    assert np.max(np.abs(dense.bwd_unit(xt, xt @ q))) < 1e-12


def test_rope_relative_position_invariance():
    """Shifting all RoPE positions by a constant leaves Q/Q relations unchanged."""
    u = torch.randn(64, 16, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    pos = torch.arange(64, dtype=torch.float64)
    a = workload.rope_rotate(u, pos, 1e4).numpy()
    b = workload.rope_rotate(u, pos + 37.5, 1e4).numpy()
    assert np.max(np.abs(dense.fwd_unit(a, b)["kl"])) < 1e-12
    c = workload.rope_rotate(u, pos / 4.0, 1e4).numpy()     # PI: a real change
    assert np.max(dense.fwd_unit(a, c)["kl"]) > 1e-4


def test_row0_causal_is_zero_and_m_is_shared_max():
    xt, xs = _rand_pair(20, 8, seed=12)
    r = dense.fwd_unit(xt, xs)
    assert r["kl"][0] == 0.0
    s = 1 / math.sqrt(8)
    for i in (0, 7, 19):
        zt = s * xt[i] @ xt[: i + 1].T
        zs = s * xs[i] @ xs[: i + 1].T
        assert r["m"][i] == max(zt.max(), zs.max())


# --------------------------------------------- linear-memory exactness (tiled)

@pytest.mark.parametrize("N,tm,tn,causal", [(1, 4, 4, True), (2, 4, 4, True), (63, 16, 8, True),
                                            (64, 16, 16, True), (65, 16, 32, True),
                                            (130, 32, 16, False), (200, 64, 64, True)])
def test_two_phase_equals_dense(N, tm, tn, causal):
    xt, xs = _rand_pair(N, 8, seed=N + tm)
    dkl = np.cos(np.arange(N)) / N
    ref = dense.fwd_unit(xt, xs, causal=causal)
    tp = tiled.two_phase(xt, xs, dkl=dkl, causal=causal, tile_m=tm, tile_n=tn)
    for k in ("kl", "lse_t", "lse_s"):
        np.testing.assert_allclose(tp[k], ref[k], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(tp["dx"], dense.bwd_unit(xt, xs, dkl=dkl, causal=causal),
                               rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("N,tm,tn,causal", [(1, 4, 4, True), (65, 16, 32, True), (130, 32, 16, False),
                                            (257, 128, 128, True)])
def test_one_pass_shared_max_equals_dense(N, tm, tn, causal):
    xt, xs = _rand_pair(N, 8, seed=N + 1, noise=0.1)
    ref = dense.fwd_unit(xt, xs, causal=causal)
    op = tiled.one_pass_shared_max(xt, xs, causal=causal, tile_m=tm, tile_n=tn)
    for k in ("kl", "lse_t", "lse_s", "w", "m"):
        np.testing.assert_allclose(op[k], ref[k], rtol=1e-11, atol=1e-13)


def test_slabs_and_sampled_rows_equal_one_slab():
    xt, xs = _rand_pair(150, 8, seed=21)
    dkl = np.sin(np.arange(150)) / 150
    for causal in (True, False):
        one = dense.fwd_unit(xt, xs, causal=causal, slab=150)
        many = dense.fwd_unit(xt, xs, causal=causal, slab=7)
        for k in one:
            np.testing.assert_allclose(many[k], one[k], rtol=1e-13, atol=1e-15)
        full = dense.bwd_unit(xt, xs, dkl=dkl, causal=causal, slab=150)
        np.testing.assert_allclose(dense.bwd_unit(xt, xs, dkl=dkl, causal=causal, slab=11), full,
                                   rtol=1e-12, atol=1e-16)
        rows = [0, 1, 63, 64, 149]
        np.testing.assert_allclose(dense.bwd_rows(xt, xs, rows, dkl=dkl, causal=causal), full[rows],
                                   rtol=1e-12, atol=1e-16)
        sub = dense.fwd_rows(xt, xs, rows, causal=causal)
        for k in sub:
            np.testing.assert_allclose(sub[k], one[k][rows], rtol=1e-13, atol=1e-15)


def test_batched_wrappers():
    xt = torch.randn(2, 3, 20, 8, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    xs = xt + 0.3 * torch.randn(2, 3, 20, 8, generator=torch.Generator().manual_seed(2),
                                dtype=torch.float64)
    r = dense.fwd(xt, xs)
    dx = dense.bwd(xt, xs)
    for b, h in ((0, 0), (1, 2)):
        u = dense.fwd_unit(xt[b, h], xs[b, h])
        np.testing.assert_array_equal(r["kl"][b, h], u["kl"])
        np.testing.assert_array_equal(dx[b, h], dense.bwd_unit(xt[b, h], xs[b, h]))


# ------------------------------------------------- the pins have teeth

def _pins_pass(mod):
    """Re-run a compact version of the pins against module ``mod``."""
    ok = True
    xt, xs = _rand_pair(9, 4, seed=77)
    dkl = np.linspace(-1, 1, 9)
    for causal in (True, False):
        kl_ref, dx_ref = _torch_reference(xt, xs, dkl, causal)
        r = mod.fwd_unit(xt, xs, causal=causal)
        ok &= np.allclose(r["kl"], kl_ref, rtol=1e-9, atol=1e-12)
        ok &= np.allclose(mod.bwd_unit(xt, xs, dkl=dkl, causal=causal), dx_ref, rtol=1e-8, atol=1e-12)
    return bool(ok)


def test_planted_mistakes_are_caught(monkeypatch):
    import importlib
    assert _pins_pass(dense)
    src = open(dense.__file__).read()
    mutations = {
        "kl direction": ("diff_logp = np.where(ok, logp_t - logp_s, 0.0)",
                         "diff_logp = np.where(ok, logp_s - logp_t, 0.0)"),
        "diagonal excluded": ("return cols[None, :] <= rows[:, None]",
                              "return cols[None, :] < rows[:, None]"),
        "dropped G^T term": ("dx[:ncol] += s * (g.T @ xs[rows])", "pass"),
        "gradient sign": ("np.exp(logp_s) - np.exp(logp_t)", "np.exp(logp_t) - np.exp(logp_s)"),
        "teacher operand in G X": ("dx[rows] += s * (g @ xs[:ncol])", "dx[rows] += s * (g @ xt[:ncol])"),
        "missing scale": ("return scale * (x_rows @ x_all.T)", "return (x_rows @ x_all.T)"),
    }
    for name, (a, b) in mutations.items():
        assert a in src, name
        mod = type(dense)("oracle_mutant")
        exec(compile(src.replace(a, b), "oracle_mutant", "exec"), mod.__dict__)
        assert not _pins_pass(mod), f"planted mistake not caught: {name}"


# ------------------------------------------------------- right padding

def _padded_pair(B, H, N, d, seed):
    gen = torch.Generator().manual_seed(seed)
    xt = torch.randn(B, H, N, d, generator=gen, dtype=torch.float64)
    xs = xt + 0.4 * torch.randn(B, H, N, d, generator=gen, dtype=torch.float64)
    return xt, xs


def test_lengths_equal_to_n_change_nothing():
    xt, xs = _padded_pair(2, 2, 11, 4, 41)
    full = np.array([11, 11])
    for causal in (True, False):
        a, b = dense.fwd(xt, xs, causal), dense.fwd(xt, xs, causal, lengths=full)
        for k in a:
            np.testing.assert_array_equal(a[k], b[k])
        np.testing.assert_array_equal(dense.bwd(xt, xs, None, causal),
                                      dense.bwd(xt, xs, None, causal, lengths=full))


def test_padding_values_do_not_leak():
    xt, xs = _padded_pair(3, 1, 12, 4, 42)
    lengths = np.array([12, 7, 0])
    yt, ys = xt.clone(), xs.clone()
    for b, L in enumerate(lengths):
        yt[b, :, L:] = 1e3
        ys[b, :, L:] = -2e3
    for causal in (True, False):
        a, b = dense.fwd(xt, xs, causal, lengths=lengths), dense.fwd(yt, ys, causal, lengths=lengths)
        np.testing.assert_array_equal(a["kl"], b["kl"])
        assert np.all(a["kl"][1, :, 7:] == 0) and np.all(a["kl"][2] == 0)
        da = dense.bwd(xt, xs, None, causal, lengths=lengths)
        np.testing.assert_array_equal(da, dense.bwd(yt, ys, None, causal, lengths=lengths))
        assert np.all(da[1, :, 7:] == 0) and np.all(da[2] == 0)


@pytest.mark.parametrize("causal", [True, False])
def test_lengths_match_torch_key_padding_mask(causal):
    # independent formulation: full-length tensors, a key-padding mask on the
    # columns, padded rows dropped from the loss, per-sequence mean over valid rows
    B, H, N, d = 3, 2, 9, 4
    xt, xs = _padded_pair(B, H, N, d, 43)
    lengths = [9, 5, 1]
    xs_var = xs.clone().requires_grad_(True)
    s = 1.0 / np.sqrt(d)
    loss = 0.0
    kl_ref = torch.zeros(B, H, N, dtype=torch.float64)
    for b in range(B):
        L = lengths[b]
        col_ok = torch.arange(N)[None, :] < L
        ok = col_ok & (torch.tril(torch.ones(N, N, dtype=torch.bool)) if causal else True)
        zt = (xt[b] @ xt[b].transpose(-1, -2) * s).masked_fill(~ok, float("-inf"))
        zs = (xs_var[b] @ xs_var[b].transpose(-1, -2) * s).masked_fill(~ok, float("-inf"))
        lt, ls = torch.log_softmax(zt[:, :L], -1), torch.log_softmax(zs[:, :L], -1)
        kl = torch.nn.functional.kl_div(ls, lt, log_target=True, reduction="none").nan_to_num(0.0)
        kl = kl.sum(-1)                        # [H, L]
        kl_ref[b, :, :L] = kl.detach()
        loss = loss + kl.sum() / L
    loss.backward()
    r = dense.fwd(xt, xs, causal, lengths=np.array(lengths))
    np.testing.assert_allclose(r["kl"], kl_ref.numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(dense.bwd(xt, xs, None, causal, lengths=np.array(lengths)),
                               xs_var.grad.numpy(), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_row_partition_contributions_sum_to_the_gradient(causal):
    """dX_s is linear in G and G's rows are independent: the contributions of
    the rows of any partition add up to the whole gradient (the basis of
    splitting one unit's rows over devices), and one part alone is not it."""
    N, d = 23, 8
    xt, xs = _rand_pair(N, d, seed=91)
    dkl = np.linspace(-0.5, 1.0, N)
    full = dense.bwd_unit(xt, xs, dkl, causal)
    rng = np.random.default_rng(4)
    owner = rng.integers(0, 3, size=N)
    parts = [dense.bwd_contrib(xt, xs, np.flatnonzero(owner == k), dkl, causal) for k in range(3)]
    np.testing.assert_allclose(sum(parts), full, rtol=1e-12, atol=1e-15)
    assert np.abs(parts[0] - full).max() > 1e-3 * np.abs(full).max()
    # one part's rows: its row side and column side, written out for one row
    i = int(np.flatnonzero(owner == 1)[0])
    one = dense.bwd_contrib(xt, xs, [i], dkl, causal)
    s = 1.0 / math.sqrt(d)
    p_t, p_s = dense.relation_probs(xt, xs, causal)
    g_i = dkl[i] * (p_s[i] - p_t[i])
    want = np.outer(g_i, xs[i]) * s
    want[i] += s * (g_i @ xs)
    np.testing.assert_allclose(one, want, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("causal", [True, False])
def test_packed_sequences_equal_separate_batches(causal):
    """Packed sequences of equal length L are a batch [n_seq, H, L, d] laid on one
    token axis: the packed oracle must equal the batched one on the reshaped
    tensors (pins the packing's index arithmetic), and a sequence must not see
    its neighbours (changing one sequence leaves the others' rows unchanged)."""
    n_seq, H, L, d = 3, 2, 9, 4
    xt, xs = workload.gaussian_pair((n_seq, H, L, d), seed=61, noise=0.5, dtype=torch.float64)
    packed_t = xt.permute(1, 0, 2, 3).reshape(1, H, n_seq * L, d)
    packed_s = xs.permute(1, 0, 2, 3).reshape(1, H, n_seq * L, d)
    cu = [0, L, 2 * L, 3 * L]
    dkl = torch.linspace(-1.0, 1.0, n_seq * H * L, dtype=torch.float64).reshape(n_seq, H, L)
    dkl_packed = dkl.permute(1, 0, 2).reshape(1, H, n_seq * L)
    ref = dense.fwd(xt, xs, causal)
    got = dense.fwd_varlen(packed_t, packed_s, cu, causal)
    for k in ("kl", "lse_t", "lse_s", "w", "m"):
        np.testing.assert_allclose(got[k].reshape(H, n_seq, L).transpose(1, 0, 2), ref[k],
                                   rtol=1e-13, atol=1e-15)
    ref_dx = dense.bwd(xt, xs, dkl, causal)
    got_dx = dense.bwd_varlen(packed_t, packed_s, cu, dkl_packed, causal)
    np.testing.assert_allclose(got_dx.reshape(H, n_seq, L, d).transpose(1, 0, 2, 3), ref_dx,
                               rtol=1e-12, atol=1e-15)
    # default upstream gradient: 1/L per row of each sequence
    np.testing.assert_allclose(dense.bwd_varlen(packed_t, packed_s, cu, None, causal)
                               .reshape(H, n_seq, L, d).transpose(1, 0, 2, 3),
                               dense.bwd(xt, xs, None, causal), rtol=1e-12, atol=1e-15)
    # isolation: perturb sequence 1 only
    pt2 = packed_t.clone()
    pt2[:, :, L:2 * L] += 1.0
    other = dense.fwd_varlen(pt2, packed_s, cu, causal)["kl"]
    np.testing.assert_array_equal(other[:, :, :L], got["kl"][:, :, :L])
    np.testing.assert_array_equal(other[:, :, 2 * L:], got["kl"][:, :, 2 * L:])
    assert np.abs(other[:, :, L:2 * L] - got["kl"][:, :, L:2 * L]).max() > 1e-3


def test_packed_sequences_ragged_and_empty():
    """Unequal lengths, an empty sequence and tokens past the last sequence."""
    H, N, d = 1, 30, 4
    xt, xs = workload.gaussian_pair((1, H, N, d), seed=62, noise=0.5, dtype=torch.float64)
    cu = [0, 7, 7, 20, 26]
    got = dense.fwd_varlen(xt, xs, cu)
    for a, b in ((0, 7), (7, 20), (20, 26)):
        np.testing.assert_allclose(got["kl"][0, 0, a:b], dense.fwd_unit(xt[0, 0, a:b],
                                                                        xs[0, 0, a:b])["kl"],
                                   rtol=1e-13, atol=1e-15)
    assert np.all(got["kl"][0, 0, 26:] == 0)
    dx = dense.bwd_varlen(xt, xs, cu)
    assert np.all(dx[0, 0, 26:] == 0)
    with pytest.raises(ValueError):
        dense.fwd_varlen(xt, xs, [0, 5, 3])
