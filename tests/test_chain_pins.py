"""Pins of the float64 chain-rule oracle (RoPE backward, weight gradient).

Each check rests on something other than the oracle's own formulas: the
adjoint and orthogonality of the rotation against the workload's forward RoPE,
a one-hot closed form of the weight gradient, central finite differences of
the whole loss, and fp64 torch autograd through the whole chain.  A last test
plants mistakes in a copy of the oracle and checks that the pins catch them.
"""
import numpy as np
import pytest
import torch

import workload
from oracle import chain, dense


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------ RoPE backward

@pytest.mark.parametrize("d,base", [(4, 1e4), (8, 500.0), (64, 1e4)])
def test_rope_backward_is_the_adjoint_of_the_rotation(d, base):
    N = 11
    pos = np.arange(N) / 3.0
    x, y = _rand((2, N, d), 1), _rand((2, N, d), 2)
    fx = workload.rope_rotate(torch.from_numpy(x), torch.from_numpy(pos), base).numpy()
    lhs = np.sum(fx * y)
    rhs = np.sum(x * chain.rope_backward(y, pos, base))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_rope_backward_inverts_the_rotation_and_is_identity_at_zero():
    d, N, base = 16, 9, 1e4
    pos = np.arange(N, dtype=np.float64) * 7.5
    x = _rand((3, N, d), 3)
    fx = workload.rope_rotate(torch.from_numpy(x), torch.from_numpy(pos), base).numpy()
    np.testing.assert_allclose(chain.rope_backward(fx, pos, base), x, rtol=0, atol=1e-12)
    z = chain.rope_backward(x, np.zeros(N), base)
    np.testing.assert_array_equal(z, x)


# ------------------------------------------------------------- weight grad

def test_weight_grad_one_hot_rows_select_token_gradients():
    # h[b, n] = e_{k(b,n)}: row k of dW is the sum of the gradients of the tokens mapped to k
    B, N, D, cols = 2, 5, 6, 7
    k = np.array([[0, 3, 3, 5, 1], [2, 0, 4, 4, 4]])
    h = np.zeros((B, N, D))
    for b in range(B):
        for n in range(N):
            h[b, n, k[b, n]] = 1.0
    g = _rand((B, N, cols), 4)
    dw = chain.weight_grad(h, g)
    for r in range(D):
        np.testing.assert_allclose(dw[r], g[k == r].sum(axis=0), rtol=0, atol=1e-14)


def test_heads_to_tokens_layout():
    x = np.arange(2 * 3 * 4 * 5, dtype=np.float64).reshape(2, 3, 4, 5)
    t = chain.heads_to_tokens(x)
    assert t.shape == (2, 4, 15)
    assert t[1, 2, 2 * 5 + 3] == x[1, 2, 2, 3]


# ------------------------------------------------------- the whole chain

def _tiny():
    return workload.ChainWorkload("pin", B=1, N=10, D=8, H=2, H_kv=1, d=4, rope_base=100.0,
                                  pi_factor=4.0, h_noise=0.3, seed=5)


def _draw_f64(cw, seed):
    rng = np.random.default_rng(seed)
    ht = rng.standard_normal((cw.B, cw.N, cw.D))
    hs = ht + cw.h_noise * rng.standard_normal((cw.B, cw.N, cw.D))
    w = {r: rng.standard_normal((cw.D, cw.heads(r) * cw.d)) / np.sqrt(cw.D) for r in "qkv"}
    return ht, hs, w


def _project(h, w, cw, rel, pos):
    x = (h @ w).reshape(cw.B, cw.N, cw.heads(rel), cw.d).transpose(0, 2, 1, 3)
    if rel != "v":
        x = workload.rope_rotate(torch.from_numpy(np.ascontiguousarray(x)), torch.from_numpy(pos),
                                 cw.rope_base).numpy()
    return x


def _loss(ht, hs, wt, ws, cw, causal=True):
    """Sum over relations and units of (1/N) sum_i kl_i, teacher weights frozen."""
    pos_t = np.arange(cw.N, dtype=np.float64)
    pos_s = pos_t / cw.pi_factor
    total = 0.0
    for rel in "qkv":
        r = dense.fwd(_project(ht, wt[rel], cw, rel, pos_t), _project(hs, ws[rel], cw, rel, pos_s),
                      causal)
        total += float(r["kl"].sum()) / cw.N
    return total


def _oracle_grads(ht, hs, wt, ws, cw, causal=True, mod=chain):
    pos_t = np.arange(cw.N, dtype=np.float64)
    pos_s = pos_t / cw.pi_factor
    x = {rel: (_project(ht, wt[rel], cw, rel, pos_t), _project(hs, ws[rel], cw, rel, pos_s))
         for rel in "qkv"}
    return mod.projection_grads(x, hs, pos_s, cw.rope_base, causal=causal)


@pytest.mark.parametrize("causal", [True, False])
def test_chain_matches_central_finite_differences(causal):
    cw = _tiny()
    ht, hs, wt = _draw_f64(cw, 6)
    ws = {r: wt[r] + 0.05 * _rand(wt[r].shape, 7) for r in "qkv"}
    g = _oracle_grads(ht, hs, wt, ws, cw, causal)
    rng = np.random.default_rng(8)
    h = 1e-6
    for rel in "qkv":
        for _ in range(4):
            i, j = rng.integers(ws[rel].shape[0]), rng.integers(ws[rel].shape[1])
            wp = {r: v.copy() for r, v in ws.items()}
            wm = {r: v.copy() for r, v in ws.items()}
            wp[rel][i, j] += h
            wm[rel][i, j] -= h
            fd = (_loss(ht, hs, wt, wp, cw, causal) - _loss(ht, hs, wt, wm, cw, causal)) / (2 * h)
            assert abs(fd - g[rel][i, j]) <= 1e-6 * max(1e-3, abs(fd)), (rel, i, j, fd, g[rel][i, j])


def test_chain_matches_torch_autograd():
    cw = workload.ChainWorkload("pin2", B=2, N=14, D=12, H=4, H_kv=2, d=6, rope_base=50.0,
                                pi_factor=8.0, h_noise=0.2, seed=9)
    ht, hs, wt = _draw_f64(cw, 10)
    ws = {r: wt[r] + 0.1 * _rand(wt[r].shape, 11) for r in "qkv"}
    pos_t = torch.arange(cw.N, dtype=torch.float64)
    pos_s = pos_t / cw.pi_factor
    wst = {r: torch.tensor(ws[r], requires_grad=True) for r in "qkv"}
    mask = torch.tril(torch.ones(cw.N, cw.N, dtype=torch.bool))
    loss = 0.0
    for rel in "qkv":
        hd = cw.heads(rel)

        def proj(h, w, pos):
            x = (torch.as_tensor(h) @ w).reshape(cw.B, cw.N, hd, cw.d).permute(0, 2, 1, 3)
            return workload.rope_rotate(x, pos, cw.rope_base) if rel != "v" else x

        xt = proj(ht, torch.tensor(wt[rel]), pos_t)
        xs = proj(hs, wst[rel], pos_s)
        zt = (xt @ xt.transpose(-1, -2) / cw.d ** 0.5).masked_fill(~mask, float("-inf"))
        zs = (xs @ xs.transpose(-1, -2) / cw.d ** 0.5).masked_fill(~mask, float("-inf"))
        lt, ls = torch.log_softmax(zt, -1), torch.log_softmax(zs, -1)
        kl = torch.nn.functional.kl_div(ls, lt, log_target=True, reduction="none")
        loss = loss + kl.nan_to_num(0.0).sum() / cw.N
    loss.backward()
    g = _oracle_grads(ht, hs, wt, ws, cw)
    for rel in "qkv":
        np.testing.assert_allclose(g[rel], wst[rel].grad.numpy(), rtol=1e-9, atol=1e-12)


# ------------------------------------------------- the pins have teeth

def _pins_pass(mod):
    cw = _tiny()
    ht, hs, wt = _draw_f64(cw, 12)
    ws = {r: wt[r] + 0.05 * _rand(wt[r].shape, 13) for r in "qkv"}
    try:
        g = _oracle_grads(ht, hs, wt, ws, cw, mod=mod)
    except Exception:
        return False
    h = 1e-6
    ok = True
    for rel, (i, j) in (("q", (1, 2)), ("k", (3, 1)), ("v", (5, 3))):
        wp = {r: v.copy() for r, v in ws.items()}
        wm = {r: v.copy() for r, v in ws.items()}
        wp[rel][i, j] += h
        wm[rel][i, j] -= h
        fd = (_loss(ht, hs, wt, wp, cw) - _loss(ht, hs, wt, wm, cw)) / (2 * h)
        ok &= abs(fd - g[rel][i, j]) <= 1e-6 * max(1e-3, abs(fd))
    return bool(ok)


def test_planted_mistakes_are_caught():
    assert _pins_pass(chain)
    src = open(chain.__file__).read()
    mutations = {
        "forward rotation instead of its transpose": (
            "(ga * c + gb * s, gb * c - ga * s)", "(ga * c - gb * s, gb * c + ga * s)"),
        "halves swapped": ("ga, gb = g[..., : d // 2], g[..., d // 2:]",
                           "gb, ga = g[..., : d // 2], g[..., d // 2:]"),
        "rotation applied to V": ('        if rel != "v":\n            dx = rope_backward',
                                  '        if True:\n            dx = rope_backward'),
        "hidden states scaled": ("out[rel] = weight_grad(h_s, heads_to_tokens(dx))",
                                 "out[rel] = weight_grad(h_s * 1.1, heads_to_tokens(dx))"),
        "teacher positions (PI factor 4 undone)": ("dx = rope_backward(dx, pos_s, rope_base)",
                                                   "dx = rope_backward(dx, pos_s * 4.0, rope_base)"),
        "head-major instead of token-major rows": (
            "return a.transpose(0, 2, 1, 3).reshape(B, N, Hh * d)", "return a.reshape(B, N, Hh * d)"),
        "frequency exponent": ("* 2.0 / d)", "* 1.0 / d)"),
    }
    for name, (a, b) in mutations.items():
        assert a in src, name
        mod = type(chain)("oracle.chain_mutant")
        mod.__dict__["__package__"] = "oracle"
        exec(compile(src.replace(a, b), "oracle_chain_mutant", "exec"), mod.__dict__)
        assert not _pins_pass(mod), f"planted mistake not caught: {name}"
