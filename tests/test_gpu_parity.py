"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs, element by element.

Small cases span several 128-row tiles with a ragged tail; the workload-sized
cases run the fused Q/K/V launch the bench times and compare sampled units
(and, for dX, sampled rows) that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from oracle import dense
from parity import DX_TOL_BF16, assert_dx, assert_kl, assert_stats, fp32_dx_tolerance, to_np

FP32 = "fp32"   # dx_tol marker: derive the fp32-path tolerance from the input

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rk.relkl_set_wait_timeout_ns(2_000_000_000)


def _device_ok():
    code, where = rk.relkl_get_device_error()
    assert code == 0, f"device wait ran out at site {where}"


def check_full(xt, xs, causal=True, dkl=None, dx_tol=DX_TOL_BF16, path=None, scale=0.0):
    """Run fwd+bwd on the GPU and compare every output with the oracle.
    ``scale`` is the desc's logit scale (0: 1/sqrt(d)); dx_tol=FP32 derives
    the fp32-path tolerance from the input's own arithmetic."""
    dev = "cuda"
    gt, gs = xt.to(dev), xs.to(dev)
    if path is not None:
        assert rk.relkl_path_for(gt, causal, scale) == path
    kl, st = rk.relkl_fwd(gt, gs, causal, scale)
    dx = rk.relkl_bwd(gt, gs, st, None if dkl is None else dkl.to(dev), causal, scale)
    torch.cuda.synchronize()
    _device_ok()
    oscale = scale if scale else None
    ref = dense.fwd(xt, xs, causal, oscale)
    assert_kl(to_np(kl), ref["kl"])
    assert_stats(to_np(st), ref)
    if dx_tol == FP32:
        dx_tol = fp32_dx_tolerance(xt, xs, dkl, causal, oscale)
    assert_dx(to_np(dx), dense.bwd(xt, xs, dkl, causal, oscale), dx_tol)


def q_inputs(B, H, N, d, dtype="bf16", seed=0, causal=True, pi=4.0):
    w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=seed, pi_factor=pi, causal=causal, B=B, H=H)
    return workload.generate(w)["q"]


# ----------------------------------------------------------- small shapes

def test_tc_single_tile():
    xt, xs = workload.gaussian_pair((1, 1, 128, 128), seed=1, noise=0.3, dtype=torch.bfloat16)
    check_full(xt, xs, path=1)


@pytest.mark.parametrize("N,d,causal,B,H", [
    (1, 128, True, 1, 1), (2, 64, True, 1, 1), (127, 128, True, 1, 2), (129, 128, True, 2, 1),
    (300, 64, True, 1, 2), (300, 128, False, 1, 2), (513, 64, False, 1, 1), (1000, 128, True, 1, 1),
])
def test_tc_shapes_rope_pi(N, d, causal, B, H):
    xt, xs = q_inputs(B, H, N, d, seed=N + d, causal=causal)
    check_full(xt, xs, causal=causal, path=1)


# N > 4096 takes the backward that pairs adjacent 128-row blocks: odd block
# counts (a last pair with one block), ragged tails, both masks.
@pytest.mark.parametrize("N,causal,B,H", [
    (4200, True, 1, 2), (4352, False, 1, 1), (4097, True, 2, 1), (4480, True, 1, 1),
])
def test_tc_paired_row_blocks(N, causal, B, H):
    xt, xs = q_inputs(B, H, N, 128, seed=N, causal=causal)
    check_full(xt, xs, causal=causal, path=1)


def test_tc_paired_row_blocks_upstream_gradient_and_zero():
    xt, xs = q_inputs(1, 1, 4300, 128, seed=31)
    dkl = torch.randn(1, 1, 4300, generator=torch.Generator().manual_seed(3)) / 4300
    check_full(xt, xs, dkl=dkl)
    g = xt.cuda()
    kl, st = rk.relkl_fwd(g, g.clone())
    dx = rk.relkl_bwd(g, g.clone(), st)
    torch.cuda.synchronize()
    assert torch.all(kl == 0) and torch.all(dx == 0)


def test_tc_value_relation_small_kl():
    # V-like: student = teacher + small noise, KL ~ 1e-3 per row
    xt, xs = workload.gaussian_pair((1, 2, 640, 128), seed=5, noise=0.05, dtype=torch.bfloat16)
    check_full(xt, xs)


# ------------------------------------------------- explicit logit scale
# The desc's scale replaces 1/sqrt(d) everywhere: in the logits, the LSEs and
# the factor s of dX = s (G + G^T) X_s.  Every kernel family, both masks.
@pytest.mark.parametrize("N,d,scale,causal,path", [
    (700, 128, 0.05, True, 1), (700, 128, 0.3, False, 1),      # one-block backward
    (4200, 128, 0.05, False, 1), (4200, 128, 0.3, True, 1),    # paired-block backward
    (513, 64, 0.05, True, 1), (513, 64, 0.3, False, 1),        # d = 64
    (150, 64, 0.05, True, 2), (150, 64, 0.3, False, 2),        # CUDA-core fp32
])
def test_explicit_scale(N, d, scale, causal, path):
    dtype = "bf16" if path == 1 else "fp32"
    xt, xs = q_inputs(1, 2 if N < 1000 else 1, N, d, dtype=dtype, seed=N + int(1000 * scale),
                      causal=causal)
    if scale * d > 20:
        # keep the rows spread: at scale 0.3 and d = 128 unit-variance rows give a
        # diagonal logit of ~38 against off-diagonal ones of ~3, every row is one-hot
        # to 1e-11 and its KL (~1e-7) lies below what float32 logits of that size
        # resolve, which would leave nothing but rounding noise to compare
        t = xt.float() * 0.4
        xt, xs = t.to(xt.dtype), (xs.float() * 0.4).to(xs.dtype)
    check_full(xt, xs, causal=causal, path=path, scale=scale,
               dx_tol=DX_TOL_BF16 if path == 1 else FP32)


# ------------------------------------------------- large logits
# Rows clustered around a few shared directions: logits reach ~70-100 across
# whole clusters (not only on the diagonal), so the shared running maximum
# moves by tens between tiles, most exponentials underflow and the KL stays
# of order 0.3.  Both masks, both backwards at d = 128, d = 64 and fp32.
@pytest.mark.parametrize("N,d,causal,dtype", [
    (4200, 128, True, "bf16"), (4200, 128, False, "bf16"), (1000, 128, True, "bf16"),
    (700, 64, False, "bf16"), (4300, 64, True, "bf16"), (200, 64, True, "fp32"),
])
def test_large_logits(N, d, causal, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    xt, xs = workload.clustered_pair((1, 1, N, d), seed=N + d, amplitude=2.5 if d == 128 else 3.0,
                                     dtype=tdt)
    ref_m = dense.fwd_rows(xt[0, 0], xs[0, 0], range(0, N, 97), causal)["m"]
    assert ref_m.max() > 60.0     # the case really has large logits
    check_full(xt, xs, causal=causal, path=1 if dtype == "bf16" else 2,
               dx_tol=DX_TOL_BF16 if dtype == "bf16" else FP32)


def test_simt_fp32_tiny_config():
    w = workload.CONFIGS["tiny_fp32_n256"]
    xt, xs = workload.generate(w)["q"]
    check_full(xt, xs, dx_tol=FP32, path=2)


def test_simt_bf16_unsupported_head_dim():
    xt, xs = q_inputs(1, 2, 200, 96, seed=3)
    check_full(xt, xs, dx_tol=FP32, path=2)


@pytest.mark.parametrize("N,d", [(700, 128), (4480, 128), (513, 64), (4300, 64)])
def test_full_mask_upstream_gradient(N, d):
    """Full masks run the symmetric schedule: each off-diagonal tile also forms
    the transposed entry's gradient from the column row's statistics and
    upstream gradient, so a row-dependent dkl must reach both orientations."""
    xt, xs = q_inputs(1, 1, N, d, seed=N + 3 * d, causal=False)
    dkl = torch.randn(1, 1, N, generator=torch.Generator().manual_seed(N)) / N
    check_full(xt, xs, causal=False, dkl=dkl, path=1)


def test_upstream_gradient():
    xt, xs = q_inputs(2, 2, 260, 128, seed=11)
    dkl = torch.randn(2, 2, 260, generator=torch.Generator().manual_seed(2)) / 260
    check_full(xt, xs, dkl=dkl)
    xt32, xs32 = q_inputs(1, 1, 70, 64, dtype="fp32", seed=12)
    check_full(xt32, xs32, dkl=torch.linspace(-1, 1, 70).reshape(1, 1, 70), dx_tol=FP32)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_identical_inputs_give_exact_zero(dtype):
    xt, _ = q_inputs(1, 2, 333, 128 if dtype == "bf16" else 64, dtype=dtype, seed=4)
    g = xt.cuda()
    kl, st = rk.relkl_fwd(g, g.clone())
    dx = rk.relkl_bwd(g, g.clone(), st)
    torch.cuda.synchronize()
    assert torch.all(kl == 0) and torch.all(dx == 0)


def test_strided_inputs():
    # [B, N, H, d] storage (a fused projection output) viewed as [B, H, N, d]
    gen = torch.Generator().manual_seed(9)
    base_t = torch.randn(1, 384, 3, 128, generator=gen).to(torch.bfloat16)
    base_s = (base_t.float() + 0.2 * torch.randn(1, 384, 3, 128, generator=gen)).to(torch.bfloat16)
    xt, xs = base_t.permute(0, 2, 1, 3), base_s.permute(0, 2, 1, 3)
    assert not xt.is_contiguous()
    kl, st = rk.relkl_fwd(base_t.cuda().permute(0, 2, 1, 3), base_s.cuda().permute(0, 2, 1, 3))
    dx = rk.relkl_bwd(base_t.cuda().permute(0, 2, 1, 3), base_s.cuda().permute(0, 2, 1, 3), st)
    torch.cuda.synchronize()
    ref = dense.fwd(xt, xs)
    assert_kl(to_np(kl), ref["kl"])
    assert_dx(to_np(dx), dense.bwd(xt, xs), DX_TOL_BF16)


def test_fused_qkv_gqa_small():
    g = workload.Workload("gqa_small", B=2, H=4, H_kv=2, N=300, d=128, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=5e5, pi_factor=4.0, v_noise=0.05,
                          seed=21)
    x = workload.generate(g)
    pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in "qkv"]
    outs = rk.relkl_fwd_qkv(pairs)
    dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs])
    torch.cuda.synchronize()
    _device_ok()
    for r, (kl, st), dx in zip("qkv", outs, dxs):
        ref = dense.fwd(*x[r])
        assert_kl(to_np(kl), ref["kl"], what=f"kl[{r}]")
        assert_stats(to_np(st), ref)
        assert_dx(to_np(dx), dense.bwd(*x[r]), DX_TOL_BF16)


def test_fused_qkv_gqa_paired_blocks():
    g = workload.Workload("gqa_paired", B=1, H=2, H_kv=1, N=4200, d=128, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=5e5, pi_factor=4.0, v_noise=0.05,
                          seed=23)
    x = workload.generate(g)
    pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in "qkv"]
    outs = rk.relkl_fwd_qkv(pairs)
    dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs])
    torch.cuda.synchronize()
    _device_ok()
    for r, (kl, st), dx in zip("qkv", outs, dxs):
        ref = dense.fwd(*x[r])
        assert_kl(to_np(kl), ref["kl"], what=f"kl[{r}]")
        assert_dx(to_np(dx), dense.bwd(*x[r]), DX_TOL_BF16)


def test_forward_is_deterministic():
    xt, xs = q_inputs(1, 4, 700, 128, seed=13)
    gt, gs = xt.cuda(), xs.cuda()
    a = rk.relkl_fwd(gt, gs)
    b = rk.relkl_fwd(gt, gs)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_binding_rejects_wrong_outputs():
    xt, xs = q_inputs(1, 2, 200, 128, seed=19)
    gt, gs = xt.cuda(), xs.cuda()
    good_kl = torch.empty(1, 2, 200, device="cuda")
    good_st = torch.empty(1, 2, 200, 4, device="cuda")
    with pytest.raises(ValueError):
        rk.relkl_fwd(gt, gs, kl=torch.empty(1, 2, 199, device="cuda"), stats=good_st)
    with pytest.raises(ValueError):
        rk.relkl_fwd(gt, gs, kl=good_kl, stats=torch.empty(1, 2, 200, 3, device="cuda"))
    with pytest.raises(ValueError):
        rk.relkl_fwd(gt, gs, kl=good_kl)                       # stats missing
    with pytest.raises(ValueError):
        rk.relkl_fwd_noalloc(gt, gs, kl=good_kl.double(), stats=good_st)
    with pytest.raises(ValueError):
        rk.relkl_fwd_noalloc(gt, gs, kl=good_kl, stats=good_st.transpose(0, 1))
    kl, st = rk.relkl_fwd(gt, gs, kl=good_kl, stats=good_st)
    with pytest.raises(ValueError):
        rk.relkl_bwd(gt, gs, st, dx_s=torch.empty(1, 2, 200, 128, device="cuda").half())
    torch.cuda.synchronize()


def test_autograd_wrapper():
    xt, xs = q_inputs(1, 2, 200, 128, seed=17)
    gt = xt.cuda()
    gs = xs.cuda().requires_grad_(True)
    kl = rk.relation_kl(gt, gs)
    kl.mean().backward()
    torch.cuda.synchronize()
    # mean over B*H*N rows: dkl = 1/(B*H*N) per row
    dkl = torch.full((1, 2, 200), 1.0 / (2 * 200))
    assert_dx(to_np(gs.grad), dense.bwd(xt, xs, dkl), DX_TOL_BF16)


# ------------------------------------------------------ workload sizes

SAMPLE_ROWS = (0, 1, 127, 128, 129)


def _dx_rows(N):
    """Rows whose dX is compared at workload size: first, second, middle and last
    rows of the 128-row blocks that the first, a middle and the last work item
    of the paired-block backward hold (blocks 2k and 2k+1 of its two pair
    sequences k = npb-1-m and k = m), plus the unit's last two rows."""
    nblk = (N + 127) // 128
    npb = (nblk + 1) // 2
    items = (npb + 1) // 2
    blocks = set()
    for m in sorted({0, items // 2, items - 1}):
        for k in (npb - 1 - m, m):
            blocks.update(b for b in (2 * k, 2 * k + 1) if 0 <= b < nblk)
    rows = set()
    for b in blocks:
        r0 = b * 128
        rows.update(r for r in (r0, r0 + 1, r0 + 63, r0 + 64, r0 + 126, r0 + 127) if r < N)
    rows.update(r for r in (N - 2, N - 1) if r >= 0)
    return sorted(rows)


def test_dx_rows_cover_pair_items():
    rows = _dx_rows(32768)
    assert len(rows) >= 64
    blocks = {r // 128 for r in rows}
    # first item: pairs 127 and 0; middle (m = 32): 95 and 32; last (m = 63): 64 and 63
    assert blocks == {254, 255, 0, 1, 190, 191, 64, 65, 128, 129, 126, 127}


def _sampled(w: workload.Workload, units, dx_units):
    """Fused Q/K/V launch of the whole workload; oracle on sampled units."""
    x = workload.generate(w)
    pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in w.relations]
    outs = rk.relkl_fwd_qkv(pairs, w.causal)
    dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs], None, w.causal)
    torch.cuda.synchronize()
    _device_ok()
    rel_idx = {r: i for i, r in enumerate(w.relations)}
    N = w.N
    rows = sorted(set([r for r in SAMPLE_ROWS if r < N] + [N // 2, N - 129, N - 2, N - 1]))
    for (rel, b, h) in units:
        xt, xs = x[rel][0][b, h], x[rel][1][b, h]
        kl, st = outs[rel_idx[rel]]
        full = (rel, b, h) in dx_units
        slab = 2048 if N <= 32768 else 512
        ref = (dense.fwd_unit(xt, xs, w.causal, slab=slab) if full
               else dense.fwd_rows(xt, xs, rows, w.causal))
        sel = slice(None) if full else rows
        assert_kl(to_np(kl[b, h])[sel], ref["kl"], what=f"kl[{rel},{b},{h}]")
        assert_stats(to_np(st[b, h])[sel], ref)
        if full:
            dx_rows = _dx_rows(N)
            ref_dx = dense.bwd_rows(xt, xs, dx_rows, causal=w.causal, lse=ref)
            got = to_np(dxs[rel_idx[rel]][b, h])[dx_rows]
            assert_dx(got, ref_dx, DX_TOL_BF16)


def test_config_llama2_h32_n4k():
    w = workload.CONFIGS["llama2_h32_n4k"]
    units = [("q", 0, 0), ("q", 0, 31), ("k", 0, 7), ("v", 0, 0), ("v", 0, 31)]
    _sampled(w, units, dx_units=set(units))


def test_config_gqa_llama3_n16k():
    w = workload.CONFIGS["gqa_llama3_n16k"]
    units = [("q", 1, 31), ("k", 0, 3), ("v", 1, 7)]
    _sampled(w, units, dx_units=set(units))


def test_config_ext_h32_n32k():
    w = workload.CONFIGS["ext_h32_n32k"]
    units = [("q", 0, 0), ("k", 0, 17), ("v", 0, 31)]
    _sampled(w, units, dx_units=set(units))


def test_config_d64_h32_n32k():
    # head dimension 64 at the 32K shape: kl on every row and dX on the
    # sampled rows of one unit of each relation
    w = workload.CONFIGS["d64_h32_n32k"]
    units = [("q", 0, 0), ("k", 0, 17), ("v", 0, 31)]
    _sampled(w, units, dx_units=set(units))


def test_config_full_h32_n16k():
    # full mask at 16K (the symmetric paired-block backward)
    w = workload.CONFIGS["full_h32_n16k"]
    units = [("q", 0, 5), ("k", 0, 17), ("v", 0, 31)]
    _sampled(w, units, dx_units=set(units))


@pytest.mark.parametrize("N", [2048, 4096])
def test_config_sweep_short_sequences(N):
    # the sweep's short-sequence points (B*N = 65536): enough units that the
    # launch picks the paired-block backward at 16 and 32 row blocks
    import bench
    w = workload.sweep_config(N)
    assert bench.bwd_kernel_name(w) == "relkl_bwd_pair_kernel"
    units = [("q", 0, 0), ("k", w.B // 2, 17), ("v", w.B - 1, 31)]
    _sampled(w, units, dx_units=set(units))


def test_config_sweep_n64k():
    # the largest point of the sequence-length sweep: B=1, H=32, N=65536
    w = workload.sweep_config(65536)
    units = [("q", 0, 0), ("k", 0, 9), ("v", 0, 31)]
    _sampled(w, units, dx_units=set(units))


# ------------------------------------------------------ right padding

def _padded_inputs(B, H, N, d, dtype, seed, lengths):
    w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=seed, pi_factor=4.0, B=B, H=H)
    xt, xs = workload.generate(w)["q"]
    xt, xs = xt.clone(), xs.clone()
    for b, L in enumerate(lengths):          # garbage in the padding must not leak
        xt[b, :, L:] = 30.0
        xs[b, :, L:] = -45.0
    return xt, xs


@pytest.mark.parametrize("B,H,N,d,dtype,causal,lengths,path", [
    (3, 2, 300, 128, "bf16", True, [300, 263, 0], 1),
    (3, 2, 300, 128, "bf16", False, [300, 177, 1], 1),
    (2, 1, 513, 64, "bf16", False, [513, 200], 1),
    (2, 1, 4200, 128, "bf16", True, [4200, 3001], 1),      # pair backward
    (2, 1, 4200, 128, "bf16", False, [2100, 4200], 1),
    (2, 2, 150, 64, "fp32", True, [150, 61], 2),           # CUDA-core path
    (2, 2, 150, 64, "fp32", False, [97, 150], 2),
])
def test_padded_lengths(B, H, N, d, dtype, causal, lengths, path):
    xt, xs = _padded_inputs(B, H, N, d, dtype, N + d + len(lengths), lengths)
    lens = torch.tensor(lengths, dtype=torch.int32)
    gt, gs, gl = xt.cuda(), xs.cuda(), lens.cuda()
    assert rk.relkl_path_for(gt, causal) == path
    kl, st = rk.relkl_fwd(gt, gs, causal, lengths=gl)
    dx = rk.relkl_bwd(gt, gs, st, None, causal, lengths=gl)
    torch.cuda.synchronize()
    _device_ok()
    ref = dense.fwd(xt, xs, causal, lengths=lengths)
    assert_kl(to_np(kl), ref["kl"])
    for b, L in enumerate(lengths):
        assert np.all(to_np(kl[b, :, L:]) == 0) and np.all(to_np(st[b, :, L:]) == 0)
        if L:
            assert_stats(to_np(st[b, :, :L]), {k: v[b, :, :L] for k, v in ref.items()})
    tol = DX_TOL_BF16 if path == 1 else fp32_dx_tolerance(xt, xs, None, causal, lengths=lengths)
    ref_dx = dense.bwd(xt, xs, None, causal, lengths=lengths)
    assert_dx(to_np(dx), ref_dx, tol)
    for b, L in enumerate(lengths):
        assert np.all(to_np(dx[b, :, L:]) == 0)


def test_fused_qkv_gqa_padded():
    g = workload.Workload("gqa_pad", B=2, H=4, H_kv=2, N=320, d=128, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=5e5, pi_factor=4.0, v_noise=0.05,
                          seed=29)
    x = workload.generate(g)
    lengths = [320, 190]
    lens = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in "qkv"]
    outs = rk.relkl_fwd_qkv(pairs, lengths=lens)
    dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs], lengths=lens)
    torch.cuda.synchronize()
    _device_ok()
    for r, (kl, _), dx in zip("qkv", outs, dxs):
        ref = dense.fwd(*x[r], lengths=lengths)
        assert_kl(to_np(kl), ref["kl"], what=f"kl[{r}]")
        assert_dx(to_np(dx), dense.bwd(*x[r], lengths=lengths), DX_TOL_BF16)
