"""GPU parity of the chain rule to the student's projection weights (RoPE
backward with the head/token transpose, and the weight-gradient GEMM) against
the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from oracle import chain
from parity import DX_TOL_BF16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _expected_pre(dx, base, scale, offset, apply):
    N = dx.shape[2]
    pos = offset + np.arange(N, dtype=np.float64) * scale
    g = chain.rope_backward(dx, pos, base) if apply else dx.astype(np.float64)
    return g.transpose(0, 2, 1, 3)   # [B, N, H, d]


@pytest.mark.parametrize("B,H,N,d,base,scale,offset", [
    (2, 3, 300, 64, 1e4, 0.25, 0.0), (1, 4, 257, 128, 5e5, 0.125, 3.0),
    (1, 2, 70000, 128, 1e4, 1.0, 0.0),      # angles up to ~7e4 rad
    (1, 5, 33, 96, 500.0, 1.0, 11.5),
])
def test_rope_bwd_fp32_and_bf16(B, H, N, d, base, scale, offset):
    gen = torch.Generator().manual_seed(N + d)
    dx = torch.randn(B, H, N, d, generator=gen)
    ref = _expected_pre(dx.numpy(), base, scale, offset, True)
    big = float(np.abs(dx.numpy()).max())
    out32 = rk.relkl_rope_bwd(dx.cuda(), base, scale, offset, True, torch.float32)
    out16 = rk.relkl_rope_bwd(dx.cuda(), base, scale, offset, True, torch.bfloat16)
    torch.cuda.synchronize()
    assert out32.shape == (B, N, H, d)
    err32 = np.abs(to_np(out32) - ref)
    assert err32.max() <= 1e-6 * big, err32.max()
    err16 = np.abs(to_np(out16) - ref)
    assert np.all(err16 <= 2.0 ** -8 * np.abs(ref) + 1e-6 * big), err16.max()


def test_rope_bwd_without_rotation_is_an_exact_transpose_and_cast():
    gen = torch.Generator().manual_seed(3)
    dx = torch.randn(2, 3, 190, 128, generator=gen)
    out32 = rk.relkl_rope_bwd(dx.cuda(), 1e4, 0.5, 0.0, False, torch.float32)
    out16 = rk.relkl_rope_bwd(dx.cuda(), 1e4, 0.5, 0.0, False, torch.bfloat16)
    torch.cuda.synchronize()
    want = dx.permute(0, 2, 1, 3).contiguous()
    assert torch.equal(out32.cpu(), want)
    assert torch.equal(out16.cpu(), want.to(torch.bfloat16))   # round to nearest even


# (1000, 1280, 3968) and (1000, 1280, 3904): the last 256-column block reaches past the
# matrix edge by half (3968: its last four 32-column boxes are not stored) or more (3904),
# and the 1000 token rows end inside a 64-row K chunk
@pytest.mark.parametrize("rows,D,cols", [(600, 192, 256), (32768, 256, 128), (40, 8, 8),
                                         (1000, 1280, 3968), (1000, 1280, 3904)])
def test_weight_grad_matches_float64(rows, D, cols):
    gen = torch.Generator().manual_seed(rows + D)
    h = torch.randn(rows, D, generator=gen).to(torch.bfloat16)
    dx = torch.randn(rows, cols, generator=gen).to(torch.bfloat16)
    dw = rk.relkl_weight_grad(h.cuda(), dx.cuda())
    torch.cuda.synchronize()
    ref = h.double().numpy().T @ dx.double().numpy()
    rel = np.abs(to_np(dw) - ref).max() / np.abs(ref).max()
    assert rel <= 1e-4, rel


def test_student_weight_grads_small_chain():
    cw = workload.CHAIN_CONFIGS["chain_small"]
    c = workload.generate_chain(cw)
    pairs = {r: (c["x"][r][0].cuda(), c["x"][r][1].cuda()) for r in "qkv"}
    got = rk.student_weight_grads(pairs, c["h_s"].cuda(), cw.rope_base, 1.0 / cw.pi_factor,
                                  cw.causal)
    torch.cuda.synchronize()
    ref = chain.projection_grads(c["x"], c["h_s"], c["pos_s"].numpy(), cw.rope_base,
                                 causal=cw.causal)
    for r in "qkv":
        g, w = to_np(got[r]), ref[r]
        assert g.shape == w.shape
        rel = np.abs(g - w).max() / np.abs(w).max()
        assert rel <= DX_TOL_BF16, (r, rel)


def test_chain_full_layer_shape_sampled():
    # LLaMA2-7B layer (D = 4096, 32 heads of 128) at N = 32768: the RoPE backward on
    # sampled tokens and the GEMM on sampled weight columns, each against float64
    # arithmetic on the GPU's own input to that step.
    cw = workload.CHAIN_CONFIGS["chain_llama2_n32k"]
    c = workload.generate_chain(cw)
    rel = "k"
    xt, xs = c["x"][rel][0].cuda(), c["x"][rel][1].cuda()
    (kl, st), = rk.relkl_fwd_qkv([(xt, xs)])
    dx, = rk.relkl_bwd_qkv([(xt, xs)], [st])
    pre = rk.relkl_rope_bwd(dx, cw.rope_base, 1.0 / cw.pi_factor, 0.0, True, torch.bfloat16)
    hs = c["h_s"].cuda()
    dw = rk.relkl_weight_grad(hs, pre)
    torch.cuda.synchronize()
    toks = np.array([0, 1, 127, 4096, 20000, cw.N - 1])
    dx_np = dx[:, :, toks].cpu().numpy()
    pos = c["pos_s"].numpy()[toks]
    want = chain.rope_backward(dx_np, pos, cw.rope_base).transpose(0, 2, 1, 3)
    got = pre[:, toks].float().cpu().numpy()
    big = float(np.abs(dx_np).max())
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6 * big)
    cols = np.array([0, 5, 127, 128, 2049, 4095])
    pre_np = pre.reshape(-1, pre.shape[2] * pre.shape[3])[:, cols].double().cpu().numpy()
    ref = c["h_s"].reshape(-1, cw.D).double().numpy().T @ pre_np
    rel_err = np.abs(dw[:, cols].double().cpu().numpy() - ref).max() / np.abs(ref).max()
    assert rel_err <= 1e-4, rel_err


def test_rope_bwd_scalar_path_odd_quads_and_misaligned_output():
    # d % 8 != 0, or an output that is not 8-byte aligned, takes the one-pair-per-thread kernel
    gen = torch.Generator().manual_seed(17)
    dx = torch.randn(1, 3, 45, 6, generator=gen)
    ref = _expected_pre(dx.numpy(), 1e4, 0.5, 0.0, True)
    out = rk.relkl_rope_bwd(dx.cuda(), 1e4, 0.5, 0.0, True, torch.float32)
    dx2 = torch.randn(2, 2, 33, 64, generator=gen)
    ref2 = _expected_pre(dx2.numpy(), 1e4, 0.25, 0.0, True)
    raw = torch.empty(dx2.numel() + 1, dtype=torch.bfloat16, device="cuda")
    view = raw[1:].view(2, 33, 2, 64)          # 2-byte aligned
    rk.relkl_rope_bwd(dx2.cuda(), 1e4, 0.25, 0.0, True, torch.bfloat16, out=view)
    torch.cuda.synchronize()
    assert np.abs(to_np(out) - ref).max() <= 1e-6 * float(np.abs(dx.numpy()).max())
    big = float(np.abs(dx2.numpy()).max())
    assert np.all(np.abs(to_np(view) - ref2) <= 2.0 ** -8 * np.abs(ref2) + 1e-6 * big)
