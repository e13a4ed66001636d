"""Parity margins of the CUDA path against the float64 oracle, as a table.

    python tests/parity_report.py [--full] > parity.md

For each case: the worst per-row KL error as a fraction of its tolerance
(1e-3 |kl| + 1e-6), the relative error of the total KL, and the max-norm
relative dX error against its tolerance (2e-2 for bf16 inputs; for the fp32
path the per-input bound of parity.fp32_dx_tolerance).  --full adds the workload-sized cases (sampled units and rows),
which take a few minutes of oracle time.  Needs a CUDA device.
"""
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import attention_relation_kl_b200 as rk  # noqa: E402
import workload  # noqa: E402
from oracle import dense  # noqa: E402
from parity import DX_TOL_BF16, KL_ATOL, KL_RTOL, fp32_dx_tolerance, to_np  # noqa: E402


def margins(kl, ref_kl, dx, ref_dx, dx_tol):
    kl, ref_kl = np.asarray(kl, np.float64), np.asarray(ref_kl, np.float64)
    kl_frac = float(np.max(np.abs(kl - ref_kl) / (KL_RTOL * np.abs(ref_kl) + KL_ATOL)))
    tot = float(abs(kl.sum() - ref_kl.sum()) / max(abs(ref_kl.sum()), 1e-30))
    dx_rel = float(np.max(np.abs(dx - ref_dx)) / max(np.max(np.abs(ref_dx)), 1e-30))
    return kl_frac, tot, dx_rel, dx_rel / dx_tol


def small_cases():
    cases = []
    for (N, d, causal, B, H, dtype) in [(128, 128, True, 1, 1, "bf16"), (300, 64, True, 1, 2, "bf16"),
                                        (1000, 128, True, 1, 1, "bf16"), (513, 64, False, 1, 1, "bf16"),
                                        (256, 64, True, 1, 1, "fp32"), (200, 96, True, 1, 2, "bf16")]:
        w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=N + d, causal=causal, B=B, H=H)
        xt, xs = workload.generate(w)["q"]
        cases.append((f"Q/Q RoPE PI4x N={N} d={d} {'causal' if causal else 'full'} {dtype}",
                      xt, xs, causal))
    xt, xs = workload.gaussian_pair((1, 2, 640, 128), seed=5, noise=0.05, dtype=torch.bfloat16)
    cases.append(("V/V sigma=0.05 N=640 d=128 bf16", xt, xs, True))
    return cases


def small_cases_more():
    """Explicit logit scale, clustered large logits (|z| ~ 70-100) and full masks
    (the symmetric schedule)."""
    cases = []
    for (N, d, scale, causal) in [(4200, 128, 0.3, True), (513, 64, 0.05, False),
                                  (150, 64, 0.3, False)]:
        dtype = "fp32" if N == 150 else "bf16"
        w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=N + int(1000 * scale), causal=causal)
        xt, xs = workload.generate(w)["q"]
        spread = ""
        if scale * d > 20:
            # the inputs of test_explicit_scale: rows kept spread, since at scale 0.3
            # and d = 128 unit-variance rows are one-hot to 1e-11
            xt, xs = (xt.float() * 0.4).to(xt.dtype), (xs.float() * 0.4).to(xs.dtype)
            spread = " (inputs x0.4)"
        cases.append((f"scale={scale}{spread} N={N} d={d} {'causal' if causal else 'full'} {dtype}",
                      xt, xs, causal, scale))
    for (N, d, causal) in [(4200, 128, True), (4200, 128, False), (4300, 64, True)]:
        xt, xs = workload.clustered_pair((1, 1, N, d), seed=N + d,
                                         amplitude=2.5 if d == 128 else 3.0)
        cases.append((f"large logits N={N} d={d} {'causal' if causal else 'full'} bf16",
                       xt, xs, causal, 0.0))
    return cases


def run_small(out):
    for name, xt, xs, causal, *rest in [c + (0.0,) for c in small_cases()] + small_cases_more():
        scale = rest[0]
        gt, gs = xt.cuda(), xs.cuda()
        path = "tcgen05" if rk.relkl_path_for(gt, causal) == 1 else "CUDA-core fp32"
        kl, st = rk.relkl_fwd(gt, gs, causal, scale)
        dx = rk.relkl_bwd(gt, gs, st, None, causal, scale)
        torch.cuda.synchronize()
        osc = scale if scale else None
        tol = DX_TOL_BF16 if path == "tcgen05" else fp32_dx_tolerance(xt, xs, None, causal, osc)
        m = margins(to_np(kl), dense.fwd(xt, xs, causal, osc)["kl"], to_np(dx),
                    dense.bwd(xt, xs, None, causal, osc), tol)
        out.append((name, path, "all rows", *m))


def run_packed(out):
    """Packed variable-length sequences (garbage in the tokens of no sequence)."""
    for lens, d, causal in [([300, 0, 1, 129, 700, 57], 128, True),
                            ([4300, 200, 4097, 5], 128, False), ([513, 64, 1000], 64, True)]:
        total = sum(lens) + 11
        w = workload.tiny_custom(N=total, d=d, dtype="bf16", seed=sum(lens) + d, H=2)
        xt, xs = workload.generate(w)["q"]
        xt, xs = xt.clone(), xs.clone()
        xt[:, :, total - 11:] = 30.0
        xs[:, :, total - 11:] = -45.0
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        gcu = torch.from_numpy(cu).cuda()
        gt, gs = xt.cuda(), xs.cuda()
        kl, st = rk.relkl_fwd(gt, gs, causal, cu_seqlens=gcu, max_seqlen=max(lens))
        dx = rk.relkl_bwd(gt, gs, st, None, causal, cu_seqlens=gcu, max_seqlen=max(lens))
        torch.cuda.synchronize()
        m = margins(to_np(kl), dense.fwd_varlen(xt, xs, cu, causal)["kl"], to_np(dx),
                    dense.bwd_varlen(xt, xs, cu, None, causal), DX_TOL_BF16)
        out.append((f"packed d={d} {'causal' if causal else 'full'} lengths={lens}", "tcgen05",
                    "all rows", *m))


def run_padded(out):
    """Right-padded batches (garbage in the padding) on every kernel family."""
    for (B, H, N, d, dtype, causal, lengths) in [(3, 2, 300, 128, "bf16", True, [300, 263, 0]),
                                                 (3, 2, 300, 128, "bf16", False, [300, 177, 1]),
                                                 (2, 1, 4200, 128, "bf16", True, [4200, 3001]),
                                                 (2, 2, 150, 64, "fp32", False, [97, 150])]:
        w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=N + d, causal=causal, B=B, H=H)
        xt, xs = workload.generate(w)["q"]
        xt, xs = xt.clone(), xs.clone()
        for b, L in enumerate(lengths):
            xt[b, :, L:] = 30.0
            xs[b, :, L:] = -45.0
        gl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
        gt, gs = xt.cuda(), xs.cuda()
        path = "tcgen05" if rk.relkl_path_for(gt, causal) == 1 else "CUDA-core fp32"
        kl, st = rk.relkl_fwd(gt, gs, causal, lengths=gl)
        dx = rk.relkl_bwd(gt, gs, st, None, causal, lengths=gl)
        torch.cuda.synchronize()
        tol = DX_TOL_BF16 if path == "tcgen05" else fp32_dx_tolerance(xt, xs, None, causal,
                                                                       lengths=lengths)
        m = margins(to_np(kl), dense.fwd(xt, xs, causal, lengths=lengths)["kl"], to_np(dx),
                    dense.bwd(xt, xs, None, causal, lengths=lengths), tol)
        out.append((f"padded N={N} d={d} {'causal' if causal else 'full'} {dtype} lengths={lengths}",
                    path, "all rows", *m))


def run_chain(out):
    """dW_q, dW_k, dW_v of the small chain workload (kl columns: not applicable)."""
    from oracle import chain
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
        rel = float(np.abs(g - w).max() / np.abs(w).max())
        out.append((f"chain_small dW_{r} [{w.shape[0]}x{w.shape[1]}]", "RoPE bwd + tcgen05 GEMM",
                    "every weight", float("nan"), float("nan"), rel, rel / DX_TOL_BF16))


def run_full(out):
    from test_gpu_parity import _dx_rows
    for cfg, units in (("llama2_h32_n4k", [("q", 0, 0), ("v", 0, 31)]),
                       ("gqa_llama3_n16k", [("k", 0, 3), ("v", 1, 7)]),
                       ("ext_h32_n32k", [("q", 0, 0), ("k", 0, 17), ("v", 0, 31)]),
                       ("d64_h32_n32k", [("q", 0, 0), ("v", 0, 31)]),
                       ("full_h32_n16k", [("q", 0, 5), ("v", 0, 31)])):
        w = workload.get_config(cfg)
        x = workload.generate(w)
        pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in w.relations]
        outs = rk.relkl_fwd_qkv(pairs, w.causal)
        dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs], None, w.causal)
        torch.cuda.synchronize()
        ri = {r: i for i, r in enumerate(w.relations)}
        for rel, b, h in units:
            xt, xs = x[rel][0][b, h], x[rel][1][b, h]
            ref = dense.fwd_unit(xt, xs, w.causal)
            rows = _dx_rows(w.N)
            ref_dx = dense.bwd_rows(xt, xs, rows, causal=w.causal, lse=ref)
            m = margins(to_np(outs[ri[rel]][0][b, h]), ref["kl"],
                        to_np(dxs[ri[rel]][b, h])[rows], ref_dx, DX_TOL_BF16)
            out.append((f"{cfg} unit ({rel}, b={b}, h={h})", "tcgen05 fused QKV",
                        f"kl all {w.N} rows, dX on {len(rows)} rows of the first, middle and "
                        f"last work items", *m))


def main():
    out = []
    t0 = time.time()
    run_small(out)
    run_padded(out)
    run_packed(out)
    run_chain(out)
    if "--full" in sys.argv:
        run_full(out)
    print(f"# Parity margins against the float64 oracle ({torch.cuda.get_device_name(0)})\n")
    print("Fractions are of the tolerance: < 1 passes.\n")
    print("| case | path | compared | worst kl err / tol | total kl rel err | dX max-norm rel err | dX err / tol |")
    print("|---|---|---|---|---|---|---|")
    for name, path, cmp, klf, tot, dxr, dxf in out:
        print(f"| {name} | {path} | {cmp} | {klf:.3f} | {tot:.2e} | {dxr:.2e} | {dxf:.3f} |")
    print(f"\n({time.time() - t0:.0f} s)")


if __name__ == "__main__":
    main()
