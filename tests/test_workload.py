"""The seeded input generator: shapes, dtypes, determinism, draw order, RoPE."""
import torch

import workload


def test_shapes_and_dtypes():
    w = workload.CONFIGS["tiny_fp32_n256"]
    x = workload.generate(w)
    assert list(x) == ["q"]
    assert x["q"][0].shape == (1, 1, 256, 64) and x["q"][0].dtype == torch.float32
    g = workload.Workload("g", B=2, H=4, H_kv=2, N=16, d=8, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=5e5, pi_factor=4.0, v_noise=0.05,
                          seed=4)
    x = workload.generate(g)
    assert x["q"][1].shape == (2, 4, 16, 8) and x["k"][0].shape == (2, 2, 16, 8)
    assert x["v"][1].dtype == torch.bfloat16 and x["v"][1].is_contiguous()
    assert g.n_units == 2 * (4 + 2 + 2) and len(workload.unit_list(g)) == g.n_units


def test_deterministic_and_subset_independent():
    g = workload.Workload("g", B=1, H=2, H_kv=2, N=32, d=16, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=1e4, pi_factor=8.0, v_noise=0.1,
                          seed=7)
    a, b = workload.generate(g), workload.generate(g)
    for r in "qkv":
        assert torch.equal(a[r][0], b[r][0]) and torch.equal(a[r][1], b[r][1])
    only_v = workload.generate(workload.Workload(**{**g.__dict__, "relations": ("v",)}))
    assert torch.equal(only_v["v"][1], a["v"][1])


def test_rope_and_pi():
    g = workload.tiny_custom(N=64, d=8, dtype="fp32", seed=3, pi_factor=4.0)
    xt, xs = workload.generate(g)["q"]
    # position 0 is not rotated: teacher and student agree there
    assert torch.equal(xt[..., 0, :], xs[..., 0, :])
    assert not torch.equal(xt[..., 5, :], xs[..., 5, :])
    # rotation preserves norms (up to the final rounding to fp32)
    torch.testing.assert_close(xt.norm(dim=-1), xs.norm(dim=-1), rtol=1e-6, atol=1e-6)
    # student at p/4 equals a teacher-style rotation at p/4
    u = torch.randn(1, 1, 64, 8, generator=torch.Generator().manual_seed(3))
    ref = workload.rope_rotate(u, torch.arange(64, dtype=torch.float64) / 4.0, 1e4).float()
    torch.testing.assert_close(xs, ref, rtol=0, atol=0)


def test_v_noise_level():
    w = workload.Workload("v", B=1, H=2, H_kv=2, N=512, d=64, dtype="fp32", causal=True,
                          relations=("v",), rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=2)
    vt, vs = workload.generate(w)["v"]
    assert abs(float((vs - vt).std()) - 0.1) < 0.005


def test_chain_workload_shapes_determinism_and_projection():
    cw = workload.CHAIN_CONFIGS["chain_small"]
    a, b = workload.generate_chain(cw), workload.generate_chain(cw)
    assert torch.equal(a["h_s"], b["h_s"]) and torch.equal(a["x"]["k"][1], b["x"]["k"][1])
    assert a["h_t"].shape == (cw.B, cw.N, cw.D) and a["h_t"].dtype == torch.bfloat16
    assert a["w"]["q"].shape == (cw.D, cw.H * cw.d) and a["w"]["v"].shape == (cw.D, cw.H_kv * cw.d)
    for rel in "qkv":
        xt, xs = a["x"][rel]
        assert xt.shape == (cw.B, cw.heads(rel), cw.N, cw.d) and xt.is_contiguous()
    # V is the plain projection of the rounded hidden states; K is its rotation at p / s
    hv = (a["h_s"].float() @ a["w"]["v"].float()).reshape(cw.B, cw.N, cw.H_kv, cw.d).permute(0, 2, 1, 3)
    assert torch.equal(a["x"]["v"][1], hv.to(torch.bfloat16))
    hk = (a["h_s"].float() @ a["w"]["k"].float()).reshape(cw.B, cw.N, cw.H_kv, cw.d).permute(0, 2, 1, 3)
    rk = workload.rope_rotate(hk, a["pos_s"], cw.rope_base).to(torch.bfloat16)
    assert torch.equal(a["x"]["k"][1], rk)
    # student hidden states differ from the teacher's by the configured noise
    diff = (a["h_s"].float() - a["h_t"].float()).std().item()
    assert 0.08 < diff < 0.12


def test_bench_names_the_backward_kernel_the_library_launches():
    # bench.py asks the library (relkl_bwd_kernel_for) which backward a workload runs
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    want = {"ext_h32_n32k": "relkl_bwd_pair_kernel", "gqa_llama3_n16k": "relkl_bwd_pair_kernel",
            "llama2_h32_n4k": "relkl_bwd_tc64_kernel",      # 96 units: 11 one-block rounds, 6 paired
            "sweep_n4096": "relkl_bwd_pair_kernel", "sweep_n2048": "relkl_bwd_pair_kernel",
            "sweep_n1024": "relkl_bwd_tc64_kernel", "full_h32_n16k": "relkl_bwd_pair_kernel",
            "d64_h32_n32k": "relkl_bwd_pair64_kernel", "tiny_fp32_n256": "relkl_bwd_simt_kernel"}
    for name, kernel in want.items():
        assert bench.bwd_kernel_name(workload.get_config(name), n_sms=148) == kernel, name


def test_bench_reference_arm_prints_its_line_on_the_host():
    # bench.py --impl reference times the float64 oracle on the host cores (no GPU)
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-prefix", "128"],
                         capture_output=True, text=True, cwd=root, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["config"]["workload"] == "ext_h32_n32k" and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
