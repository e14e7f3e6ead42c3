"""The FLOP / parameter / byte model against the figures the pages print."""
import json
import os

import pytest

from token_mixing_feature_b200 import roofline, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_appendix_b_flops():
    """Three Mixer layers at B=256, T=8, d=256, h=1024 -> 6.442451 GFLOPs (Appendix B)."""
    with open(os.path.join(GOLDEN, "appendix_b_flops.json")) as f:
        g = json.load(f)
    flops = g["L"] * roofline.dense_block_flops(g["B"], g["T"], g["D"], g["hidden"])
    assert round(flops / 1e9, 6) == g["gflops"]
    for row in g["rows"]:
        # the TFLOP/s column is the GFLOPs over the ms column, which the table
        # prints rounded to 1 us: the printed rate lies inside that interval
        lo = flops / ((row["ms"] + 5e-4) * 1e-3) / 1e12
        hi = flops / ((row["ms"] - 5e-4) * 1e-3) / 1e12
        assert lo - 5e-4 <= row["tflops"] <= hi + 5e-4


def test_pffn_param_formula():
    """Per-token FFN parameters 2 T k D^2: T times a shared FFN's 2 k D^2."""
    assert roofline.pffn_params(1, 768, 4 * 768) * 16 == roofline.pffn_params(16, 768, 4 * 768)
    assert roofline.pffn_params(16, 768, 3072) == 2 * 16 * 4 * 768 ** 2


@pytest.mark.parametrize("name,params", [("rm100m", 151e6), ("rm1b", 1.2e9)])
def test_workload_param_counts(name, params):
    wl = synth.WORKLOADS[name]
    p = wl.L * roofline.pffn_params(wl.T, wl.D, wl.hidden)
    assert abs(p - params) / params < 0.02


def test_stack_flops_and_bytes_1b():
    wl = synth.WORKLOADS["rm1b"]
    assert roofline.stack_flops(wl) == 2 * 4 * 512 * 32 * 1536 * 6144
    wbytes = 2 * 2 * 32 * 1536 * 6144 * 2
    assert roofline.stack_bytes(wl) > wbytes
    assert roofline.stack_bytes(wl) < wbytes * 1.1


def test_moe_flops_need_active_counts():
    wl = synth.WORKLOADS["moe"]
    with pytest.raises(ValueError):
        roofline.stack_flops(wl)
    f = roofline.stack_flops(wl, [1000, 2000])
    assert f == 3000 * 4 * 768 * 768 + 2 * (2 * 2048 * 16 * 768 * 8)


def test_code_digest_ignores_comments_only(tmp_path):
    """The benchmark reports the committed ncu traffic only while the GEMM's
    code is the captured one; comment or whitespace edits are not changes."""
    import bench
    a = tmp_path / "a.cu"
    a.write_text("int f(int x) {\n    return x + 1;  // one\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("/* header */\nint f(int x) {\n  return x + 1;\n}  // trailing\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) {\n    return x + 2;\n}\n")
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))


def _fake_tree(tmp_path, workload, family_file, source, digest_of_source=True, bytes_line="gemm1 = 123456"):
    import bench
    csrc = tmp_path / "token_mixing_feature_b200" / "csrc"
    csrc.mkdir(parents=True, exist_ok=True)
    (csrc / source).write_text("int kernel() { return 1; }  // v1\n")
    digest = bench.code_digest(str(csrc / source)) if digest_of_source else "0" * 16
    prof = tmp_path / "profiles"
    prof.mkdir(exist_ok=True)
    (prof / family_file.format(workload=workload)).write_text(
        f"code sha256[:16]: {digest}\n\ndram_bytes_per_launch {bytes_line}\n")
    return str(tmp_path)


PEAKS = {"bf16_tflops": 1617.4, "bf16_tflops_sustained": 1372.7, "hbm_gbs": 6543.4}


def test_top_kernel_roofline_tensor_traffic_per_workload(tmp_path):
    """The GEMM roofline takes its traffic from the summary of the same
    workload, only while that summary's code digest matches the source."""
    import bench
    wl = synth.WORKLOADS["padsplit"]
    root = _fake_tree(tmp_path, "padsplit", "ncu_gemm_tc_{workload}.md", "rm_gemm_tc.cu")
    r = bench.top_kernel_roofline(wl, "gemm1", 0.08, None, PEAKS, "measured", 148, 1965.0, root)
    assert r["bound"] == "tensor" and r["traffic"] == 123456.0
    flops = 2.0 * wl.B * wl.T * wl.D * wl.hidden
    assert abs(r["achieved"] - flops / 0.08e-3 / 1e12) < 1e-9
    # a short timed region: the burst peak is the ceiling, sustained and spec beside it
    assert abs(r["frac"] - r["achieved"] / 1617.4) < 1e-12
    assert abs(r["frac_of_sustained"] - r["achieved"] / 1372.7) < 1e-12
    assert abs(r["frac_of_spec"] - r["achieved"] / 2250.0) < 1e-12
    # another workload has no summary here: no traffic
    r2 = bench.top_kernel_roofline(synth.WORKLOADS["rm1b"], "gemm1", 0.3, None, PEAKS, "measured", 148, 1965.0, root)
    assert r2["traffic"] is None
    # a summary of other code: no traffic
    root3 = _fake_tree(tmp_path / "stale", "padsplit", "ncu_gemm_tc_{workload}.md", "rm_gemm_tc.cu",
                       digest_of_source=False)
    assert bench.top_kernel_roofline(wl, "gemm1", 0.08, None, PEAKS, "m", 148, 1965.0, root3)["traffic"] is None


def test_top_kernel_roofline_alu_and_hbm(tmp_path):
    import bench
    wl = synth.WORKLOADS["padsplit"]
    root = _fake_tree(tmp_path, "padsplit", "ncu_gemm_tc_{workload}.md", "rm_gemm_tc.cu")
    # the fp32 path runs on CUDA cores: FFMA peak of 148 SMs x 128 lanes x 2 x 1965 MHz
    tiny = synth.WORKLOADS["tiny_f32"]
    a = bench.top_kernel_roofline(tiny, "gemm2", 0.01, None, PEAKS, "measured", 148, 1965.0, root)
    assert a["bound"] == "alu" and abs(a["peak"] - 148 * 128 * 2 * 1965e6 / 1e12) < 1e-9
    h = bench.top_kernel_roofline(wl, "mix_ln", 0.04, None, PEAKS, "measured", 148, 1965.0, root)
    nbytes = roofline.kernel_work(wl, "mix_ln")[1]
    assert h["bound"] == "hbm" and abs(h["achieved"] - nbytes / 0.04e-3 / 1e9) < 1e-6
    assert abs(h["frac"] - h["achieved"] / 6543.4) < 1e-12


KERNELS_BY_WORKLOAD = {
    "rm1b": ["mix_ln", "gemm1", "gemm2", "ln_pool"],
    "rm100m": ["mix_ln", "gemm1", "gemm2", "ln_pool"],
    "padsplit": ["mix_ln", "gemm1", "gemm2", "ln_pool", "padsplit", "head"],
    "moe": ["mix_ln", "gemm1", "gemm2", "ln_pool", "moe_route", "moe_gather", "moe_combine"],
    "appendix_b": ["mix_ln", "gemm1", "gemm2", "ln_pool"],
    "tiny_f32": ["mix_ln", "gemm1", "gemm2", "ln_pool"],
}


@pytest.mark.parametrize("name", sorted(KERNELS_BY_WORKLOAD))
def test_per_kernel_rooflines_cover_every_kernel(name):
    """Every kernel kind the stack launches gets an achieved rate against its
    own bound (HBM for the memory-bound kinds, tensor or fp32 FFMA for the
    FFN contractions)."""
    import bench
    wl = synth.WORKLOADS[name]
    kinds = KERNELS_BY_WORKLOAD[name]
    kern = {k: {"ms_avg": 0.05, "launches": 2, "share": 0.1} for k in kinds}
    active = [wl.B * wl.T * 2, wl.B * wl.T * 2] if wl.n_experts else None
    out = bench.per_kernel_rooflines(wl, kern, active, PEAKS, 148, 1965.0)
    for k, e in out.items():
        assert e["frac"] > 0 and e["achieved"] > 0, k
        if k in ("gemm1", "gemm2"):
            assert e["unit"] == "TFLOP/s" and e["bound"] == ("alu" if wl.dtype == "f32" else "tensor")
        else:
            assert e["unit"] == "GB/s" and e["bound"] == "hbm"


def test_kernel_work_figures():
    """Algorithmic bytes of the memory-bound kinds at the 1B-scale and
    Pad-Split sizes, by hand: X in + S out, plus half the launches reading
    the previous block's 24 LayerNorm partials per row."""
    rm1b = synth.WORKLOADS["rm1b"]
    act = 512 * 32 * 1536 * 2
    assert roofline.kernel_work(rm1b, "mix_ln") == ("bytes", 2 * act + 512 * 32 * 24 * 8 * 0.5)
    assert roofline.kernel_work(rm1b, "ln_pool") == ("bytes", act + 512 * 32 * 24 * 8 + 512 * 1536 * 4)
    ps = synth.WORKLOADS["padsplit"]
    assert roofline.kernel_work(ps, "padsplit") == ("bytes", 4096 * 4800 * 2 + 4096 * 16 * 320 * 2)
    assert roofline.kernel_work(ps, "gemm1") == ("flops", 2.0 * 4096 * 16 * 320 * 1280)
    with pytest.raises(KeyError):
        roofline.kernel_work(ps, "no_such_kernel")
