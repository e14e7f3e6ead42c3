"""Whole-stack parity on the five synthetic workloads, through the C ABI.

The small fp32 stack is compared in full.  The bf16 stacks run at their full
batch in the launch configuration the benchmark times (rm_stack_forward over
the whole batch); the oracle recomputes a sample of rows one by one (samples
are independent), and every block output X_l, the last block output and the
pooled output of those rows are compared.
"""
import numpy as np
import pytest
import torch

from gpu_common import assert_close, dev, host64, sample_rows
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rm():
    from token_mixing_feature_b200 import rankmixer
    return rankmixer


def _stack(wl, d):
    from token_mixing_feature_b200.stack import RankMixerStack
    return RankMixerStack(wl, d["blocks"], d.get("head"))


@pytest.mark.parametrize("name", ["tiny_f32", "appendix_b"])
def test_small_stack_full(rm, O, name):
    """Every sample: the fp32 stack, and the Appendix B three-layer ReLU Mixer (bf16)."""
    wl = synth.WORKLOADS[name]
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    X0 = dev(d["X0"])
    Xlast = st.empty_act(wl.B)
    pooled = st.forward(X0, Xlast=Xlast)
    xs = [X0]
    for l in range(wl.L):
        xs.append(st.block(l, xs[-1]))
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    ref = O.stack(d["X0"], d["blocks"], want_all=True, gelu=wl.act)
    for l in range(wl.L):
        assert_close(host64(xs[l + 1]), ref["Xall"][l], wl.dtype, f"X_{l + 1}")
    assert_close(host64(Xlast), ref["Xlast"], wl.dtype, "Xlast")
    assert_close(host64(pooled), ref["pooled"], wl.dtype, "pooled")
    st.close()


@pytest.mark.parametrize("dtype,T,D,hidden,B,mix_addnorm", [
    ("bf16", 5, 80, 64, 37, True),      # odd T; several samples per staged chunk, ragged last chunk
    ("f32", 3, 24, 16, 11, True),       # odd T, fp32, dh = 8 bytes pieces
    ("bf16", 16, 320, 256, 70, True),   # Pad-Split width: dh = 20 (8-byte pieces)
    ("bf16", 8, 128, 64, 3, True),      # fewer samples than one chunk holds
    ("bf16", 5, 80, 64, 37, False),     # no Add & Norm after mixing
    ("bf16", 16, 16, 32, 5, True),      # dh = 1
    ("bf16", 64, 1536, 64, 2, True),    # T = 64 at D = 1536 (a 195 KB staged sample)
    ("bf16", 32, 2048, 64, 3, True),    # D = 2048, the largest bf16 width
    ("f32", 16, 1024, 32, 2, True),     # D = 1024, the largest fp32 width
])
def test_stack_small_shapes_full(rm, O, dtype, T, D, hidden, B, mix_addnorm):
    """Two-block stacks compared in full on shapes that exercise the staged
    chunks of several samples, odd T and the narrow-piece mixing paths."""
    wl = synth.Workload("small", B=B, T=T, D=D, hidden=hidden, L=2, dtype=dtype, ln_params="perturbed",
                        mix_addnorm=mix_addnorm)
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    X0 = dev(d["X0"])
    Xlast = st.empty_act(wl.B)
    pooled = st.forward(X0, Xlast=Xlast)
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    ref = O.stack(d["X0"], d["blocks"], want_all=False, mix_addnorm=mix_addnorm)
    assert_close(host64(Xlast), ref["Xlast"], dtype, "Xlast")
    assert_close(host64(pooled), ref["pooled"], dtype, "pooled")
    st.close()


@pytest.mark.parametrize("name,nsamp", [("rm100m", 16), ("rm1b", 8), ("moe", 16)])
def test_bf16_stack_sampled(rm, O, name, nsamp):
    wl = synth.WORKLOADS[name]
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    X0 = dev(d["X0"])
    Xlast = st.empty_act(wl.B)
    pooled = st.forward(X0, Xlast=Xlast)
    xs = [X0]
    for l in range(wl.L):
        xs.append(st.block(l, xs[-1]))
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    idx = sample_rows(wl.B, nsamp)
    ref = O.stack(synth.make_x0(wl, samples=idx), d["blocks"], want_all=True)
    for l in range(wl.L):
        assert_close(host64(xs[l + 1][idx.to("cuda")]), ref["Xall"][l], "bf16", f"X_{l + 1}")
    assert_close(host64(Xlast[idx.to("cuda")]), ref["Xlast"], "bf16", "Xlast")
    assert_close(host64(pooled[idx.to("cuda")]), ref["pooled"], "bf16", "pooled")
    st.close()


def test_padsplit_stack_sampled(rm, O):
    wl = synth.WORKLOADS["padsplit"]
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    X0 = st.tokenize([dev(g) for g in d["groups"]])
    pooled = st.forward(X0)
    prob = st.head_forward(pooled)
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    idx = sample_rows(wl.B, 24)
    groups = synth.make_groups(wl, samples=idx)
    X0ref = O.padsplit(groups, wl.padded_width).reshape(len(idx), wl.T, wl.D)
    np.testing.assert_array_equal(host64(X0[idx.to("cuda")]), X0ref)
    ref = O.stack(X0ref.astype(np.float32), d["blocks"], want_all=False)
    assert_close(host64(pooled[idx.to("cuda")]), ref["pooled"], "bf16", "pooled")
    pref = O.head(ref["pooled"], d["head"]["w"], float(d["head"]["b"][0]))
    np.testing.assert_allclose(host64(prob[idx.to("cuda")]), pref, rtol=0, atol=2e-3)
    st.close()


def test_host_entry_matches_device_entry(rm):
    wl = synth.WORKLOADS["rm100m"].with_batch(200)
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    pooled_dev = st.forward(dev(d["X0"]))
    X0h = d["X0"].pin_memory()
    pooled_h = torch.empty(wl.B, wl.D, dtype=torch.float32).pin_memory()
    st.forward_host(X0h, pooled_h)
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    assert torch.equal(pooled_dev.cpu(), pooled_h)
    st.close()


def test_host_async_pipeline_matches_device_entry(rm):
    """Back-to-back asynchronous host calls (two device buffer sets used in
    turn, so the third call reuses the first set): each call's pooled output
    equals the device entry point's on the same input."""
    wl = synth.WORKLOADS["rm100m"].with_batch(160)
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    inputs = [synth.random_activations((wl.B, wl.T, wl.D), "bf16", seed=40 + i) for i in range(3)]
    expect = [st.forward(dev(x)).cpu() for x in inputs]
    hosts = [x.pin_memory() for x in inputs]
    outs = [torch.full((wl.B, wl.D), float("nan"), dtype=torch.float32).pin_memory() for _ in range(3)]
    for xh, oh in zip(hosts, outs):
        st.forward_host_async(xh, oh)
    st.host_wait()
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    for i in range(3):
        assert torch.equal(outs[i], expect[i]), f"call {i}"
    st.close()


def test_programmatic_launch_changes_no_bits(rm, tmp_path):
    """Kernels overlap their launch with the previous kernel's tail
    (programmatic dependent launch); a process with it switched off
    (RM_NO_PDL) computes bit-identical stacks (dense, MoE, Pad-Split + head)."""
    import os
    import subprocess
    import sys
    script = tmp_path / "run.py"
    script.write_text(
        "import sys, torch\n"
        "sys.path.insert(0, %r)\n"
        "from token_mixing_feature_b200 import synth\n"
        "from token_mixing_feature_b200.stack import RankMixerStack\n"
        "out = {}\n"
        "for name, B in (('rm100m', 96), ('moe', 128), ('padsplit', 200)):\n"
        "    wl = synth.WORKLOADS[name].with_batch(B)\n"
        "    d = synth.make_inputs(wl)\n"
        "    st = RankMixerStack(wl, d['blocks'], d.get('head'))\n"
        "    X0 = st.tokenize([g.cuda() for g in d['groups']]) if wl.group_widths else d['X0'].cuda()\n"
        "    pooled = st.forward(X0)\n"
        "    out[name] = (st.head_forward(pooled) if wl.head else pooled).cpu()\n"
        "    st.close()\n"
        "torch.save(out, sys.argv[1])\n" % os.getcwd())
    results = []
    for env_extra in ({}, {"RM_NO_PDL": "1"}):
        env = dict(os.environ)
        env.pop("RM_NO_PDL", None)
        env.update(env_extra)
        path = tmp_path / f"out{len(results)}.pt"
        subprocess.run([sys.executable, str(script), str(path)], check=True, env=env, timeout=600)
        results.append(torch.load(path))
    for name in results[0]:
        assert torch.equal(results[0][name], results[1][name]), name


@pytest.mark.parametrize("name,B", [("rm100m", 96), ("moe", 128)])
def test_cuda_graph_replay_equals_direct_launch(rm, name, B):
    """The stack captured once in a CUDA graph (kernel launches, programmatic
    dependencies and the router's memset become graph nodes) and replayed on
    new inputs copied into the captured buffer gives the direct launches'
    bits."""
    wl = synth.WORKLOADS[name].with_batch(B)
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    X0 = dev(d["X0"])
    pooled = torch.empty(wl.B, wl.D, dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        st.forward(X0, pooled, stream=side.cuda_stream)
        side.synchronize()
        with torch.cuda.graph(g, stream=side):
            st.forward(X0, pooled, stream=side.cuda_stream)
    torch.cuda.synchronize()
    for i in range(2):
        x = synth.random_activations((wl.B, wl.T, wl.D), "bf16", seed=60 + i)
        X0.copy_(dev(x))
        g.replay()
        torch.cuda.synchronize()
        got = pooled.clone()
        expect = st.forward(dev(x))
        torch.cuda.synchronize()
        assert rm.rm_sync_status(st.h) == rm.RM_OK
        assert torch.equal(got, expect), f"replay {i}"
    del g
    st.close()


def test_moe_router_masks_at_workload_constants(rm, O, record_property):
    """Router masks of the sparse-MoE workload at its own constants (B 2048,
    T 16, D 768, 8 experts per token, router weights N(0, 0.02), bias -0.5),
    on the S the library's LayerNorm produces for every block of the stack.
    The ReLU routing equation (fun-rec "Rankmixer: 硬件效率优化", section
    Sparse MoE扩展) opens expert j iff its logit is > 0: the masks must equal
    the oracle's wherever |logit| >= 1e-3 (the kernel decides in fp32, the
    oracle in fp64), the undecided band must stay small, the gates must equal
    ReLU(logit), and the expert output V must match on sampled rows."""
    wl = synth.WORKLOADS["moe"]
    d = synth.make_inputs(wl)
    st = _stack(wl, d)
    x = dev(d["X0"])
    G = torch.empty(wl.B, wl.T, wl.n_experts, dtype=torch.float32, device="cuda")
    V = torch.empty_like(x)
    idx = sample_rows(wl.B, 16)
    for l in range(wl.L):
        blk = st.blocks[l]
        M = torch.empty_like(x)
        rm.rm_token_mix(st.h, x, M, wl.B)
        S = torch.empty_like(x)
        rm.rm_layernorm(st.h, M, x, blk["ln1_g"], blk["ln1_b"], S, wl.B * wl.T)
        rm.rm_moe_forward(st.h, blk, S, V, G, wl.B)
        assert rm.rm_sync_status(st.h) == rm.RM_OK
        S_h = S.cpu()
        logits = O.router(S_h, d["blocks"][l]["Wr"], d["blocks"][l]["br"])
        g = host64(G)
        decided = np.abs(logits) >= 1e-3
        excluded = int((~decided).sum())
        rate = float((g > 0).mean())
        record_property(f"block{l}_undecided_entries", excluded)
        record_property(f"block{l}_active_rate", rate)
        print(f"block {l}: {excluded} of {logits.size} router entries within 1e-3 of zero, "
              f"active rate {rate:.4f}")
        assert excluded < 0.005 * logits.size
        np.testing.assert_array_equal((g > 0)[decided], (logits > 0)[decided])
        np.testing.assert_allclose(g, np.maximum(logits, 0), rtol=0, atol=1e-4)
        assert 0.1 < rate < 0.3          # about 18 % for logits ~ N(-0.5, 0.55^2)
        Vref, _ = O.moe(S_h[idx], d["blocks"][l])
        assert_close(host64(V[idx.to("cuda")]), Vref, "bf16", f"moe V, block {l}", raw=True)
        x = st.block(l, x)
    st.close()
