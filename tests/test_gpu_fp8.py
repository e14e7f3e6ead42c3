"""Stack with e4m3 (fp8) FFN weights: rm_quantize_fp8 against the definition
of e4m3 rounding, and rm_stack_forward_fp8 against the oracle and against the
bf16 stack.

Tolerance.  e4m3 keeps 3 mantissa bits: rounding x / scale to it has a
relative error of at most 2^-4 (half an ulp at the bottom of a binade) and
about 2.4 % RMS over a binade.  Each projection multiplies two rounded
operands (the row-quantised activations and the channel-quantised weights):
about sqrt(2) x 2.4 % = 3.4 % relative error of its output; the second
projection adds the rounding of H: V ~ sqrt(3.4^2 + 2.4^2 + 3.4^2) % = 5.4 %;
the block output LN(V + S) halves that when |V| ~ |S| (S is exact), ~4 %, and
two blocks compound to ~5 %.  The bound is 1e-1 relative L2 on the pooled
output and the last block's output (twice the estimate); the bf16 stack's
own 1e-2 bound is for bf16 configurations only.
"""
import numpy as np
import pytest
import torch

from gpu_common import dev, host64, rel_l2, sample_rows
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu
FP8_REL_L2 = 1e-1


@pytest.fixture(scope="module")
def rm():
    from token_mixing_feature_b200 import rankmixer
    return rankmixer


def _e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest e4m3 value (3 mantissa bits, exponent bias 7,
    subnormals below 2^-6), ties to even; |x| <= 448 here."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -6)))
    ulp = 2.0 ** (e - 3)
    q = ax / ulp
    r = np.floor(q)
    frac = q - r
    r = np.where((frac > 0.5) | ((frac == 0.5) & (r % 2 == 1)), r + 1, r)
    return np.sign(x) * r * ulp


@pytest.mark.parametrize("rows,K", [
    (40, 96),        # 12 vectors a row: one partial warp, four rows a CTA
    (24, 1536),      # S rows at D = 1536: 192 threads, one vector each, four rows a CTA
    (25, 1536),      # the last CTA's four rows ragged
    (9, 2064),       # 258 vectors: two a thread, the second ragged
    (12, 6144),      # H rows at kD = 6144: three vectors a thread
    (5, 12304),      # 1538 vectors: the eight-vector form with seven in use
    (3, 16384),      # the largest row
])
def test_quantize_rows_matches_definition(rm, rows, K):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(rows, K, generator=g) * torch.logspace(-3, 2, rows).unsqueeze(1)).to(torch.bfloat16)
    x[rows // 2] = 0                                            # an all-zero row gets scale 1
    q = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, device="cuda")
    rm.rm_quantize_fp8(dev(x), q, sc, rows, K)
    torch.cuda.synchronize()
    xf = x.float().numpy().astype(np.float64)
    absmax = np.abs(xf).max(axis=1)
    want_sc = np.where(absmax > 0, (absmax.astype(np.float32) / np.float32(448.0)), 1.0)
    assert np.array_equal(sc.cpu().numpy(), want_sc.astype(np.float32))
    dec = q.cpu().view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    inv = (np.float32(1.0) / sc.cpu().numpy()).astype(np.float64)
    ref = _e4m3_round((xf.astype(np.float32) * inv[:, None].astype(np.float32)).astype(np.float64))
    assert np.array_equal(dec, ref)


def _quantize_block(rm, blk, T, D, Hd):
    q = {}
    for k, rows, K in (("W1", T * Hd, D), ("W2", T * D, Hd)):
        w = dev(blk[k])
        q[k + "q"] = torch.empty(rows * K, dtype=torch.uint8, device="cuda")
        q[k + "s"] = torch.empty(rows, device="cuda")
        rm.rm_quantize_fp8(w, q[k + "q"], q[k + "s"], rows, K)
    return q


@pytest.mark.parametrize("B,T,D,hidden,L,act", [
    (48, 8, 256, 512, 2, "tanh"),
    (130, 4, 128, 256, 1, "erf"),      # ragged batch: several M tiles and a partial one
    (64, 16, 768, 3072, 2, "tanh"),    # the 100M-scale widths
])
def test_fp8_stack(rm, O, B, T, D, hidden, L, act):
    from token_mixing_feature_b200.stack import RankMixerStack
    wl = synth.Workload("fp8", B=B, T=T, D=D, hidden=hidden, L=L, ln_params="perturbed", act=act)
    d = synth.make_inputs(wl, seed=B + T)
    st = RankMixerStack(wl, d["blocks"])
    qblocks = [_quantize_block(rm, blk, T, D, hidden) for blk in d["blocks"]]
    X0 = dev(d["X0"])
    pooled8 = torch.empty(B, D, device="cuda")
    rm.rm_stack_forward_fp8(st.h, st.blocks, qblocks, X0, pooled8, B)
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    pooled16 = st.forward(X0)
    torch.cuda.synchronize()
    ref = O.stack(d["X0"], d["blocks"], want_all=False, want_last=False, gelu=act)
    r_or = rel_l2(host64(pooled8), ref["pooled"])
    r_bf = rel_l2(host64(pooled8), host64(pooled16))
    assert np.all(np.isfinite(host64(pooled8)))
    assert r_or <= FP8_REL_L2, f"fp8 vs oracle: rel L2 {r_or:.3e}"
    assert r_bf <= FP8_REL_L2, f"fp8 vs bf16 stack: rel L2 {r_bf:.3e}"
    assert r_or > 1e-3   # the quantisation is really in the path
    st.close()


def test_fp8_stack_rm1b_graph_sampled(rm, O):
    """The rm1b stack with e4m3 FFN operands as the benchmark runs it: weights
    quantised once, the step captured in a CUDA graph on a side stream and
    replayed there; the replay equals a direct launch bit for bit, and sampled
    rows of the pooled output stay within the e4m3 bound of the oracle."""
    from token_mixing_feature_b200.stack import RankMixerStack
    wl = synth.WORKLOADS["rm1b"]
    B, T, D, Hd = wl.B, wl.T, wl.D, wl.hidden
    d = synth.make_inputs(wl)
    st = RankMixerStack(wl, d["blocks"])
    qblocks = [_quantize_block(rm, blk, T, D, Hd) for blk in d["blocks"]]
    X0 = dev(d["X0"])
    pooled = torch.empty(B, D, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        rm.rm_stack_forward_fp8(st.h, st.blocks, qblocks, X0, pooled, B, side)
        side.synchronize()
        with torch.cuda.graph(g, stream=side):
            rm.rm_stack_forward_fp8(st.h, st.blocks, qblocks, X0, pooled, B, side)
    torch.cuda.synchronize()
    pooled.zero_()
    with torch.cuda.stream(side):
        g.replay()
    torch.cuda.synchronize()
    got = pooled.clone()
    direct = torch.empty_like(pooled)
    rm.rm_stack_forward_fp8(st.h, st.blocks, qblocks, X0, direct, B)
    torch.cuda.synchronize()
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    assert torch.equal(got, direct)
    idx = sample_rows(B, 8)
    ref = O.stack(synth.make_x0(wl, samples=idx), d["blocks"], want_all=False, want_last=False)
    r = rel_l2(host64(got[idx.to("cuda")]), ref["pooled"])
    assert 1e-3 < r <= FP8_REL_L2, f"fp8 rm1b vs oracle: rel L2 {r:.3e}"
    del g
    st.close()


def test_quantize_rejects_unsupported(rm):
    x = torch.zeros(2, 16400, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(2, 16400, dtype=torch.uint8, device="cuda")
    sc = torch.empty(2, device="cuda")
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_quantize_fp8(x, q, sc, 2, 16400)          # rows longer than 16384
    assert e.value.status == rm.RM_ERR_UNSUPPORTED
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_quantize_fp8(x, q, sc, 2, 24)             # K not a multiple of 16
    assert e.value.status == rm.RM_ERR_INVALID_ARG
    rm.rm_quantize_fp8(x, q, sc, 0, 16)                 # no rows: nothing to do
