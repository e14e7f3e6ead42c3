"""Token-sharded stack forward (the mixing as an all-to-all between ranks
that each own T / G tokens), G ranks run in one process on one GPU with the
exchanges as device copies (tokshard.run_local), against the single-GPU
stack and the oracle.  The NCCL path (tokshard.run_distributed) performs the
same exchanges with torch.distributed; its exchange layout is tested on CPU
ranks with gloo (tests/test_tokshard_gloo.py)."""
import numpy as np
import pytest
import torch

from gpu_common import assert_close, dev, host64, rel_l2
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,D,hidden,L,world", [
    (24, 8, 256, 128, 2, 1),
    (24, 8, 256, 128, 2, 2),
    (24, 8, 256, 128, 2, 4),
    (24, 8, 256, 128, 2, 8),      # one token per rank
    (40, 16, 768, 256, 3, 4),     # the 100M-scale width, three blocks
])
def test_token_sharded_forward(O, B, T, D, hidden, L, world):
    from token_mixing_feature_b200 import tokshard
    from token_mixing_feature_b200.stack import RankMixerStack
    wl = synth.Workload("tokshard", B=B, T=T, D=D, hidden=hidden, L=L, ln_params="perturbed")
    d = synth.make_inputs(wl, seed=B + world)
    X0 = dev(d["X0"])
    ranks = [tokshard.TokenShardedRank(wl, d["blocks"], r, world) for r in range(world)]
    pooled = tokshard.run_local(ranks, [tokshard.shard_rows(X0, r, world) for r in range(world)], B)
    torch.cuda.synchronize()
    for r in ranks:   # every rank holds the same pooled output
        assert torch.equal(r.pooled, pooled)
    ref = O.stack(d["X0"], d["blocks"], want_all=False, want_last=False)
    assert_close(host64(pooled), ref["pooled"], "bf16", "pooled")
    st = RankMixerStack(wl, d["blocks"])
    single = st.forward(X0)
    torch.cuda.synchronize()
    assert rel_l2(host64(pooled), host64(single)) <= 1e-2
    st.close()
    for r in ranks:
        r.close()


def test_token_sharded_rejects_unsupported():
    from token_mixing_feature_b200 import rankmixer as rm
    from token_mixing_feature_b200 import tokshard
    wl = synth.Workload("tokshard", B=8, T=8, D=256, hidden=128, L=1)
    d = synth.make_inputs(wl)
    with pytest.raises(ValueError):
        tokshard.TokenShardedRank(wl, d["blocks"], 0, 3)        # T % world != 0
    r = tokshard.TokenShardedRank(wl, d["blocks"], 0, 2)
    z = torch.zeros(8 * 4 * 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RankMixerError) as e:                 # (D / G) % 8 != 0 for G = 64
        rm.rm_tokshard_pack(r.h, z, None, None, None, z, z, 8, 64)
    assert e.value.status == rm.RM_ERR_UNSUPPORTED
    r.close()
