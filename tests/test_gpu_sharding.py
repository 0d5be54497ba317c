"""Sharding on one GPU: each rank's share computed in turn with the library's kernels, then
reassembled as the gather would; checked against the unsharded call and the oracle."""
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def test_head_shares_reassemble_to_the_hybrid(orc):
    import linear_video_world_b200 as h
    from linear_video_world_b200.sharding import assemble_heads, global_heads, head_plan
    wl = hi.Workload("t", B=2, Hs=3, Hd=2, Hg=3, d=128, T=4, N=150, w_swa=3, w_dswa=2, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=61)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    world = 3
    plan = head_plan(wl.Hs, wl.Hd, wl.Hg, world)
    parts, states = [], []
    for pr in plan:                      # the work of rank r, on this GPU
        (s0, ns), (d0, nd), (g0, ng) = pr
        idx = torch.tensor(global_heads(pr, wl.Hs, wl.Hd), device="cuda")
        gi = torch.arange(g0, g0 + ng, device="cuda")
        o, S = h.hybrid(q.index_select(1, idx).contiguous(), k.index_select(1, idx).contiguous(),
                        v.index_select(1, idx).contiguous(), a.index_select(1, gi).contiguous(),
                        b.index_select(1, gi).contiguous(), ns, nd, ng, wl.T, wl.N, wl.w_swa,
                        wl.w_dswa, wl.r)
        parts.append(o)
        states.append(S)
    o_full = assemble_heads(parts, plan, wl.Hs, wl.Hd)
    S_full = torch.cat(states, dim=1)
    torch.cuda.synchronize()
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg, wl.T,
                              wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o_full, o_ref) <= TOL
    assert maxabs(S_full, S_ref) <= TOL
    # the unsharded call gives the same values up to rounding
    o1, S1 = h.hybrid(q, k, v, a, b, wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    torch.cuda.synchronize()
    assert float((o1.float() - o_full.float()).abs().max()) <= TOL


def test_rollout_shares_equal_one_cache():
    """Rollouts are independent: two caches holding rollouts [0, 2) and [2, 5) give exactly the
    outputs and states of one 5-rollout cache."""
    import linear_video_world_b200 as h
    wl = hi.Workload("t", B=5, Hs=1, Hd=1, Hg=1, d=128, T=6, N=130, w_swa=3, w_dswa=3, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=62)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    full = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r)
    shares = [(0, 2), (2, 3)]
    parts = [h.Stream(n, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r) for _, n in shares]
    for f in range(wl.T):
        s = slice(f * wl.N, (f + 1) * wl.N)
        o_full = full.step(*(t[:, :, s].contiguous() for t in (q, k, v, a, b)))
        o_parts = [st.step(*(t[b0:b0 + n, :, s].contiguous() for t in (q, k, v, a, b)))
                   for (b0, n), st in zip(shares, parts)]
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(o_parts, dim=0), o_full), f
    assert torch.equal(torch.cat([st.state_tensor() for st in parts], dim=0), full.state_tensor())
    for st in parts + [full]:
        st.close()
