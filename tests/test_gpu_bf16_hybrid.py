"""GPU parity of the bf16 gated-delta path, the hybrid operator and the streaming step
against the CPU oracle, max-abs <= 2e-2 (bf16 I/O, fp32 accumulation, fp32 state)."""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _gdn_wl(B, H, L, decay=1.0):
    return hi.Workload("t", B=B, Hs=0, Hd=0, Hg=H, d=128, T=L, N=1, w_swa=1, w_dswa=1, r=1,
                       chunk=64, dtype="bf16", decay=decay)


@pytest.mark.parametrize("B,H,L,decay", [(1, 1, 64, 1.0), (2, 2, 150, 1.0), (1, 1, 1, 1.0),
                                         (1, 2, 1000, 0.05), (1, 1, 4097, 1.0)])
def test_gdn_bf16_full(h, orc, B, H, L, decay):
    wl = _gdn_wl(B, H, L, decay)
    x = hi.make_inputs(wl, seed=L + H)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    S0 = hi.random_state(B, H, 128, seed=3, scale=0.1)
    o, S = h.gdn(q, k, v, a, b, S0=dev(S0), out=poison_like(q))
    torch.cuda.synchronize()
    o_ref, S_ref = orc.gdn(x["q"], x["k"], x["v"], x["a"], x["b"], S0.double().numpy())
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(S, S_ref) <= TOL


@pytest.mark.parametrize("B,H,L,decay", [(1, 8, 32760, 1.0), (1, 2, 8360, 0.05)])
def test_gdn_bf16_segment_scan(h, orc, B, H, L, decay):
    """Heads long enough for the two-level scan: 480P's 8 heads of 512 chunks (16 segments
    of 32 chunks: segment maps, their composition and the replay), and 131 chunks in 5
    segments with a ragged last segment and a ragged last chunk under slow decay (the maps
    carry the start state far)."""
    wl = _gdn_wl(B, H, L, decay)
    x = hi.make_inputs(wl, seed=L + H)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    S0 = hi.random_state(B, H, 128, seed=4, scale=0.1)
    o, S = h.gdn(q, k, v, a, b, S0=dev(S0), out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    o_ref, S_ref = orc.gdn(x["q"], x["k"], x["v"], x["a"], x["b"], S0.double().numpy())
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(S, S_ref) <= TOL


def test_gdn_bf16_zero_gate_write_keeps_zero_state(h):
    """b = 0 from a zero state: the memory stays exactly zero (no write ever happens)."""
    wl = _gdn_wl(1, 1, 300)
    x = hi.make_inputs(wl, seed=1)
    q, k, v, a = (dev(x[n]) for n in "qkva")
    b = torch.zeros_like(a)
    o, S = h.gdn(q, k, v, a, b, out=poison_like(q))
    torch.cuda.synchronize()
    assert torch.count_nonzero(o) == 0 and torch.count_nonzero(S) == 0


def _hybrid_check(h, orc, wl, rows_count, seed=0):
    x = hi.make_inputs(wl, seed=seed)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    o = poison_like(q)
    o, S = h.hybrid(q, k, v, a, b, wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r,
                    out=o)
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert torch.isfinite(o).all()
    if rows_count is None:
        o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                                  wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
        assert maxabs(o, o_ref) <= TOL
        assert maxabs(S, S_ref) <= TOL
        return
    rows = hi.sample_rows(wl.L, wl.N, rows_count, seed=seed + 1).numpy()
    o_s, o_d, o_g, S_ref = orc.hybrid_rows(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs,
                                           wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r,
                                           rows)
    ridx = torch.from_numpy(rows).cuda()
    assert maxabs(o[:, :wl.Hs, ridx], o_s) <= TOL
    assert maxabs(o[:, wl.Hs:wl.Hs + wl.Hd, ridx], o_d) <= TOL
    assert maxabs(o[:, wl.Hs + wl.Hd:], o_g) <= TOL
    assert maxabs(S, S_ref) <= TOL


def test_hybrid_small_full(h, orc):
    wl = hi.Workload("t", B=2, Hs=1, Hd=2, Hg=1, d=128, T=6, N=100, w_swa=3, w_dswa=3, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    _hybrid_check(h, orc, wl, None, seed=4)


def test_hybrid_480p(h, orc):
    """The 480P workload (1x24 heads, T=21, N=1560): softmax heads on sampled rows, every
    GDN output and the final state in full."""
    _hybrid_check(h, orc, hi.WORKLOADS["480p"], 192)


def test_hybrid_480p_long_sampled(h, orc):
    """Long 480P rollout (T=61, DSWA w=4 r=6, slow decay a = exp(-0.05 softplus))."""
    _hybrid_check(h, orc, hi.WORKLOADS["480p_long"], 64)


def test_hybrid_720p_long_geometry_sampled(h, orc):
    """The 720P long rollout's geometry (T=61 frames of N=3600 tokens, L=219600: ragged key
    tiles, row indices past 2^17; SWA w=3, DSWA w=4 r=6) on two heads per branch: softmax heads
    on sampled rows, the GDN heads over the whole 219600-token recurrence."""
    wl = hi.WORKLOADS["720p_long"].with_(Hs=2, Hd=2, Hg=2)
    _hybrid_check(h, orc, wl, 48)


def test_stream_steps_equal_hybrid_bf16(h, orc):
    """Successive streaming steps from empty caches reproduce the hybrid operator on the
    concatenated clip (frame by frame) and its final state; rings wrap several times."""
    wl = hi.Workload("t", B=2, Hs=1, Hd=1, Hg=1, d=128, T=14, N=130, w_swa=3, w_dswa=4, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=9)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r)
    outs = []
    for f in range(wl.T):
        s = slice(f * wl.N, (f + 1) * wl.N)
        outs.append(st.step(q[:, :, s].contiguous(), k[:, :, s].contiguous(),
                            v[:, :, s].contiguous(), a[:, :, s].contiguous(),
                            b[:, :, s].contiguous()))
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=2)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    st.close()


def test_stream_steps_streaming_workload_geometry_sampled(h, orc):
    """The streaming workload's geometry: B=8 rollouts, frames of N=1560 tokens (key tiles
    end partly filled at every frame), SWA w=3, DSWA w=4 r=6 (a ring of r(w-1)+1 = 19 frame slots), d=128, one
    head per branch. 26 single-frame steps from empty caches, so every ring slot is reused and
    the last eight steps see all DSWA taps. Each step's softmax outputs on sampled rows of
    every frame, every GDN output and the final state are compared with the oracle's hybrid
    over the concatenated 26-frame clip."""
    wl = hi.WORKLOADS["stream_480p"].with_(Hs=1, Hd=1, Hg=1, T=26, streaming=False)
    assert wl.r * (wl.w_dswa - 1) + 1 == 19
    x = hi.make_inputs(wl, seed=41)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r)
    outs = []
    for f in range(wl.T):
        s = slice(f * wl.N, (f + 1) * wl.N)
        outs.append(st.step(q[:, :, s].contiguous(), k[:, :, s].contiguous(),
                            v[:, :, s].contiguous(), a[:, :, s].contiguous(),
                            b[:, :, s].contiguous(), out=poison_like(q[:, :, s].contiguous())))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    o = torch.cat(outs, dim=2)
    assert torch.isfinite(o).all()
    rows = hi.sample_rows(wl.L, wl.N, 256, seed=42).numpy()
    o_s, o_d, o_g, S_ref = orc.hybrid_rows(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs,
                                           wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r,
                                           rows)
    ridx = torch.from_numpy(rows).cuda()
    assert maxabs(o[:, :1, ridx], o_s) <= TOL
    assert maxabs(o[:, 1:2, ridx], o_d) <= TOL
    assert maxabs(o[:, 2:], o_g) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    st.close()


@pytest.mark.parametrize("groups", [(3, 1, 4, 2, 4), (1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1), (4, 4, 4, 2)])
def test_stream_multi_frame_steps_equal_hybrid_bf16(h, orc, groups):
    """Steps appending several frames per rollout at once (ragged group sizes, up to the
    cache's maximum) reproduce the hybrid operator on the concatenated clip."""
    wl = hi.Workload("t", B=2, Hs=1, Hd=1, Hg=1, d=128, T=sum(groups), N=130, w_swa=3, w_dswa=4,
                     r=2, chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=19)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r,
                  max_step_frames=max(groups))
    outs, f0 = [], 0
    for g in groups:
        s = slice(f0 * wl.N, (f0 + g) * wl.N)
        outs.append(st.step_frames(q[:, :, s].contiguous(), k[:, :, s].contiguous(),
                                   v[:, :, s].contiguous(), a[:, :, s].contiguous(),
                                   b[:, :, s].contiguous(), g))
        f0 += g
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert st.state()[1] == wl.T
    o = torch.cat(outs, dim=2)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    st.close()


def test_stream_step_frames_rejects_too_many_frames(h):
    wl = hi.Workload("t", B=1, Hs=1, Hd=1, Hg=1, d=128, T=3, N=64, w_swa=2, w_dswa=2, r=1,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=2)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r, max_step_frames=2)
    with pytest.raises(h.HltaError):
        st.step_frames(q, k, v, a, b, 3)
    assert st.state()[1] == 0                  # nothing was appended
    st.close()


def _frame_counter(st):
    ptr = st.frame_counter()

    class _View:
        __cuda_array_interface__ = {"shape": (1,), "typestr": "<i4", "data": (ptr, False),
                                    "version": 2}
    return int(torch.as_tensor(_View(), device="cuda").item())


def test_stream_step_graph_replay_equals_hybrid_bf16(h, orc):
    """A step captured once into a CUDA graph and replayed for successive frames (inputs
    written into the captured buffers before each replay), with eager steps before and after,
    reproduces the hybrid operator on the concatenated clip: the frame index the ring appends
    and the attention read comes from the cache's device counter, advanced by every replay."""
    F = 2
    wl = hi.Workload("t", B=2, Hs=1, Hd=1, Hg=1, d=128, T=16, N=130, w_swa=3, w_dswa=4, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=23)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r,
                  max_step_frames=F)

    def part(t, f0):
        return t[:, :, f0 * wl.N:(f0 + F) * wl.N].contiguous()

    outs = [st.step_frames(*(part(t, 0) for t in (q, k, v, a, b)), F)]     # eager, frames 0-1
    static = [part(t, 0).clone() for t in (q, k, v, a, b)]
    so = torch.empty_like(static[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        st.step_frames(*static, F, out=so)                                  # captured, not run
    assert _frame_counter(st) == F                                         # capture ran nothing
    f0 = F
    while f0 < wl.T - F:                                                   # replays, frames 2-13
        for buf, t in zip(static, (q, k, v, a, b)):
            buf.copy_(part(t, f0))
        g.replay()
        outs.append(so.clone())
        f0 += F
    outs.append(st.step_frames(*(part(t, f0) for t in (q, k, v, a, b)), F))  # eager again
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert _frame_counter(st) == wl.T
    o = torch.cat(outs, dim=2)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    del g
    st.close()


def test_hybrid_and_gdn_backward_graph_replay(h):
    """The hybrid forward (three branches on the library's fork/join streams) and the bf16 GDN
    backward (state passes on side streams) captured into CUDA graphs: replays reproduce the
    eager results bit for bit, after the inputs are rewritten in place."""
    wl = hi.Workload("t", B=1, Hs=1, Hd=1, Hg=1, d=128, T=5, N=200, w_swa=3, w_dswa=2, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x0, x1 = hi.make_inputs(wl, seed=31), hi.make_inputs(wl, seed=32)
    q, k, v, a, b = (dev(x0[n]) for n in "qkvab")
    gq, gk, gv = (t[:, 2:3].contiguous() for t in (q, k, v))
    ga, gb = a[:, :1].contiguous(), b[:, :1].contiguous()
    dO = torch.randn_like(gq)
    o = torch.empty_like(q)
    S = torch.empty((1, 1, 128, 128), device="cuda")
    wsh = torch.empty(h.hlta_hybrid_workspace_bytes(1, 1, wl.T, wl.N, 128, 64, h.HLTA_BF16),
                      dtype=torch.uint8, device="cuda")
    wsb = torch.empty(h.hlta_gdn_bwd_workspace_bytes(1, 1, wl.L), dtype=torch.uint8, device="cuda")
    grads = [torch.empty_like(gq) for _ in range(3)] + [torch.empty_like(ga) for _ in range(2)] + \
            [torch.empty_like(S)]

    def run():
        h.hlta_hybrid_fwd(q, k, v, a, b, o, None, S, 1, 1, 1, 1, wl.T, wl.N, 128, wl.w_swa,
                          wl.w_dswa, wl.r, 64, 0.0, wsh)
        h.hlta_gdn_chunk_bwd(gq, gk, gv, ga, gb, None, dO, None, *grads, 1, 1, wl.L, 128, 64, wsb)

    def snapshot():
        return [t.clone() for t in [o, S] + grads]

    run()
    torch.cuda.synchronize()
    eager0 = snapshot()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        run()
    for t in [o, S] + grads:
        t.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    for got, ref in zip(snapshot(), eager0):
        assert torch.equal(got, ref)
    # new inputs written into the captured buffers: the replay follows them
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (a, "a"), (b, "b")):
        t.copy_(dev(x1[n]))
    for t, src in ((gq, q[:, 2:3]), (gk, k[:, 2:3]), (gv, v[:, 2:3]), (ga, a[:, :1]), (gb, b[:, :1])):
        t.copy_(src)
    g.replay()
    torch.cuda.synchronize()
    replay1 = snapshot()
    run()
    torch.cuda.synchronize()
    for got, ref in zip(replay1, snapshot()):
        assert torch.equal(got, ref)
    del g


def test_stream_graph_replay_beside_other_attention(h, orc):
    """Replays of a captured streaming step run while 70 other window attention launches run
    on a second stream each time. Those launches cycle through the library's 64 shared work
    counters; the step's persistent attention uses the cache's own counter, so no launch takes
    another's units: the replayed frames reproduce the hybrid operator and every side launch
    reproduces its eager result bit for bit."""
    wl = hi.Workload("t", B=2, Hs=1, Hd=1, Hg=1, d=128, T=7, N=130, w_swa=3, w_dswa=4, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=41)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    side_wl = hi.Workload("s", B=1, Hs=0, Hd=2, Hg=0, d=128, T=3, N=300, w_swa=2, w_dswa=2, r=1,
                          chunk=64, dtype="bf16", decay=1.0)
    xs = hi.make_inputs(side_wl, seed=42)
    sq, sk, sv = (dev(xs[n]) for n in "qkv")
    side_ref = h.swa(sq, sk, sv, side_wl.T, side_wl.N, 2)
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r)

    def frame(t, f):
        return t[:, :, f * wl.N:(f + 1) * wl.N].contiguous()

    outs = [st.step(*(frame(t, 0) for t in (q, k, v, a, b)))]
    static = [frame(t, 0).clone() for t in (q, k, v, a, b)]
    so = torch.empty_like(static[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        st.step(*static, out=so)
    side = torch.cuda.Stream()
    side_outs = []
    for f in range(1, wl.T):
        for buf, t in zip(static, (q, k, v, a, b)):
            buf.copy_(frame(t, f))
        side.wait_stream(torch.cuda.current_stream())
        g.replay()
        with torch.cuda.stream(side):
            for _ in range(70):
                side_outs.append(h.swa(sq, sk, sv, side_wl.T, side_wl.N, 2, out=poison_like(sq)))
        outs.append(so.clone())
        torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    for o_side in side_outs:
        assert torch.equal(o_side, side_ref)
    o = torch.cat(outs, dim=2)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    del g
    st.close()
