"""Forward + backward captured into a CUDA graph: the library's calls are
stream-ordered (side streams joined by events, no host synchronisation), so a
captured step replays the whole path.  Replays are compared with eager calls bit
for bit (the kernels are deterministic), before and after the inputs change in
place."""
import pytest
import torch

import exact_relative_position_b200 as rp
from synth import small_workload

from relpos_harness import lmap, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    dict(map_kind="truncated", clip=16, N=300, B=2, H=2, terms=("aQ", "aK", "b"), key_len=[300, 171]),
    dict(map_kind="log", num_buckets=32, max_distance=128, N=384, B=1, H=3, terms=("aQ", "aK"),
         per_head_tables=True, causal=True),
    dict(map_kind="t5", num_buckets=32, max_distance=128, N=257, B=1, H=2, terms=("b",)),
]


def _step(w, dev, ws, outs):
    o, lse = outs[0], outs[1]
    rp.relpos_attn_fwd(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], tau=w.tau, map=lmap(w),
                       causal=w.causal, key_len=dev["key_len"], workspace=ws, o=o, lse=lse)
    rp.relpos_attn_bwd(dev["do"], dev["q"], dev["k"], dev["v"], o, lse, dev["aq"], dev["ak"], dev["b"], tau=w.tau,
                       map=lmap(w), causal=w.causal, key_len=dev["key_len"], workspace=ws, grads=tuple(outs[2:]),
                       reuse_forward=True)


def _buffers(w, dev):
    q = dev["q"]
    f32 = lambda t: None if t is None else torch.empty(t.shape, device="cuda", dtype=torch.float32)
    outs = [torch.empty_like(q), torch.empty(q.shape[:3], device="cuda", dtype=torch.float32),
            torch.empty_like(q), torch.empty_like(dev["k"]), torch.empty_like(dev["v"]),
            f32(dev["aq"]), f32(dev["ak"]), f32(dev["b"])]
    fws, bws = rp.workspace_size(q, dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w), causal=w.causal,
                                 key_len=dev["key_len"])
    return outs, torch.empty(max(fws, bws), device="cuda", dtype=torch.uint8)


def _snapshot(outs):
    return [None if t is None else t.clone() for t in outs]


def _same(a, b):
    for x, y in zip(a, b):
        assert (x is None) == (y is None)
        if x is not None:
            assert torch.equal(x, y)


@pytest.mark.parametrize("spec", CASES, ids=["shaw-padding", "deberta-causal", "t5-bias"])
def test_captured_step_replays_bit_exact(spec):
    w = small_workload(**spec)
    dev = to_dev(w)
    outs, ws = _buffers(w, dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                 # eager warm-up (creates the library's side streams)
        _step(w, dev, ws, outs)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = _snapshot(outs)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(w, dev, ws, outs)
    for t in outs:
        if t is not None:
            t.zero_()
    g.replay()
    torch.cuda.synchronize()
    _same(outs, eager)
    assert rp.check_workspace(ws) == 0

    # new values in the captured input buffers: the replay follows them
    gen = torch.Generator(device="cuda").manual_seed(11)
    for name in ("q", "k", "v", "do"):
        dev[name].copy_(torch.randn(dev[name].shape, device="cuda", generator=gen).to(dev[name].dtype))
    g.replay()
    torch.cuda.synchronize()
    replayed = _snapshot(outs)
    _step(w, dev, ws, outs)
    torch.cuda.synchronize()
    _same(replayed, outs)
    assert not torch.equal(replayed[0], eager[0])
