"""The call captured in a CUDA graph.

A caller that replays a fixed step (a serving loop, a training step) captures
deltanet_fwd once, after one call on the capturing stream has set up that
stream's workspace, and replays it: the replays must reproduce eager calls bit
for bit.  For packed input the schedule is built on the device from the
contents of cu_seqlens, so a replay after the boundaries changed (same number
of sequences, same total length) follows the new boundaries.
"""
import pytest
import torch

import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def to_dev(x):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def capture(g, out, fs, stream, seg_chunks):
    def call():
        dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"], g["cu_seqlens"],
                        out=out, final_state=fs, stream=stream, seg_chunks=seg_chunks)

    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        call()  # sets up this stream's workspace outside the capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    return graph


@pytest.mark.parametrize("seg_chunks", [0, 2])
def test_graph_replay_dense(seg_chunks):
    w = wl.custom(2, 700, 4, 128, 128, torch.bfloat16, init_state=True)
    g = to_dev(wl.generate(w, seed=3))
    ref_o, ref_s = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                                   seg_chunks=seg_chunks)
    torch.cuda.synchronize()
    out = torch.empty_like(ref_o)
    fs = torch.empty_like(ref_s)
    stream = torch.cuda.Stream(DEV)
    graph = capture(g, out, fs, stream, seg_chunks)
    for _ in range(2):
        out.zero_()
        fs.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o)
        assert torch.equal(fs, ref_s)
    assert dn.get_error(stream) == 0


def test_graph_replay_follows_new_seqlens():
    lens_a = (300, 1000, 64, 900)
    lens_b = (1000, 900, 300, 64)  # same count and total, other boundaries
    w = wl.custom(1, 0, 4, 128, 128, torch.bfloat16, init_state=True, seqlens=lens_a)
    g = to_dev(wl.generate(w, seed=4))
    cu_b = torch.tensor([0] + list(torch.tensor(lens_b).cumsum(0)), dtype=torch.int32, device=DEV)
    out = torch.empty(g["q"].shape[:3] + (128,), dtype=torch.bfloat16, device=DEV)
    fs = torch.empty((len(lens_a), 4, 128, 128), dtype=torch.float32, device=DEV)
    stream = torch.cuda.Stream(DEV)
    graph = capture(g, out, fs, stream, seg_chunks=3)
    for cu in (g["cu_seqlens"].clone(), cu_b):
        ref_o, ref_s = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"], cu,
                                       seg_chunks=3)
        torch.cuda.synchronize()
        g["cu_seqlens"].copy_(cu)
        out.zero_()
        fs.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o)
        assert torch.equal(fs, ref_s)
    assert dn.get_error(stream) == 0
