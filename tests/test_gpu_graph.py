"""The forward can be captured in a CUDA graph: its launch path makes no
synchronising or allocating call once a device is initialised, so replays
give the eager results bit for bit (static and dynamic schedules, the
dynamic one clearing its work counter inside the graph)."""

import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_122_b200 as m
    from exact_attention_122_b200 import build
    build.build()
    return m


@pytest.mark.parametrize("schedule", ["static", "dynamic"])
@pytest.mark.parametrize("shape", [(2, 3, 300, 128, True), (1, 5, 513, 64, False)],
                         ids=["d128c", "d64"])
def test_graph_replay_matches_eager(fa, schedule, shape):
    B, H, N, d, causal = shape
    q, k, v = (t.cuda() for t in synth.draw_qkv(B, H, N, d, seed=4400 + N))
    scale = 1 / math.sqrt(d)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()    # the inputs were copied on the default stream
    o_ref, l_ref = fa.fa_fwd(q, k, v, causal=causal, scale=scale, stream=s, schedule=schedule)
    s.synchronize()
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(3):      # several launches: the dynamic counter is cleared before each
            fa.fa_fwd(q, k, v, causal=causal, scale=scale, out=o, lse=lse, stream=s,
                      schedule=schedule)
    for _ in range(2):
        with torch.cuda.stream(s):
            o.zero_()
            lse.zero_()
            g.replay()
        s.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    st, word = fa.device_status(s.cuda_stream)
    assert st == fa.FA_OK, (fa.status_string(st), hex(word))
    del g
