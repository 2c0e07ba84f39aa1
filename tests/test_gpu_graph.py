"""A forward captured in a CUDA graph: replays give the stream-launch result,
and per-class timing events recorded inside the graph are read after replays."""
import pytest
import torch

import synth
import transformer_encoder_albert_b200 as tea

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_stream_forward_and_times_a_class():
    w = synth.make_weights(seed=1234, bf16=True)
    wl = synth.WORKLOADS["b8_T128"]
    ids, mask, L = synth.make_batch(wl)
    ids_d, mask_d = torch.as_tensor(ids).cuda(), torch.as_tensor(mask).cuda()
    enc = tea.Encoder(w, synth.ARCH, max_tokens=wl.B * wl.T)
    ref = enc.forward(ids_d, mask_d).clone()
    out = torch.empty_like(ref)
    enc.profile(["gemm_qkv"])
    enc.profile_retain(True)
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        enc.forward(ids_d, mask_d, out)
    g.replay()           # the captured events exist once a replay has recorded them
    enc.profile_reset()
    launches = []
    for _ in range(3):
        out.zero_()
        g.replay()
        launches.append(enc.profile_read()["gemm_qkv"])
    assert enc.status() == 0
    assert torch.equal(out, ref)
    # each replay adds the 12 Q|K|V launches recorded in the graph, with positive times
    assert [n for n, _ in launches] == [12, 24, 36]
    assert 0 < launches[0][1] < launches[1][1] < launches[2][1]
    enc.profile_retain(False)
    enc.profile([])
    del g
    enc.close()
