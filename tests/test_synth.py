"""The seeded input generators (no GPU): reproducible, the stated distributions and
shapes, and the workload dimensions the configurations name."""
import torch

from nf4_layer_streamed_b200 import synth


def test_generators_are_reproducible_and_layer_streams_independent():
    s = synth.TINY
    a, b = synth.layer_weights(s, 3, 7), synth.layer_weights(s, 3, 7)
    assert all(torch.equal(a[k], b[k]) for k in a)
    c = synth.layer_weights(s, 4, 7)
    assert not torch.equal(a["q"], c["q"])
    assert torch.equal(synth.token_ids(100, 2, 9, 5, step=1), synth.token_ids(100, 2, 9, 5, step=1))
    assert not torch.equal(synth.token_ids(100, 2, 9, 5, step=1), synth.token_ids(100, 2, 9, 5, step=2))


def test_stated_distributions():
    s = synth.LLAMA_8B
    w = synth.layer_weights(s, 0, 1234)
    assert w["q"].dtype == torch.bfloat16 and tuple(w["q"].shape) == (s.q_dim, s.hidden)
    q = w["q"].float()
    assert abs(q.std().item() - 0.02) < 0.0005 and abs(q.mean().item()) < 1e-4
    assert torch.equal(w["norm_in"], torch.ones(s.hidden, dtype=torch.bfloat16))
    lo = synth.lora_params(s, 0, 1234)
    assert lo["A_q"].dtype == torch.float32 and abs(lo["A_q"].std().item() - 0.02) < 0.001
    assert torch.count_nonzero(lo["B_q"]) == 0 and torch.count_nonzero(lo["B_v"]) == 0
    lr = synth.lora_params(s, 0, 1234, b_random=True)
    assert torch.count_nonzero(lr["B_q"]) == lr["B_q"].numel() and torch.equal(lr["A_q"], lo["A_q"])
    x = synth.hidden_states(s, 1, 512, 1234).float()
    assert abs(x.std().item() - 1.0) < 0.01
    ids = synth.token_ids(128256, 4, 512, 1234)
    assert ids.dtype == torch.int32 and int(ids.min()) >= 0 and int(ids.max()) < 128256
    assert len(torch.unique(ids)) > 1900   # 2048 draws from 128256 values: few repeats


def test_workload_dimensions():
    s8 = synth.LLAMA_8B
    assert (s8.hidden, s8.inter, s8.n_q, s8.n_kv, s8.head_dim) == (4096, 14336, 32, 8, 128)
    assert s8.n_params() == 218103808      # seven frozen linears of one Llama-8B layer
    wl = synth.WORKLOADS["llama8b_32L_b4s512"]
    assert (wl.n_layers, wl.batch, wl.seq, wl.vocab, wl.tied, wl.tokens) == (32, 4, 512, 128256, False, 2048)
    ws = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    assert (ws.n_layers, ws.vocab, ws.tied, ws.shape.hidden, ws.shape.head_dim) == (30, 49152, True, 576, 64)
    s32 = synth.WORKLOADS["qwen32b_4L_b1s1024"].shape
    assert (s32.hidden, s32.inter, s32.n_q, s32.n_kv) == (5120, 27648, 40, 8)
