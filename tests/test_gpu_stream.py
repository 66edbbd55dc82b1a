"""Streaming checks (GPU): the pool's copy / reuse bookkeeping, the 30-layer
SmolLM2-shaped training run streamed at depth 2 and 3 against the HBM-resident run
(25 AdamW steps, loss curves and adapters bit-equal; first step against the oracle),
the poisoned-pool run, and the 32B-class layers above the 165 MiB aliasing threshold
whose LoRA gradients after buffer reuse must equal the resident gradients exactly.
These are the gate-record checks of "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.2 (streamed
= resident, n=2 = n=3, same-seed reruns, nonzero LoRA gradients in every layer) and the
Issue #331 scenario of the layer-streaming review's bug history."""
import ctypes
import os

import numpy as np
import pytest
import torch

from nf4_layer_streamed_b200 import api, binding as B, synth
from oracle import model as omodel
from tests.helpers import LOSS_RTOL, TOL, close, f64, oracle_lora, oracle_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_pool_copies_hits_and_slot_contents():
    shape = synth.SMOLLM2_135M
    cfg = api.layer_cfg(shape, 1, 512)
    nb = api.shard_bytes(cfg)
    slot = (nb + 255) // 256 * 256
    store = torch.empty(3 * slot, dtype=torch.uint8).pin_memory()
    for i in range(3):
        w = synth.layer_weights(shape, i, 1234, device=DEV)
        store[i * slot:i * slot + nb].copy_(api.nf4_quantize_shard(cfg, w).cpu())
    pool = api.Pool(store, [0, slot, 2 * slot], [nb] * 3, depth=2)
    try:
        seen = {}
        for i in range(3):                          # forward order
            p = pool.stream_prefetch(i)
            if i + 1 < 3:
                pool.prefetch(i + 1)
            seen[i] = pool.view(p, nb).clone()
            pool.release(i)
        for i in (2, 1, 0):                         # backward order
            p = pool.stream_prefetch(i)
            if i - 1 >= 0:
                pool.prefetch(i - 1)
            assert torch.equal(pool.view(p, nb).cpu(), store[i * slot:i * slot + nb])
            pool.release(i)
        torch.cuda.synchronize()
        for i in range(3):
            assert torch.equal(seen[i].cpu(), store[i * slot:i * slot + nb])
        assert pool.wait(0, 1000) == 0
        s = pool.stats()
        assert s["copies"] == 4 and s["bytes_copied"] == 4 * nb
        assert s["acquisitions"] == 6 and s["hits"] == 5
    finally:
        pool.destroy()


def test_pool_wait_times_out_while_the_slot_is_still_read():
    """A copy into a slot waits for the release event of the slot's last reader; a
    bounded host wait on that copy returns TIMEOUT while the reader is still busy
    (a GPU spin of about a second, which ends by itself) and OK afterwards."""
    shape = synth.SMOLLM2_135M
    cfg = api.layer_cfg(shape, 1, 512)
    nb = api.shard_bytes(cfg)
    slot = (nb + 255) // 256 * 256
    store = torch.zeros(3 * slot, dtype=torch.uint8).pin_memory()
    pool = api.Pool(store, [0, slot, 2 * slot], [nb] * 3, depth=2)
    try:
        pool.stream_prefetch(0)
        torch.cuda._sleep(2_000_000_000)      # the reader of layer 0 stays busy ~1 s
        pool.release(0)
        pool.stream_prefetch(1)
        pool.release(1)
        assert pool.prefetch(2) == 0          # goes into layer 0's slot, after its release
        assert pool.wait(2, 20) == -7         # TIMEOUT
        assert pool.wait(2, 10000) == 0
        torch.cuda.synchronize()
    finally:
        pool.destroy()


def _train(wl, depth, resident, steps, poison=False, b_random=False):
    m = api.StreamedModel(wl, depth=depth, resident=resident, b_random=b_random)
    if poison and m.pool is not None:
        m.pool.set_poison(True)
    losses, first_grads = [], None
    try:
        for s in range(steps):
            ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=s, device=DEV)
            m.forward_backward(ids)
            if s == 0:
                first_grads = m.grads.clone()
            losses.append(m.loss.clone())
            m.adamw_step()
        torch.cuda.synchronize()
        st, err = api.device_error()
        assert st == 0, err
        stats = m.pool.stats() if m.pool is not None else None
        return torch.cat(losses), m.lora.clone(), first_grads, m, stats
    finally:
        m.close()


def test_smollm2_30_layers_streamed_equals_resident_and_depths():
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    steps = wl.steps
    l_res, p_res, g_res, m, _ = _train(wl, 2, True, steps)
    l_2, p_2, g_2, _, st2 = _train(wl, 2, False, steps)
    l_3, p_3, g_3, _, _ = _train(wl, 3, False, steps)
    assert torch.equal(l_res, l_2) and torch.equal(l_2, l_3)
    assert torch.equal(p_res, p_2) and torch.equal(p_2, p_3)
    assert torch.equal(g_res, g_2) and torch.equal(g_2, g_3)
    l_again, p_again, _, _, _ = _train(wl, 2, False, steps)
    assert torch.equal(l_again, l_2) and torch.equal(p_again, p_2)
    # every layer is read twice per step, minus the layers the backward finds resident
    assert st2["copies"] <= 2 * wl.n_layers * steps
    # uniform random targets: the loss stays near ln V (nothing to learn), finite throughout
    assert torch.all(torch.isfinite(l_2))
    assert torch.all(torch.abs(l_2 - np.log(wl.vocab)) < 1.0)


def test_smollm2_30_layers_first_step_against_oracle():
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    shape = wl.shape
    m = api.StreamedModel(wl, depth=2, resident=False)
    try:
        ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=0, device=DEV)
        m.forward_backward(ids)
        torch.cuda.synchronize()
        loss_gpu = float(m.loss.item())
        grads = [m.grad_views(i) for i in range(wl.n_layers)]
        # B = 0 at initialisation: dB is nonzero in every layer, dA is exactly zero
        for g in grads:
            assert torch.count_nonzero(g["dB_q"]) > 0 and torch.count_nonzero(g["dB_v"]) > 0
            assert torch.count_nonzero(g["dA_q"]) == 0
        # the model drew its weights on the GPU: regenerate them there, then hand them to the oracle
        layers = [oracle_weights(synth.layer_weights(shape, i, wl.seed, device=DEV)) for i in range(wl.n_layers)]
        loras = [oracle_lora(synth.lora_params(shape, i, wl.seed)) for i in range(wl.n_layers)]
        emb = f64(m.embed)
        loss, og, _ = omodel.forward_backward(ids.cpu().numpy(), layers, loras, emb, None,
                                              np.ones(shape.hidden), shape, wl.batch, wl.seq, rnd=True)
        assert abs(loss_gpu - loss) <= LOSS_RTOL * abs(loss), (loss_gpu, loss)
        # through 30 layers the oracle's own bf16 roundings move the first layer's dB by
        # about 1.6% of max|ref| (its run with and without them); where twice that exceeds
        # 2e-2 it is the bound, as for the 8B two-layer model (tests/test_gpu_oracle_parity.py)
        _, ex, _ = omodel.forward_backward(ids.cpu().numpy(), layers, loras, emb, None,
                                           np.ones(shape.hidden), shape, wl.batch, wl.seq, rnd=False)
        for i in (0, wl.n_layers - 1):
            for k in ("dB_q", "dB_v"):
                floor = float(np.max(np.abs(og[i][k] - ex[i][k])))
                tol = max(TOL, 2.0 * floor / float(np.max(np.abs(og[i][k]))))
                close(grads[i][k], og[i][k], tol, what=f"layer {i} {k} (noise floor {floor:.3e})")
        # second step: B is now nonzero, so dA is nonzero in every layer
        m.adamw_step()
        ids2 = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=1, device=DEV)
        m.forward_backward(ids2)
        torch.cuda.synchronize()
        for i in range(wl.n_layers):
            assert torch.count_nonzero(m.grad_views(i)["dA_q"]) > 0, i
    finally:
        m.close()


def test_adapter_off_reference_pass():
    """The DPO/KTO reference model is the same streamed base with the adapter off
    ("Soup v0.72.4 技术解析" §3.1): nf4ls_forward_loss(lora_on = 0) over the streamed
    layers equals the resident run bit for bit, differs from the adapter-on loss when
    B is nonzero, and matches the oracle's adapter-free forward."""
    wl = synth.Workload("smollm2_4L_tied", synth.SMOLLM2_135M, 4, 1, 512, vocab=49152, tied=True)
    m_res = api.StreamedModel(wl, resident=True, b_random=True)
    m_str = api.StreamedModel(wl, depth=2, resident=False, b_random=True)
    try:
        ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=0, device=DEV)
        off_res = m_res.forward_loss(ids, lora_on=False).clone()
        off_str = m_str.forward_loss(ids, lora_on=False).clone()
        on_str = m_str.forward_loss(ids, lora_on=True).clone()
        torch.cuda.synchronize()
        assert torch.equal(off_res, off_str)
        assert not torch.equal(off_str, on_str)
        shape = wl.shape
        layers = [oracle_weights(synth.layer_weights(shape, i, wl.seed, device=DEV)) for i in range(wl.n_layers)]
        loss, _, _ = omodel.forward_backward(ids.cpu().numpy(), layers, [None] * wl.n_layers, f64(m_str.embed), None,
                                             np.ones(shape.hidden), shape, wl.batch, wl.seq, rnd=True)
        assert abs(float(off_str.item()) - loss) <= LOSS_RTOL * abs(loss)
    finally:
        m_res.close()
        m_str.close()


def test_poisoned_pool_still_equals_resident():
    wl = synth.Workload("smollm2_6L_tied", synth.SMOLLM2_135M, 6, 1, 512, vocab=49152, tied=True)
    l_res, p_res, _, _, _ = _train(wl, 2, True, 3, b_random=True)
    l_poi, p_poi, _, _, _ = _train(wl, 2, False, 3, poison=True, b_random=True)
    assert torch.equal(l_res, l_poi) and torch.equal(p_res, p_poi)


def _stack_grads(shape, n_layers, batch, seq, depth, resident, poison=False):
    cfg = api.layer_cfg(shape, batch, seq)
    nb = api.shard_bytes(cfg)
    slot = (nb + 255) // 256 * 256
    shards = []
    if resident:
        buf = torch.empty(n_layers * slot, dtype=torch.uint8, device=DEV)
    else:
        store = torch.empty(n_layers * slot, dtype=torch.uint8).pin_memory()
    for i in range(n_layers):
        w = synth.layer_weights(shape, i, 1234, device=DEV)
        if resident:
            api.nf4_quantize_shard(cfg, w, out=buf[i * slot:(i + 1) * slot])
            shards.append(buf[i * slot:(i + 1) * slot])
        else:
            store[i * slot:i * slot + nb].copy_(api.nf4_quantize_shard(cfg, w).cpu())
        del w
    pool = None if resident else api.Pool(store, [i * slot for i in range(n_layers)], [nb] * n_layers, depth)
    if pool is not None and poison:
        pool.set_poison(True)

    def get(i, nxt):
        if resident:
            return shards[i]
        p = pool.stream_prefetch(i)
        if 0 <= nxt < n_layers:
            pool.prefetch(nxt)
        return pool.view(p, nb)

    try:
        ws = api.LayerWorkspace(cfg)
        loras = [synth.lora_params(shape, i, 1234, b_random=True, device=DEV) for i in range(n_layers)]
        xs = [synth.hidden_states(shape, batch, seq, 1234, device=DEV).view(batch * seq, shape.hidden)]
        for i in range(n_layers):
            s = get(i, i + 1)
            xs.append(api.layer_forward(cfg, s, loras[i], xs[-1], ws))
            if pool:
                pool.release(i)
        _, dy = api.mse_loss(xs[-1])
        grads = [None] * n_layers
        for i in range(n_layers - 1, -1, -1):
            s = get(i, i - 1)
            dy, grads[i] = api.layer_backward(cfg, s, loras[i], xs[i], dy, ws)
            if pool:
                pool.release(i)
        torch.cuda.synchronize()
        return grads, dy
    finally:
        if pool is not None:
            pool.destroy()


def test_32b_class_layers_over_165mib_gradients_after_reuse_equal_resident():
    wl = synth.WORKLOADS["qwen32b_4L_b1s1024"]
    shape = wl.shape
    assert api.shard_bytes(api.layer_cfg(shape, 1, 1024)) > 165 * 2 ** 20
    g_res, dx_res = _stack_grads(shape, wl.n_layers, wl.batch, wl.seq, 2, True)
    g_str, dx_str = _stack_grads(shape, wl.n_layers, wl.batch, wl.seq, 2, False, poison=True)
    assert torch.equal(dx_res, dx_str)
    for i in range(wl.n_layers):
        for k in g_res[i]:
            assert torch.equal(g_res[i][k], g_str[i][k]), (i, k)
            assert torch.count_nonzero(g_res[i][k]) > 0
    st, err = api.device_error()
    assert st == 0, err


def test_adapter_checkpoint_resume_is_bit_exact(tmp_path):
    """Six streamed steps in one run equal three steps, a save, a new model that
    loads the file and three more steps: losses, adapter and both AdamW moments
    bit-equal ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §3.2: an adapter that was
    saved must come back, not load as a no-op)."""
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    ids = [synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=s, device=DEV) for s in range(6)]

    def run(m, steps):
        out = []
        for s in steps:
            out.append(m.train_step(ids[s]).clone())
        torch.cuda.synchronize()
        return out

    m = api.StreamedModel(wl, depth=2, resident=False, b_random=True)
    try:
        l_full = run(m, range(6))
        full = (m.lora.clone(), m.adam_m.clone(), m.adam_v.clone(), m.step_count)
    finally:
        m.close()

    path = str(tmp_path / "adapter.bin")
    m = api.StreamedModel(wl, depth=2, resident=False, b_random=True)
    try:
        l_a = run(m, range(3))
        m.save_adapter(path)
        saved = m.lora.clone()
    finally:
        m.close()
    assert os.path.getsize(path) == B.lib().nf4ls_adapter_file_bytes(ctypes.byref(m.cfg))

    m = api.StreamedModel(wl, depth=2, resident=False, b_random=True)
    try:
        assert not torch.equal(m.lora, saved)   # a fresh adapter: loading must change it
        assert m.load_adapter(path) == 3
        assert torch.equal(m.lora, saved)
        l_b = run(m, range(3, 6))
        resumed = (m.lora.clone(), m.adam_m.clone(), m.adam_v.clone(), m.step_count)
        st, err = api.device_error()
        assert st == 0, err
    finally:
        m.close()
    assert torch.equal(torch.cat(l_full), torch.cat(l_a + l_b))
    for a, b in zip(full[:3], resumed[:3]):
        assert torch.equal(a, b)
    assert full[3] == resumed[3] == 6
    assert torch.count_nonzero(full[2]) > 0


def test_step_log_on_the_streamed_run(tmp_path):
    """The per-step log of a streamed run: one line per step, the step's copies
    (every layer read, some backward reads served by the slot still holding it), the
    loss the step returned, the event time and phases with library profiling on."""
    import json
    from nf4_layer_streamed_b200 import steplog
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    m = api.StreamedModel(wl, depth=2, resident=False)
    path = str(tmp_path / "steps.jsonl")
    api.profile(True)
    try:
        log = steplog.StepLog(m, path, tokens_per_step=wl.batch * wl.seq)
        losses = []
        for s in range(2):
            ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=s, device=DEV)
            losses.append(log.step(ids)["loss"])
        log.close()
    finally:
        api.profile(False)
        api.profile_reset()
        m.close()
    recs = [json.loads(l) for l in open(path)]
    assert [r["step"] for r in recs] == [1, 2]
    for r, l in zip(recs, losses):
        assert r["loss"] == l and np.isfinite(l)
        assert r["step_ms"] > 0 and r["peak_mem_bytes"] > 0
        assert wl.n_layers <= r["copies"] <= 2 * wl.n_layers
        assert 0 < r["hits"] <= 2 * wl.n_layers   # prefetched or still-resident layers
        assert r["h2d_bytes"] >= r["copies"] * api.shard_bytes(m.cfg.layer)
        assert set(r["phases_ms"]) >= {"layers_forward", "layers_backward"}


def test_llama8b_32_layers_b4s512_streamed_equals_resident():
    """The bench workload at full size (32 Llama-8B-shaped layers, untied vocab 128256,
    batch 4 x 512), streamed at depth 2 as the bench times it, against every shard
    resident in HBM: two AdamW steps with bit-equal losses, LoRA gradients and adapters;
    the loss at initialisation sits near ln V (uniform targets)."""
    wl = synth.WORKLOADS["llama8b_32L_b4s512"]
    out = {}
    for resident in (False, True):
        m = api.StreamedModel(wl, depth=2, resident=resident)
        try:
            losses = []
            for s in range(2):
                ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=s, device=DEV)
                m.forward_backward(ids)
                losses.append(m.loss.clone())
                m.adamw_step()
            torch.cuda.synchronize()
            st, err = api.device_error()
            assert st == 0, err
            out[resident] = (torch.cat(losses), m.grads.clone(), m.lora.clone())
        finally:
            m.close()
    for a, b in zip(out[False], out[True]):
        assert torch.equal(a, b)
    l0 = float(out[False][0][0])
    assert np.isfinite(l0) and abs(l0 - np.log(wl.vocab)) < 1.0
