"""C-ABI library checks that need no GPU: the library loads, exports every symbol the
header declares, builds code tables equal to the oracle's, sizes shards by the byte
identity, and refuses bad headers, sizes and pool depths on the host."""
import ctypes
import os
import re

import numpy as np
import pytest

from nf4_layer_streamed_b200 import api, binding as B, synth
from oracle import account, codebooks

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nf4ls.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\([^;{]*\)\s*;", text)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    declared = _declared_functions()
    assert len(declared) >= 30
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(B.SIGNATURES), set(declared) ^ set(B.SIGNATURES)


def test_code_tables_equal_oracle_bit_for_bit():
    nf4, c8, h = api.codebooks()
    assert np.array_equal(nf4.view(np.uint32), codebooks.nf4_table().view(np.uint32))
    assert np.array_equal(c8.view(np.uint32), codebooks.code8_table().view(np.uint32))
    assert h == codebooks.codebook_hash()


@pytest.mark.parametrize("shape", [synth.SMOLLM2_135M, synth.LLAMA_8B, synth.QWEN_32B_CLASS])
def test_shard_sizes_follow_byte_identity(shape):
    cfg = api.layer_cfg(shape, 1, 512)
    assert api.shard_quantized_bytes(cfg) == account.layer_shard_bytes(shape)
    total = api.shard_bytes(cfg)
    # header + descriptors + 256-byte alignment of 30 regions + two bf16 norm vectors
    assert account.layer_shard_bytes(shape) < total <= account.layer_shard_bytes(shape) + 1024 + 30 * 256 + \
        4 * shape.hidden + 512


def _header(cfg, fp=7, magic=0x5334464E, version=1, chash=None):
    h = np.zeros(1024, np.uint8)
    u32 = h[:48].view(np.uint32)
    u32[:] = [magic, version, 1, 64, 256, 9, cfg.hidden, cfg.inter, cfg.n_q, cfg.n_kv, cfg.head_dim, 0]
    u64 = h[48:80].view(np.uint64)
    u64[0] = codebooks.codebook_hash() if chash is None else chash
    u64[1] = fp
    u64[2] = api.shard_bytes(cfg)
    return h


def test_shard_header_checks():
    cfg = api.layer_cfg(synth.SMOLLM2_135M, 1, 512)
    ok = _header(cfg)
    st = B.call_status("nf4ls_shard_check", ok.ctypes.data, ctypes.byref(cfg), 7)
    assert st == B.OK, B.last_error()
    assert B.call_status("nf4ls_shard_check", ok.ctypes.data, ctypes.byref(cfg), 8) == -5   # fingerprint
    bad = _header(cfg, chash=123)
    assert B.call_status("nf4ls_shard_check", bad.ctypes.data, ctypes.byref(cfg), 0) == -4  # code tables
    bad = _header(cfg, magic=0)
    assert B.call_status("nf4ls_shard_check", bad.ctypes.data, ctypes.byref(cfg), 0) == -1
    other = api.layer_cfg(synth.LLAMA_8B, 1, 512)
    assert B.call_status("nf4ls_shard_check", ok.ctypes.data, ctypes.byref(other), 0) == -2  # shape


def test_pool_rejects_bad_depth_and_sizes_without_touching_a_gpu():
    store = np.zeros(4096, np.uint8)
    offs = (ctypes.c_size_t * 2)(0, 2048)
    sizes = (ctypes.c_size_t * 2)(1024, 1024)
    out = ctypes.c_void_p()
    fake_dev = ctypes.c_void_p(1 << 20)  # never dereferenced: arguments are rejected first
    for depth in (1, 9):
        st = B.call_status("nf4ls_pool_create", store.ctypes.data, ctypes.cast(offs, ctypes.c_void_p),
                           ctypes.cast(sizes, ctypes.c_void_p), 2, depth, fake_dev, 2048, ctypes.byref(out))
        assert st == -1 and "depth" in B.last_error()
    st = B.call_status("nf4ls_pool_create", store.ctypes.data, ctypes.cast(offs, ctypes.c_void_p),
                       ctypes.cast(sizes, ctypes.c_void_p), 2, 2, fake_dev, 512, ctypes.byref(out))
    assert st == -1 and "exceeds slot" in B.last_error()
    st = B.call_status("nf4ls_pool_create", store.ctypes.data, ctypes.cast(offs, ctypes.c_void_p),
                       ctypes.cast(sizes, ctypes.c_void_p), 2, 2, ctypes.c_void_p((1 << 20) + 8), 2048,
                       ctypes.byref(out))
    assert st == -3


def test_workspace_queries_and_options():
    cfg = api.layer_cfg(synth.LLAMA_8B, 4, 512)
    assert B.lib().nf4ls_workspace_bytes(ctypes.byref(cfg)) > 0
    assert B.lib().nf4ls_lora_stride(ctypes.byref(cfg)) == 16 * (2 * 4096 + 4096 + 1024)
    assert B.call_status("nf4ls_set_gemm_path", 3) == -1
    assert B.call_status("nf4ls_set_gemm_path", 0) == 0
    assert B.lib().nf4ls_quantize_scratch_bytes(64 * 1000) >= 4000


def test_layer_calls_validate_config_on_host():
    cfg = api.layer_cfg(synth.SMOLLM2_135M, 1, 512)
    cfg.head_dim = 96
    st = B.call_status("layer_forward", ctypes.byref(cfg), ctypes.c_void_p(256), None, ctypes.c_void_p(256),
                       ctypes.c_void_p(256), ctypes.c_void_p(256), 1 << 30, None)
    assert st == -2


def test_streamed_head_config_checked_on_host():
    """The model refuses a streamed head whose chunk is not a multiple of 64 rows, or
    that has no head pool, before it touches any buffer."""
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    fake = ctypes.c_void_p(256)
    for rows, pool, want in ((100, fake, -2), (8192, None, -1)):
        cfg = B.ModelCfg(api.layer_cfg(wl.shape, wl.batch, wl.seq), wl.n_layers, wl.vocab, 1, 2e-4, 0.9, 0.999,
                         1e-8, 0.0, rows)
        ws = B.lib().nf4ls_model_workspace_bytes(ctypes.byref(cfg))
        m = B.Model(None, None, 256, 256, 256, 256, 256, 256, None, 256, ws, pool, 256)
        st = B.call_status("nf4ls_forward_loss", ctypes.byref(cfg), ctypes.byref(m), fake, 1, fake, None)
        assert st == want, (rows, st)
    # the streamed head needs one vocab chunk of logits, not all of them
    cfg_res = B.ModelCfg(api.layer_cfg(wl.shape, wl.batch, wl.seq), wl.n_layers, wl.vocab, 1, 2e-4, 0.9, 0.999,
                         1e-8, 0.0, 0)
    cfg_str = B.ModelCfg(api.layer_cfg(wl.shape, wl.batch, wl.seq), wl.n_layers, wl.vocab, 1, 2e-4, 0.9, 0.999,
                         1e-8, 0.0, 8192)
    res = B.lib().nf4ls_model_workspace_bytes(ctypes.byref(cfg_res))
    strm = B.lib().nf4ls_model_workspace_bytes(ctypes.byref(cfg_str))
    assert strm < res


def test_layer_sharded_fetch_arguments_on_host():
    nid = api.nccl_unique_id()
    assert len(nid) == 128 and any(nid)
    buf = (ctypes.c_uint8 * 128).from_buffer_copy(nid)
    idp = ctypes.cast(buf, ctypes.c_void_p)
    assert B.call_status("nf4ls_pool_share", None, 0, 2, idp) == -1
    assert B.call_status("nf4ls_pool_share", ctypes.c_void_p(256), 2, 2, idp) == -1
    assert B.call_status("nf4ls_pool_share", ctypes.c_void_p(256), 0, 0, idp) == -1


def _fnv1a64(data: bytes) -> int:
    h = 0xCBF29CE484222325
    for b in data:
        h = ((h ^ b) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def test_adapter_load_refuses_bad_files_before_touching_the_device(tmp_path):
    """An adapter file that is not exactly what this model saved is refused on the
    host, before any copy to the (here fake) device pointers: wrong magic or version,
    another shape or alpha, a short, over-long or corrupted body, a missing file."""
    import struct
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    lc = api.layer_cfg(wl.shape, wl.batch, wl.seq)
    n_layers = 2
    cfg = B.ModelCfg(lc, n_layers, wl.vocab, 1, 2e-4, 0.9, 0.999, 1e-8, 0.0, 0)
    stride = B.lib().nf4ls_lora_stride(ctypes.byref(lc))
    n = n_layers * stride
    assert B.lib().nf4ls_adapter_file_bytes(ctypes.byref(cfg)) == 64 + 12 * n
    assert B.lib().nf4ls_adapter_file_bytes(None) == 0
    m = B.Model(256, None, 256, 256, 256, 256, 256, 256, None, 256, 0, None, None)
    body = np.arange(3 * n, dtype=np.float32).tobytes()

    def header(**kw):
        # the checksum covers the header (checksum field zero) and then the body
        f = dict(magic=0x41344E46, version=2, hidden=lc.hidden, inter=lc.inter, n_q=lc.n_q, n_kv=lc.n_kv,
                 head_dim=lc.head_dim, r=lc.lora_r, layers=n_layers, alpha=lc.lora_alpha, step=7, n=n,
                 csum=None)
        f.update(kw)

        def pack(c):
            return struct.pack("<IIiiiiiiifiIQQ", f["magic"], f["version"], f["hidden"], f["inter"], f["n_q"],
                               f["n_kv"], f["head_dim"], f["r"], f["layers"], f["alpha"], f["step"], 0, f["n"], c)
        return pack(_fnv1a64(pack(0) + body) if f["csum"] is None else f["csum"])

    csum = _fnv1a64(header(csum=0) + body)

    assert len(header()) == 64
    step = ctypes.c_int32(-1)
    cases = [
        ("magic", header(magic=0x12345678) + body, -1),
        ("version", header(version=3) + body, -1),
        ("hidden", header(hidden=lc.hidden * 2) + body, -2),
        ("rank", header(r=lc.lora_r * 2) + body, -2),
        ("alpha", header(alpha=lc.lora_alpha + 1) + body, -2),
        ("layers", header(layers=n_layers + 1) + body, -2),
        ("count", header(n=n - 1) + body, -2),
        ("short_header", header()[:40], -11),
        ("truncated", header() + body[:-4], -11),
        ("trailing", header() + body + b"\0", -11),
        ("corrupt", header() + body[:-1] + bytes([body[-1] ^ 1]), -11),
        ("checksum", header(csum=csum ^ 1) + body, -11),
        # a damaged step (still >= 0) or alpha with the checksum of the intact header
        ("step", header(step=8, csum=csum) + body, -11),
        ("version1", header(version=1) + body, -1),
    ]
    assert header(csum=None) == header(csum=csum)
    for name, blob, want in cases:
        p = tmp_path / f"{name}.adapter"
        p.write_bytes(blob)
        st = B.call_status("nf4ls_adapter_load", os.fsencode(str(p)), ctypes.byref(cfg), ctypes.byref(m),
                           ctypes.byref(step), None)
        assert st == want, (name, st, B.last_error())
        assert step.value == -1, name
    missing = os.fsencode(str(tmp_path / "missing.adapter"))
    assert B.call_status("nf4ls_adapter_load", missing, ctypes.byref(cfg), ctypes.byref(m), ctypes.byref(step),
                         None) == -11
    # null arguments
    good = tmp_path / "good.adapter"
    good.write_bytes(header() + body)
    g = os.fsencode(str(good))
    assert B.call_status("nf4ls_adapter_load", g, ctypes.byref(cfg), ctypes.byref(m), None, None) == -1
    assert B.call_status("nf4ls_adapter_load", None, ctypes.byref(cfg), ctypes.byref(m), ctypes.byref(step),
                         None) == -1
    no_moments = B.Model(256, None, 256, 256, 256, None, 256, 256, None, 256, 0, None, None)
    assert B.call_status("nf4ls_adapter_load", g, ctypes.byref(cfg), ctypes.byref(no_moments), ctypes.byref(step),
                         None) == -1
    assert B.call_status("nf4ls_adapter_save", g, ctypes.byref(cfg), ctypes.byref(m), -1, None) == -1


def test_wait_probe_refuses_bad_arguments_on_the_host():
    # the limits are checked before any device work, so these run without a GPU
    for limit in (0, -5, 1_000_001):
        assert B.call_status("nf4ls_wait_probe", limit, ctypes.c_void_p(256), None) == -1, limit
    assert B.call_status("nf4ls_wait_probe", 1000, None, None) == -1
    assert "limit_us" in B.last_error()
