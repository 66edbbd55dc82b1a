"""Python face of libnf4ls: the C-ABI calls with torch tensors as buffers.

Marshalling only: torch allocates device and pinned memory and supplies streams;
every computation is a call into libnf4ls.so (binding.py).  Function names follow
the C ABI (include/nf4ls.h): nf4_quantize_shard, layer_forward, layer_backward,
stream_prefetch and the pool, model and building-block calls.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

from . import binding as B
from .synth import LayerShape, Workload

LAYER_TENSORS = ("q", "k", "v", "o", "gate", "up", "down", "norm_in", "norm_post")


def _p(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _s(stream=None) -> ctypes.c_void_p:
    st = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(st.cuda_stream)


def _aligned(t: torch.Tensor, a: int = 256) -> torch.Tensor:
    assert t.data_ptr() % a == 0, "buffer is not aligned"
    return t


def _buffer(nbytes: int, device="cuda") -> torch.Tensor:
    return _aligned(torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device))


# The library takes raw device pointers and cannot see a wrong dtype, size, layout or
# device itself, so each call below first checks every tensor's dtype, size and layout,
# then that all of them live on a CUDA device, and only then passes the pointers.
def _need(t, name: str, dtype, numel: int | None = None, contiguous: bool = True) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t


def _need_rows(t, name: str, rows: int, ld: int, width: int) -> torch.Tensor:
    """A bf16 row-major view of `rows` rows of `width` elements, `ld` elements apart."""
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.dim() != 2:
        raise ValueError(f"{name}: expected a 2-D bf16 tensor")
    if t.shape[0] < rows or t.shape[1] < width or t.stride(1) != 1 or (rows > 1 and t.stride(0) != ld):
        raise ValueError(f"{name}: shape {tuple(t.shape)} / strides {t.stride()} do not hold {rows} rows "
                         f"of {width} elements {ld} apart")
    return t


def _need_cuda(**tensors) -> None:
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name}: must be a CUDA tensor")


def _need_shard(shard, cfg: B.LayerCfg) -> None:
    if not isinstance(shard, torch.Tensor):
        raise TypeError("shard: expected a torch.Tensor")
    if shard.numel() * shard.element_size() < shard_bytes(cfg):
        raise ValueError(f"shard: {shard.numel() * shard.element_size()} bytes, the layer needs {shard_bytes(cfg)}")


def _need_lora(lora: dict | None, cfg: B.LayerCfg, grads: bool = False) -> dict:
    if lora is None:
        return {}
    r, H, qd, kvd = cfg.lora_r, cfg.hidden, cfg.n_q * cfg.head_dim, cfg.n_kv * cfg.head_dim
    p = "d" if grads else ""
    for k, n in (("A_q", r * H), ("B_q", qd * r), ("A_v", r * H), ("B_v", kvd * r)):
        _need(lora[p + k], p + k, torch.float32, n)
    return {p + k: lora[p + k] for k in ("A_q", "B_q", "A_v", "B_v")}


def layer_cfg(shape: LayerShape, batch: int, seq: int) -> B.LayerCfg:
    return B.LayerCfg(shape.hidden, shape.inter, shape.n_q, shape.n_kv, shape.head_dim, batch, seq,
                      shape.rope_theta, shape.rms_eps, shape.lora_r, shape.lora_alpha)


def codebooks():
    nf4 = np.zeros(16, np.float32)
    c8 = np.zeros(256, np.float32)
    h = ctypes.c_uint64()
    B.call("nf4ls_codebooks", nf4.ctypes.data, c8.ctypes.data, ctypes.byref(h))
    return nf4, c8, h.value


def set_gemm_path(path: int) -> None:
    B.call("nf4ls_set_gemm_path", path)


def set_gemm_pair(on: bool) -> None:
    B.call("nf4ls_set_gemm_pair", int(on))


def set_attention_path(tc: bool) -> None:
    """True: tcgen05 attention forward where the shape allows; False: the mma.sync kernel."""
    B.call("nf4ls_set_attention_path", int(tc))


def set_gemm_half(mode: int) -> None:
    """0: per-launch choice of the pair-tile schedule; 1: always 512 tokens; 2: always 256;
    3: 512 for the whole waves, 256 for the last partial wave (nf4ls_set_gemm_half)."""
    B.call("nf4ls_set_gemm_half", int(mode))


def launch_count() -> int:
    return int(B.lib().nf4ls_launch_count())


def profile(on: bool) -> None:
    B.call("nf4ls_profile", int(on))


def profile_read(sel: int) -> dict:
    """Aggregate of the timed records since the last reset: sel 0 dense GEMMs, 1 NF4-decode
    GEMMs, 2 step phases; sel >= 1000 one detail (see nf4ls_profile_read in the header)."""
    out = (ctypes.c_double * 3)()
    B.call("nf4ls_profile_read", sel, ctypes.cast(out, ctypes.c_void_p))
    return {"launches": int(out[0]), "ms": float(out[1]), "flops": float(out[2])}


def profile_reset() -> None:
    B.call("nf4ls_profile_reset")


GEMM_DETAILS = {}
for _dec, _dn in ((0, "dense"), (1, "nf4")):
    for _dg, _gn in ((0, "fwd"), (1, "dgrad")):
        for _e, _en in enumerate(("store", "resid", "rope", "swiglu", "dswiglu")):
            GEMM_DETAILS[1000 + 100 * _dec + 10 * _dg + _e] = f"{_dn}_{_gn}_{_en}"
PHASES = {2000: "layers_forward", 2001: "head_forward_loss", 2002: "head_backward", 2003: "layers_backward"}


def device_error():
    out = (ctypes.c_int32 * 4)()
    st = B.call_status("nf4ls_device_error", ctypes.cast(out, ctypes.c_void_p))
    return st, list(out)


def wait_probe(limit_us: int, result: torch.Tensor, stream=None) -> None:
    """Launches the bounded-wait expiry probe (a wait that nothing ends) on the
    stream; result: int32 [2] on the device, 0 per warp whose wait gave up."""
    _need(result, "result", torch.int32, 2)
    _need_cuda(result=result)
    B.call("nf4ls_wait_probe", int(limit_us), _p(result), _s(stream))


# ----------------------------------------------------------------------------- NF4 tensors

def nf4_quantize_tensor(w: torch.Tensor, stream=None) -> dict:
    """bf16 device tensor -> dict(packed, q8, nested, offset) of device tensors."""
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    n = w.numel()
    dev = w.device
    packed = _buffer(n // 2, dev)[: n // 2]
    q8 = _buffer(n // 64, dev)[: n // 64]
    nested = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=dev)
    offset = torch.empty(1, dtype=torch.float32, device=dev)
    scratch_bytes = B.lib().nf4ls_quantize_scratch_bytes(n)
    scratch = _buffer(scratch_bytes, dev)
    B.call("nf4_quantize_tensor", _p(w), n, _p(packed), _p(q8), _p(nested), _p(offset), _p(scratch),
           scratch_bytes, _s(stream))
    return {"packed": packed, "q8": q8, "nested": nested, "offset": offset, "n": n, "_scratch": scratch}


def nf4_dequantize_tensor(q: dict, stream=None) -> torch.Tensor:
    n = q["n"]
    out = torch.empty(n, dtype=torch.bfloat16, device=q["packed"].device)
    B.call("nf4_dequantize_tensor", _p(q["packed"]), _p(q["q8"]), _p(q["nested"]), _p(q["offset"]), n, _p(out),
           _s(stream))
    return out


# ----------------------------------------------------------------------------- shards

def shard_bytes(cfg: B.LayerCfg) -> int:
    return B.lib().nf4ls_shard_bytes(ctypes.byref(cfg))


def shard_quantized_bytes(cfg: B.LayerCfg) -> int:
    return B.lib().nf4ls_shard_quantized_bytes(ctypes.byref(cfg))


def nf4_quantize_shard(cfg: B.LayerCfg, weights: dict, fingerprint: int = 0, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Quantises one layer (dict of bf16 device tensors) into a device shard (uint8)."""
    nbytes = shard_bytes(cfg)
    dev = weights["q"].device
    shard = out if out is not None else _buffer(nbytes, dev)
    ptrs = (ctypes.c_void_p * 9)(*[weights[n].contiguous().data_ptr() for n in LAYER_TENSORS])
    sb = B.lib().nf4ls_shard_scratch_bytes(ctypes.byref(cfg))
    scratch = _buffer(sb, dev)
    used = ctypes.c_size_t()
    B.call("nf4_quantize_shard", ctypes.byref(cfg), ctypes.cast(ptrs, ctypes.c_void_p), fingerprint, _p(shard),
           shard.numel(), ctypes.byref(used), _p(scratch), sb, _s(stream))
    return shard[:nbytes] if out is None else shard


def shard_check(header: torch.Tensor, cfg: B.LayerCfg | None, fingerprint: int = 0) -> int:
    h = header[:1024].cpu().contiguous()
    return B.call_status("nf4ls_shard_check", _p(h), ctypes.byref(cfg) if cfg is not None else None, fingerprint)


# ----------------------------------------------------------------------------- layer calls

def _lora_struct(lora: dict | None):
    if lora is None:
        return None
    return B.Lora(lora["A_q"].data_ptr(), lora["B_q"].data_ptr(), lora["A_v"].data_ptr(), lora["B_v"].data_ptr())


class LayerWorkspace:
    def __init__(self, cfg: B.LayerCfg, device="cuda"):
        self.nbytes = B.lib().nf4ls_workspace_bytes(ctypes.byref(cfg))
        self.buf = _buffer(self.nbytes, device)


def layer_forward(cfg: B.LayerCfg, shard: torch.Tensor, lora: dict | None, x: torch.Tensor,
                  ws: LayerWorkspace | None = None, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    MH = cfg.batch * cfg.seq * cfg.hidden
    _need(x, "x", torch.bfloat16, MH)
    _need_shard(shard, cfg)
    lt = _need_lora(lora, cfg)
    if y is not None:
        _need(y, "y", torch.bfloat16, MH)
    _need_cuda(x=x, shard=shard, y=y, **lt)
    ws = ws or LayerWorkspace(cfg, x.device)
    y = torch.empty_like(x) if y is None else y
    lo = _lora_struct(lora)
    B.call("layer_forward", ctypes.byref(cfg), _p(shard), ctypes.byref(lo) if lo else None, _p(x), _p(y),
           _p(ws.buf), ws.nbytes, _s(stream))
    return y


def layer_backward(cfg: B.LayerCfg, shard: torch.Tensor, lora: dict | None, x: torch.Tensor, dy: torch.Tensor,
                   ws: LayerWorkspace | None = None, dx: torch.Tensor | None = None, grads: dict | None = None,
                   stream=None):
    MH = cfg.batch * cfg.seq * cfg.hidden
    _need(x, "x", torch.bfloat16, MH)
    _need(dy, "dy", torch.bfloat16, MH)
    _need_shard(shard, cfg)
    lt = _need_lora(lora, cfg)
    if dx is not None:
        _need(dx, "dx", torch.bfloat16, MH)
    gt = _need_lora(grads, cfg, grads=True) if (lora is not None and grads is not None) else {}
    _need_cuda(x=x, dy=dy, shard=shard, dx=dx, **lt, **gt)
    ws = ws or LayerWorkspace(cfg, x.device)
    dx = torch.empty_like(x) if dx is None else dx
    lo = _lora_struct(lora)
    gs = None
    if lora is not None:
        if grads is None:
            grads = {"dA_q": torch.empty_like(lora["A_q"]), "dB_q": torch.empty_like(lora["B_q"]),
                     "dA_v": torch.empty_like(lora["A_v"]), "dB_v": torch.empty_like(lora["B_v"])}
        gs = B.LoraGrads(grads["dA_q"].data_ptr(), grads["dB_q"].data_ptr(), grads["dA_v"].data_ptr(),
                         grads["dB_v"].data_ptr())
    B.call("layer_backward", ctypes.byref(cfg), _p(shard), ctypes.byref(lo) if lo else None, _p(x), _p(dy), _p(dx),
           ctypes.byref(gs) if gs else None, _p(ws.buf), ws.nbytes, _s(stream))
    return dx, grads


def mse_loss(out: torch.Tensor, stream=None):
    """loss = mean(out^2) (fp32 device scalar), dout = bf16(2 out / n)."""
    _need(out, "out", torch.bfloat16)
    _need_cuda(out=out)
    n = out.numel()
    dout = torch.empty_like(out)
    loss = torch.empty(1, dtype=torch.float32, device=out.device)
    npart = 256
    partial = torch.empty(npart, dtype=torch.float32, device=out.device)
    B.call("nf4ls_mse_loss", _p(out), n, _p(dout), _p(loss), _p(partial), npart, _s(stream))
    return loss, dout


def gemm_bf16(A: torch.Tensor, Bm: torch.Tensor, b_trans: bool = False, stream=None) -> torch.Tensor:
    """out = A B^T (B [N, K]) or, with b_trans, out = A B (B [K, N]); tcgen05 kernel."""
    if A.dim() != 2 or Bm.dim() != 2 or Bm.shape[0 if b_trans else 1] != A.shape[1]:
        raise ValueError(f"gemm_bf16: A {tuple(A.shape)} and B {tuple(Bm.shape)} (b_trans={b_trans}) do not match")
    _need(A, "A", torch.bfloat16)
    _need(Bm, "B", torch.bfloat16)
    _need_cuda(A=A, B=Bm)
    M, K = A.shape
    N = Bm.shape[1] if b_trans else Bm.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    B.call("nf4ls_gemm_bf16", _p(A), _p(Bm), _p(out), M, N, K, int(b_trans), N, _s(stream))
    return out


def gemm_nf4(A: torch.Tensor, q: dict, rows: int, cols: int, dgrad: bool = False, stream=None) -> torch.Tensor:
    """out = A W^T (forward) or A W (dgrad) with W [rows, cols] given as an NF4 tensor dict."""
    K = rows if dgrad else cols
    _need_rows(A, "A", A.shape[0] if A.dim() == 2 else 0, A.stride(0) if A.dim() == 2 else 0, K)
    if A.shape[1] != K:
        raise ValueError(f"gemm_nf4: A has {A.shape[1]} columns, the product needs {K}")
    if q.get("n") != rows * cols:
        raise ValueError(f"gemm_nf4: the NF4 tensor holds {q.get('n')} weights, not {rows} x {cols}")
    _need_cuda(A=A, **{k: q[k] for k in ("packed", "q8", "nested", "offset")})
    M = A.shape[0]
    N = cols if dgrad else rows
    out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    B.call("nf4ls_gemm_nf4", _p(A), A.stride(0), M, _p(q["packed"]), _p(q["q8"]), _p(q["nested"]),
           _p(q["offset"]), rows, cols, int(dgrad), _p(out), N, _s(stream))
    return out


def attention_fwd(cfg: B.LayerCfg, q, k, v, ld_q: int, ld_kv: int, stream=None):
    M = cfg.batch * cfg.seq
    _need_rows(q, "q", M, ld_q, cfg.n_q * cfg.head_dim)
    _need_rows(k, "k", M, ld_kv, cfg.n_kv * cfg.head_dim)
    _need_rows(v, "v", M, ld_kv, cfg.n_kv * cfg.head_dim)
    _need_cuda(q=q, k=k, v=v)
    o = torch.empty(M, cfg.n_q * cfg.head_dim, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(cfg.batch, cfg.n_q, cfg.seq, dtype=torch.float32, device=q.device)
    B.call("nf4ls_attention_fwd", ctypes.byref(cfg), _p(q), _p(k), _p(v), ld_q, ld_kv, _p(o), _p(lse), _s(stream))
    return o, lse


def attention_bwd(cfg: B.LayerCfg, q, k, v, ld_q: int, ld_kv: int, o, do, lse, stream=None):
    """Gradients (dq, dk, dv) of the causal GQA attention and delta = rowsum(do * o)."""
    M = cfg.batch * cfg.seq
    qd, kvd = cfg.n_q * cfg.head_dim, cfg.n_kv * cfg.head_dim
    _need_rows(q, "q", M, ld_q, qd)
    _need_rows(k, "k", M, ld_kv, kvd)
    _need_rows(v, "v", M, ld_kv, kvd)
    _need(o, "o", torch.bfloat16, M * qd)
    _need(do, "do", torch.bfloat16, M * qd)
    _need(lse, "lse", torch.float32, cfg.batch * cfg.n_q * cfg.seq)
    _need_cuda(q=q, k=k, v=v, o=o, do=do, lse=lse)
    dq = torch.empty(M, qd, dtype=torch.bfloat16, device=q.device)
    dk = torch.empty(M, kvd, dtype=torch.bfloat16, device=q.device)
    dv = torch.empty(M, kvd, dtype=torch.bfloat16, device=q.device)
    delta = torch.empty(cfg.batch, cfg.n_q, cfg.seq, dtype=torch.float32, device=q.device)
    B.call("nf4ls_attention_bwd", ctypes.byref(cfg), _p(q), _p(k), _p(v), ld_q, ld_kv, _p(o), _p(do), _p(lse),
           _p(delta), _p(dq), _p(dk), _p(dv), _s(stream))
    return dq, dk, dv, delta


# ----------------------------------------------------------------------------- streaming pool

class Pool:
    """n-deep HBM slot pool filled from a pinned host store (nf4ls_pool_*)."""

    def __init__(self, store: torch.Tensor, offsets, sizes, depth: int, slot_bytes: int | None = None,
                 device="cuda"):
        assert store.is_pinned(), "the host store must be page-locked"
        self.store = store
        n = len(offsets)
        self.offsets = (ctypes.c_size_t * n)(*offsets)
        self.sizes = (ctypes.c_size_t * n)(*sizes)
        self.slot_bytes = slot_bytes or (max(sizes) + 255) // 256 * 256
        self.slots = _buffer(depth * self.slot_bytes, device)
        self.handle = ctypes.c_void_p()
        B.call("nf4ls_pool_create", _p(store), ctypes.cast(self.offsets, ctypes.c_void_p),
               ctypes.cast(self.sizes, ctypes.c_void_p), n, depth, _p(self.slots), self.slot_bytes,
               ctypes.byref(self.handle))

    @classmethod
    def from_file(cls, path: str, offsets, sizes, depth: int, slot_bytes: int | None = None, device="cuda"):
        """A pool whose store is a file (the disk stream source): a library thread reads
        each layer into pinned staging and copies it into its slot."""
        self = cls.__new__(cls)
        self.store = None
        n = len(offsets)
        self.offsets = (ctypes.c_size_t * n)(*offsets)
        self.sizes = (ctypes.c_size_t * n)(*sizes)
        self.slot_bytes = slot_bytes or (max(sizes) + 255) // 256 * 256
        self.slots = _buffer(depth * self.slot_bytes, device)
        nst = B.lib().nf4ls_pool_file_staging_bytes(ctypes.cast(self.sizes, ctypes.c_void_p), n)
        raw = torch.empty(nst + 4096, dtype=torch.uint8).pin_memory()
        skip = (-raw.data_ptr()) % 4096
        self.staging = raw[skip:skip + nst]
        self.handle = ctypes.c_void_p()
        B.call("nf4ls_pool_create_file", path.encode(), ctypes.cast(self.offsets, ctypes.c_void_p),
               ctypes.cast(self.sizes, ctypes.c_void_p), n, depth, _p(self.slots), self.slot_bytes,
               _p(self.staging), nst, ctypes.byref(self.handle))
        return self

    def prefetch(self, layer: int) -> int:
        return B.call_status("nf4ls_pool_prefetch", self.handle, layer)

    def stream_prefetch(self, layer: int, stream=None) -> int:
        out = ctypes.c_void_p()
        B.call("stream_prefetch", self.handle, layer, _s(stream), ctypes.byref(out))
        return out.value

    def release(self, layer: int, stream=None) -> None:
        B.call("nf4ls_pool_release", self.handle, layer, _s(stream))

    def wait(self, layer: int, timeout_ms: int) -> int:
        return B.call_status("nf4ls_wait", self.handle, layer, timeout_ms)

    def set_poison(self, on: bool) -> None:
        B.call("nf4ls_pool_set_poison", self.handle, int(on))

    def stats(self) -> dict:
        s = B.PoolStats()
        B.call("nf4ls_pool_get_stats", self.handle, ctypes.byref(s))
        return {"bytes_copied": s.bytes_copied, "copies": s.copies, "hits": s.hits, "acquisitions": s.acquisitions,
                "peer_bytes": s.peer_bytes}

    def share(self, rank: int, world: int, nccl_id: bytes) -> None:
        """Layer-sharded fetch across ranks (every rank calls this at the same time)."""
        buf = (ctypes.c_uint8 * 128).from_buffer_copy(nccl_id)
        B.call("nf4ls_pool_share", self.handle, rank, world, ctypes.cast(buf, ctypes.c_void_p))

    def synchronize(self) -> None:
        B.call("nf4ls_pool_synchronize", self.handle)

    def destroy(self) -> None:
        if self.handle:
            B.call("nf4ls_pool_destroy", self.handle)
            self.handle = ctypes.c_void_p()

    def __enter__(self) -> "Pool":
        return self

    def __exit__(self, *exc) -> None:
        self.destroy()

    def view(self, ptr: int, nbytes: int) -> torch.Tensor:
        """A uint8 view of the slot at device address ptr (for reading a streamed shard)."""
        off = ptr - self.slots.data_ptr()
        return self.slots[off: off + nbytes]


class SlotPlan:
    """The pool's slot decisions on the host (no device work): prefetch / acquire /
    release return what the pool does for the same call (slot, hit, fill, wait for
    the slot's release, owner rank, host read, broadcast) as a dict."""

    def __init__(self, n_layers: int, depth: int):
        h = ctypes.c_void_p()
        B.call("nf4ls_plan_create", n_layers, depth, ctypes.byref(h))
        self.handle = h

    @staticmethod
    def _dict(st: B.PlanStep) -> dict:
        return {k: int(getattr(st, k)) for k, _ in B.PlanStep._fields_}

    def share(self, rank: int, world: int) -> None:
        B.call("nf4ls_plan_share", self.handle, rank, world)

    def prefetch(self, layer: int):
        """The step dict, or None when the pool would answer BUFFER_BUSY."""
        st = B.PlanStep()
        r = B.call_status("nf4ls_plan_prefetch", self.handle, layer, ctypes.byref(st))
        if r == -6:
            return None
        B.check(r)
        return self._dict(st)

    def acquire(self, layer: int) -> dict:
        st = B.PlanStep()
        B.call("nf4ls_plan_acquire", self.handle, layer, ctypes.byref(st))
        return self._dict(st)

    def release(self, layer: int) -> None:
        B.call("nf4ls_plan_release", self.handle, layer)

    def close(self) -> None:
        if self.handle:
            B.lib().nf4ls_plan_destroy(self.handle)
            self.handle = None

    def __enter__(self) -> "SlotPlan":
        return self

    def __exit__(self, *exc) -> None:
        self.close()


PASS_OPS = ("acquire", "prefetch", "run", "release")


def step_pass_ops(n_layers: int, direction: int) -> list:
    """[(op name, layer)] of the pool calls one pass of the model step makes."""
    n = ctypes.c_int32(0)
    B.call_status("nf4ls_step_pass_ops", n_layers, direction, None, None, 0, ctypes.byref(n))
    ops = (ctypes.c_int32 * n.value)()
    layers = (ctypes.c_int32 * n.value)()
    B.call("nf4ls_step_pass_ops", n_layers, direction, ops, layers, n.value, ctypes.byref(n))
    return [(PASS_OPS[o], l) for o, l in zip(ops, layers)]


def nccl_unique_id() -> bytes:
    buf = (ctypes.c_uint8 * 128)()
    B.call("nf4ls_nccl_unique_id", ctypes.cast(buf, ctypes.c_void_p))
    return bytes(buf)


def disk_probe(path: str, probe_bytes: int = 1 << 30) -> dict:
    info = B.DiskInfo()
    B.call("nf4ls_disk_probe", path.encode(), probe_bytes, ctypes.byref(info))
    return {"read_gbs": info.read_gbs, "block_device": bool(info.block_device), "nvme": bool(info.nvme),
            "rotational": bool(info.rotational), "direct_io": bool(info.direct_io)}


def disk_accept(info: dict, min_gbs: float = 1.5) -> int:
    """NF4LS_OK, or NF4LS_SOURCE_REFUSED for a spinning / non-NVMe / slow device."""
    d = B.DiskInfo(info["read_gbs"], int(info["block_device"]), int(info["nvme"]), int(info["rotational"]),
                   int(info.get("direct_io", False)))
    return B.call_status("nf4ls_disk_accept", ctypes.byref(d), float(min_gbs))


def choose_source(store_bytes: int, reserve_bytes: int = 8 << 30) -> str:
    """stream_source: auto -- 'ram' when the store fits in available host memory."""
    out = ctypes.c_int32()
    B.call("nf4ls_choose_source", store_bytes, reserve_bytes, ctypes.byref(out))
    return "disk" if out.value else "ram"


# ----------------------------------------------------------------------------- whole model

@dataclass
class TrainConfig:
    lr: float = 2e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


class StreamedModel:
    """All buffers of one n-layer model: pinned NF4 store (or resident shards), the
    resident bf16 embedding / lm_head, LoRA masters, gradients and AdamW moments, and
    the step workspace.  Quantisation runs through nf4_quantize_shard on the GPU."""

    def __init__(self, wl: Workload, depth: int = 2, resident: bool = False, b_random: bool = False,
                 train: TrainConfig = TrainConfig(), device="cuda", weights_device=None, fingerprint: int = 1234,
                 head_chunk_rows: int = 0, source: str = "ram", store_path: str | None = None,
                 min_disk_gbs: float | None = None):
        """head_chunk_rows > 0: the embedding and lm_head stay in pinned host memory; the
        output matrix streams through a depth-2 pool in chunks of that many vocab rows.
        source: 'ram' (pinned store), 'disk' (the shard set written once to store_path and
        read back by the pool's reader thread; with min_disk_gbs set, the device is probed
        first and a spinning, non-NVMe or slower device is refused) or 'auto' (RAM when the
        store fits in available memory)."""
        self.wl = wl
        shape = wl.shape
        self.cfg = B.ModelCfg(layer_cfg(shape, wl.batch, wl.seq), wl.n_layers, wl.vocab, int(wl.tied), train.lr,
                              train.beta1, train.beta2, train.eps, train.weight_decay, head_chunk_rows)
        lc = self.cfg.layer
        from . import synth
        wdev = weights_device or device
        self.shard_nbytes = shard_bytes(lc)
        self.slot_bytes = (self.shard_nbytes + 255) // 256 * 256
        L = wl.n_layers
        self.resident = resident
        self.pool = None
        shards = []
        file_stride = (self.slot_bytes + 4095) // 4096 * 4096
        if source == "auto":
            source = choose_source(L * self.slot_bytes)
        self.source = "resident" if resident else source
        if resident:
            self.shard_buf = _buffer(L * self.slot_bytes, device)
        elif source == "disk":
            if not store_path:
                raise ValueError("the disk stream source needs store_path")
            fh = open(store_path, "wb")
            fh.truncate(L * file_stride)
            host = torch.empty(self.slot_bytes, dtype=torch.uint8).pin_memory()
        else:
            self.store = torch.empty(L * self.slot_bytes, dtype=torch.uint8).pin_memory()
        tmp = _buffer(self.slot_bytes, device)
        for i in range(L):
            w = synth.layer_weights(shape, i, wl.seed, device=wdev)
            w = {k: v.to(device) for k, v in w.items()}
            if resident:
                dst = self.shard_buf[i * self.slot_bytes:(i + 1) * self.slot_bytes]
                nf4_quantize_shard(lc, w, fingerprint, out=dst)
                shards.append(dst.data_ptr())
            else:
                nf4_quantize_shard(lc, w, fingerprint, out=tmp)
                torch.cuda.synchronize()
                if source == "disk":
                    host.copy_(tmp)
                    fh.seek(i * file_stride)
                    fh.write(host.numpy().tobytes())
                else:
                    self.store[i * self.slot_bytes:(i + 1) * self.slot_bytes].copy_(tmp)
            del w
        del tmp
        if resident:
            self.shard_ptrs = (ctypes.c_void_p * L)(*shards)
        elif source == "disk":
            fh.close()
            del host
            self.disk = None
            if min_disk_gbs is not None:
                self.disk = disk_probe(store_path)
                st = disk_accept(self.disk, min_disk_gbs)
                if st != 0:
                    raise B.NF4LSError(st, B.lib().nf4ls_last_error().decode())
            offs = [i * file_stride for i in range(L)]
            self.pool = Pool.from_file(store_path, offs, [self.shard_nbytes] * L, depth, self.slot_bytes, device)
        else:
            offs = [i * self.slot_bytes for i in range(L)]
            self.pool = Pool(self.store, offs, [self.shard_nbytes] * L, depth, self.slot_bytes, device)
        self.head_pool = None
        if head_chunk_rows > 0:
            self.embed = synth.embedding(wl.vocab, shape.hidden, wl.seed, 0, device=wdev).cpu().pin_memory()
            self.lm_head = None if wl.tied else \
                synth.embedding(wl.vocab, shape.hidden, wl.seed, 1, device=wdev).cpu().pin_memory()
            out = self.embed if wl.tied else self.lm_head
            row_bytes = shape.hidden * 2
            n_chunks = (wl.vocab + head_chunk_rows - 1) // head_chunk_rows
            offs = [i * head_chunk_rows * row_bytes for i in range(n_chunks)]
            sizes = [min(head_chunk_rows, wl.vocab - i * head_chunk_rows) * row_bytes for i in range(n_chunks)]
            self.head_pool = Pool(out, offs, sizes, 2, None, device)
        else:
            self.embed = synth.embedding(wl.vocab, shape.hidden, wl.seed, 0, device=wdev).to(device)
            self.lm_head = None if wl.tied else \
                synth.embedding(wl.vocab, shape.hidden, wl.seed, 1, device=wdev).to(device)
        self.norm_final = torch.ones(shape.hidden, dtype=torch.bfloat16, device=device)
        self.stride = B.lib().nf4ls_lora_stride(ctypes.byref(lc))
        self.lora = torch.zeros(L * self.stride, dtype=torch.float32, device=device)
        for i in range(L):
            lp = synth.lora_params(shape, i, wl.seed, b_random=b_random, device="cpu")
            flat = torch.cat([lp["A_q"].reshape(-1), lp["B_q"].reshape(-1), lp["A_v"].reshape(-1),
                              lp["B_v"].reshape(-1)])
            self.lora[i * self.stride:(i + 1) * self.stride].copy_(flat)
        self.grads = torch.zeros_like(self.lora)
        self.adam_m = torch.zeros_like(self.lora)
        self.adam_v = torch.zeros_like(self.lora)
        self.ws_bytes = B.lib().nf4ls_model_workspace_bytes(ctypes.byref(self.cfg))
        self.ws = _buffer(self.ws_bytes, device)
        self.loss = torch.zeros(1, dtype=torch.float32, device=device)
        streamed = self.head_pool is not None
        self.model = B.Model(None if streamed else self.embed.data_ptr(),
                             None if (streamed or self.lm_head is None) else self.lm_head.data_ptr(),
                             self.norm_final.data_ptr(), self.lora.data_ptr(), self.grads.data_ptr(),
                             self.adam_m.data_ptr(), self.adam_v.data_ptr(),
                             self.pool.handle.value if self.pool else None,
                             ctypes.cast(self.shard_ptrs, ctypes.c_void_p) if resident else None,
                             self.ws.data_ptr(), self.ws_bytes,
                             self.head_pool.handle.value if streamed else None,
                             self.embed.data_ptr() if streamed else None)
        self.step_count = 0

    def lora_views(self, layer: int) -> dict:
        sh = self.wl.shape
        r, H = sh.lora_r, sh.hidden
        base = self.lora[layer * self.stride:(layer + 1) * self.stride]
        a = r * H
        bq = sh.q_dim * r
        return {"A_q": base[:a].view(r, H), "B_q": base[a:a + bq].view(sh.q_dim, r),
                "A_v": base[a + bq:2 * a + bq].view(r, H), "B_v": base[2 * a + bq:].view(sh.kv_dim, r)}

    def grad_views(self, layer: int) -> dict:
        sh = self.wl.shape
        r, H = sh.lora_r, sh.hidden
        base = self.grads[layer * self.stride:(layer + 1) * self.stride]
        a = r * H
        bq = sh.q_dim * r
        return {"dA_q": base[:a].view(r, H), "dB_q": base[a:a + bq].view(sh.q_dim, r),
                "dA_v": base[a + bq:2 * a + bq].view(r, H), "dB_v": base[2 * a + bq:].view(sh.kv_dim, r)}

    def train_step(self, ids: torch.Tensor, stream=None) -> torch.Tensor:
        self.step_count += 1
        B.call("nf4ls_train_step", ctypes.byref(self.cfg), ctypes.byref(self.model), _p(ids), self.step_count,
               _p(self.loss), _s(stream))
        return self.loss

    def forward_backward(self, ids: torch.Tensor, stream=None) -> torch.Tensor:
        B.call("nf4ls_forward_backward", ctypes.byref(self.cfg), ctypes.byref(self.model), _p(ids), _p(self.loss),
               _s(stream))
        return self.loss

    def adamw_step(self, stream=None) -> None:
        self.step_count += 1
        B.call("nf4ls_adamw_step", ctypes.byref(self.cfg), ctypes.byref(self.model), self.step_count, _s(stream))

    def save_adapter(self, path: str, stream=None) -> None:
        """Writes the LoRA parameters, both AdamW moments and step_count to path."""
        B.call("nf4ls_adapter_save", os.fsencode(path), ctypes.byref(self.cfg), ctypes.byref(self.model),
               self.step_count, _s(stream))

    def load_adapter(self, path: str, stream=None) -> int:
        """Restores what save_adapter wrote (the same model shape is required) and
        step_count, so the next train_step continues the saved run."""
        step = ctypes.c_int32(0)
        B.call("nf4ls_adapter_load", os.fsencode(path), ctypes.byref(self.cfg), ctypes.byref(self.model),
               ctypes.byref(step), _s(stream))
        self.step_count = step.value
        return self.step_count

    def forward_loss(self, ids: torch.Tensor, lora_on: bool = True, stream=None) -> torch.Tensor:
        B.call("nf4ls_forward_loss", ctypes.byref(self.cfg), ctypes.byref(self.model), _p(ids), int(lora_on),
               _p(self.loss), _s(stream))
        return self.loss

    def close(self) -> None:
        if self.pool is not None:
            self.pool.destroy()
            self.pool = None
        if self.head_pool is not None:
            self.head_pool.destroy()
            self.head_pool = None

    def __enter__(self) -> "StreamedModel":
        return self

    def __exit__(self, *exc) -> None:
        self.close()
