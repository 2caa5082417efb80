"""B200 (sm_100a) DeepSeek Sparse Attention hot path: Python binding of libdsa.so.

Argument marshalling only: every step runs in the library's CUDA kernels. Functions take torch
CUDA tensors (PyTorch is used for device memory and streams) and pass raw pointers and the current
stream through the C ABI declared in include/dsa.h. A non-OK status raises DsaError. There is no
CPU fallback: if libdsa.so is missing, loading fails with an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdsa.so")
PAGE_SIZE = 64
D_INDEX = 128
D_LATENT = 576
D_V = 512
D_QK_MHA = 192
D_V_MHA = 128

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported size", 3: "workspace too small", 4: "CUDA error",
          5: "a kernel wait timed out", 6: "a kernel met an out-of-range index",
          7: "a kernel met a non-finite input value"}


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class DsaBatchC(ctypes.Structure):
    _fields_ = [("num_requests", ctypes.c_int32), ("total_q", ctypes.c_int32), ("max_q", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32), ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("seq_lens", ctypes.c_void_p), ("cu_q", ctypes.c_void_p), ("block_table", ctypes.c_void_p)]


EXPORTS = ("dsa_abi_version", "dsa_status_string", "dsa_plan_workspace_size", "dsa_plan", "dsa_status_read",
           "dsa_index_scores", "dsa_index_topk_supported", "dsa_index_topk", "dsa_topk_workspace_size", "dsa_topk", "dsa_sparse_mla_workspace_size", "dsa_sparse_mla",
           "dsa_layer_workspace_size", "dsa_layer", "dsa_layer_noalloc", "dsa_layer_noalloc_status_read", "dsa_cache_write",
           "dsa_masked_mha_workspace_size", "dsa_masked_mha")

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdsa.so (built by `python -m sparse_attention_12_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libdsa.so not found at {path}; build it with `python -m sparse_attention_12_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    BP = ctypes.POINTER(DsaBatchC)
    sig = {
        "dsa_abi_version": (I, []),
        "dsa_status_string": (ctypes.c_char_p, [I]),
        "dsa_plan_workspace_size": (SZ, [BP, I]),
        "dsa_plan": (I, [BP, I, P, SZ, P]),
        "dsa_status_read": (I, [P, P]),
        "dsa_index_scores": (I, [BP, P, P, P, P, I, P, P, P, I64, P]),
        "dsa_index_topk_supported": (I, [BP, I, I]),
        "dsa_index_topk": (I, [BP, P, P, P, P, I, P, P, I, P, P]),
        "dsa_topk_workspace_size": (SZ, [BP, I]),
        "dsa_topk": (I, [BP, P, P, I64, I, P, P, SZ, P]),
        "dsa_sparse_mla_workspace_size": (SZ, [BP, I, I]),
        "dsa_sparse_mla": (I, [BP, P, P, I, P, P, I, ctypes.c_float, P, P, P, SZ, P]),
        "dsa_layer_workspace_size": (SZ, [BP, I, I, I]),
        "dsa_layer": (I, [BP, P, P, P, I, P, P, P, I, P, I, ctypes.c_float, P, P, P, P, SZ, P]),
        "dsa_layer_noalloc": (I, [BP, P, P, P, I, P, P, P, I, P, I, ctypes.c_float, P, P, P, P]),
        "dsa_layer_noalloc_status_read": (I, [P]),
        "dsa_cache_write": (I, [BP, P, P, P, P, P, P, P]),
        "dsa_masked_mha_workspace_size": (SZ, [BP, I, I]),
        "dsa_masked_mha": (I, [BP, P, P, P, P, I, P, I, ctypes.c_float, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(x: Optional[torch.Tensor]) -> Optional[int]:
    return None if x is None else x.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise DsaError(status, where)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


class Batch:
    """A ragged batch: device seq_lens [B], cu_q [B+1], block_table [B, max_pages] (int32) plus the
    host-side sizes the launches need."""

    def __init__(self, seq_lens: torch.Tensor, cu_q: torch.Tensor, block_table: torch.Tensor, num_pages: int,
                 total_q: int, max_q: int, max_seq_len: int):
        for n, t in (("seq_lens", seq_lens), ("cu_q", cu_q), ("block_table", block_table)):
            _need(t, n, torch.int32)
        self.seq_lens, self.cu_q, self.block_table = seq_lens, cu_q, block_table
        self.c = DsaBatchC(int(seq_lens.shape[0]), int(total_q), int(max_q), int(max_seq_len),
                           int(block_table.shape[1]), int(num_pages), seq_lens.data_ptr(), cu_q.data_ptr(),
                           block_table.data_ptr())

    @classmethod
    def from_host(cls, seq_lens, cu_q, block_table, num_pages: int, device="cuda"):
        """From host int arrays (numpy or lists); copies them to the device."""
        import numpy as np
        sl = np.asarray(seq_lens, np.int32)
        cq = np.asarray(cu_q, np.int32)
        bt = np.asarray(block_table, np.int32)
        m = np.diff(cq)
        return cls(torch.from_numpy(sl).to(device), torch.from_numpy(cq).to(device), torch.from_numpy(bt).to(device),
                   num_pages, int(cq[-1]), int(m.max()) if m.size else 0, int(sl.max()) if sl.size else 0)

    @property
    def total_q(self) -> int:
        return self.c.total_q

    def ref(self):
        return ctypes.byref(self.c)


def plan_workspace_size(batch: Batch, nhI: int) -> int:
    return load().dsa_plan_workspace_size(batch.ref(), nhI)


def plan(batch: Batch, nhI: int, plan_ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Compute the batch plan into `plan_ws` (uint8, allocated if None) and return it."""
    lib = load()
    n = lib.dsa_plan_workspace_size(batch.ref(), nhI)
    if plan_ws is None:
        plan_ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    _check(lib.dsa_plan(batch.ref(), nhI, plan_ws.data_ptr(), plan_ws.numel(), _stream()), "dsa_plan")
    return plan_ws


def status_read(plan_ws: torch.Tensor) -> int:
    """Synchronise the current stream and return (and clear) the kernels' status word."""
    return load().dsa_status_read(plan_ws.data_ptr(), _stream())


def cache_write(batch: Batch, plan_ws, k_new, c_new, kI_cache, kI_scale, kv_cache) -> None:
    """Store every query row's new indexer key (fp32 [T, 128], quantised to FP8 + scale) and latent
    row (bf16 [T, 576]) at its own position of the paged caches (dsa_cache_write)."""
    T = batch.total_q
    _need(k_new, "k_new", torch.float32, (T, D_INDEX))
    _need(c_new, "c_new", torch.bfloat16, (T, D_LATENT))
    _need(kI_cache, "kI_cache", torch.float8_e4m3fn)
    _need(kI_scale, "kI_scale", torch.float32)
    _need(kv_cache, "kv_cache", torch.bfloat16)
    _check(load().dsa_cache_write(batch.ref(), plan_ws.data_ptr(), k_new.data_ptr(), c_new.data_ptr(),
                                  kI_cache.data_ptr(), kI_scale.data_ptr(), kv_cache.data_ptr(), _stream()),
           "dsa_cache_write")


def index_scores(batch: Batch, plan_ws, qI, qI_scale, wI, kI_cache, kI_scale, scores=None, ld=None) -> torch.Tensor:
    T = batch.total_q
    nhI = int(qI.shape[1])
    _need(qI, "qI", torch.float8_e4m3fn, (T, nhI, D_INDEX))
    _need(qI_scale, "qI_scale", torch.float32, (T,))
    _need(wI, "wI", torch.float32, (T, nhI))
    _need(kI_cache, "kI_cache", torch.float8_e4m3fn)
    _need(kI_scale, "kI_scale", torch.float32)
    if ld is None:
        ld = (batch.c.max_seq_len + 127) // 128 * 128
    if scores is None:
        scores = torch.empty((T, ld), dtype=torch.float32, device="cuda")
    _need(scores, "scores", torch.float32, (T, ld))
    _check(load().dsa_index_scores(batch.ref(), plan_ws.data_ptr(), qI.data_ptr(), qI_scale.data_ptr(),
                                   wI.data_ptr(), nhI, kI_cache.data_ptr(), kI_scale.data_ptr(), scores.data_ptr(),
                                   ld, _stream()), "dsa_index_scores")
    return scores


def index_topk_supported(batch: Batch, nhI: int, k: int) -> bool:
    return bool(load().dsa_index_topk_supported(batch.ref(), nhI, k))


def index_topk(batch: Batch, plan_ws, qI, qI_scale, wI, kI_cache, kI_scale, k: int, S=None) -> torch.Tensor:
    """Indexer scores and top-k fused (dsa_index_topk): S [T, k] int32 without score rows in memory."""
    T = batch.total_q
    nhI = int(qI.shape[1])
    _need(qI, "qI", torch.float8_e4m3fn, (T, nhI, D_INDEX))
    _need(qI_scale, "qI_scale", torch.float32, (T,))
    _need(wI, "wI", torch.float32, (T, nhI))
    _need(kI_cache, "kI_cache", torch.float8_e4m3fn)
    _need(kI_scale, "kI_scale", torch.float32)
    if S is None:
        S = torch.empty((T, k), dtype=torch.int32, device="cuda")
    _need(S, "S", torch.int32, (T, k))
    _check(load().dsa_index_topk(batch.ref(), plan_ws.data_ptr(), qI.data_ptr(), qI_scale.data_ptr(), wI.data_ptr(),
                                 nhI, kI_cache.data_ptr(), kI_scale.data_ptr(), k, S.data_ptr(), _stream()),
           "dsa_index_topk")
    return S


def topk(batch: Batch, plan_ws, scores: torch.Tensor, k: int, S=None, ws=None) -> torch.Tensor:
    T = batch.total_q
    _need(scores, "scores", torch.float32)
    if S is None:
        S = torch.empty((T, k), dtype=torch.int32, device="cuda")
    _need(S, "S", torch.int32, (T, k))
    lib = load()
    need = lib.dsa_topk_workspace_size(batch.ref(), k)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    _check(lib.dsa_topk(batch.ref(), plan_ws.data_ptr(), scores.data_ptr(), int(scores.shape[1]), k, S.data_ptr(),
                        _ptr(ws), 0 if ws is None else ws.numel(), _stream()), "dsa_topk")
    return S


def sparse_mla(batch: Batch, plan_ws, q, kv_cache, S, softmax_scale: float, out=None, lse=None, ws=None):
    T = batch.total_q
    H = int(q.shape[1])
    k = int(S.shape[1])
    _need(q, "q", torch.bfloat16, (T, H, D_LATENT))
    _need(kv_cache, "kv_cache", torch.bfloat16)
    _need(S, "S", torch.int32, (T, k))
    lib = load()
    if out is None:
        out = torch.empty((T, H, D_V), dtype=torch.bfloat16, device="cuda")
    _need(out, "out", torch.bfloat16, (T, H, D_V))
    if lse is not None:
        _need(lse, "lse", torch.float32, (T, H))
    need = lib.dsa_sparse_mla_workspace_size(batch.ref(), H, k)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    _check(lib.dsa_sparse_mla(batch.ref(), plan_ws.data_ptr(), q.data_ptr(), H, kv_cache.data_ptr(), S.data_ptr(),
                              k, float(softmax_scale), out.data_ptr(), _ptr(lse), _ptr(ws),
                              0 if ws is None else ws.numel(), _stream()), "dsa_sparse_mla")
    return out


def masked_mha(batch: Batch, plan_ws, q, k, v, S, softmax_scale: float, out=None, lse=None, ws=None):
    """Masked MHA mode for short prefill (dsa_masked_mha): expanded q, k [T, H, 192] and v [T, H, 128]
    (bf16, every request a whole prefill), index sets S [T, topk]. Returns out [T, H, 128] bf16."""
    T = batch.total_q
    H = int(q.shape[1])
    topk = int(S.shape[1])
    _need(q, "q", torch.bfloat16, (T, H, D_QK_MHA))
    _need(k, "k", torch.bfloat16, (T, H, D_QK_MHA))
    _need(v, "v", torch.bfloat16, (T, H, D_V_MHA))
    _need(S, "S", torch.int32, (T, topk))
    lib = load()
    if out is None:
        out = torch.empty((T, H, D_V_MHA), dtype=torch.bfloat16, device="cuda")
    _need(out, "out", torch.bfloat16, (T, H, D_V_MHA))
    if lse is not None:
        _need(lse, "lse", torch.float32, (T, H))
    need = lib.dsa_masked_mha_workspace_size(batch.ref(), H, topk)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    _check(lib.dsa_masked_mha(batch.ref(), plan_ws.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), H,
                              S.data_ptr(), topk, float(softmax_scale), out.data_ptr(), _ptr(lse), ws.data_ptr(),
                              ws.numel(), _stream()), "dsa_masked_mha")
    return out


def layer_workspace_size(batch: Batch, nhI: int, H: int, k: int) -> int:
    return load().dsa_layer_workspace_size(batch.ref(), nhI, H, k)


def layer(batch: Batch, qI, qI_scale, wI, kI_cache, kI_scale, q, kv_cache, k: int, softmax_scale: float,
          out=None, lse=None, S_out=None, ws=None):
    """The whole path (plan, indexer, top-k, sparse MLA). Returns out [T, H, 512] bf16."""
    T = batch.total_q
    nhI = int(qI.shape[1])
    H = int(q.shape[1])
    _need(qI, "qI", torch.float8_e4m3fn, (T, nhI, D_INDEX))
    _need(qI_scale, "qI_scale", torch.float32, (T,))
    _need(wI, "wI", torch.float32, (T, nhI))
    _need(kI_cache, "kI_cache", torch.float8_e4m3fn)
    _need(kI_scale, "kI_scale", torch.float32)
    _need(q, "q", torch.bfloat16, (T, H, D_LATENT))
    _need(kv_cache, "kv_cache", torch.bfloat16)
    lib = load()
    if out is None:
        out = torch.empty((T, H, D_V), dtype=torch.bfloat16, device="cuda")
    _need(out, "out", torch.bfloat16, (T, H, D_V))
    if S_out is not None:
        _need(S_out, "S_out", torch.int32, (T, k))
    if lse is not None:
        _need(lse, "lse", torch.float32, (T, H))
    need = lib.dsa_layer_workspace_size(batch.ref(), nhI, H, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    _check(lib.dsa_layer(batch.ref(), qI.data_ptr(), qI_scale.data_ptr(), wI.data_ptr(), nhI, kI_cache.data_ptr(),
                         kI_scale.data_ptr(), q.data_ptr(), H, kv_cache.data_ptr(), k, float(softmax_scale),
                         out.data_ptr(), _ptr(lse), _ptr(S_out), ws.data_ptr(), ws.numel(), _stream()), "dsa_layer")
    return out


# ---------------------------------------------------------------------------------------------
# device copies of a synthetic batch

class DeviceBatch:
    """The tensors of a synth.Batch on the GPU, typed for the library."""

    def __init__(self, hb, device="cuda"):
        dev = torch.device(device)
        self.host = hb
        self.batch = Batch.from_host(hb.seq_lens, hb.cu_q, hb.block_table, hb.num_pages, device=dev)
        f8 = lambda a: torch.from_numpy(a).to(dev).view(torch.float8_e4m3fn)
        bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
        self.qI = f8(hb.qI)
        self.qI_scale = torch.from_numpy(hb.qI_scale).to(dev)
        self.wI = torch.from_numpy(hb.wI).to(dev)
        self.kI_cache = f8(hb.kI_cache)
        self.kI_scale = torch.from_numpy(hb.kI_scale).to(dev)
        self.q = bf(hb.q)
        self.kv_cache = bf(hb.kv_cache)
        self.nhI = int(hb.qI.shape[1])
        self.H = int(hb.q.shape[1])
        self.k = hb.wl.topk
        self.softmax_scale = hb.wl.softmax_scale
