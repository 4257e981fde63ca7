"""Thin Python front end of libsoup: passes torch device pointers and streams through the
C-ABI.  PyTorch supplies device memory (through the allocator callback) and streams; every
step of the computation runs in libsoup's CUDA kernels.
"""
from __future__ import annotations

import ctypes
from ctypes import byref, c_float, c_int, c_size_t, c_void_p

import numpy as np
import torch

from . import _lib
from ._lib import PROJ, Batch, ModelConfig, Stats, check, lib


def make_config(cfg: dict, mode: str = "streamed", n_layer_buffers: int = 2, max_tokens: int | None = None,
                device: int = 0, source: str = "ram", stack_path: str | None = None) -> ModelConfig:
    c = ModelConfig()
    for k in ("n_layers", "hidden", "n_heads", "n_kv_heads", "head_dim", "intermediate", "vocab", "lora_r"):
        setattr(c, k, int(cfg[k]))
    c.rms_eps = float(cfg["rms_eps"])
    c.rope_theta = float(cfg["rope_theta"])
    c.lora_alpha = float(cfg["lora_alpha"])
    c.mode = _lib.SOUP_STREAMED if mode == "streamed" else _lib.SOUP_RESIDENT
    c.n_layer_buffers = int(n_layer_buffers)
    c.max_tokens = int(max_tokens if max_tokens is not None else cfg["batch"] * cfg["seq"])
    c.device = int(device)
    c.stream_source = {"ram": _lib.SOUP_SOURCE_RAM, "file": _lib.SOUP_SOURCE_FILE, "auto": _lib.SOUP_SOURCE_AUTO}[source]
    c.stack_path = stack_path.encode() if stack_path else None
    return c


def blob_bytes(cfg: dict) -> int:
    n = c_size_t()
    check(lib.soup_layer_blob_bytes(byref(make_config(cfg)), byref(n)))
    return n.value


def blob_part(cfg: dict, proj: int, part: int):
    off, sz = c_size_t(), c_size_t()
    check(lib.soup_layer_blob_part(byref(make_config(cfg)), proj, part, byref(off), byref(sz)))
    return off.value, sz.value


def lora_numel(cfg: dict) -> int:
    n = c_size_t()
    check(lib.soup_lora_numel(byref(make_config(cfg)), byref(n)))
    return n.value


def lora_offset(cfg: dict, layer: int, proj: int, which_b: int):
    off, r, c = c_size_t(), c_int(), c_int()
    check(lib.soup_lora_offset(byref(make_config(cfg)), layer, proj, which_b, byref(off), byref(r), byref(c)))
    return off.value, r.value, c.value


def codebook() -> np.ndarray:
    out = (c_float * 16)()
    check(lib.soup_nf4_codebook(out))
    return np.frombuffer(out, dtype=np.float32).copy()


def _stream_ptr(stream=None) -> c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> c_void_p:
    return c_void_p(t.data_ptr()) if t is not None else c_void_p(None)


class _TorchAllocator:
    """Routes the library's device allocations to PyTorch's caching allocator."""

    def __init__(self, device: int):
        self.device = device

        def _alloc(nbytes, user):
            try:
                return torch.cuda.caching_allocator_alloc(int(nbytes), self.device)
            except Exception:  # the library reports SOUP_ERR_OOM
                return None

        def _free(p, user):
            torch.cuda.caching_allocator_delete(int(p))

        self._alloc = _lib.ALLOC_FN(_alloc)
        self._free = _lib.FREE_FN(_free)
        self.struct = _lib.Allocator(self._alloc, self._free, None)


class SoupModel:
    def __init__(self, cfg: dict, mode: str = "streamed", n_layer_buffers: int = 2, max_tokens: int | None = None,
                 device: int = 0, torch_alloc: bool = True, source: str = "ram", stack_path: str | None = None):
        """source: "ram" (page-locked host stack), "file" (stack file at stack_path, streamed
        through page-locked staging) or "auto" (RAM if it fits, else the file)."""
        self.cfg = dict(cfg)
        self.ccfg = make_config(cfg, mode, n_layer_buffers, max_tokens, device, source, stack_path)
        self.device = torch.device("cuda", device)
        self._allocator = _TorchAllocator(device) if torch_alloc else None
        h = c_void_p()
        check(lib.soup_model_create(byref(self.ccfg), byref(self._allocator.struct) if self._allocator else None,
                                    byref(h)))
        self.h = h
        self.blob_bytes = blob_bytes(cfg)
        self._keep = {}
        self.lora_n = lora_numel(cfg)

    # ------------------------------------------------------------------ lifecycle
    def close(self):
        if getattr(self, "h", None):
            torch.cuda.synchronize(self.device)
            check(lib.soup_model_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _ck(self, status):
        check(status, self.h)

    # ------------------------------------------------------------------ weights
    def quantize_layer(self, layer: int, w: dict, gamma_attn: torch.Tensor, gamma_mlp: torch.Tensor):
        """w[p]: fp32 cuda tensors [out, in]; gammas: bf16 cuda tensors [hidden]."""
        ptrs = (c_void_p * 7)(*[w[p].data_ptr() for p in PROJ])
        self._ck(lib.soup_model_quantize_layer(self.h, layer, ptrs, _ptr(gamma_attn), _ptr(gamma_mlp), _stream_ptr()))

    def load_layer(self, layer: int, w: dict, gamma_attn: np.ndarray, gamma_mlp: np.ndarray):
        """w[p]: host fp32 arrays [out, in]; gammas: host bf16 bit patterns (uint16) [hidden].
        The library quantises on the host into its page-locked layer stack."""
        arrs = [np.ascontiguousarray(w[p], dtype=np.float32) for p in PROJ]
        ga = np.ascontiguousarray(gamma_attn, dtype=np.uint16)
        gm = np.ascontiguousarray(gamma_mlp, dtype=np.uint16)
        ptrs = (c_void_p * 7)(*[a.ctypes.data for a in arrs])
        self._ck(lib.soup_model_load_layer(self.h, layer, ptrs, ga.ctypes.data_as(c_void_p),
                                           gm.ctypes.data_as(c_void_p)))

    def load_layer_nf4(self, layer: int, blob: np.ndarray):
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        self._ck(lib.soup_model_load_layer_nf4(self.h, layer, blob.ctypes.data_as(c_void_p), blob.nbytes))

    def read_layer_nf4(self, layer: int) -> np.ndarray:
        out = np.empty(self.blob_bytes, dtype=np.uint8)
        self._ck(lib.soup_model_read_layer_nf4(self.h, layer, out.ctypes.data_as(c_void_p), out.nbytes))
        return out

    def set_head(self, embed: torch.Tensor, final_gamma: torch.Tensor, lm_head: torch.Tensor):
        self._keep["head"] = (embed, final_gamma, lm_head)
        self._ck(lib.soup_model_set_head(self.h, _ptr(embed), _ptr(final_gamma), _ptr(lm_head)))

    def set_lora(self, params: torch.Tensor):
        """params: flat fp32 cuda tensor of lora_numel elements (layout of include/soup.h)."""
        assert params.numel() == self.lora_n and params.dtype == torch.float32 and params.is_cuda
        self.lora_params = params
        self.lora_grads = torch.zeros_like(params)
        self.adam_m = torch.zeros_like(params)
        self.adam_v = torch.zeros_like(params)
        self._ck(lib.soup_model_set_lora(self.h, _ptr(self.lora_params), _ptr(self.lora_grads), _ptr(self.adam_m),
                                         _ptr(self.adam_v)))

    def set_lora_proj(self, layer: int, proj: str, A: torch.Tensor, B: torch.Tensor):
        """Copies one projection's fp32 adapters (cuda or cpu tensors) into the parameter buffer."""
        A = A.to(torch.float32).contiguous()
        B = B.to(torch.float32).contiguous()
        self._ck(lib.soup_model_set_lora_proj(self.h, layer, PROJ.index(proj), _ptr(A), _ptr(B), _stream_ptr()))
        torch.cuda.current_stream().synchronize()

    def refresh_lora(self):
        """Call after changing lora_params outside the library (refreshes its bf16 copy)."""
        self._ck(lib.soup_model_refresh_lora(self.h, _stream_ptr()))

    def lora_view(self, flat: torch.Tensor, layer: int, proj: str, which_b: int) -> torch.Tensor:
        off, r, c = lora_offset(self.cfg, layer, PROJ.index(proj), which_b)
        return flat[off:off + r * c].view(r, c)

    def set_lora_enabled(self, enabled: bool):
        self._ck(lib.soup_set_lora_enabled(self.h, 1 if enabled else 0))

    def merge_lora(self, layer: int, proj: str, out: torch.Tensor | None = None) -> torch.Tensor:
        """bf16 [out_features, in_features]: the projection's NF4 base fused with its adapter."""
        j = PROJ.index(proj)
        rows, cols = self._proj_shape(j)
        if out is None:
            out = torch.empty(rows, cols, dtype=torch.bfloat16, device=self.device)
        assert out.dtype == torch.bfloat16 and out.is_contiguous() and tuple(out.shape) == (rows, cols)
        self._ck(lib.soup_model_merge_lora(self.h, layer, j, _ptr(out), _stream_ptr()))
        return out

    def _proj_shape(self, j: int):
        c = self.cfg
        qd, kvd = c["n_heads"] * c["head_dim"], c["n_kv_heads"] * c["head_dim"]
        h, I = c["hidden"], c["intermediate"]
        return [(qd, h), (kvd, h), (kvd, h), (h, qd), (I, h), (I, h), (h, I)][j]

    # ------------------------------------------------------------------ compute
    def layer_fwd(self, layer: int, x: torch.Tensor, B: int, S: int, out: torch.Tensor | None = None):
        y = out if out is not None else torch.empty_like(x)
        self._ck(lib.soup_layer_fwd(self.h, layer, _ptr(x), _ptr(y), B, S, _stream_ptr()))
        return y

    def layer_bwd(self, layer: int, dy: torch.Tensor, B: int, S: int, out: torch.Tensor | None = None):
        dx = out if out is not None else torch.empty_like(dy)
        self._ck(lib.soup_layer_bwd(self.h, layer, _ptr(dy), _ptr(dx), B, S, _stream_ptr()))
        return dx

    def step(self, ids, loss: str = "sft", mask=None, n_pairs: int = 0, prefix_len: int = 0, beta: float = 0.1,
             lr: float = 2e-5, apply_optimizer: bool = True, dpo_shared_load: bool = False, labels=None,
             gamma: float = 0.0, lambda_or: float = 0.1, lambda_d: float = 1.0, lambda_u: float = 1.0,
             share_prefix: bool = False) -> float:
        """ids: int32 [B, S] as a cuda tensor, or as host memory (numpy / cpu tensor: copied by the
        library); mask (SFT) and labels (KTO, uint8 [B]) in the same memory space as ids."""
        b = Batch()
        on_host = not (isinstance(ids, torch.Tensor) and ids.is_cuda)
        keep = []

        def _host_u8(a):
            t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a, np.uint8))
            t = t.contiguous()
            keep.append(t)
            return t.data_ptr()

        if on_host:
            ids_h = ids if isinstance(ids, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(ids, np.int32))
            ids_h = ids_h.contiguous()
            assert ids_h.dtype == torch.int32
            b.ids = ids_h.data_ptr()
            keep.append(ids_h)
            if mask is not None:
                b.loss_mask = _host_u8(mask)
            if labels is not None:
                b.labels = _host_u8(labels)
            B, S = ids_h.shape
        else:
            assert ids.dtype == torch.int32
            b.ids = ids.data_ptr()
            if mask is not None:
                b.loss_mask = mask.data_ptr()
            if labels is not None:
                if not (isinstance(labels, torch.Tensor) and labels.is_cuda):
                    labels = torch.as_tensor(np.ascontiguousarray(labels, np.uint8)).to(ids.device)
                assert labels.dtype == torch.uint8
                keep.append(labels)
                b.labels = labels.data_ptr()
            B, S = ids.shape
        b.B, b.S = int(B), int(S)
        b.ids_on_host = 1 if on_host else 0
        b.n_pairs, b.prefix_len, b.beta = int(n_pairs), int(prefix_len), float(beta)
        b.lr, b.apply_optimizer = float(lr), 1 if apply_optimizer else 0
        b.dpo_shared_load = 1 if dpo_shared_load else 0
        b.gamma, b.lambda_or, b.lambda_d, b.lambda_u = float(gamma), float(lambda_or), float(lambda_d), float(lambda_u)
        b.share_prefix = 1 if share_prefix else 0
        out = c_float()
        self._ck(lib.soup_step(self.h, _lib.LOSS_KINDS[loss], byref(b), byref(out), _stream_ptr()))
        return out.value

    def optimizer_step(self, lr: float):
        self._ck(lib.soup_optimizer_step(self.h, float(lr), _stream_ptr()))

    def last_logps(self, n: int):
        pi, ref = (c_float * n)(), (c_float * n)()
        self._ck(lib.soup_last_logps(self.h, pi, ref, n))
        return np.array(pi[:]), np.array(ref[:])

    def stats(self) -> dict:
        s = Stats()
        self._ck(lib.soup_get_stats(self.h, byref(s)))
        return {k: getattr(s, k) for k, _ in Stats._fields_}

    def h2d_probe(self, reps: int = 20) -> float:
        """GB/s of back-to-back layer copies on the streamer's own copy path."""
        out = ctypes.c_double()
        self._ck(lib.soup_h2d_probe(self.h, int(reps), byref(out)))
        return out.value

    def set_profiling(self, enabled: bool):
        self._ck(lib.soup_set_profiling(self.h, 1 if enabled else 0))

    def profile(self, reset: bool = False) -> dict:
        arr = (_lib.ProfileEntry * 64)()
        n = c_int()
        self._ck(lib.soup_get_profile(self.h, arr, 64, byref(n), 1 if reset else 0))
        return {arr[i].name.decode(): dict(launches=arr[i].launches, total_ms=arr[i].total_ms, flops=arr[i].flops,
                                           bytes=arr[i].bytes) for i in range(n.value)}

    def set_timed_category(self, name: str | None):
        """Event pairs around every launch of one profile category ("all": every category) in
        ordinary (graph-replayed) calls; None turns them off."""
        self._ck(lib.soup_set_timed_category(self.h, (name or "").encode()))

    def timed_category(self, reset: bool = False) -> dict:
        e = _lib.ProfileEntry()
        self._ck(lib.soup_get_timed_category(self.h, byref(e), 1 if reset else 0))
        return dict(name=e.name.decode(), launches=e.launches, total_ms=e.total_ms, flops=e.flops, bytes=e.bytes)

    def timed_profile(self, reset: bool = False) -> dict:
        arr = (_lib.ProfileEntry * 64)()
        n = c_int()
        self._ck(lib.soup_get_timed_profile(self.h, arr, 64, byref(n), 1 if reset else 0))
        return {arr[i].name.decode(): dict(launches=arr[i].launches, total_ms=arr[i].total_ms, flops=arr[i].flops,
                                           bytes=arr[i].bytes) for i in range(n.value)}

    def reset_stats(self):
        self._ck(lib.soup_reset_stats(self.h))

    def check_device(self):
        self._ck(lib.soup_check_device(self.h, _stream_ptr()))


# ---------------------------------------------------------------------- single ops
def nf4_quantize(w: torch.Tensor) -> dict:
    """NF4 + double quant of a cuda fp32 tensor; returns device tensors."""
    n = w.numel()
    nb = (n + 63) // 64
    ng = (nb + 255) // 256
    dev = w.device
    out = dict(codes=torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
               q8=torch.empty(nb, dtype=torch.int8, device=dev),
               scales=torch.empty(ng, dtype=torch.float32, device=dev),
               mean=torch.empty(1, dtype=torch.float32, device=dev))
    scratch = torch.empty(nb, dtype=torch.float32, device=dev)
    check(lib.soup_nf4_quantize(_ptr(w), n, _ptr(out["codes"]), _ptr(out["q8"]), _ptr(out["scales"]),
                                _ptr(out["mean"]), _ptr(scratch), _stream_ptr()))
    out["n"] = n
    out["shape"] = tuple(w.shape)
    return out


def nf4_quantize_host(w: np.ndarray, threads: int = 0) -> dict:
    """NF4 + double quant of a host fp32 array on the host (no GPU); numpy outputs."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n = w.size
    nb = (n + 63) // 64
    ng = (nb + 255) // 256
    out = dict(codes=np.empty((n + 1) // 2, np.uint8), q8=np.empty(nb, np.int8), scales=np.empty(ng, np.float32),
               mean=np.empty(1, np.float32))
    p = lambda a: a.ctypes.data_as(c_void_p)
    check(lib.soup_nf4_quantize_host(p(w), n, p(out["codes"]), p(out["q8"]), p(out["scales"]), p(out["mean"]),
                                     int(threads)))
    return out


def nf4_dequantize(q: dict) -> torch.Tensor:
    """bf16 (as int16 bit patterns viewed as bfloat16) tensor of shape q['shape']."""
    out = torch.empty(q["n"], dtype=torch.bfloat16, device=q["codes"].device)
    check(lib.soup_nf4_dequantize(_ptr(q["codes"]), _ptr(q["q8"]), _ptr(q["scales"]), _ptr(q["mean"]), q["n"],
                                  _ptr(out), _stream_ptr()))
    return out.view(q["shape"])


def gemm_plan(M: int, N: int, K: int, nf4: bool = True, transposed: bool = False, sms: int = 148) -> dict:
    """How the library schedules y[M, N] = x[M, K] W^T (host only; see soup_gemm_plan)."""
    info = _lib.GemmPlanInfo()
    check(lib.soup_gemm_plan(M, N, K, 1 if nf4 else 0, 1 if transposed else 0, sms, byref(info)))
    return {f: getattr(info, f) for f, _ in _lib.GemmPlanInfo._fields_}


def stream_k_pieces(tiles: int, kblocks_per_tile: int, ctas: int, cta: int) -> list:
    """(tile, kb_lo, kb_hi, slot) of each piece of one stream-K CTA (slot -1: whole tile)."""
    cap = 64
    arrs = [(c_int * cap)() for _ in range(4)]
    n = c_int()
    check(lib.soup_gemm_stream_k_pieces(tiles, kblocks_per_tile, ctas, cta, cap, *arrs, byref(n)))
    return [tuple(a[i] for a in arrs) for i in range(min(n.value, cap))]


def stream_k_shares(tiles: int, kblocks_per_tile: int, ctas: int, tile: int) -> list:
    """(cta, slot) of each share of one stream-K tile, in k order (slot -1: one CTA alone)."""
    cap = 64
    cta, slot, n = (c_int * cap)(), (c_int * cap)(), c_int()
    check(lib.soup_gemm_stream_k_shares(tiles, kblocks_per_tile, ctas, tile, cap, cta, slot, byref(n)))
    return [(cta[i], slot[i]) for i in range(min(n.value, cap))]


def nf4_matmul(x: torch.Tensor, q: dict, transpose_w: bool = False, residual: torch.Tensor | None = None):
    """y = x W^T (W = NF4 tensor [N, K]) or y = x W when transpose_w; bf16 in/out."""
    N, K = q["shape"]
    M = x.shape[0]
    y = torch.empty((M, K if transpose_w else N), dtype=torch.bfloat16, device=x.device)
    check(lib.soup_nf4_matmul(_ptr(x), M, N, K, _ptr(q["codes"]), _ptr(q["q8"]), _ptr(q["scales"]), _ptr(q["mean"]),
                              1 if transpose_w else 0, _ptr(residual), _ptr(y), _stream_ptr()))
    return y
