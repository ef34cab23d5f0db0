"""B200-native Compressed Sparse Attention (CSA) and Heavily Compressed Attention (HCA).

Thin Python binding over the C ABI of ``libcsa.so`` (declared in include/csa.h).
Every function here only checks tensor metadata, allocates outputs and scratch
with torch (device memory is torch's job here) and calls the library entry point
of the same name; all arithmetic runs in the library's CUDA kernels.  There is
no CPU or PyTorch fallback: a missing library raises.

Shapes (B sequences, Tq query rows, N entries, H heads in {16, 64}):
  csa_compress / hca_compress: x bf16 [B, T, d] -> bf16 [B, N, d], or with
      ``fp8=True`` (d == 192) the split cache (nope e4m3 as uint8 [B, N, 128],
      rope bf16 [B, N, 64], scale fp32 [B, N]).
  csa_indexer_topk: qI bf16 [B, Tq, 4, 64], wI fp32 [B, Tq, 4], kIc bf16
      [B, N, 64] -> idx int32 [B, Tq, k] (ascending, -1 padded).
  csa_sparse_mqa / hca_dense_mqa: q bf16 [B, Tq, H, 192] -> (out bf16
      [B, Tq, H, 128], lse fp32 [B, Tq, H]).
  grouped_out_proj: out bf16 [..., H, 128], w bf16 [G, d_g, (H/G)*128] ->
      y bf16 [..., G, d_g].
"""
from __future__ import annotations

import ctypes
import dataclasses

import torch

from . import _lib

__all__ = ["CsaError", "KVCache", "Window", "csa_compress", "hca_compress", "csa_indexer_topk", "csa_indexer_topk_e4m3",
           "csa_indexer_topk_workspace_size", "csa_sparse_mqa", "csa_sparse_mqa_workspace_size", "hca_dense_mqa",
           "hca_dense_mqa_workspace_size", "grouped_out_proj", "launch_count", "version", "Packed", "csa_compress_append",
           "hca_compress_append", "csa_compress_packed", "hca_compress_packed", "csa_indexer_topk_packed",
           "csa_sparse_mqa_packed", "hca_dense_mqa_packed", "csa_indexer_topk_e2m1"]


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        msg = lib.csa_last_error().decode()
        super().__init__(f"{where}: {lib.csa_status_string(status).decode()} ({msg})")
        self.status = status


def _check(status: int, where: str):
    if status != _lib.CSA_OK:
        raise CsaError(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def version() -> str:
    return _lib.load().csa_version().decode()


def launch_count() -> int:
    """Kernels the library has enqueued in this process (graph captures count once)."""
    return int(_lib.load().csa_launch_count())


@dataclasses.dataclass
class KVCache:
    """A compressed cache: bf16 (k, optional v) or split FP8 (nope, rope, scale)."""
    k: torch.Tensor | None = None
    v: torch.Tensor | None = None
    nope: torch.Tensor | None = None
    rope: torch.Tensor | None = None
    scale: torch.Tensor | None = None

    @property
    def split(self) -> bool:
        return self.nope is not None

    @property
    def n_entries(self) -> int:
        # entries per sequence ([B, N, ...]), or all entries of packed sequences ([total_entries, ...])
        return (self.nope if self.split else self.k).shape[-2]

    def desc(self) -> _lib.KVCacheDesc:
        d = _lib.KVCacheDesc()
        d.layout = _lib.CSA_KV_SPLIT_FP8 if self.split else _lib.CSA_KV_BF16
        d.reserved = 0
        d.n_entries = self.n_entries
        d.k, d.v = _ptr(self.k), _ptr(self.v)
        d.nope, d.rope, d.scale = _ptr(self.nope), _ptr(self.rope), _ptr(self.scale)
        return d


@dataclasses.dataclass
class Window:
    """Raw tokens for the sliding-window branch: rows hold positions pos0, pos0+1, ..."""
    k: torch.Tensor | None
    v: torch.Tensor | None = None
    pos0: int = 0
    length: int = 128

    def desc(self) -> _lib.WindowDesc:
        d = _lib.WindowDesc()
        d.k, d.v = _ptr(self.k), _ptr(self.v)
        d.pos0 = self.pos0
        # rows per sequence ([B, rows, 192]), or all packed tokens ([total_tokens, 192])
        d.rows = 0 if self.k is None else self.k.shape[-2]
        d.len = self.length
        d.reserved = 0
        return d


def _compress(fn_name, x, w, b_pos, stride, fp8, out, stream):
    lib = _lib.load()
    B, T, d = x.shape
    N = -(-T // stride)
    if fp8:
        nope, rope, scale = out if out is not None else (
            torch.empty(B, N, 128, dtype=torch.uint8, device=x.device),
            torch.empty(B, N, 64, dtype=torch.bfloat16, device=x.device),
            torch.empty(B, N, dtype=torch.float32, device=x.device))
        st = getattr(lib, fn_name)(_ptr(x), B, T, d, stride, _ptr(w), _ptr(b_pos), _lib.CSA_KV_SPLIT_FP8,
                                   _ptr(nope), _ptr(rope), _ptr(scale), _stream(stream))
        _check(st, fn_name)
        return nope, rope, scale
    y = out if out is not None else torch.empty(B, N, d, dtype=torch.bfloat16, device=x.device)
    st = getattr(lib, fn_name)(_ptr(x), B, T, d, stride, _ptr(w), _ptr(b_pos), _lib.CSA_KV_BF16, _ptr(y), None,
                               None, _stream(stream))
    _check(st, fn_name)
    return y


def csa_compress(x, w, b_pos, m, *, fp8=False, out=None, stream=None):
    """CSA compression: overlapping 2m-token windows with stride m."""
    return _compress("csa_compress", x, w, b_pos, m, fp8, out, stream)


def hca_compress(x, w, b_pos, m_prime, *, fp8=False, out=None, stream=None):
    """HCA compression: non-overlapping m'-token windows."""
    return _compress("hca_compress", x, w, b_pos, m_prime, fp8, out, stream)


def csa_indexer_topk_workspace_size(B, Tq, N, k) -> int:
    return int(_lib.load().csa_indexer_topk_workspace_size(B, Tq, N, k))


def csa_indexer_topk_coded_workspace_size(B, Tq, N, k) -> int:
    """Workspace of the E4M3 / E2M1 key calls and of csa_indexer_topk_with_scores."""
    return int(_lib.load().csa_indexer_topk_coded_workspace_size(B, Tq, N, k))


def csa_indexer_topk(qI, wI, kIc, m, k, *, q_pos0=0, idx=None, workspace=None, stream=None):
    """Lightning-indexer scores and top-k entry ids (int32 [B, Tq, k], ascending, -1 padded)."""
    lib = _lib.load()
    B, Tq = qI.shape[0], qI.shape[1]
    N = kIc.shape[1]
    if idx is None:
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=qI.device)
    need = csa_indexer_topk_workspace_size(B, Tq, N, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=qI.device)
    st = lib.csa_indexer_topk(_ptr(qI), _ptr(wI), _ptr(kIc), B, Tq, N, q_pos0, m, k, _ptr(idx), _ptr(workspace),
                              workspace.numel(), _stream(stream))
    _check(st, "csa_indexer_topk")
    return idx


def csa_indexer_topk_e4m3(qI, wI, kI_codes, kI_scale, m, k, *, q_pos0=0, idx=None, workspace=None, stream=None):
    """csa_indexer_topk over FP8 keys: kI_codes uint8 [B, N, 64] (E4M3), kI_scale fp32 [B, N]."""
    lib = _lib.load()
    B, Tq = qI.shape[0], qI.shape[1]
    N = kI_codes.shape[1]
    if idx is None:
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=qI.device)
    need = csa_indexer_topk_coded_workspace_size(B, Tq, N, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=qI.device)
    st = lib.csa_indexer_topk_e4m3(_ptr(qI), _ptr(wI), _ptr(kI_codes), _ptr(kI_scale), B, Tq, N, q_pos0, m, k,
                                   _ptr(idx), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "csa_indexer_topk_e4m3")
    return idx


def csa_indexer_topk_e2m1(qI, wI, kI_codes, kI_scale, m, k, *, q_pos0=0, idx=None, workspace=None, stream=None):
    """csa_indexer_topk over FP4 keys: kI_codes uint8 [B, N, 32] (E2M1, two per byte, low nibble = even
    dimension), kI_scale fp32 [B, N]."""
    lib = _lib.load()
    B, Tq = qI.shape[0], qI.shape[1]
    N = kI_codes.shape[1]
    if idx is None:
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=qI.device)
    need = csa_indexer_topk_coded_workspace_size(B, Tq, N, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=qI.device)
    st = lib.csa_indexer_topk_e2m1(_ptr(qI), _ptr(wI), _ptr(kI_codes), _ptr(kI_scale), B, Tq, N, q_pos0, m, k,
                                   _ptr(idx), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "csa_indexer_topk_e2m1")
    return idx


def csa_sparse_mqa_workspace_size(B, Tq, H, k, win_len) -> int:
    return int(_lib.load().csa_sparse_mqa_workspace_size(B, Tq, H, k, win_len))


def hca_dense_mqa_workspace_size(B, Tq, H, N, win_len) -> int:
    return int(_lib.load().hca_dense_mqa_workspace_size(B, Tq, H, N, win_len))


def _attn_out(q, out, lse):
    B, Tq, H, _ = q.shape
    if out is None:
        out = torch.empty(B, Tq, H, 128, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, Tq, H, dtype=torch.float32, device=q.device)
    return out, lse


def csa_sparse_mqa(q, cache: KVCache, m, idx, win: Window | None, scale, *, q_pos0=0, out=None, lse=None,
                   workspace=None, stream=None):
    """CSA core attention over the selected entries plus the sliding window (one softmax)."""
    lib = _lib.load()
    B, Tq, H, _ = q.shape
    k = idx.shape[-1]
    out, lse = _attn_out(q, out, lse)
    wlen = win.length if win is not None else 0
    need = csa_sparse_mqa_workspace_size(B, Tq, H, k, wlen)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    cd = cache.desc()
    wd = win.desc() if win is not None else None
    st = lib.csa_sparse_mqa(_ptr(q), B, Tq, H, q_pos0, ctypes.byref(cd), m, _ptr(idx), k,
                            ctypes.byref(wd) if wd is not None else None, float(scale), _ptr(out), _ptr(lse),
                            _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "csa_sparse_mqa")
    return out, lse


def hca_dense_mqa(q, cache: KVCache, m_prime, win: Window | None, scale, *, q_pos0=0, out=None, lse=None,
                  workspace=None, stream=None, max_sms=0):
    """HCA core attention over every visible entry plus the sliding window (one softmax).

    ``max_sms`` > 0 keeps the 64-head decode launch to that many SMs (``hca_dense_mqa_budget``), leaving the
    rest to work the caller runs beside it on another stream."""
    lib = _lib.load()
    B, Tq, H, _ = q.shape
    out, lse = _attn_out(q, out, lse)
    wlen = win.length if win is not None else 0
    need = hca_dense_mqa_workspace_size(B, Tq, H, cache.n_entries, wlen)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    cd = cache.desc()
    wd = win.desc() if win is not None else None
    wsz = 0 if workspace is None else workspace.numel()
    if max_sms:
        st = lib.hca_dense_mqa_budget(_ptr(q), B, Tq, H, q_pos0, ctypes.byref(cd), m_prime,
                                      ctypes.byref(wd) if wd is not None else None, float(scale), _ptr(out), _ptr(lse),
                                      int(max_sms), _ptr(workspace), wsz, _stream(stream))
        _check(st, "hca_dense_mqa_budget")
    else:
        st = lib.hca_dense_mqa(_ptr(q), B, Tq, H, q_pos0, ctypes.byref(cd), m_prime,
                               ctypes.byref(wd) if wd is not None else None, float(scale), _ptr(out), _ptr(lse),
                               _ptr(workspace), wsz, _stream(stream))
        _check(st, "hca_dense_mqa")
    return out, lse


def grouped_out_proj(o, w, *, y=None, stream=None):
    """Grouped output projection: heads in G groups of H/G, group g's outputs times w[g]^T.

    o bf16 [..., H, 128] (attention output), w bf16 [G, d_g, (H/G)*128] -> y bf16 [..., G, d_g].
    """
    lib = _lib.load()
    H = o.shape[-2]
    G, dg = w.shape[0], w.shape[1]
    lead = tuple(o.shape[:-2])
    R = 1
    for n in lead:
        R *= n
    if y is None:
        y = torch.empty(*lead, G, dg, dtype=torch.bfloat16, device=o.device)
    st = lib.csa_grouped_out_proj(_ptr(o), R, H, G, dg, _ptr(w), _ptr(y), _stream(stream))
    _check(st, "csa_grouped_out_proj")
    return y


class Packed:
    """Packed sequences (e.g. the documents of a packed pre-training batch) for one stride.

    Built from the host-side sequence lengths: sequence s owns packed tokens [cu_tokens[s], cu_tokens[s+1])
    and entries [cu_entries[s], cu_entries[s+1]) (ceil(len / stride) of them).  The offsets are uploaded once.
    """

    def __init__(self, lengths, stride, device="cuda"):
        lens = [int(n) for n in lengths]
        if any(n < 0 for n in lens):
            raise ValueError("sequence lengths must be >= 0")
        ent = [-(-n // stride) for n in lens]
        cu_t, cu_e = [0], [0]
        for n, e in zip(lens, ent):
            cu_t.append(cu_t[-1] + n)
            cu_e.append(cu_e[-1] + e)
        self.lengths, self.stride = lens, stride
        self.cu_tokens_host, self.cu_entries_host = cu_t, cu_e
        self.cu_tokens = torch.tensor(cu_t, dtype=torch.int32, device=device)
        self.cu_entries = torch.tensor(cu_e, dtype=torch.int32, device=device)
        self.total_tokens, self.total_entries = cu_t[-1], cu_e[-1]
        self.max_tokens = max(lens) if lens else 0

    def desc(self) -> _lib.PackedDesc:
        d = _lib.PackedDesc()
        d.cu_tokens, d.cu_entries = _ptr(self.cu_tokens), _ptr(self.cu_entries)
        d.n_seqs = len(self.lengths)
        d.max_tokens = self.max_tokens
        d.total_tokens, d.total_entries = self.total_tokens, self.total_entries
        return d


def _compress_append(fn_name, x, x_pos0, t, w, b_pos, stride, cache, stream):
    lib = _lib.load()
    B, rows, d = x.shape
    if isinstance(cache, KVCache) and cache.split:
        st = getattr(lib, fn_name)(_ptr(x), B, rows, x_pos0, t, d, stride, _ptr(w), _ptr(b_pos),
                                   _lib.CSA_KV_SPLIT_FP8, _ptr(cache.nope), _ptr(cache.rope), _ptr(cache.scale),
                                   cache.nope.shape[1], _stream(stream))
    else:
        k = cache.k if isinstance(cache, KVCache) else cache
        st = getattr(lib, fn_name)(_ptr(x), B, rows, x_pos0, t, d, stride, _ptr(w), _ptr(b_pos), _lib.CSA_KV_BF16,
                                   _ptr(k), None, None, k.shape[1], _stream(stream))
    _check(st, fn_name)


def csa_compress_append(x, x_pos0, t, w, b_pos, m, cache, *, stream=None):
    """Decode-time append: if token t completes CSA entry i = (t+1)/m - 1, write it into cache slot i.

    x bf16 [B, rows, d] holds raw tokens at positions x_pos0 ..; cache is a bf16 tensor [B, n_cap, d] or a split
    FP8 KVCache (nope [B, n_cap, 128], rope, scale)."""
    _compress_append("csa_compress_append", x, x_pos0, t, w, b_pos, m, cache, stream)


def hca_compress_append(x, x_pos0, t, w, b_pos, m_prime, cache, *, stream=None):
    """Decode-time append of the HCA entry that token t completes (t + 1 a multiple of m')."""
    _compress_append("hca_compress_append", x, x_pos0, t, w, b_pos, m_prime, cache, stream)


def _compress_packed(fn_name, x, packed: Packed, w, b_pos, stride, fp8, stream):
    lib = _lib.load()
    d = x.shape[-1]
    E = packed.total_entries
    pd = packed.desc()
    if fp8:
        nope = torch.empty(E, 128, dtype=torch.uint8, device=x.device)
        rope = torch.empty(E, 64, dtype=torch.bfloat16, device=x.device)
        scale = torch.empty(E, dtype=torch.float32, device=x.device)
        st = getattr(lib, fn_name)(_ptr(x), ctypes.byref(pd), d, stride, _ptr(w), _ptr(b_pos), _lib.CSA_KV_SPLIT_FP8,
                                   _ptr(nope), _ptr(rope), _ptr(scale), _stream(stream))
        _check(st, fn_name)
        return nope, rope, scale
    y = torch.empty(E, d, dtype=torch.bfloat16, device=x.device)
    st = getattr(lib, fn_name)(_ptr(x), ctypes.byref(pd), d, stride, _ptr(w), _ptr(b_pos), _lib.CSA_KV_BF16, _ptr(y),
                               None, None, _stream(stream))
    _check(st, fn_name)
    return y


def csa_compress_packed(x, packed: Packed, w, b_pos, m, *, fp8=False, stream=None):
    """CSA compression of packed sequences x bf16 [total_tokens, d] -> entries [total_entries, d]."""
    if packed.stride != m:
        raise ValueError("packed descriptor was built for another stride")
    return _compress_packed("csa_compress_packed", x, packed, w, b_pos, m, fp8, stream)


def hca_compress_packed(x, packed: Packed, w, b_pos, m_prime, *, fp8=False, stream=None):
    """HCA compression of packed sequences x bf16 [total_tokens, d] -> entries [total_entries, d]."""
    if packed.stride != m_prime:
        raise ValueError("packed descriptor was built for another stride")
    return _compress_packed("hca_compress_packed", x, packed, w, b_pos, m_prime, fp8, stream)


def csa_indexer_topk_packed(qI, wI, kIc, packed: Packed, m, k, *, idx=None, workspace=None, stream=None):
    """Indexer top-k over packed sequences: qI [total_tokens, 4, 64] -> idx int32 [total_tokens, k] of entry
    indices within each row's own sequence (ascending, -1 padded)."""
    lib = _lib.load()
    if packed.stride != m:
        raise ValueError("packed descriptor was built for another stride")
    pd = packed.desc()
    if idx is None:
        idx = torch.empty(packed.total_tokens, k, dtype=torch.int32, device=qI.device)
    need = int(lib.csa_indexer_topk_packed_workspace_size(ctypes.byref(pd), m, k))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=qI.device)
    st = lib.csa_indexer_topk_packed(_ptr(qI), _ptr(wI), _ptr(kIc), ctypes.byref(pd), m, k, _ptr(idx),
                                     _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "csa_indexer_topk_packed")
    return idx


def _packed_window(k, v, packed, length):
    return Window(k=k, v=v, pos0=0, length=length)


def csa_sparse_mqa_packed(q, packed: Packed, cache: KVCache, m, idx, win_k, win_v, win_len, scale, *, out=None,
                          lse=None, workspace=None, stream=None):
    """CSA attention over packed sequences: q [total_tokens, H, 192]; the window is read from the packed raw
    tokens win_k [total_tokens, 192] (win_v [total_tokens, 128] or None)."""
    lib = _lib.load()
    TT, H = q.shape[0], q.shape[1]
    k = idx.shape[-1]
    out = out if out is not None else torch.empty(TT, H, 128, dtype=torch.bfloat16, device=q.device)
    lse = lse if lse is not None else torch.empty(TT, H, dtype=torch.float32, device=q.device)
    need = csa_sparse_mqa_workspace_size(1, TT, H, k, win_len)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    pd, cd, wd = packed.desc(), cache.desc(), _packed_window(win_k, win_v, packed, win_len).desc()
    st = lib.csa_sparse_mqa_packed(_ptr(q), H, ctypes.byref(pd), ctypes.byref(cd), m, _ptr(idx), k, ctypes.byref(wd),
                                   float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "csa_sparse_mqa_packed")
    return out, lse


def hca_dense_mqa_packed(q, packed: Packed, cache: KVCache, m_prime, win_k, win_v, win_len, scale, *, out=None,
                         lse=None, workspace=None, stream=None):
    """HCA attention over packed sequences (every visible entry of the row's own sequence + its window)."""
    lib = _lib.load()
    TT, H = q.shape[0], q.shape[1]
    out = out if out is not None else torch.empty(TT, H, 128, dtype=torch.bfloat16, device=q.device)
    lse = lse if lse is not None else torch.empty(TT, H, dtype=torch.float32, device=q.device)
    need = hca_dense_mqa_workspace_size(1, TT, H, -(-packed.max_tokens // m_prime), win_len)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    pd, cd, wd = packed.desc(), cache.desc(), _packed_window(win_k, win_v, packed, win_len).desc()
    st = lib.hca_dense_mqa_packed(_ptr(q), H, ctypes.byref(pd), ctypes.byref(cd), m_prime, ctypes.byref(wd),
                                  float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "hca_dense_mqa_packed")
    return out, lse
