"""Seeded synthetic inputs for CSA / HCA workloads.

This module only draws random numbers and lays them out; it holds none of the
attention method's arithmetic.  Both the CUDA path's tests/benchmark and the CPU
oracle read the arrays it produces, so the two sides always see identical bytes.

Every named array has its own random stream: ``PCG64(SeedSequence([seed,
array_id, chunk]))`` over fixed-size chunks of the flattened array, so a single
array (or a slice of rows) can be regenerated without drawing the others, and
generation parallelises over chunks.

Distributions (standard deviations, not variances):
  * activations q, K, V, qI, kI and decode caches: N(0, 1), rounded to bf16 (RNE);
  * compression weights w: N(0, 0.02), fp32; position bias b: N(0, 0.1), fp32;
  * indexer head weights wI: U(0, 1), fp32.

The decode KV cache uses the split storage the DeepSeek-V4 pages describe
(paper summary, hyper.ai, section "Method": RoPE dims kept in BF16, the other
dims in FP8): the 128 "nope" channels of each entry are stored as OCP FP8 E4M3
with one fp32 scale per entry (max |x| / 448), the 64 RoPE channels as bf16.
The E4M3 encoding here is torch's own ``float8_e4m3fn`` cast after clamping to
the finite range, i.e. a library conversion, not this project's code.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

D_QK = 192
D_NOPE = 128
D_ROPE = 64
D_V = 128
H_I = 4
D_I = 64
E4M3_MAX = 448.0

_CHUNK = 1 << 22
_POOL = None

# stream ids: fixed forever, so that adding arrays never changes existing ones
_IDS = {
    "q": 1, "k": 2, "v": 3, "qI": 4, "kI": 5, "wI": 6,
    "w_k": 7, "b_k": 8, "w_v": 9, "b_v": 10, "w_i": 11, "b_i": 12,
    "cache": 20, "kIc": 21, "win_k": 22,
    "hca_q": 30, "hca_cache": 31, "hca_win_k": 32,
}


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=8)
    return _POOL


def _draw(seed: int, name: str, n: int, kind: str, std: float = 1.0, sub: int = -1) -> np.ndarray:
    """Flat float32 array of n draws ('normal' N(0,std) or 'uniform' U(0,1)).

    ``sub`` >= 0 selects a per-sequence sub-stream (decode caches are drawn one
    sequence at a time so that batch shards are slices of the full batch).
    """
    key = [seed, _IDS[name]] + ([sub + 1] if sub >= 0 else [])
    nchunks = max(1, -(-n // _CHUNK))
    out = np.empty(n, dtype=np.float32)

    def fill(c):
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(key + [c])))
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        if kind == "normal":
            out[lo:hi] = g.standard_normal(hi - lo, dtype=np.float32)
            if std != 1.0:
                out[lo:hi] *= np.float32(std)
        else:
            out[lo:hi] = g.random(hi - lo, dtype=np.float32)

    if nchunks == 1:
        fill(0)
    else:
        list(_pool().map(fill, range(nchunks)))
    return out


def normal_bf16(seed, name, shape, std=1.0) -> torch.Tensor:
    n = int(np.prod(shape))
    return torch.from_numpy(_draw(seed, name, n, "normal", std)).to(torch.bfloat16).reshape(shape)


def normal_f32(seed, name, shape, std=1.0) -> torch.Tensor:
    n = int(np.prod(shape))
    return torch.from_numpy(_draw(seed, name, n, "normal", std)).reshape(shape)


def uniform_f32(seed, name, shape) -> torch.Tensor:
    n = int(np.prod(shape))
    return torch.from_numpy(_draw(seed, name, n, "uniform")).reshape(shape)


def split_fp8_cache(x: torch.Tensor):
    """Store K entries [..., 192] (fp32) as (nope e4m3 bytes, rope bf16, per-entry scale).

    scale = max |nope| / 448 per entry (1 when the entry's nope channels are all
    zero); the nope channels are divided by the scale, clamped to +-448 and cast
    with torch's float8_e4m3fn conversion (round to nearest even).
    """
    nope = x[..., :D_NOPE].float()
    rope = x[..., D_NOPE:].to(torch.bfloat16).contiguous()
    amax = nope.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).float()
    qv = (nope / scale[..., None]).clamp(-E4M3_MAX, E4M3_MAX)
    codes = qv.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return codes, rope, scale.contiguous()


def fp8_rows(x: torch.Tensor):
    """Store rows [..., d] (fp32) as E4M3 codes with one scale per row (max |x| / 448, 1 if zero)."""
    x = x.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).float()
    qv = (x / scale[..., None]).clamp(-E4M3_MAX, E4M3_MAX)
    return qv.to(torch.float8_e4m3fn).view(torch.uint8).contiguous(), scale.contiguous()


E2M1_MAX = 6.0
_E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])  # between adjacent E2M1 magnitudes


def fp4_rows(x: torch.Tensor):
    """Store rows [..., d] (fp32, d even) as OCP MX E2M1 codes, two per byte (dimension 2j in the low
    nibble of byte j), with one scale per row (max |x| / 6, 1 if zero); magnitudes round to the nearest
    E2M1 value, ties to the even code.  Returns (uint8 [..., d/2], fp32 [...])."""
    x = x.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E2M1_MAX, torch.ones_like(amax)).float()
    v = (x / scale[..., None]).numpy()
    a = np.minimum(np.abs(v), E2M1_MAX)
    code = np.searchsorted(_E2M1_MIDS, a, side="left")            # a <= mids[code]: the lower neighbour on a tie
    tie = (code < 7) & (a == _E2M1_MIDS[np.minimum(code, 6)])
    code = np.where(tie & (code % 2 == 1), code + 1, code)         # ties go to the even code
    nib = (code | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return torch.from_numpy(np.ascontiguousarray(packed)), scale.contiguous()


@dataclasses.dataclass(frozen=True)
class Prefill:
    """One prefill workload: B sequences of T tokens, all queries attend."""
    name: str
    kind: str          # "csa" or "hca"
    B: int
    T: int
    H: int
    m: int             # compression stride (CSA m, HCA m')
    k: int = 0         # top-k (CSA only)
    win: int = 128     # sliding window of raw tokens

    @property
    def cwin(self):    # compression window: CSA overlaps 2m, HCA m' (no overlap)
        return 2 * self.m if self.kind == "csa" else self.m

    @property
    def N(self):
        return -(-self.T // self.m)


@dataclasses.dataclass(frozen=True)
class Decode:
    """One decode workload: B sequences, one new query each at position L-1."""
    name: str
    kind: str          # "csa" or "hybrid" (a CSA layer then an HCA layer)
    B: int
    L: int
    H: int
    m: int
    k: int
    win: int = 128
    m_hca: int = 128
    indexer_fp8: bool = False  # indexer keys stored as E4M3 codes + per-entry scale
    indexer_fp4: bool = False  # indexer keys stored as E2M1 codes (two per byte) + per-entry scale

    @property
    def N(self):
        return self.L // self.m

    @property
    def N_hca(self):
        return self.L // self.m_hca


WORKLOADS = {
    "csa_prefill_t2048": Prefill("csa_prefill_t2048", "csa", B=1, T=2048, H=16, m=4, k=64),
    "hca_prefill_t8192": Prefill("hca_prefill_t8192", "hca", B=2, T=8192, H=16, m=128),
    "csa_decode_l131072": Decode("csa_decode_l131072", "csa", B=64, L=131072, H=64, m=4, k=2048),
    "csa_prefill_t65536": Prefill("csa_prefill_t65536", "csa", B=1, T=65536, H=64, m=4, k=2048),
    # the same shapes at a quarter of the length (for counter captures: inputs above L2, ~1 GB in all)
    "csa_prefill_t16384": Prefill("csa_prefill_t16384", "csa", B=1, T=16384, H=64, m=4, k=2048),
    "hybrid_decode_l1m": Decode("hybrid_decode_l1m", "hybrid", B=8, L=1 << 20, H=64, m=4, k=2048),
    # the same workload with FP8 (E4M3 + per-entry scale) lightning-indexer keys
    "hybrid_decode_l1m_fp8idx": Decode("hybrid_decode_l1m_fp8idx", "hybrid", B=8, L=1 << 20, H=64, m=4, k=2048,
                                       indexer_fp8=True),
    # ... and with FP4 (E2M1 + per-entry scale) lightning-indexer keys
    "hybrid_decode_l1m_fp4idx": Decode("hybrid_decode_l1m_fp4idx", "hybrid", B=8, L=1 << 20, H=64, m=4, k=2048,
                                       indexer_fp4=True),
}


def prefill_inputs(w: Prefill, seed: int = 0) -> dict:
    """Raw tokens and parameters for a prefill workload (torch CPU tensors)."""
    B, T, H, cw = w.B, w.T, w.H, w.cwin
    out = {
        "q": normal_bf16(seed, "q", (B, T, H, D_QK)),
        "k": normal_bf16(seed, "k", (B, T, D_QK)),
        "v": normal_bf16(seed, "v", (B, T, D_V)),
        "w_k": normal_f32(seed, "w_k", (D_QK,), 0.02),
        "b_k": normal_f32(seed, "b_k", (cw, D_QK), 0.1),
        "w_v": normal_f32(seed, "w_v", (D_V,), 0.02),
        "b_v": normal_f32(seed, "b_v", (cw, D_V), 0.1),
    }
    if w.kind == "csa":
        out.update({
            "qI": normal_bf16(seed, "qI", (B, T, H_I, D_I)),
            "kI": normal_bf16(seed, "kI", (B, T, D_I)),
            "wI": uniform_f32(seed, "wI", (B, T, H_I)),
            "w_i": normal_f32(seed, "w_i", (D_I,), 0.02),
            "b_i": normal_f32(seed, "b_i", (cw, D_I), 0.1),
        })
    return out


def decode_inputs(w: Decode, seed: int = 0, batch: slice | None = None) -> dict:
    """Query, resident caches and raw window for a decode workload.

    ``batch`` selects a contiguous range of sequences (the stream layout is
    per-sequence, so a shard draws exactly the rows the full batch would).
    """
    bs = batch or slice(0, w.B)
    b0, b1 = bs.start, bs.stop
    B = b1 - b0

    def rows(name, per_seq_shape, kind="normal_bf16"):
        # one stream per sequence so shards are slices of the full batch
        parts = []
        for b in range(b0, b1):
            n = int(np.prod(per_seq_shape))
            flat = _draw(seed, name, n, "uniform" if kind == "uniform" else "normal", sub=b)
            t = torch.from_numpy(flat).reshape(per_seq_shape)
            if kind == "normal_bf16":
                t = t.to(torch.bfloat16)
            parts.append(t)
        return torch.stack(parts)

    cache_f = rows("cache", (w.N, D_QK), kind="normal_f32")
    nope, rope, scale = split_fp8_cache(cache_f)
    del cache_f
    out = {
        "q": rows("q", (1, w.H, D_QK)),
        "qI": rows("qI", (1, H_I, D_I)),
        "wI": rows("wI", (1, H_I), kind="uniform"),
        "nope": nope, "rope": rope, "scale": scale,
        "win_k": rows("win_k", (w.win, D_QK)),
    }
    if w.indexer_fp8:
        out["kI_codes"], out["kI_scale"] = fp8_rows(rows("kIc", (w.N, D_I), kind="normal_f32"))
    elif w.indexer_fp4:
        out["kI_codes"], out["kI_scale"] = fp4_rows(rows("kIc", (w.N, D_I), kind="normal_f32"))
    else:
        out["kIc"] = rows("kIc", (w.N, D_I))
    if w.kind == "hybrid":
        hc = rows("hca_cache", (w.N_hca, D_QK), kind="normal_f32")
        hn, hr, hs = split_fp8_cache(hc)
        del hc
        out.update({
            "hca_q": rows("hca_q", (1, w.H, D_QK)),
            "hca_nope": hn, "hca_rope": hr, "hca_scale": hs,
            "hca_win_k": rows("hca_win_k", (w.win, D_QK)),
        })
    assert out["q"].shape[0] == B
    return out
