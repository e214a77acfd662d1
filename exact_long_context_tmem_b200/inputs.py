"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Every tensor is produced on the CPU from a
``torch.Generator`` so that the GPU path and the float64 oracle see the same
bits.  The workloads mirror the long-context LLM inference shapes the pages
discuss (grouped-query heads, 64K-128K token caches, FP8 KV caches, streamed
million-token prefill); the values are N(0, 1) because the pages name no data
set the path needs.

Draw order within one workload is fixed: Q, K, V, then lengths.
"""
from __future__ import annotations

import dataclasses
import math

import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark / parity workload, named by what it is."""

    name: str
    kind: str  # "prefill" | "decode" | "stream"
    B: int
    Hq: int
    Hkv: int
    D: int
    S: int = 1  # query length (prefill / stream)
    T: int = 0  # KV length (prefill), max padded length (decode)
    causal: bool = True
    len_lo: int = 0  # ragged decode lengths, closed interval
    len_hi: int = 0
    kv_fp8: bool = False
    kv_bits: int = 0  # 8 or 4: INT8 / INT4 KV cache (0: not an integer cache)
    chunk_tokens: int = 0  # streamed prefill
    budget_bytes: int = 0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


WORKLOADS = {
    "prefill_b1_h4g2_d64_s256": Workload(
        "prefill_b1_h4g2_d64_s256", "prefill", B=1, Hq=4, Hkv=2, D=64, S=256, T=256, seed=1000),
    "prefill_b2_h32g8_d128_s8192": Workload(
        "prefill_b2_h32g8_d128_s8192", "prefill", B=2, Hq=32, Hkv=8, D=128, S=8192, T=8192, seed=1001),
    "decode_b4_h32g8_d128_ragged64k_128k": Workload(
        "decode_b4_h32g8_d128_ragged64k_128k", "decode", B=4, Hq=32, Hkv=8, D=128,
        len_lo=65536, len_hi=131072, seed=1002),
    "decode_fp8_b16_h32g8_d128_t32768": Workload(
        "decode_fp8_b16_h32g8_d128_t32768", "decode", B=16, Hq=32, Hkv=8, D=128,
        len_lo=32768, len_hi=32768, kv_fp8=True, seed=1003),
    "decode_int8_b16_h32g8_d128_t32768": Workload(
        "decode_int8_b16_h32g8_d128_t32768", "decode", B=16, Hq=32, Hkv=8, D=128,
        len_lo=32768, len_hi=32768, kv_bits=8, seed=1006),
    "decode_int4_b16_h32g8_d128_t32768": Workload(
        "decode_int4_b16_h32g8_d128_t32768", "decode", B=16, Hq=32, Hkv=8, D=128,
        len_lo=32768, len_hi=32768, kv_bits=4, seed=1007),
    "prefill_varlen_b16_h32g8_d128_ragged512_2048": Workload(
        "prefill_varlen_b16_h32g8_d128_ragged512_2048", "prefill_varlen", B=16, Hq=32, Hkv=8, D=128,
        len_lo=512, len_hi=2048, seed=1005),
    "stream_b1_h32g8_d128_s1m_chunk64k": Workload(
        "stream_b1_h32g8_d128_s1m_chunk64k", "stream", B=1, Hq=32, Hkv=8, D=128,
        S=1 << 20, T=1 << 20, chunk_tokens=65536, budget_bytes=16 * 10**9, seed=1004),
    "stream_b1_h32g8_d128_s128k_chunk16k": Workload(
        "stream_b1_h32g8_d128_s128k_chunk16k", "stream", B=1, Hq=32, Hkv=8, D=128, S=131072, T=131072,
        chunk_tokens=16384, budget_bytes=2_500_000_000, seed=1005),
}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def randn_bf16(shape, g: torch.Generator, out: torch.Tensor | None = None,
               block_rows: int = 1 << 16) -> torch.Tensor:
    """N(0,1) float32 draws rounded to bf16 (round-to-nearest-even).

    Large tensors are filled in blocks along dim 1 so the float32 temporary
    stays small; the draw sequence depends only on ``shape`` and ``block_rows``.
    ``out`` may be a preallocated (e.g. pinned) bf16 tensor of ``shape``.
    """
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16)
    if len(shape) < 2 or shape[1] <= block_rows:
        out.copy_(torch.randn(shape, generator=g, dtype=torch.float32))
        return out
    for r0 in range(0, shape[1], block_rows):
        r1 = min(shape[1], r0 + block_rows)
        sub = (shape[0], r1 - r0) + tuple(shape[2:])
        out[:, r0:r1].copy_(torch.randn(sub, generator=g, dtype=torch.float32))
    return out


def prefill_inputs(w: Workload, S: int | None = None, T: int | None = None, seed: int | None = None):
    """Q [B,S,Hq,D], K and V [B,T,Hkv,D], all bf16, token-major (BSHD)."""
    S = w.S if S is None else S
    T = w.T if T is None else T
    g = generator(w.seed if seed is None else seed)
    q = randn_bf16((w.B, S, w.Hq, w.D), g)
    k = randn_bf16((w.B, T, w.Hkv, w.D), g)
    v = randn_bf16((w.B, T, w.Hkv, w.D), g)
    return q, k, v


def ragged_lengths(w: Workload, g: torch.Generator, B: int | None = None) -> torch.Tensor:
    B = w.B if B is None else B
    return torch.randint(w.len_lo, w.len_hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def quantize_e4m3_per_token(x: torch.Tensor):
    """Synthetic FP8 KV cache: codes + one float32 scale per (batch, token, head).

    scale = absmax over the head dimension / 448 (1 for an all-zero row); codes are
    x / scale clamped to +-448 and rounded to nearest-even E4M3 by torch's
    float8_e4m3fn cast.  Returns (codes uint8 [..., D], scale float32 [...]).
    """
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (xf / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.contiguous()


def quantize_int_per_token(x: torch.Tensor, bits: int):
    """Synthetic INT8 / INT4 KV cache: symmetric codes + one float32 scale per (batch, token,
    head).  qmax = 127 (INT8) or 7 (INT4); scale = absmax over the head dimension / qmax (1 for
    an all-zero row); codes = x / scale rounded half-to-even and clamped to +-qmax.  INT8 codes are
    int8 [..., D]; INT4 codes are packed two per byte, element 2i in the low nibble of byte i and
    element 2i+1 in the high nibble, uint8 [..., D/2].
    """
    qmax = {8: 127.0, 4: 7.0}[bits]
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / qmax, torch.ones_like(amax))
    c = torch.round(xf / scale.unsqueeze(-1)).clamp(-qmax, qmax).to(torch.int32)
    if bits == 8:
        return c.to(torch.int8).contiguous(), scale.contiguous()
    n = c & 0xF
    packed = (n[..., 0::2] | (n[..., 1::2] << 4)).to(torch.uint8)
    return packed.contiguous(), scale.contiguous()


def decode_inputs(w: Workload, B: int | None = None, Tmax: int | None = None, seed: int | None = None,
                  lens: torch.Tensor | None = None, pad_value: float = float("nan")):
    """Decode workload.

    Returns a dict with q [B,Hq,D] bf16, kv_lens int32 [B], and either
    k, v bf16 [B,Tmax,Hkv,D] or k_codes, v_codes (uint8 E4M3 [B,Tmax,Hkv,D]; int8
    [B,Tmax,Hkv,D] for INT8; packed uint8 [B,Tmax,Hkv,D/2] for INT4, with kv_bits) and
    k_scale, v_scale float32 [B,Tmax,Hkv].  Cache slots at or beyond a
    sequence's length hold ``pad_value`` (NaN by default; code 0x7f for FP8 and
    the integer caches, whose pad scales are NaN), so any read of padding shows up
    in the output.
    """
    B = w.B if B is None else B
    g = generator(w.seed if seed is None else seed)
    q = randn_bf16((B, w.Hq, w.D), g)
    if lens is None:
        # lengths are drawn after Q, K, V in the fixed order, so draw K, V first
        # at the maximal padded size and then the lengths.
        Tmax = w.len_hi if Tmax is None else Tmax
    else:
        Tmax = int(lens.max()) if Tmax is None else Tmax
    kf = randn_bf16((B, Tmax, w.Hkv, w.D), g)
    vf = randn_bf16((B, Tmax, w.Hkv, w.D), g)
    if lens is None:
        lens = ragged_lengths(w, g, B)
        lens = torch.clamp(lens, max=Tmax)
    lens = lens.to(torch.int32)
    out = {"q": q, "kv_lens": lens, "Tmax": Tmax}
    pad = torch.arange(Tmax).unsqueeze(0) >= lens.long().unsqueeze(1)  # [B, Tmax]
    if w.kv_bits:
        kc, ks = quantize_int_per_token(kf, w.kv_bits)
        vc, vs = quantize_int_per_token(vf, w.kv_bits)
        kc[pad] = 0x7F
        vc[pad] = 0x7F
        ks[pad] = pad_value
        vs[pad] = pad_value
        out.update(k_codes=kc, v_codes=vc, k_scale=ks, v_scale=vs, kv_bits=w.kv_bits)
    elif w.kv_fp8:
        kc, ks = quantize_e4m3_per_token(kf)
        vc, vs = quantize_e4m3_per_token(vf)
        code_pad = 0x7F if pad_value != pad_value else 0
        kc[pad] = code_pad
        vc[pad] = code_pad
        ks[pad] = pad_value
        vs[pad] = pad_value
        out.update(k_codes=kc, v_codes=vc, k_scale=ks, v_scale=vs)
    else:
        kf[pad] = pad_value
        vf[pad] = pad_value
        out.update(k=kf, v=vf)
    return out


def varlen_inputs(w: Workload, seed: int | None = None):
    """Packed batch of w.B sequences, each with U{len_lo..len_hi} tokens (queries = keys: plain
    causal prefill).  Returns q [total, Hq, D], k, v [total, Hkv, D] bf16, lengths int32 [B] and
    cumulative lengths cu int32 [B + 1]; Q, K, V are drawn in that order, then the lengths."""
    g = generator(w.seed if seed is None else seed)
    lens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=g, dtype=torch.int64)
    total = int(lens.sum())
    q = randn_bf16((total, w.Hq, w.D), g)
    k = randn_bf16((total, w.Hkv, w.D), g)
    v = randn_bf16((total, w.Hkv, w.D), g)
    cu = torch.zeros(w.B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    return {"q": q, "k": k, "v": v, "lens": lens.to(torch.int32), "cu": cu}


def paged_inputs(d: dict, page_size: int, seed: int, spare_frac: float = 0.125):
    """Lay a decode_inputs() cache out as a page pool plus a page table (no arithmetic, only
    copies).  Each sequence's pages covering [0, len) go to pool pages in a seeded random order;
    table entries past them are -1; a few spare pool pages and every slot past a length hold
    the padding (NaN, code 0x7f for FP8), so any read of an unmapped page shows up.

    Returns a dict with q, kv_lens, page_table int32 [B, max_pages], page_size, num_pages and
    k_pool, v_pool [num_pages, page_size, Hkv, D] (bf16) or k_codes/v_codes pools with
    k_scale/v_scale pools [num_pages, page_size, Hkv].
    """
    fp8 = "k_codes" in d
    names = ("k_codes", "v_codes", "k_scale", "v_scale") if fp8 else ("k", "v")
    lens = d["kv_lens"].long()
    B, Tmax = d[names[0]].shape[0], d[names[0]].shape[1]
    max_pages = (Tmax + page_size - 1) // page_size
    need = [(int(x) + page_size - 1) // page_size for x in lens]
    total = sum(need)
    spare = max(2, int(total * spare_frac))
    g = generator(seed)
    perm = torch.randperm(total + spare, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    out = {"q": d["q"], "kv_lens": d["kv_lens"], "page_size": page_size, "num_pages": total + spare}
    if "kv_bits" in d:
        out["kv_bits"] = d["kv_bits"]
    for name in names:
        src = d[name]
        pad_val = 0x7F if src.dtype in (torch.uint8, torch.int8) else float("nan")
        pool = torch.full((total + spare, page_size) + tuple(src.shape[2:]), pad_val, dtype=src.dtype)
        padded = torch.full((B, max_pages * page_size) + tuple(src.shape[2:]), pad_val, dtype=src.dtype)
        padded[:, :Tmax] = src
        k = 0
        for b in range(B):
            for i in range(need[b]):
                pool[perm[k]] = padded[b, i * page_size:(i + 1) * page_size]
                table[b, i] = int(perm[k])
                k += 1
        out[name] = pool
    out["page_table"] = table
    return out


def sample_rows(S: int, n_random: int, seed: int, edges=()) -> list[int]:
    """Seeded query-row sample for checks on workloads too big for the full oracle."""
    g = generator(seed)
    rows = torch.randint(0, S, (n_random,), generator=g).tolist()
    rows += [r for r in edges if 0 <= r < S]
    return sorted(set(rows))
