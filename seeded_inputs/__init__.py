"""Seeded synthetic inputs shared by the fp64 oracle and the CUDA path.

This module only draws random numbers and rounds them to the storage type the
kernels read.  It holds none of the attention arithmetic: no dot products, no
softmax, no rotation.  Both sides of every parity check consume the exact bytes
produced here, so the oracle sees the bf16-rounded values the GPU sees.

Generator: numpy's PCG64 seeded through ``SeedSequence(seed, spawn_key=(stream,))``
(one independent stream per tensor).  Normals are numpy's ``standard_normal``
in float32, scaled by the requested standard deviation in float32.  bf16 values
come from fp32 by round-to-nearest-even on the bit pattern, which is the
rounding ``torch.Tensor.to(torch.bfloat16)`` performs for finite inputs.

Workload shapes follow the five attention configurations the pages' workloads
suggest (single fp32 head; MHA causal prefill; GQA 32/8 causal prefill with
RoPE, the LFM2-2.6B attention shape from whisper-apr ``lfm2/gqa.rs``
``GqaConfig::lfm2_2_6b``; GQA flash-decode against a long cache; long-context
D=128 causal prefill with peaked scores).
"""
from __future__ import annotations

import dataclasses
import numpy as np

# Stream ids, one per tensor of a workload.
STREAM_Q, STREAM_K, STREAM_V, STREAM_SEQLENS = 0, 1, 2, 3
# Decode caches draw one stream per sequence so each sequence's size is free.
STREAM_KCACHE_BASE, STREAM_VCACHE_BASE = 1000, 2000

BF16_NAN_BITS = 0x7FC0


def rng(seed: int, stream: int) -> np.random.Generator:
    """Independent PCG64 stream ``stream`` of master seed ``seed``."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream,))))


def normal_f32(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    """iid N(0, std^2) as float32."""
    x = rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns the uint16 bit patterns.

    NaN stays NaN (quiet); infinities stay infinite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = BF16_NAN_BITS
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to the float32 values they encode (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_normal(seed: int, stream: int, shape, std: float = 1.0):
    """iid N(0, std^2) rounded to bf16: returns (bits uint16, values float32)."""
    bits = f32_to_bf16_bits(normal_f32(seed, stream, shape, std))
    return bits, bf16_bits_to_f32(bits)


def uniform_int(seed: int, stream: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n iid integers uniform on [lo, hi] (inclusive), as int32."""
    return rng(seed, stream).integers(lo, hi + 1, size=n, dtype=np.int64).astype(np.int32)


# ----------------------------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Prefill:
    name: str
    dtype: str            # "fp32" or "bf16": storage type of q, k, v and o
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    causal: bool
    scale: float
    rope_base: float = 0.0   # <= 0: no RoPE
    q_pos0: int = 0          # position of query row 0 (keys sit at 0..Skv-1)
    qk_std: float = 1.0
    v_std: float = 1.0
    seed: int = 0

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*D per unmasked (query, key) pair."""
        return 4.0 * self.D * self.unmasked_pairs * self.B * self.Hq

    @property
    def unmasked_pairs(self) -> int:
        """Unmasked (query, key) pairs of one (batch, head); bottom-right causal alignment."""
        if not self.causal:
            return self.Sq * self.Skv
        off = self.Skv - self.Sq
        tot = 0
        # row i sees keys 0..i+off, clipped to [0, Skv]
        for i in range(self.Sq):
            tot += min(max(i + off + 1, 0), self.Skv)
        return tot

    @property
    def io_bytes(self) -> int:
        """Algorithmic bytes: q, k, v read once, o written once, lse written once."""
        es = 4 if self.dtype == "fp32" else 2
        return (es * self.D * (2 * self.B * self.Sq * self.Hq + 2 * self.B * self.Skv * self.Hkv)
                + 4 * self.B * self.Hq * self.Sq)


@dataclasses.dataclass(frozen=True)
class Decode:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Smax: int
    len_lo: int
    len_hi: int
    scale: float
    num_splits: int
    seed: int = 0

    def seqlens(self) -> np.ndarray:
        return uniform_int(self.seed, STREAM_SEQLENS, self.B, self.len_lo, self.len_hi)


C1 = Prefill("c1_fp32_B1_H1_S128_D64", "fp32", 1, 1, 1, 128, 128, 64, False, 1.0 / 8.0, seed=1001)
C2 = Prefill("c2_bf16_mha_causal_B4_H8_S2048_D64", "bf16", 4, 8, 8, 2048, 2048, 64, True, 1.0 / 8.0,
             seed=1002)
C3 = Prefill("c3_bf16_gqa32x8_causal_rope_B2_S4096_D64", "bf16", 2, 32, 8, 4096, 4096, 64, True,
             1.0 / 8.0, rope_base=10000.0, seed=1003)
# num_splits = 16: with the split policy (each split covers >= 512 keys) a sequence of L keys
# uses min(L / 512, 16) splits of >= 1024 keys for every L >= 8192.
C4 = Decode("c4_bf16_decode_B16_Hq32_Hkv8_D64_Smax32768", 16, 32, 8, 64, 32768, 1024, 32768,
            1.0 / 8.0, 16, seed=1004)
C5 = Prefill("c5_bf16_mha_causal_B1_H16_S16384_D128_peaked", "bf16", 1, 16, 16, 16384, 16384, 128,
             True, 1.0 / np.sqrt(128.0), qk_std=3.0, seed=1005)

# Beyond the five configurations: the pages' second prefill workload and the cache-offset case.
# Whisper encoder self-attention (whisper-apr: 1500 audio frames, 6 heads of 64, no mask), and a
# chunked prefill -- 512 new query rows at positions 3584..4095 against a 4096-key cache,
# bottom-right causal, GQA 32/8 with RoPE (scirs2-neural grouped_query_attention.rs
# forward_with_cache: the cache offset shifts both the mask and the query positions).
F2_WHISPER = Prefill("f2_bf16_whisper_encoder_B1_H6_S1500_D64", "bf16", 1, 6, 6, 1500, 1500, 64, False,
                     1.0 / 8.0, seed=1006)
F2_CHUNK = Prefill("f2_bf16_chunked_prefill_gqa32x8_rope_B2_Sq512_Skv4096_D64", "bf16", 2, 32, 8, 512, 4096,
                   64, True, 1.0 / 8.0, rope_base=10000.0, q_pos0=3584, seed=1007)

WORKLOADS = {w.name: w for w in (C1, C2, C3, C4, C5, F2_WHISPER, F2_CHUNK)}


def prefill_inputs(w: Prefill):
    """q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D].

    Returns a dict with float32 value arrays ``q, k, v`` (exactly the values the
    kernel reads) and, for bf16 workloads, the bf16 bit arrays ``q_bits`` etc.
    """
    shp_q = (w.B, w.Sq, w.Hq, w.D)
    shp_kv = (w.B, w.Skv, w.Hkv, w.D)
    out = {}
    for name, stream, shp, std in (("q", STREAM_Q, shp_q, w.qk_std), ("k", STREAM_K, shp_kv, w.qk_std),
                                   ("v", STREAM_V, shp_kv, w.v_std)):
        if w.dtype == "fp32":
            out[name] = normal_f32(w.seed, stream, shp, std)
        else:
            bits, vals = bf16_normal(w.seed, stream, shp, std)
            out[name + "_bits"] = bits
            out[name] = vals
    return out


def decode_inputs(w: Decode, fill_tail_nan: bool = True, seqlens=None):
    """q [B,Hq,D]; kcache/vcache [B,Smax,Hkv,D] bf16; seqlens int32 [B].

    Cache rows at positions >= seqlens[b] are never part of the attention; they
    hold bf16 NaN (``fill_tail_nan``) so that any read past a sequence's end
    poisons the output.  ``seqlens`` overrides the workload's drawn lengths.
    """
    seqlens = w.seqlens() if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    q_bits, q = bf16_normal(w.seed, STREAM_Q, (w.B, w.Hq, w.D))
    fill = BF16_NAN_BITS if fill_tail_nan else 0
    kb = np.full((w.B, w.Smax, w.Hkv, w.D), fill, dtype=np.uint16)
    vb = np.full((w.B, w.Smax, w.Hkv, w.D), fill, dtype=np.uint16)
    for b in range(w.B):
        L = int(min(max(seqlens[b], 0), w.Smax))
        kb[b, :L] = bf16_normal(w.seed, STREAM_KCACHE_BASE + b, (L, w.Hkv, w.D))[0]
        vb[b, :L] = bf16_normal(w.seed, STREAM_VCACHE_BASE + b, (L, w.Hkv, w.D))[0]
    return {"q_bits": q_bits, "q": q, "k_bits": kb, "v_bits": vb, "seqlens": seqlens}


def decode_kv_bytes(seqlens: np.ndarray, Hkv: int, D: int) -> int:
    """Algorithmic KV-cache bytes one decode call must read: K and V rows up to each length."""
    return int(np.sum(seqlens.astype(np.int64))) * Hkv * D * 2 * 2
