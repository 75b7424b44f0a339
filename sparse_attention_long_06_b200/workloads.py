"""Seeded synthetic inputs for the NSA forward pass.

This module only draws random inputs; it contains none of the method's
arithmetic.  Both the CUDA path (tests, bench) and the fp64 oracle are fed
from here, so a parity test compares the two on identical bits.

Recipe (shapes and distributions follow the NSA configuration knobs on the
"DeepSeek NSA config.toml" page, section 3: bfloat16 activations, block sizes
64, top-16, window 512, 64k context):
  * Q, K, V: float32 N(0, 1), rounded to bf16 (round to nearest even).
  * gates:   float32 U(0, 1), shape [T, Hq, 3], order (cmp, slc, win).
  * W_K, W_V: float32 N(0, 1 / (l * D)), shape [Hkv, D, l * D].
  * varlen:  8 lengths ~ U[4096, 32768], all redrawn until the sum is
    <= 131072; per sequence a unit direction u; queries become
    (z + sqrt(D) * u) / sqrt(2); 5 % of the key blocks (length l') of each
    sequence get every key rotated to cosine 0.8 with u, norm preserved.
  * decode:  KV cache and compressed-KV cache drawn N(0, 1) in bf16.
Every tensor draws from its own numpy PCG64 stream keyed by
(seed, tensor id, sequence index), so any single sequence can be regenerated
alone.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_STREAM = {"q": 1, "k": 2, "v": 3, "gates": 4, "wk": 5, "wv": 6, "lens": 7, "plant": 8,
           "kc": 9, "vc": 10, "dseq": 11}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class NsaConfig:
    name: str
    seed: int
    head_dim: int
    num_q_heads: int
    num_kv_heads: int
    cmp_block: int
    cmp_stride: int
    sel_block: int
    top_n: int
    window: int
    seqlens: tuple = ()          # prefill: per-sequence lengths (filled for varlen by draw)
    decode_batch: int = 0        # decode: number of sequences
    decode_len: int = 0          # decode: tokens in the cache including the new one
    varlen: bool = False
    planted: bool = False

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


CONFIGS = {
    "tiny": NsaConfig("tiny", 1, 64, 4, 1, 32, 32, 32, 4, 128, seqlens=(1024,)),
    "prefill_8k": NsaConfig("prefill_8k", 2, 128, 64, 4, 64, 64, 64, 16, 512, seqlens=(8192,)),
    "prefill_64k": NsaConfig("prefill_64k", 3, 128, 64, 4, 64, 64, 64, 16, 512, seqlens=(65536,)),
    "decode_64k": NsaConfig("decode_64k", 4, 128, 64, 4, 64, 64, 64, 16, 512,
                            decode_batch=32, decode_len=65537),
    "varlen": NsaConfig("varlen", 5, 128, 64, 4, 64, 64, 64, 16, 512, varlen=True, planted=True),
    # overlapping compression (blocks of 32 at a stride of 16) ranked over
    # selection blocks of 64, on the 8k shape: the geometry the pages leave
    # open (compression stride and selection block as separate knobs)
    "prefill_8k_overlap": NsaConfig("prefill_8k_overlap", 6, 128, 64, 4, 32, 16, 64, 16, 512,
                                    seqlens=(8192,)),
}


def _rng(seed: int, stream: str, index: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, _STREAM[stream], index])


def varlen_lengths(seed: int, n: int = 8, lo: int = 4096, hi: int = 32768,
                   total_max: int = 131072) -> list[int]:
    """8 lengths ~ U[lo, hi], all redrawn until their sum fits total_max."""
    rng = _rng(seed, "lens")
    while True:
        lens = rng.integers(lo, hi + 1, size=n)
        if int(lens.sum()) <= total_max:
            return [int(x) for x in lens]


def seqlens_of(cfg: NsaConfig) -> list[int]:
    return varlen_lengths(cfg.seed) if cfg.varlen else list(cfg.seqlens)


def compressor_weights(cfg: NsaConfig):
    """W_K, W_V: float32 [Hkv, D, l*D] ~ N(0, 1/(l*D))."""
    D, l, H = cfg.head_dim, cfg.cmp_block, cfg.num_kv_heads
    std = 1.0 / math.sqrt(l * D)
    wk = (_rng(cfg.seed, "wk").standard_normal((H, D, l * D), dtype=np.float32) * np.float32(std))
    wv = (_rng(cfg.seed, "wv").standard_normal((H, D, l * D), dtype=np.float32) * np.float32(std))
    return wk, wv


def _plant(cfg: NsaConfig, b: int, T: int, q32: np.ndarray, k32: np.ndarray,
           blocks=None) -> None:
    """Planted shared direction for the peaked-score varlen workload (in place):
    queries biased toward a per-sequence unit direction u, and the keys of
    `blocks` (default: a seeded 5 % of the key blocks) rotated to cosine 0.8
    with u, norm preserved."""
    D = cfg.head_dim
    rng = _rng(cfg.seed, "plant", b)
    u = rng.standard_normal(D).astype(np.float64)
    u /= np.linalg.norm(u)
    q32[...] = ((q32.astype(np.float64) + math.sqrt(D) * u) / math.sqrt(2.0)).astype(np.float32)
    nblk = T // cfg.sel_block
    if blocks is None:
        nplant = max(1, int(round(0.05 * nblk)))
        blocks = rng.choice(nblk, size=nplant, replace=False)
    for j in blocks:
        kb = k32[j * cfg.sel_block:(j + 1) * cfg.sel_block].astype(np.float64)  # [l', Hkv, D]
        along = kb @ u                                                            # [l', Hkv]
        perp = kb - along[..., None] * u
        norm = np.linalg.norm(kb, axis=-1, keepdims=True)
        pn = np.linalg.norm(perp, axis=-1, keepdims=True)
        pn[pn == 0] = 1.0
        kb = norm * (0.8 * u + 0.6 * perp / pn)
        k32[j * cfg.sel_block:(j + 1) * cfg.sel_block] = kb.astype(np.float32)


def sequence_inputs(cfg: NsaConfig, b: int, T: int) -> dict:
    """Q/K/V (bf16 bits) and gates (fp32) of sequence b with T tokens."""
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    q32 = _rng(cfg.seed, "q", b).standard_normal((T, Hq, D), dtype=np.float32)
    k32 = _rng(cfg.seed, "k", b).standard_normal((T, Hkv, D), dtype=np.float32)
    v32 = _rng(cfg.seed, "v", b).standard_normal((T, Hkv, D), dtype=np.float32)
    if cfg.planted:
        _plant(cfg, b, T, q32, k32)
    gates = _rng(cfg.seed, "gates", b).random((T, Hq, 3), dtype=np.float32)
    return {"q": bf16_bits(q32), "k": bf16_bits(k32), "v": bf16_bits(v32), "gates": gates}


def prefill_inputs(cfg: NsaConfig, seqlens: list[int] | None = None) -> dict:
    """Packed prefill batch: q [T,Hq,D], k/v [T,Hkv,D] bf16 bits, gates, W, cu_seqlens."""
    lens = list(seqlens) if seqlens is not None else seqlens_of(cfg)
    parts = [sequence_inputs(cfg, b, T) for b, T in enumerate(lens)]
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    wk, wv = compressor_weights(cfg)
    out = {key: np.concatenate([p[key] for p in parts], axis=0) for key in ("q", "k", "v", "gates")}
    out.update(w_k=wk, w_v=wv, cu_seqlens=cu, seqlens=lens)
    return out


def lane_planted_prefill_inputs(cfg: NsaConfig, residues=(0, 1, 2), modulus: int = 32) -> dict:
    """prefill_inputs with the planted direction of the varlen recipe on the
    key blocks j with j % modulus in `residues` (every such block of every
    sequence): the strongest blocks of a query all share a few residues, the
    tie-heavy case for warp-level selections that deal blocks to lanes by
    j % 32."""
    lens = seqlens_of(cfg)
    parts = []
    for b, T in enumerate(lens):
        D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
        q32 = _rng(cfg.seed, "q", b).standard_normal((T, Hq, D), dtype=np.float32)
        k32 = _rng(cfg.seed, "k", b).standard_normal((T, Hkv, D), dtype=np.float32)
        v32 = _rng(cfg.seed, "v", b).standard_normal((T, Hkv, D), dtype=np.float32)
        nblk = T // cfg.sel_block
        _plant(cfg, b, T, q32, k32, blocks=[j for j in range(nblk) if j % modulus in residues])
        gates = _rng(cfg.seed, "gates", b).random((T, Hq, 3), dtype=np.float32)
        parts.append({"q": bf16_bits(q32), "k": bf16_bits(k32), "v": bf16_bits(v32), "gates": gates})
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    wk, wv = compressor_weights(cfg)
    out = {key: np.concatenate([p[key] for p in parts], axis=0) for key in ("q", "k", "v", "gates")}
    out.update(w_k=wk, w_v=wv, cu_seqlens=cu, seqlens=lens)
    return out


def mean_pool_weights(cfg: NsaConfig):
    """W_K = W_V = [I/l, ..., I/l] per KV head ([Hkv, D, l*D] fp32): the
    compressor that averages a block's keys, so that a block of keys aligned
    with a direction gives a compressed key aligned with it too."""
    D, l, H = cfg.head_dim, cfg.cmp_block, cfg.num_kv_heads
    w = np.zeros((H, D, l * D), dtype=np.float32)
    for p in range(l):
        w[:, np.arange(D), p * D + np.arange(D)] = np.float32(1.0 / l)
    return w, w.copy()


def make_keys_periodic(cfg: NsaConfig, inputs: dict, period_blocks: int) -> dict:
    """Copies of prefill inputs whose keys repeat every `period_blocks` key
    blocks inside each sequence (K[t] = K[t mod (period_blocks * l)]), so that
    equal blocks give bit-identical compressed keys and exactly equal block
    scores: the exact-tie case of the selection."""
    out = dict(inputs)
    k = inputs["k"].copy()
    cu = inputs["cu_seqlens"]
    span = period_blocks * cfg.cmp_block
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        idx = s + (np.arange(e - s) % span)
        k[s:e] = inputs["k"][idx]
    out["k"] = k
    return out


def decode_sequence(cfg: NsaConfig, b: int, length: int, capacity: int) -> dict:
    """One decode sequence: q [Hq,D], caches [capacity,Hkv,D] and compressed
    caches [capacity // d, Hkv, D]."""
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    ccap = capacity // cfg.cmp_stride
    rng_q = _rng(cfg.seed, "q", b)
    q = bf16_bits(rng_q.standard_normal((Hq, D), dtype=np.float32))
    k = np.zeros((capacity, Hkv, D), dtype=np.uint16)
    v = np.zeros((capacity, Hkv, D), dtype=np.uint16)
    k[:length] = bf16_bits(_rng(cfg.seed, "k", b).standard_normal((length, Hkv, D), dtype=np.float32))
    v[:length] = bf16_bits(_rng(cfg.seed, "v", b).standard_normal((length, Hkv, D), dtype=np.float32))
    kc = bf16_bits(_rng(cfg.seed, "kc", b).standard_normal((ccap, Hkv, D), dtype=np.float32))
    vc = bf16_bits(_rng(cfg.seed, "vc", b).standard_normal((ccap, Hkv, D), dtype=np.float32))
    gates = _rng(cfg.seed, "gates", b).random((Hq, 3), dtype=np.float32)
    return {"q": q, "k": k, "v": v, "kc": kc, "vc": vc, "gates": gates}


def decode_inputs(cfg: NsaConfig, lengths: list[int] | None = None, capacity: int | None = None) -> dict:
    """Batch of decode queries: every sequence's cache holds `length` tokens
    (the last one is the new token) and a precomputed compressed cache."""
    B = cfg.decode_batch
    lens = list(lengths) if lengths is not None else [cfg.decode_len] * B
    cap = capacity if capacity is not None else max(lens)
    unit = max(cfg.cmp_block, cfg.sel_block)  # both are powers of two
    cap = ((cap + unit - 1) // unit) * unit
    seqs = [decode_sequence(cfg, b, L, cap) for b, L in enumerate(lens)]
    wk, wv = compressor_weights(cfg)
    out = {key: np.stack([s[key] for s in seqs]) for key in ("q", "k", "v", "kc", "vc", "gates")}
    out.update(w_k=wk, w_v=wv, seqlens=np.asarray(lens, dtype=np.int32), capacity=cap)
    return out


def indexer_inputs(seqlens: list[int], heads: int, dim: int, seed: int) -> dict:
    """Indexer tensors of a packed batch for token-level selection: queries
    q_index [T, heads, dim] and keys k_index [T, dim] N(0,1) rounded to bf16,
    per-token head weights w_index [T, heads] ~ U(0,1)."""
    T = int(sum(seqlens))
    rng = np.random.default_rng([seed, 97])
    return {"q_index": bf16_bits(rng.standard_normal((T, heads, dim), dtype=np.float32)),
            "k_index": bf16_bits(rng.standard_normal((T, dim), dtype=np.float32)),
            "w_index": rng.random((T, heads), dtype=np.float32)}
