"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic. It only draws the tensors that both
the CUDA path and the fp64 oracle consume, so the two always see bit-identical
inputs. Every tensor is drawn i.i.d. N(0, 1) in fp32 on the CPU from
``torch.Generator().manual_seed(seed)`` in the order Q, K, V, dO and cast once
(round to nearest even) to the workload dtype.

The shapes stand in for the workloads the source pages describe (no dataset,
image or weight is used):

* a 40x40 feature map of a YOLOv12 attention block, 1600 tokens per head
  ("YOLOv12官版镜像集成Flash Attention v2", sections 2.1 and 4.1);
* an InternViT-6B-448px encoder layer: 32x32 patches + 1 CLS token = 1025
  tokens, 25 heads of width 128, with RMS normalisation of Q and K
  ("InternViT-6B-448px-V1-2 ... FlashAttention v1/v2", model specs table and
  the QK-normalisation remark);
* a packed variable-length batch addressed by ``cu_seqlens`` and ``max_s``,
  with the key-padding path realised as unpad -> varlen (same page, the
  three execution paths of its FlashAttention wrapper);
* a causal LLM prefill with grouped KV heads and a backward pass
  ("FlashAttention/zh", sections on the algorithm and on recomputation);
* LLM decode: one new query token per sequence against a long key/value cache,
  the step that dominates text generation (the Gemma-3-12b-it generation
  measurements on "Gemma-3-12b-it GPU利用率提升实测", which give no attention
  shape, so the LLM prefill shape's heads are kept), optionally through the
  paged KV cache of PagedAttention ("FlashAttention/zh", section "variants").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}

RMSNORM_EPS = 1e-6


@dataclass(frozen=True)
class FixedConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    dtype: str
    causal: bool
    seed: int
    rmsnorm: bool = False
    backward: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5


@dataclass(frozen=True)
class VarlenConfig:
    name: str
    num_seqs: int
    min_len: int
    max_len: int
    Hq: int
    Hkv: int
    d: int
    dtype: str
    causal: bool
    len_seed: int
    seed: int
    key_pad_frac: float = 0.0  # fraction of each sequence's tail keys that are padding

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5


# The five workloads, by what they are.
TINY = FixedConfig("tiny_b1_h2_n256_d64", B=1, Hq=2, Hkv=2, Nq=256, Nk=256, d=64,
                   dtype="bf16", causal=False, seed=0)
VISION = FixedConfig("vision_b32_h8_n1600_d64", B=32, Hq=8, Hkv=8, Nq=1600, Nk=1600, d=64,
                     dtype="bf16", causal=False, seed=1)
VIT_RMSNORM = FixedConfig("vit_rmsnorm_b8_h25_n1025_d128", B=8, Hq=25, Hkv=25, Nq=1025,
                          Nk=1025, d=128, dtype="bf16", causal=False, seed=2, rmsnorm=True)
VARLEN = VarlenConfig("varlen_32seq_64to4096_h32_d128_fp16", num_seqs=32, min_len=64,
                      max_len=4096, Hq=32, Hkv=32, d=128, dtype="fp16", causal=False,
                      len_seed=3, seed=4)
VARLEN_KEYPAD = VarlenConfig("varlen_keypad25_32seq_64to4096_h32_d128_fp16", num_seqs=32,
                             min_len=64, max_len=4096, Hq=32, Hkv=32, d=128, dtype="fp16",
                             causal=False, len_seed=3, seed=4, key_pad_frac=0.25)
CAUSAL_GQA = FixedConfig("causal_gqa_b2_n8192_hq32_hkv8_d128", B=2, Hq=32, Hkv=8, Nq=8192,
                         Nk=8192, d=128, dtype="bf16", causal=True, seed=5, backward=True)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int      # new query tokens per sequence
    Nk: int      # cache capacity (keys) per sequence
    d: int
    dtype: str
    causal: bool
    seed: int
    len_seed: int = -1  # >= 0: sequence lengths uniform in [min_len, Nk] from this seed; else all Nk
    min_len: int = 1

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5


DECODE = DecodeConfig("decode_b32_nk8192_hq32_hkv8_d128", B=32, Hq=32, Hkv=8, Nq=1, Nk=8192, d=128,
                      dtype="bf16", causal=False, seed=6)
DECODE_RAGGED = DecodeConfig("decode_ragged_b32_nk8192_hq32_hkv8_d128", B=32, Hq=32, Hkv=8, Nq=1, Nk=8192,
                             d=128, dtype="bf16", causal=False, seed=6, len_seed=7)
DECODE_D64 = DecodeConfig("decode_b32_nk8192_hq32_hkv8_d64", B=32, Hq=32, Hkv=8, Nq=1, Nk=8192, d=64,
                          dtype="bf16", causal=False, seed=6)
DECODE_SPEC4 = DecodeConfig("decode_spec4_b32_nk8192_hq32_hkv8_d128", B=32, Hq=32, Hkv=8, Nq=4, Nk=8192, d=128,
                            dtype="bf16", causal=True, seed=6)  # 4 speculative tokens per sequence, causal

ALL_FIXED = (TINY, VISION, VIT_RMSNORM, CAUSAL_GQA)
ALL_VARLEN = (VARLEN, VARLEN_KEYPAD)


def _normal(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def rms_normalise_rows(x: torch.Tensor, eps: float = RMSNORM_EPS) -> torch.Tensor:
    """Per-head RMS normalisation with unit gain, computed in fp64.

    Input preparation for the QK-normalised ViT workload: the page on the
    InternViT wrapper says Q and K pass through an RMSNorm before attention
    but gives neither epsilon nor dtype, so this takes eps = 1e-6, the
    mean over the head dimension, and fp64 arithmetic on the fp32 draws.
    """
    x64 = x.to(torch.float64)
    ms = (x64 * x64).mean(dim=-1, keepdim=True)
    return x64 / torch.sqrt(ms + eps)


@dataclass
class FixedInputs:
    cfg: FixedConfig
    q: torch.Tensor  # [B, Nq, Hq, d]  (bf16 / fp16, CPU)
    k: torch.Tensor  # [B, Nk, Hkv, d]
    v: torch.Tensor  # [B, Nk, Hkv, d]
    do: torch.Tensor | None = None  # [B, Nq, Hq, d]


def make_fixed(cfg: FixedConfig, with_do: bool | None = None, **override) -> FixedInputs:
    """Draw Q, K, V (and dO) for a fixed-length workload.

    ``override`` replaces fields of the config (used by tests for small or
    ragged shapes that follow the same recipe).
    """
    if override:
        cfg = FixedConfig(**{**cfg.__dict__, **override})
    dt = DTYPES[cfg.dtype]
    g = torch.Generator().manual_seed(cfg.seed)
    q = _normal(g, (cfg.B, cfg.Nq, cfg.Hq, cfg.d))
    k = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d))
    v = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d))
    want_do = cfg.backward if with_do is None else with_do
    do = _normal(g, (cfg.B, cfg.Nq, cfg.Hq, cfg.d)) if want_do else None
    if cfg.rmsnorm:
        q = rms_normalise_rows(q)
        k = rms_normalise_rows(k)
    return FixedInputs(cfg, q.to(dt), k.to(dt), v.to(dt), None if do is None else do.to(dt))


@dataclass
class VarlenInputs:
    cfg: VarlenConfig
    seqlens_q: list[int]
    seqlens_k: list[int]
    cu_seqlens_q: torch.Tensor  # int32 [num_seqs + 1]
    cu_seqlens_k: torch.Tensor  # int32 [num_seqs + 1]
    max_seqlen_q: int
    max_seqlen_k: int
    q: torch.Tensor  # [total_q, Hq, d]
    k: torch.Tensor  # [total_k, Hkv, d]  (padding keys already removed)
    v: torch.Tensor  # [total_k, Hkv, d]
    k_padded: torch.Tensor = field(repr=False, default=None)  # [total_q, Hkv, d] before unpad
    v_padded: torch.Tensor = field(repr=False, default=None)
    do: torch.Tensor | None = None  # [total_q, Hq, d] when drawn (with_do=True)


def _cumsum(lengths: list[int]) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    return torch.tensor(cu, dtype=torch.int32)


def make_varlen(cfg: VarlenConfig, lengths: list[int] | None = None, with_do: bool = False,
                **override) -> VarlenInputs:
    """Draw a packed variable-length batch.

    Lengths are i.i.d. uniform integers in [min_len, max_len] from their own
    generator (``len_seed``). Every sequence keeps all its queries. With
    ``key_pad_frac`` > 0 the last floor(frac * L) keys of each sequence are
    padding: the full packed K/V is drawn, then the padding rows are removed
    (the unpad step), and ``cu_seqlens_k`` addresses the unpadded buffer.
    With ``with_do`` the output gradient dO is drawn last, after V, so Q, K
    and V are the same with or without it.
    """
    if override:
        cfg = VarlenConfig(**{**cfg.__dict__, **override})
    if lengths is None:
        gl = torch.Generator().manual_seed(cfg.len_seed)
        lengths = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.num_seqs,), generator=gl).tolist()
    lengths = [int(n) for n in lengths]
    total = sum(lengths)
    dt = DTYPES[cfg.dtype]
    g = torch.Generator().manual_seed(cfg.seed)
    q = _normal(g, (total, cfg.Hq, cfg.d)).to(dt)
    kf = _normal(g, (total, cfg.Hkv, cfg.d)).to(dt)
    vf = _normal(g, (total, cfg.Hkv, cfg.d)).to(dt)
    do = _normal(g, (total, cfg.Hq, cfg.d)).to(dt) if with_do else None
    lk = [n - int(cfg.key_pad_frac * n) for n in lengths]
    cu_q = _cumsum(lengths)
    if cfg.key_pad_frac > 0:
        keep = torch.cat([torch.arange(int(cu_q[s]), int(cu_q[s]) + lk[s]) for s in range(len(lengths))]) \
            if total else torch.zeros(0, dtype=torch.long)
        k = kf.index_select(0, keep).contiguous()
        v = vf.index_select(0, keep).contiguous()
    else:
        k, v = kf, vf
    return VarlenInputs(cfg, lengths, lk, cu_q, _cumsum(lk), max(lengths, default=0),
                        max(lk, default=0), q, k, v, kf, vf, do)



@dataclass
class DecodeInputs:
    cfg: DecodeConfig
    q: torch.Tensor        # [B, Nq, Hq, d]
    k: torch.Tensor        # [B, Nk, Hkv, d]  contiguous caches; rows past a sequence's length hold NaN
    v: torch.Tensor
    seqlens: list[int] | None  # None: every sequence fills the cache
    page_size: int = 0
    k_pages: torch.Tensor | None = None  # [num_pages, page_size, Hkv, d]; unused rows NaN
    v_pages: torch.Tensor | None = None
    block_table: torch.Tensor | None = None  # int32 [B, max_pages]; unused entries -1


def make_decode(cfg: DecodeConfig, lengths: list[int] | None = None, page_size: int = 0, spare_pages: int = 3,
                **override) -> DecodeInputs:
    """Draw a decode batch: Q, then the K and V caches (all rows drawn, in that
    order), then the rows past each sequence's length are overwritten with NaN
    (a cache slot not yet written may hold anything). Lengths: ``lengths``, else
    uniform in [min_len, Nk] from ``len_seed``, else all Nk (``seqlens`` None).

    With ``page_size`` the same caches are also laid out as page pools: the
    pages of every sequence, plus ``spare_pages`` unused ones, are placed in a
    random order (generator seed + 1) in pools filled with NaN, and block_table
    row b lists the pages of sequence b in key order (-1 past its last page)."""
    if override:
        cfg = DecodeConfig(**{**cfg.__dict__, **override})
    dt = DTYPES[cfg.dtype]
    g = torch.Generator().manual_seed(cfg.seed)
    q = _normal(g, (cfg.B, cfg.Nq, cfg.Hq, cfg.d)).to(dt)
    k = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d)).to(dt)
    v = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d)).to(dt)
    if lengths is None and cfg.len_seed >= 0:
        gl = torch.Generator().manual_seed(cfg.len_seed)
        lengths = torch.randint(cfg.min_len, cfg.Nk + 1, (cfg.B,), generator=gl).tolist()
    seqlens = None if lengths is None else [int(n) for n in lengths]
    if seqlens is not None:
        for b, n in enumerate(seqlens):
            k[b, n:] = float("nan")
            v[b, n:] = float("nan")
    out = DecodeInputs(cfg, q, k, v, seqlens)
    if page_size:
        lens = seqlens if seqlens is not None else [cfg.Nk] * cfg.B
        counts = [(n + page_size - 1) // page_size for n in lens]
        max_pages = max(1, (cfg.Nk + page_size - 1) // page_size)
        n_pages = sum(counts) + spare_pages
        order = torch.randperm(n_pages, generator=torch.Generator().manual_seed(cfg.seed + 1)).tolist()
        kp = torch.full((n_pages, page_size, cfg.Hkv, cfg.d), float("nan"), dtype=dt)
        vp = torch.full_like(kp, float("nan"))
        table = torch.full((cfg.B, max_pages), -1, dtype=torch.int32)
        nxt = 0
        for b, (n, c) in enumerate(zip(lens, counts)):
            for i in range(c):
                page = order[nxt]
                nxt += 1
                table[b, i] = page
                rows = min(page_size, n - i * page_size)
                kp[page, :rows] = k[b, i * page_size:i * page_size + rows]
                vp[page, :rows] = v[b, i * page_size:i * page_size + rows]
        out.page_size, out.k_pages, out.v_pages, out.block_table = page_size, kp, vp, table
    return out


@dataclass
class Fp8Inputs:
    cfg: FixedConfig
    q: torch.Tensor        # uint8 E4M3 codes [B, Nq, Hq, d]
    k: torch.Tensor        # [B, Nk, Hkv, d]
    v: torch.Tensor
    q_scale: torch.Tensor  # float32 [B, Hq, ceil(Nq / 128)]: real = scale * e4m3(code)
    k_scale: torch.Tensor  # float32 [B, Hkv, ceil(Nk / 128)]
    v_scale: torch.Tensor


def _quantise_e4m3(x: torch.Tensor, block: int = 128):
    """Block-scaled E4M3 codes of x [B, N, H, d]: per head and block of 128 tokens the
    factor amax / 448 (1 for an all-zero block), codes = round-to-nearest E4M3 of
    x / factor (torch's float8 conversion)."""
    B, N, H, d = x.shape
    nb = (N + block - 1) // block
    scales = torch.ones((B, H, nb), dtype=torch.float32)
    codes = torch.zeros((B, N, H, d), dtype=torch.uint8)
    for i in range(nb):
        blk = x[:, i * block:(i + 1) * block]
        amax = blk.abs().amax(dim=(1, 3))  # [B, H]
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        scales[:, :, i] = sc
        q = (blk / sc[:, None, :, None]).clamp(-448.0, 448.0)
        codes[:, i * block:(i + 1) * block] = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scales


def make_fp8(cfg: FixedConfig, **override) -> Fp8Inputs:
    """The fixed-length recipe (Q, K, V drawn N(0, 1) in fp32 in that order), then each
    tensor quantised to block-scaled E4M3 (per head, 128 tokens per block)."""
    if override:
        cfg = FixedConfig(**{**cfg.__dict__, **override})
    g = torch.Generator().manual_seed(cfg.seed)
    q = _normal(g, (cfg.B, cfg.Nq, cfg.Hq, cfg.d))
    k = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d))
    v = _normal(g, (cfg.B, cfg.Nk, cfg.Hkv, cfg.d))
    (q8, qs), (k8, ks), (v8, vs) = (_quantise_e4m3(t) for t in (q, k, v))
    return Fp8Inputs(cfg, q8, k8, v8, qs, ks, vs)


# The causal GQA prefill shape with E4M3 inputs (forward).
CAUSAL_GQA_FP8 = FixedConfig("causal_gqa_fp8_b2_n8192_hq32_hkv8_d128", B=2, Hq=32, Hkv=8, Nq=8192, Nk=8192, d=128,
                             dtype="bf16", causal=True, seed=5)
