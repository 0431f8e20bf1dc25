"""Seeded synthetic inputs for MLA decode over a paged latent KV cache.

This module only draws random numbers and lays them out (shapes, block tables,
length mixes, index sets, the byte layout of the FP8 cache).  It holds none of
the attention arithmetic and imports neither the CUDA binding nor the oracle,
so both sides of a parity check take their inputs from here.

Workloads (shapes and distributions as specified for this library):

* ``tiny``      dense bf16, b=2, s_q=1, h_q=16, lengths {37, 200}
* ``compute``   dense bf16, b=64, s_q=1, h_q=128, L ~ U[4096, 8192], q,k ~ 0.5 N(0,1)
* ``memory``    dense bf16, b=128, s_q=2 (causal pair), h_q=16,
                L log-uniform in [1024, 16384], q,k ~ N(0,1)
* ``fused``     s_q=1, h_q=64, d_v=576, L ~ U[2048, 32768], b in {1, 32},
                q_raw ~ N(0,1), RMSNorm gain ~ N(1, 0.1), eps 1e-6, RoPE base 1e4
* ``sparse``    b=32, s_q=1, h_q=128, 65536-token cache per sequence, topk=2048
                indices drawn without replacement, round(5%) of slots = -1,
                656-byte FP8 rows.
* ``sparse_v41`` the same shapes over the 528-byte V4.1 FP8 cache: a 512-dim
                latent, 512 e4m3 codes + 16 e8m0 (power-of-two) scales per row,
                q [b, s_q, h_q, 512].
* ``sparse_v41_fp4`` the same over 288-byte V4.1 FP4 rows: 512 e2m1 codes
                packed two per byte + 32 e4m3 scales (one per 16 values).
* ``sparse_prefill`` token-level sparse prefill, no batch dimension: s_q =
                s_kv = 4096, h_q=128, topk=2048 rows at or before each
                token's position, per-token top-k length, one sink per head.
* ``fused_sparse`` the fused decode in sparse mode: fused-workload queries
                (h_q=64, gain ~ N(1, 0.1)) over the sparse workload's FP8
                cache and indices, position L - 1.

The cache of the fused workload is specified as "already rotated at its own
positions".  A rotation of an isotropic Gaussian pair is again an isotropic
Gaussian pair, so drawing the RoPE dims N(0,1) directly gives exactly the
distribution of rotated N(0,1) dims; no rotation is applied here.

The FP8 rows are prepared the way a cache writer would: x ~ N(0,1), one fp32
scale = absmax/448 per 128-value tile, codes = torch's float8_e4m3fn cast of
x/scale; RoPE dims stored as bf16.  Byte order per row:
``[512 x e4m3][4 x fp32 little-endian][64 x bf16]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

D_QK = 576
D_NOPE = 512
D_ROPE = 64
PAGE = 64
ROW656 = 656
ROW528 = 528  # V4.1 FP8 row: 512 e4m3 codes + 16 e8m0 scales
ROW288 = 288  # V4.1 FP4 row: 512 e2m1 codes (256 bytes) + 32 e4m3 scales
D_V41 = 512   # V4.1 latent width (RoPE dims included)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


@dataclass
class DenseCase:
    q: torch.Tensor            # [b, s_q, h_q, 576] bf16
    kcache: torch.Tensor       # [num_blocks, 64, 1, 576] bf16
    block_table: torch.Tensor  # [b, max_pages] int32 (-1 = unused)
    cache_seqlens: torch.Tensor  # [b] int32
    s_q: int
    h_q: int
    d_v: int
    causal: bool
    softmax_scale: float
    name: str = ""

    @property
    def batch(self):
        return int(self.q.shape[0])


@dataclass
class FusedCase:
    q_raw: torch.Tensor        # [b, 1, h_q, 576] bf16
    gain: torch.Tensor         # [576] fp32
    eps: float
    rope_base: float
    kcache: torch.Tensor
    block_table: torch.Tensor
    cache_seqlens: torch.Tensor
    h_q: int
    softmax_scale: float
    positions: Optional[torch.Tensor] = None
    name: str = ""
    d_v: int = D_QK

    @property
    def batch(self):
        return int(self.q_raw.shape[0])


@dataclass
class SparseCase:
    q: torch.Tensor            # [b, s_q, h_q, 576] bf16 (512 for the V4.1 format)
    kcache: torch.Tensor       # [num_blocks, 64, 656] uint8 (528 for the V4.1 format)
    indices: torch.Tensor      # [b, s_q, topk] int32, physical slot or -1
    h_q: int
    s_q: int
    d_v: int
    softmax_scale: float
    topk: int
    seqlen: int
    block_table: torch.Tensor = field(default=None)  # logical -> physical (for checks)
    name: str = ""

    @property
    def batch(self):
        return int(self.q.shape[0])


def default_scale() -> float:
    return 1.0 / math.sqrt(D_QK)


def paged_block_table(seqlens, gen, spare_blocks=0, device="cpu"):
    """Random permutation of the sum(ceil(L/64)) (+spare) physical blocks dealt
    out to the sequences in order; unused table entries are -1."""
    seqlens = [int(x) for x in seqlens]
    pages = [(L + PAGE - 1) // PAGE for L in seqlens]
    total = sum(pages) + int(spare_blocks)
    max_pages = max(1, max(pages) if pages else 1)
    perm = torch.randperm(max(total, 1), generator=gen, device=gen.device).to(torch.int32)
    bt = torch.full((len(seqlens), max_pages), -1, dtype=torch.int32, device=gen.device)
    pos = 0
    for b, p in enumerate(pages):
        if p:
            bt[b, :p] = perm[pos:pos + p]
        pos += p
    return bt.to(device), max(total, 1)


def _randn_bf16(shape, gen, std=1.0, device="cpu", chunk_rows=None):
    """N(0, std^2) drawn in fp32 and rounded to bf16, optionally in row chunks
    to bound temporary memory for very large caches."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=gen.device)
    flat = out.view(shape[0], -1)
    rows = shape[0]
    step = chunk_rows or rows
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=gen, device=gen.device,
                        dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[r0:r1] = x.to(torch.bfloat16)
    return out.to(device)


def make_dense(seqlens, s_q, h_q, *, seed=0, q_std=1.0, k_std=1.0, d_v=D_NOPE, causal=True,
               spare_blocks=0, device="cpu", name="", gen_device=None):
    """Dense paged case with the given per-sequence lengths."""
    gd = gen_device or device
    g = _gen(seed, gd)
    b = len(seqlens)
    bt, nb = paged_block_table(seqlens, g, spare_blocks, device=g.device)
    kcache = _randn_bf16((nb, PAGE, 1, D_QK), g, std=k_std, chunk_rows=4096)
    q = _randn_bf16((b, s_q, h_q, D_QK), g, std=q_std)
    sl = torch.tensor([int(x) for x in seqlens], dtype=torch.int32)
    return DenseCase(q=q.to(device), kcache=kcache.to(device), block_table=bt.to(device),
                     cache_seqlens=sl.to(device), s_q=s_q, h_q=h_q, d_v=d_v, causal=causal,
                     softmax_scale=default_scale(), name=name)


# ----------------------------------------------------------- length mixes

def lengths_uniform(b, lo, hi, seed):
    g = _gen(seed + 7919, "cpu")
    return torch.randint(lo, hi + 1, (b,), generator=g).tolist()


def lengths_loguniform(b, lo, hi, seed):
    g = _gen(seed + 7919, "cpu")
    u = torch.rand((b,), generator=g, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))))
            for x in u]


# -------------------------------------------------------- named workloads

def tiny(seed=0, device="cpu"):
    return make_dense([37, 200], 1, 16, seed=seed, spare_blocks=3, device=device, name="tiny")


def compute_bound(seed=0, device="cpu", batch=64, lo=4096, hi=8192):
    sl = lengths_uniform(batch, lo, hi, seed)
    return make_dense(sl, 1, 128, seed=seed, q_std=0.5, k_std=0.5, device=device,
                      name="compute", gen_device=device)


def memory_bound(seed=0, device="cpu", batch=128, lo=1024, hi=16384):
    sl = lengths_loguniform(batch, lo, hi, seed)
    return make_dense(sl, 2, 16, seed=seed, device=device, name="memory", gen_device=device)


def fused(seed=0, device="cpu", batch=32, lo=2048, hi=32768, h_q=64, seqlens=None):
    sl = seqlens if seqlens is not None else lengths_uniform(batch, lo, hi, seed)
    g = _gen(seed, device)
    bt, nb = paged_block_table(sl, g, device=g.device)
    kcache = _randn_bf16((nb, PAGE, 1, D_QK), g, chunk_rows=4096)
    q_raw = _randn_bf16((len(sl), 1, h_q, D_QK), g)
    gain = (1.0 + 0.1 * torch.randn((D_QK,), generator=g, device=g.device,
                                    dtype=torch.float32))
    return FusedCase(q_raw=q_raw.to(device), gain=gain.to(device), eps=1e-6, rope_base=10000.0,
                     kcache=kcache.to(device), block_table=bt.to(device),
                     cache_seqlens=torch.tensor(sl, dtype=torch.int32).to(device), h_q=h_q,
                     softmax_scale=default_scale(), name=f"fused_b{len(sl)}")


def quantize_rows656(x_nope: torch.Tensor, rope_bf16: torch.Tensor) -> torch.Tensor:
    """Cache-writer layout of the 656-byte row from fp32 nope values [n, 512]
    and bf16 rope dims [n, 64]: per 128-value tile scale = absmax/448 (1 if the
    tile is all zero), codes = float8_e4m3fn cast of x/scale."""
    n = x_nope.shape[0]
    tiles = x_nope.view(n, 4, 128)
    amax = tiles.abs().amax(dim=2, keepdim=True)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (tiles / scale).to(torch.float8_e4m3fn).view(torch.uint8).view(n, 512)
    out = torch.empty((n, ROW656), dtype=torch.uint8, device=x_nope.device)
    out[:, :512] = codes
    out[:, 512:528] = scale.view(n, 4).contiguous().view(torch.uint8).view(n, 16)
    out[:, 528:] = rope_bf16.contiguous().view(torch.uint8).view(n, 128)
    return out


def _sparse_indices(sl, bt, s_q, topk, invalid_frac, g):
    """Per (sequence, query): min(topk, L) logical tokens drawn without
    replacement from [0, L), mapped through the block table to physical slots
    (block * 64 + offset); round(invalid_frac * topk) random entries -> -1."""
    n_bad = int(round(invalid_frac * topk))
    idx = torch.empty((len(sl), s_q, topk), dtype=torch.int32, device=g.device)
    for b, L in enumerate(sl):
        for i in range(s_q):
            k = min(topk, L)
            logical = torch.randperm(L, generator=g, device=g.device)[:k].to(torch.int64)
            phys = bt[b].to(torch.int64)[logical // PAGE] * PAGE + logical % PAGE
            row = torch.full((topk,), -1, dtype=torch.int64, device=g.device)
            row[:k] = phys
            if n_bad:
                bad = torch.randperm(topk, generator=g, device=g.device)[:n_bad]
                row[bad] = -1
            idx[b, i] = row.to(torch.int32)
    return idx


def sparse(seed=0, device="cpu", batch=32, h_q=128, s_q=1, seqlen=65536, topk=2048,
           invalid_frac=0.05, seqlens=None):
    """Sparse FP8 case.  Each sequence owns ceil(seqlen/64) physical blocks of
    a shuffled pool; each query's topk logical tokens are drawn without
    replacement from [0, L) and mapped through that block table to physical
    slots; round(invalid_frac * topk) random slots are set to -1."""
    gd = device
    g = _gen(seed, gd)
    sl = seqlens if seqlens is not None else [seqlen] * batch
    bt, nb = paged_block_table(sl, g, device=g.device)
    n_rows = nb * PAGE
    cache = torch.empty((n_rows, ROW656), dtype=torch.uint8, device=g.device)
    step = 1 << 16
    for r0 in range(0, n_rows, step):
        r1 = min(n_rows, r0 + step)
        x = torch.randn((r1 - r0, D_NOPE), generator=g, device=g.device, dtype=torch.float32)
        rope = torch.randn((r1 - r0, D_ROPE), generator=g, device=g.device,
                           dtype=torch.float32).to(torch.bfloat16)
        cache[r0:r1] = quantize_rows656(x, rope)
    q = _randn_bf16((len(sl), s_q, h_q, D_QK), g)
    idx = _sparse_indices(sl, bt, s_q, topk, invalid_frac, g)
    return SparseCase(q=q.to(device), kcache=cache.view(nb, PAGE, ROW656).to(device),
                      indices=idx.to(device), h_q=h_q, s_q=s_q, d_v=D_NOPE,
                      softmax_scale=default_scale(), topk=topk, seqlen=max(sl),
                      block_table=bt.to(device), name="sparse")


def quantize_rows528(x: torch.Tensor) -> torch.Tensor:
    """Cache-writer layout of the 528-byte V4.1 row from fp32 values [n, 512]:
    per 32-value group a power-of-two scale 2^e with e = ceil(log2(absmax/448))
    (e = 0 for an all-zero group), stored as the E8M0 byte e + 127 after the
    512 codes; codes = float8_e4m3fn cast of x / 2^e."""
    n = x.shape[0]
    grp = x.view(n, 16, 32)
    amax = grp.abs().amax(dim=2, keepdim=True)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    e = e.clamp(-127.0, 127.0)
    codes = (grp / torch.exp2(e)).to(torch.float8_e4m3fn).view(torch.uint8).view(n, 512)
    out = torch.empty((n, ROW528), dtype=torch.uint8, device=x.device)
    out[:, :512] = codes
    out[:, 512:] = (e + 127.0).to(torch.uint8).view(n, 16)
    return out


E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # codes 0..7 of the format


def quantize_rows288(x: torch.Tensor) -> torch.Tensor:
    """Cache-writer layout of the 288-byte V4.1 FP4 row from fp32 values
    [n, 512]: per 16-value group an e4m3 scale = float8_e4m3fn(absmax / 6)
    (1 for an all-zero group), codes = the E2M1 magnitude nearest |x| / scale
    (saturating at 6) with the sign bit; code 2i in the low nibble of byte i,
    code 2i + 1 in the high nibble; the 32 scale bytes follow the 256 code
    bytes."""
    n = x.shape[0]
    grp = x.view(n, 32, 16)
    amax = grp.abs().amax(dim=2, keepdim=True)
    scale8 = torch.where(amax > 0, amax / 6.0, torch.ones_like(amax)).to(torch.float8_e4m3fn)
    scale = scale8.to(torch.float32)
    scale = torch.where(scale > 0, scale, torch.ones_like(scale))
    scale8 = scale.to(torch.float8_e4m3fn)
    v = (grp / scale).abs().clamp(max=6.0)
    mags = torch.tensor(E2M1_MAGNITUDES, dtype=torch.float32, device=x.device)
    code = (v.unsqueeze(-1) - mags).abs().argmin(dim=-1).to(torch.uint8)
    code = code | ((grp < 0).to(torch.uint8) << 3)
    code = code.view(n, 256, 2)
    out = torch.empty((n, ROW288), dtype=torch.uint8, device=x.device)
    out[:, :256] = code[..., 0] | (code[..., 1] << 4)
    out[:, 256:] = scale8.view(torch.uint8).view(n, 32)
    return out


def sparse_v41(seed=0, device="cpu", batch=32, h_q=128, s_q=1, seqlen=65536, topk=2048,
               invalid_frac=0.05, seqlens=None, fp4=False):
    """Sparse case over the V4.1 cache: a 512-dim latent (RoPE dims
    included) in 528-byte FP8 rows, or 288-byte FP4 rows with ``fp4``;
    q [b, s_q, h_q, 512] ~ N(0,1), cache values ~ N(0,1) before quantisation,
    indices drawn as in ``sparse``; softmax scale 1/sqrt(512), d_v = 512."""
    g = _gen(seed, device)
    sl = seqlens if seqlens is not None else [seqlen] * batch
    bt, nb = paged_block_table(sl, g, device=g.device)
    n_rows = nb * PAGE
    row_bytes = ROW288 if fp4 else ROW528
    cache = torch.empty((n_rows, row_bytes), dtype=torch.uint8, device=g.device)
    step = 1 << 16
    for r0 in range(0, n_rows, step):
        r1 = min(n_rows, r0 + step)
        x = torch.randn((r1 - r0, D_V41), generator=g, device=g.device, dtype=torch.float32)
        cache[r0:r1] = quantize_rows288(x) if fp4 else quantize_rows528(x)
    q = _randn_bf16((len(sl), s_q, h_q, D_V41), g)
    idx = _sparse_indices(sl, bt, s_q, topk, invalid_frac, g)
    return SparseCase(q=q.to(device), kcache=cache.view(nb, PAGE, row_bytes).to(device),
                      indices=idx.to(device), h_q=h_q, s_q=s_q, d_v=D_V41,
                      softmax_scale=1.0 / math.sqrt(D_V41), topk=topk, seqlen=max(sl),
                      block_table=bt.to(device), name="sparse_v41_fp4" if fp4 else "sparse_v41")


def sparse_v41_fp4(seed=0, device="cpu", **kw):
    """``sparse_v41`` over 288-byte FP4 rows."""
    return sparse_v41(seed=seed, device=device, fp4=True, **kw)


@dataclass
class FusedSparseCase:
    q_raw: torch.Tensor        # [b, 1, h_q, 576] bf16
    gain: torch.Tensor         # [576] fp32
    eps: float
    rope_base: float
    positions: torch.Tensor    # [b] int32, the query's position (RoPE angle)
    kcache: torch.Tensor       # [num_blocks, 64, 656] uint8
    indices: torch.Tensor      # [b, 1, topk] int32, physical slot or -1
    h_q: int
    topk: int
    softmax_scale: float
    block_table: torch.Tensor = field(default=None)
    name: str = ""
    d_v: int = D_QK

    @property
    def batch(self):
        return int(self.q_raw.shape[0])


def fused_sparse(seed=0, device="cpu", batch=32, h_q=64, seqlen=65536, topk=2048,
                 invalid_frac=0.05, seqlens=None):
    """The fused decode in sparse mode: the fused workload's query, gain, eps
    and RoPE base over the sparse workload's 656-byte FP8 cache and indices
    (s_q = 1); each query sits at position L - 1 of its sequence."""
    g = _gen(seed, device)
    sl = seqlens if seqlens is not None else [seqlen] * batch
    bt, nb = paged_block_table(sl, g, device=g.device)
    n_rows = nb * PAGE
    cache = torch.empty((n_rows, ROW656), dtype=torch.uint8, device=g.device)
    step = 1 << 16
    for r0 in range(0, n_rows, step):
        r1 = min(n_rows, r0 + step)
        x = torch.randn((r1 - r0, D_NOPE), generator=g, device=g.device, dtype=torch.float32)
        rope = torch.randn((r1 - r0, D_ROPE), generator=g, device=g.device,
                           dtype=torch.float32).to(torch.bfloat16)
        cache[r0:r1] = quantize_rows656(x, rope)
    q_raw = _randn_bf16((len(sl), 1, h_q, D_QK), g)
    gain = (1.0 + 0.1 * torch.randn((D_QK,), generator=g, device=g.device,
                                    dtype=torch.float32))
    idx = _sparse_indices(sl, bt, 1, topk, invalid_frac, g)
    pos = torch.tensor([int(L) - 1 for L in sl], dtype=torch.int32)
    return FusedSparseCase(q_raw=q_raw.to(device), gain=gain.to(device), eps=1e-6,
                           rope_base=10000.0, positions=pos.to(device),
                           kcache=cache.view(nb, PAGE, ROW656).to(device),
                           indices=idx.to(device), h_q=h_q, topk=topk,
                           softmax_scale=default_scale(), block_table=bt.to(device),
                           name="fused_sparse")


@dataclass
class PrefillCase:
    q: torch.Tensor            # [s_q, h_q, 576] bf16
    kv: torch.Tensor           # [s_kv, 576] bf16, one latent KV head
    indices: torch.Tensor      # [s_q, topk] int32 rows of kv, -1 = unused
    topk_length: Optional[torch.Tensor]  # [s_q] int32 or None
    attn_sink: Optional[torch.Tensor]    # [h_q] fp32 or None
    h_q: int
    topk: int
    softmax_scale: float
    d_v: int = D_NOPE
    name: str = ""

    @property
    def s_q(self):
        return int(self.q.shape[0])


def sparse_prefill(seed=0, device="cpu", s_q=4096, s_kv=4096, h_q=128, topk=2048,
                   with_length=True, with_sink=True):
    """Sparse prefill without a batch dimension: query token t sits at
    position s_kv - s_q + t and draws min(topk, position + 1) distinct rows of
    kv at or before its position (the rest -1); topk_length[t] is that count;
    one attention-sink logit per head ~ N(0, 1); q, kv ~ N(0, 1) in bf16."""
    g = _gen(seed, device)
    kv = _randn_bf16((s_kv, D_QK), g, chunk_rows=4096)
    q = _randn_bf16((s_q, h_q, D_QK), g)
    idx = torch.full((s_q, topk), -1, dtype=torch.int32, device=g.device)
    lengths = torch.empty((s_q,), dtype=torch.int32)
    for t in range(s_q):
        pos = s_kv - s_q + t
        k = min(topk, pos + 1)
        idx[t, :k] = torch.randperm(pos + 1, generator=g, device=g.device)[:k].to(torch.int32)
        lengths[t] = k
    sink = torch.randn((h_q,), generator=g, device=g.device, dtype=torch.float32)
    return PrefillCase(q=q.to(device), kv=kv.to(device), indices=idx.to(device),
                       topk_length=lengths.to(device) if with_length else None,
                       attn_sink=sink.to(device) if with_sink else None, h_q=h_q, topk=topk,
                       softmax_scale=default_scale(), name="sparse_prefill")


WORKLOADS = {
    "tiny": tiny,
    "compute": compute_bound,
    "memory": memory_bound,
    "fused": fused,
    "sparse": sparse,
    "sparse_v41": sparse_v41,
    "sparse_v41_fp4": sparse_v41_fp4,
    "fused_sparse": fused_sparse,
    "sparse_prefill": sparse_prefill,
}
