"""Workload shapes and seeded random inputs.

Recipe (the same for every workload):
  * query q: N(0,1) fp32 [B, H, D] per layer.
  * raw tokens appended through the compressor (the unfinished group before the decode token,
    the decode token itself, or, for ``from_scratch`` workloads, the whole context): N(0,1)
    fp32 vectors and N(0,1) fp32 compressor logits.
  * compressed entries that already exist when the step starts: drawn directly as stored codes.
    f32: N(0,1). bf16: N(0,1) cast to bf16 by torch. nvfp4: each nibble's magnitude drawn from a
    fixed categorical over the 8 e2m1 magnitudes (the histogram of N(0,1) data at scale amax/6)
    with a fair sign; each 16-element scale code uniform in [40, 52] (0.25 .. 0.75).
  * window tokens not written by the appends: f32 N(0,1), or fp8 codes = torch's e4m3 cast of
    110*N(0,1) clamped to +-440 with an fp32 scale uniform in [0.8, 1.2]/110.
  * block tables: a seeded random permutation of the pool's block ids, dealt to the requests in
    order (``paged``), or the identity (contiguous cache). Unmapped logical blocks are -1.
  * multi-head indexer (CSA layers, 64 index heads x 128 dims unless stated): index query
    N(0,1) fp32 [B, H_I, d_I]; head weights N(0,1)/sqrt(H_I) fp32 [B, H_I]; stored index entries
    FP8 like the window (e4m3 of 110*N(0,1) clamped to +-440, scale uniform in [0.8, 1.2]/110);
    index keys appended through the compressor N(0,1) fp32 (their logits are the layer's).
  * context lengths of the mixed workload: round(LogNormal(ln 16384, 1.0)) clipped to
    [1024, 524288] for the tokens already cached, plus the decode token.

Every tensor has its own generator stream (seed * 1000 + stream id), so adding a tensor does not
shift the others.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

BLOCK_TOKENS = 256

# relative frequencies of the e2m1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for N(0,1) data whose
# 16-element block maximum is mapped to 6
NVFP4_MAGNITUDE_WEIGHTS = (7.0, 13.0, 13.0, 12.0, 15.0, 16.0, 15.0, 9.0)


@dataclass(frozen=True)
class LayerSpec:
    ratio: int              # tokens per compressed entry (4 = CSA, 128 = HCA)
    top_k: int | None       # None: dense layer, every completed entry is attended
    comp_dtype: str         # 'f32' | 'bf16' | 'nvfp4'
    win_dtype: str          # 'f32' | 'fp8'


@dataclass(frozen=True)
class Workload:
    name: str
    seq_lens: tuple         # L per request, including the decode token
    num_heads: int
    head_dim: int
    rope_dim: int
    window: int
    layers: tuple
    paged: bool             # False: identity tables (contiguous cache)
    from_scratch: bool      # True: the whole context is appended through the compressor
    seed: int
    description: str = ""

    @property
    def batch(self) -> int:
        return len(self.seq_lens)


def csa_b1_ctx4k_fp32() -> Workload:
    return Workload(
        "csa_b1_ctx4k_h16_d128_fp32", (4096,), 16, 128, 32, 128,
        (LayerSpec(4, 64, "f32", "f32"),), paged=False, from_scratch=True, seed=1001,
        description="1 CSA layer, batch 1, context 4096, H=16, D=128 (rope 32), r=4, top-k 64, "
                    "window 128, fp32, contiguous cache built by appending every token")


def csa_b8_ctx32k() -> Workload:
    return Workload(
        "csa_b8_ctx32k_h64_d512_bf16_fp8win", (32768,) * 8, 64, 512, 64, 128,
        (LayerSpec(4, 512, "bf16", "fp8"),), paged=True, from_scratch=False, seed=1002,
        description="1 CSA layer, batch 8, context 32768, H=64, D=512 (rope 64), r=4, top-k 512, "
                    "window 128; bf16 compressed cache, FP8 window, paged 256-token blocks")


def hca_b32_ctx128k() -> Workload:
    return Workload(
        "hca_b32_ctx128k_h64_d512_bf16_fp8win", (131072,) * 32, 64, 512, 64, 128,
        (LayerSpec(128, None, "bf16", "fp8"),), paged=True, from_scratch=False, seed=1003,
        description="1 HCA layer, batch 32, context 131072, H=64, D=512, r=128, 1024 entries "
                    "attended densely + 128-token FP8 window, bf16 compressed cache, paged")


def csa_b4_ctx1m() -> Workload:
    return Workload(
        "csa_b4_ctx1m_h64_d512_bf16_fp8win", (1048576,) * 4, 64, 512, 64, 128,
        (LayerSpec(4, 2048, "bf16", "fp8"),), paged=True, from_scratch=False, seed=1004,
        description="1 CSA layer, batch 4, context 1048576, H=64, D=512, r=4 (262144 entries), "
                    "top-k 2048, 128-token FP8 window, bf16 compressed cache, paged")


def csa_b4_ctx256k() -> Workload:
    return Workload(
        "csa_b4_ctx256k_h64_d512_bf16_fp8win", (262144,) * 4, 64, 512, 64, 128,
        (LayerSpec(4, 2048, "bf16", "fp8"),), paged=True, from_scratch=False, seed=1006,
        description="1 CSA layer, batch 4, context 262144, H=64, D=512, r=4 (65536 entries, 256 MiB "
                    "of keys: larger than L2), top-k 2048, FP8 window, bf16 compressed cache, paged")


def mixed_lengths(seed: int = 1005, n: int = 64) -> tuple:
    rng = np.random.Generator(np.random.PCG64(seed))
    prev = np.clip(np.rint(np.exp(rng.normal(math.log(16384.0), 1.0, size=n))), 1024, 524288)
    return tuple(int(p) + 1 for p in prev)


def mixed_64req() -> Workload:
    return Workload(
        "mixed_64req_2layer_nvfp4_fp8win", mixed_lengths(1005, 64), 64, 512, 64, 128,
        (LayerSpec(4, 2048, "nvfp4", "fp8"), LayerSpec(128, None, "nvfp4", "fp8")),
        paged=True, from_scratch=False, seed=1005,
        description="64 requests, lognormal context (median 16K, clipped 1K..512K), CSA r=4 "
                    "top-k 2048 + HCA r=128 layers, H=64, D=512, NVFP4 compressed cache, FP8 "
                    "window, per-layer paged tables, append of 1 token per request")


WORKLOADS = {
    "csa_b1_ctx4k_fp32": csa_b1_ctx4k_fp32,
    "csa_b8_ctx32k": csa_b8_ctx32k,
    "hca_b32_ctx128k": hca_b32_ctx128k,
    "csa_b4_ctx1m": csa_b4_ctx1m,
    "csa_b4_ctx256k": csa_b4_ctx256k,
    "mixed_64req": mixed_64req,
}


def scaled(w: Workload, seq_lens, name_suffix: str = "small", seed: int | None = None) -> Workload:
    """The same workload (dims, dtypes, layers) at other context lengths."""
    return Workload(w.name + "_" + name_suffix, tuple(int(x) for x in seq_lens), w.num_heads,
                    w.head_dim, w.rope_dim, w.window, w.layers, w.paged, w.from_scratch,
                    w.seed if seed is None else seed, w.description)


# ------------------------------------------------------------------------------------------------
# sizes of the stored formats (bytes), used only to size the random pools
# ------------------------------------------------------------------------------------------------

def comp_code_bytes(dtype: str, d: int) -> int:
    return {"f32": 4 * d, "bf16": 2 * d, "nvfp4": d // 2}[dtype]


def win_code_bytes(dtype: str, d: int) -> int:
    return {"f32": 4 * d, "fp8": d}[dtype]


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + stream)
    return g


def _randn(shape, g, device, chunk=1 << 26) -> torch.Tensor:
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.float32, device=device)
    for i in range(0, n, chunk):
        out[i:i + chunk] = torch.randn(min(chunk, n - i), generator=g, device=device)
    return out.view(*shape)


def _random_comp_pool(dtype, n_entries, d, g, device):
    if dtype == "f32":
        return _randn((n_entries, d), g, device).view(torch.uint8).view(n_entries, 4 * d), None
    if dtype == "bf16":
        out = torch.empty((n_entries, d), dtype=torch.bfloat16, device=device)
        step = max(1, (1 << 26) // d)
        for i in range(0, n_entries, step):
            j = min(n_entries, i + step)
            out[i:j] = torch.randn((j - i, d), generator=g, device=device).to(torch.bfloat16)
        return out.view(torch.uint8).view(n_entries, 2 * d), None
    if dtype == "nvfp4":
        w = torch.tensor(NVFP4_MAGNITUDE_WEIGHTS, dtype=torch.float32, device=device)
        n_nib = n_entries * d
        mag = torch.empty(n_nib, dtype=torch.uint8, device=device)
        step = 1 << 24
        for i in range(0, n_nib, step):
            j = min(n_nib, i + step)
            mag[i:j] = torch.multinomial(w, j - i, replacement=True, generator=g).to(torch.uint8)
        sign = torch.randint(0, 2, (n_nib,), generator=g, device=device, dtype=torch.uint8)
        nib = (mag | (sign << 3)).view(n_entries, d // 2, 2)
        codes = (nib[..., 0] | (nib[..., 1] << 4)).contiguous()
        scales = torch.randint(40, 53, (n_entries, d // 16), generator=g, device=device,
                               dtype=torch.int32).to(torch.uint8)
        return codes, scales
    raise ValueError(dtype)


def _random_win_pool(dtype, n_tokens, d, g, device):
    if dtype == "f32":
        return _randn((n_tokens, d), g, device).view(torch.uint8).view(n_tokens, 4 * d), None
    if dtype == "fp8":
        x = (_randn((n_tokens, d), g, device) * 110.0).clamp_(-440.0, 440.0)
        codes = x.to(torch.float8_e4m3fn).view(torch.uint8)
        scales = (torch.rand(n_tokens, generator=g, device=device) * 0.4 + 0.8) / 110.0
        return codes, scales
    raise ValueError(dtype)


def _deal_blocks(counts, total, paged, g, device, width, first_lblk=None):
    """Table [B, width] of physical ids; request b maps logical blocks first_lblk[b] ..
    first_lblk[b]+counts[b]-1; the rest are -1."""
    ids = torch.randperm(total, generator=g, device=device).to(torch.int32) if paged \
        else torch.arange(total, dtype=torch.int32, device=device)
    table = torch.full((len(counts), width), -1, dtype=torch.int32, device=device)
    off = 0
    for b, c in enumerate(counts):
        lo = 0 if first_lblk is None else first_lblk[b]
        table[b, lo:lo + c] = ids[off:off + c]
        off += c
    return table


def generate(w: Workload, device="cpu") -> dict:
    """All inputs of one decode step of workload w, on ``device``.

    Returns {'seq_len': int32 [B], 'layers': [per-layer dict]}. Per layer:
      q [B,H,D] f32; comp_codes uint8 [blocks, 256/r, bytes]; comp_scales uint8 or None;
      win_codes uint8 [wblocks, 256, bytes]; win_scales f32 [wblocks, 256] or None;
      comp_table / win_table int32 [B, ceil(max L/256)];
      setup_start int64 [B]: first position appended before the step (the step appends L-1);
      cu_setup int32 [B+1], kv_setup f32 [sum, D], logit_setup f32 [sum];
      kv_new f32 [B, D], logit_new f32 [B] (the decode token, position L-1).
    """
    B, H, D, W = w.batch, w.num_heads, w.head_dim, w.window
    lens = [int(x) for x in w.seq_lens]
    width = max(1, -(-max(lens) // BLOCK_TOKENS))
    out = {"seq_len": torch.tensor(lens, dtype=torch.int32, device=device), "layers": []}
    for li, ls in enumerate(w.layers):
        base = 100 * li
        g = lambda s: _gen(device, w.seed, base + s)  # noqa: E731
        lay = {"spec": ls}
        lay["q"] = _randn((B, H, D), g(1), device)
        # compressed pool: every logical block of the context has a physical block
        counts = [-(-L // BLOCK_TOKENS) for L in lens]
        n_blocks = sum(counts)
        epb = BLOCK_TOKENS // ls.ratio
        codes, scales = _random_comp_pool(ls.comp_dtype, n_blocks * epb, D, g(2), device)
        lay["comp_codes"] = codes.view(n_blocks, epb, -1)
        lay["comp_scales"] = None if scales is None else scales.view(n_blocks, epb, -1)
        lay["comp_table"] = _deal_blocks(counts, n_blocks, w.paged, g(3), device, width)
        # window pool: the blocks holding positions max(0, L-1-W) .. L-1
        lo = [max(0, L - 1 - W) // BLOCK_TOKENS for L in lens]
        hi = [(L - 1) // BLOCK_TOKENS for L in lens]
        wcounts = [h - l + 1 for l, h in zip(lo, hi)]
        n_wblocks = sum(wcounts)
        wcodes, wscales = _random_win_pool(ls.win_dtype, n_wblocks * BLOCK_TOKENS, D, g(4), device)
        lay["win_codes"] = wcodes.view(n_wblocks, BLOCK_TOKENS, -1)
        lay["win_scales"] = None if wscales is None else wscales.view(n_wblocks, BLOCK_TOKENS)
        lay["win_table"] = _deal_blocks(wcounts, n_wblocks, w.paged, g(5), device, width, lo)
        # raw tokens appended before the step: the unfinished group before position L-1
        # (or the whole context), then the decode token itself
        if w.from_scratch:
            start = [0 for _ in lens]
        else:
            start = [(L - 1) - ((L - 1) % ls.ratio) for L in lens]
        n_setup = [L - 1 - s for L, s in zip(lens, start)]
        lay["setup_start"] = torch.tensor(start, dtype=torch.int64, device=device)
        lay["cu_setup"] = torch.tensor(np.concatenate([[0], np.cumsum(n_setup)]), dtype=torch.int32,
                                       device=device)
        tot = int(sum(n_setup))
        lay["kv_setup"] = _randn((tot, D), g(6), device)
        lay["logit_setup"] = _randn((tot,), g(7), device)
        lay["kv_new"] = _randn((B, D), g(8), device)
        lay["logit_new"] = _randn((B,), g(9), device)
        out["layers"].append(lay)
    return out


def generate_index(w: Workload, gen: dict, layer: int = 0, heads: int = 64, dim: int = 128,
                   device="cpu") -> dict:
    """Inputs of the multi-head indexer for layer ``layer`` of workload w, whose other inputs
    ``gen`` holds (the index plane shares that layer's compressed blocks and table).

    Returns: q_index f32 [B, H_I, d_I]; weights f32 [B, H_I]; codes uint8 [blocks, 256/r, d_I];
    scales f32 [blocks, 256/r]; k_setup f32 [sum, d_I] and k_new f32 [B, d_I] (the index keys of
    the tokens the layer appends before and at the step)."""
    lay = gen["layers"][layer]
    B = w.batch
    n_blocks, epb = lay["comp_codes"].shape[0], lay["comp_codes"].shape[1]
    g = lambda s: _gen(device, w.seed, 100 * layer + 20 + s)  # noqa: E731
    out = {"q_index": _randn((B, heads, dim), g(1), device),
           "weights": _randn((B, heads), g(2), device) / math.sqrt(heads)}
    codes, scales = _random_win_pool("fp8", n_blocks * epb, dim, g(3), device)
    out["codes"] = codes.view(n_blocks, epb, dim)
    out["scales"] = scales.view(n_blocks, epb)
    out["k_setup"] = _randn((lay["kv_setup"].shape[0], dim), g(4), device)
    out["k_new"] = _randn((B, dim), g(5), device)
    return out
