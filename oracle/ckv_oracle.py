"""Plain CPU oracle (numpy, fp64) for compressed-KV sparse decode attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run this module. It shares no code with
the CUDA library: its codecs, rotary embedding, paging arithmetic, compressor, scoring, selection
and attention are written here from the sources below, and nothing here imports the package.

Sources, cited by page title and section:

  [HR] 24-ai.news, "vLLM uveo DeepSeek V4 s 8,7× manjim KV cacheom: milijun tokena konteksta
       na standardnom GPU hardveru" (Croatian).
       §A "Kako funkcionira optimizacija KV cachea?": one shared K=V vector per token with
          inverse RoPE; KV compression by a weighted sum of tokens (4× to 128×); sparse attention
          over the top-k compressed tokens; a local sliding window keeps full vectors.
       §B "Što je vLLM morao riješiti u integraciji?": ratio 4 (CSA) and 128 (HCA) layers; fixed
          logical blocks of 256 token positions whose logical-to-physical mapping differs per
          layer; the compressor remainder is kept as sliding-window state.
  [DE] 24-ai.news, "vLLM integriert DeepSeek V4 mit 8,7× kleinerem KV-Cache: eine Million Token
       Kontext auf Standard-GPU-Hardware" (German translation of [HR]); §A "Wie funktioniert die
       KV-Cache-Optimierung?", §B "Was musste vLLM bei der Integration lösen?".
  [CZ] aidevelopers.cz, "DeepSeek-V4.1-Flash ve vLLM: kde se vzala 5,3× vyšší propustnost"
       (Czech). §A "Proč je obnova sliding-window cache drahá": FP8 sliding-window cache of the
       last 128 positions, FP4 compressed cache. §C "Výkon nepřinesl jeden kernel": "Sparse MQA
       logits" scores only candidate positions; attention reads an NVFP4 compressed cache.

The pages print no formulas. Where they are silent the oracle takes a stated reading, marked
``reading:`` in place. Every public function is pinned by ``tests/test_oracle_*.py`` against
something other than itself (a library routine, a closed form, an invariant or brute force).

Arithmetic is fp64 unless a step is a quantisation decision: those are taken on fp32 values in
fp32 arithmetic, the precision in which the CUDA path takes the same decision.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

LOGICAL_BLOCK_TOKENS = 256  # [HR] §B: fixed logical blocks of 256 token positions


# ------------------------------------------------------------------------------------------------
# Configuration
# ------------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerCfg:
    """One attention layer of the decode path.

    num_heads: H query heads sharing one K=V vector per key ([HR] §A, MQA).
    head_dim: D, the width of the shared K=V vector.
    rope_dim: d_r, rotary dims = the LAST d_r of D (reading: interleaved pairs, base 10000).
    ratio: r tokens per compressed entry; 4 for CSA and 128 for HCA layers ([HR] §B).
    window: W most recent tokens kept uncompressed ([HR] §A; 128 in [CZ] §A).
    comp_dtype: 'f32' | 'bf16' | 'nvfp4' storage of compressed entries.
    win_dtype: 'f32' | 'fp8' storage of window tokens (fp8 = e4m3 codes + fp32 scale per token).
    sm_scale: softmax scale; 0 means 1/sqrt(D) (reading).
    rope_base: rotary base; 0 means 10000 (reading).
    """

    num_heads: int
    head_dim: int
    rope_dim: int
    ratio: int
    window: int
    comp_dtype: str
    win_dtype: str
    sm_scale: float = 0.0
    rope_base: float = 0.0

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale > 0 else 1.0 / math.sqrt(self.head_dim)

    @property
    def base(self) -> float:
        return self.rope_base if self.rope_base > 0 else 10000.0

    @property
    def entries_per_block(self) -> int:
        return LOGICAL_BLOCK_TOKENS // self.ratio


# ------------------------------------------------------------------------------------------------
# Number formats. The pages name bf16, FP8 and NVFP4 storage ([HR] lede, [CZ] §A, §C); the
# format definitions below are the public ones (IEEE binary32 upper half; OCP e4m3 "fn";
# e2m1), written from their field layouts.
# ------------------------------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 is the upper 16 bits of a binary32: decode is a 16-bit left shift."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # NaN bit patterns stay NaN; numpy only warns about them
        return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to bf16, nearest with ties to even (finite inputs only)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def _e4m3_value(code: int) -> float:
    # 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal;
    # S.1111.111 is NaN and there is no infinity ("fn" variant).
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def _e2m1_value(code: int) -> float:
    # 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal (step 0.5).
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return sign * 0.5 * m
    return sign * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_MAX = float(E4M3_TABLE[0x7E])  # 448
E2M1_MAX = float(E2M1_TABLE[0x7])   # 6


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes).astype(np.int64)]


def e2m1_decode(nibbles: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(nibbles).astype(np.int64) & 0xF]


def _round_to_grid(x: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to |x|; ties go to the even index; beyond the last grid
    value the last index is returned (saturation). ``grid`` is increasing and starts at 0."""
    a = np.abs(np.asarray(x, dtype=np.float32)).astype(np.float64)
    n = len(grid)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, n - 1)
    lo = np.clip(hi - 1, 0, n - 1)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(a >= grid[-1], n - 1, idx)


def e4m3_encode_satfinite(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 code to each fp32 value, ties to even, saturating at +-448.

    The sign bit is copied from x, so a negative value that rounds to zero gives -0 (0x80)."""
    x32 = np.asarray(x, dtype=np.float32)
    mag = _round_to_grid(x32, E4M3_TABLE[:0x7F])
    return (mag | np.where(np.signbit(x32), 0x80, 0)).astype(np.uint8)


def e2m1_encode_satfinite(x: np.ndarray) -> np.ndarray:
    """Nearest e2m1 code (a nibble, returned in a uint8) to each fp32 value, ties to even,
    saturating at +-6; the sign bit is copied from x."""
    x32 = np.asarray(x, dtype=np.float32)
    mag = _round_to_grid(x32, E2M1_TABLE[:8])
    return (mag | np.where(np.signbit(x32), 0x8, 0)).astype(np.uint8)


def quantize_fp8_token(x32: np.ndarray) -> tuple[np.ndarray, np.float32]:
    """FP8 window storage of one token ([CZ] §A: the sliding-window cache is FP8).

    reading: one fp32 scale per token, s = amax(|x|)/448 in fp32 (s = 1 when x == 0), codes =
    e4m3 round-to-nearest-even (saturating) of x/s computed as an fp32 division."""
    x32 = np.asarray(x32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    return e4m3_encode_satfinite(x32 / s), s


def dequant_fp8_token(codes: np.ndarray, scale) -> np.ndarray:
    return e4m3_decode(codes) * np.float64(np.float32(scale))


def quantize_nvfp4(x32: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4 storage of one vector ([CZ] §C: NVFP4 compressed cache): e2m1 elements with one
    e4m3 scale per 16 consecutive elements, no second-level scale.

    reading: per block, scale code = e4m3 RNE-satfinite(amax16/6) in fp32; if that scale decodes
    to 0 every element code is +0; else code_i = e2m1 RNE-satfinite(x_i / scale) (fp32 divide).
    Returns (packed codes [D/2] with element 2i in the low nibble, scale codes [D/16])."""
    x32 = np.asarray(x32, dtype=np.float32).reshape(-1, 16)
    amax = np.max(np.abs(x32), axis=1).astype(np.float32)
    sc = e4m3_encode_satfinite(amax / np.float32(6.0))
    s = e4m3_decode(sc).astype(np.float32)
    nib = np.zeros(x32.shape, dtype=np.uint8)
    nz = s > 0
    if np.any(nz):
        nib[nz] = e2m1_encode_satfinite(x32[nz] / s[nz, None])
    flat = nib.reshape(-1)
    packed = (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8)
    return packed, sc.astype(np.uint8)


def dequant_nvfp4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Element value = e2m1(code) * e4m3(scale of its 16-element block)."""
    packed = np.asarray(packed, dtype=np.uint8)
    lo = packed & 0xF
    hi = packed >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    vals = e2m1_decode(nib)
    sc = e4m3_decode(np.asarray(scales, dtype=np.uint8))
    return vals * np.repeat(sc, 16, axis=-1)


# ------------------------------------------------------------------------------------------------
# Rotary position embedding on the last d_r dims ([HR] §A: shared K=V vectors with inverse RoPE).
# reading: interleaved pairs (D-d_r+2i, D-d_r+2i+1), theta_i = base^(-2i/d_r), angle = p*theta_i
# in fp64. Keys are rotated once, at their own position, when appended; the query is rotated at
# the position of the decode token; the rotary dims of the output get the inverse rotation at
# the query position.
# ------------------------------------------------------------------------------------------------

def rope_inv_freq(rope_dim: int, base: float) -> np.ndarray:
    i = np.arange(rope_dim // 2, dtype=np.float64)
    return np.power(np.float64(base), -(2.0 * i) / rope_dim)


def rope_apply(x: np.ndarray, pos, rope_dim: int, base: float, inverse: bool = False) -> np.ndarray:
    """Rotate the last ``rope_dim`` dims of x[..., D] by the angle of position ``pos``.

    ``pos`` is a scalar or an integer array broadcastable to x.shape[:-1]; inverse=True applies
    R(-pos)."""
    x = np.array(x, dtype=np.float64, copy=True)
    if rope_dim == 0:
        return x
    d = x.shape[-1]
    ang = np.multiply.outer(np.asarray(pos, dtype=np.float64), rope_inv_freq(rope_dim, base))
    if inverse:
        ang = -ang
    c = np.cos(ang)
    s = np.sin(ang)
    a = x[..., d - rope_dim::2].copy()
    b = x[..., d - rope_dim + 1::2].copy()
    x[..., d - rope_dim::2] = a * c - b * s
    x[..., d - rope_dim + 1::2] = a * s + b * c
    return x


# ------------------------------------------------------------------------------------------------
# Paged addressing ([HR] §B: fixed 256-position logical blocks, per-layer logical->physical map).
# A layer of ratio r holds 256/r compressed entries per block; the window cache holds 256 tokens
# per block (ratio 1).
# ------------------------------------------------------------------------------------------------

def comp_entry_rows(table_row: np.ndarray, entries: np.ndarray, ratio: int) -> np.ndarray:
    """Pool row of compressed entry i: table[(i*r)//256] * (256/r) + i mod (256/r)."""
    entries = np.asarray(entries, dtype=np.int64)
    epb = LOGICAL_BLOCK_TOKENS // ratio
    phys = np.asarray(table_row, dtype=np.int64)[(entries * ratio) // LOGICAL_BLOCK_TOKENS]
    if np.any(phys < 0):
        raise ValueError("compressed entry in an unmapped logical block")
    return phys * epb + entries % epb


def window_token_rows(table_row: np.ndarray, tokens: np.ndarray) -> np.ndarray:
    """Pool row of window token t: table[t//256] * 256 + t mod 256."""
    tokens = np.asarray(tokens, dtype=np.int64)
    phys = np.asarray(table_row, dtype=np.int64)[tokens // LOGICAL_BLOCK_TOKENS]
    if np.any(phys < 0):
        raise ValueError("window token in an unmapped logical block")
    return phys * LOGICAL_BLOCK_TOKENS + tokens % LOGICAL_BLOCK_TOKENS


class BlockPool:
    """Host allocator of physical block ids for one pool.

    reading: a LIFO free list whose initial order hands out 0, 1, 2, ... ; alloc is
    all-or-nothing; freeing an id that is free or out of range is an error."""

    def __init__(self, num_blocks: int):
        self.num_blocks = num_blocks
        self._stack = list(range(num_blocks - 1, -1, -1))
        self._is_free = [True] * num_blocks

    def alloc(self, n: int):
        if n < 0:
            raise ValueError("negative count")
        if n > len(self._stack):
            return None
        out = [self._stack.pop() for _ in range(n)]
        for i in out:
            self._is_free[i] = False
        return out

    def free(self, ids) -> None:
        ids = list(ids)
        for i in ids:
            if not (0 <= i < self.num_blocks) or self._is_free[i]:
                raise ValueError(f"bad free of block {i}")
        if len(set(ids)) != len(ids):
            raise ValueError("duplicate id in free")
        for i in ids:
            self._is_free[i] = True
            self._stack.append(i)

    @property
    def num_free(self) -> int:
        return len(self._stack)


# ------------------------------------------------------------------------------------------------
# Cache state held by the oracle (same byte layout as the pools the tests hand to the GPU).
# ------------------------------------------------------------------------------------------------

def comp_entry_code_bytes(cfg: LayerCfg) -> int:
    return {"f32": 4 * cfg.head_dim, "bf16": 2 * cfg.head_dim, "nvfp4": cfg.head_dim // 2}[cfg.comp_dtype]


def win_token_code_bytes(cfg: LayerCfg) -> int:
    return {"f32": 4 * cfg.head_dim, "fp8": cfg.head_dim}[cfg.win_dtype]


@dataclass
class LayerCache:
    """Pools and tables of one layer.

    comp_codes: uint8 [comp_blocks, 256/r, entry code bytes]
    comp_scales: uint8 [comp_blocks, 256/r, D/16] (nvfp4 only)
    win_codes: uint8 [win_blocks, 256, token code bytes]
    win_scales: float32 [win_blocks, 256] (fp8 only)
    comp_table, win_table: int32 [B, max logical blocks]; -1 = unmapped
    residue: per request, the raw (un-rotated) tokens of the unfinished group as
      (position, kv fp32 [D], logit fp32) ([HR] §B: the remainder is sliding-window state).
    """

    comp_codes: np.ndarray
    comp_scales: np.ndarray | None
    win_codes: np.ndarray
    win_scales: np.ndarray | None
    comp_table: np.ndarray
    win_table: np.ndarray
    residue: list = field(default_factory=list)


def decode_comp_entries(cfg: LayerCfg, cache: LayerCache, b: int, entries) -> np.ndarray:
    rows = comp_entry_rows(cache.comp_table[b], entries, cfg.ratio)
    flat = cache.comp_codes.reshape(-1, cache.comp_codes.shape[-1])
    raw = flat[rows]
    if cfg.comp_dtype == "f32":
        return raw.view(np.float32).astype(np.float64).reshape(len(rows), cfg.head_dim)
    if cfg.comp_dtype == "bf16":
        return bf16_bits_to_f64(raw.view(np.uint16)).reshape(len(rows), cfg.head_dim)
    if cfg.comp_dtype == "nvfp4":
        sflat = cache.comp_scales.reshape(-1, cache.comp_scales.shape[-1])
        return dequant_nvfp4(raw, sflat[rows])
    raise ValueError(cfg.comp_dtype)


def decode_window_tokens(cfg: LayerCfg, cache: LayerCache, b: int, tokens) -> np.ndarray:
    rows = window_token_rows(cache.win_table[b], tokens)
    flat = cache.win_codes.reshape(-1, cache.win_codes.shape[-1])
    raw = flat[rows]
    if cfg.win_dtype == "f32":
        return raw.view(np.float32).astype(np.float64).reshape(len(rows), cfg.head_dim)
    if cfg.win_dtype == "fp8":
        sc = cache.win_scales.reshape(-1)[rows].astype(np.float64)
        return e4m3_decode(raw) * sc[:, None]
    raise ValueError(cfg.win_dtype)


def write_comp_entry(cfg: LayerCfg, cache: LayerCache, b: int, entry: int, c32: np.ndarray) -> None:
    row = int(comp_entry_rows(cache.comp_table[b], [entry], cfg.ratio)[0])
    flat = cache.comp_codes.reshape(-1, cache.comp_codes.shape[-1])
    c32 = np.asarray(c32, dtype=np.float32)
    if cfg.comp_dtype == "f32":
        flat[row] = c32.view(np.uint8)
    elif cfg.comp_dtype == "bf16":
        flat[row] = f32_to_bf16_bits(c32).view(np.uint8)
    elif cfg.comp_dtype == "nvfp4":
        packed, sc = quantize_nvfp4(c32)
        flat[row] = packed
        cache.comp_scales.reshape(-1, cache.comp_scales.shape[-1])[row] = sc
    else:
        raise ValueError(cfg.comp_dtype)


def write_window_token(cfg: LayerCfg, cache: LayerCache, b: int, t: int, x32: np.ndarray) -> None:
    row = int(window_token_rows(cache.win_table[b], [t])[0])
    flat = cache.win_codes.reshape(-1, cache.win_codes.shape[-1])
    x32 = np.asarray(x32, dtype=np.float32)
    if cfg.win_dtype == "f32":
        flat[row] = x32.view(np.uint8)
    elif cfg.win_dtype == "fp8":
        codes, s = quantize_fp8_token(x32)
        flat[row] = codes
        cache.win_scales.reshape(-1)[row] = s
    else:
        raise ValueError(cfg.win_dtype)


# ------------------------------------------------------------------------------------------------
# Step 1: KV compressor ([HR] §A: compression by weighted summation of tokens, 4x to 128x).
# reading: one scalar logit per token; the weights of a group are the softmax of its r logits;
# each token is rotated at its own position before the sum (so a one-hot weight reproduces the
# token exactly); the unfinished group is residue ([HR] §B) and is never a candidate.
# ------------------------------------------------------------------------------------------------

def softmax_weights(logits: np.ndarray) -> np.ndarray:
    """softmax over a group's logits in fp64, max-subtracted; a -inf logit gets weight 0."""
    lg = np.asarray(logits, dtype=np.float64)
    e = np.exp(lg - np.max(lg))
    return e / np.sum(e)


def compress_group(x_rot: np.ndarray, logits: np.ndarray) -> np.ndarray:
    """Entry = sum over the group's tokens, in token order, of w_t * (rotated token t)."""
    w = softmax_weights(logits)
    c = np.zeros(x_rot.shape[-1], dtype=np.float64)
    for t in range(x_rot.shape[0]):
        c = c + w[t] * x_rot[t]
    return c


def append_tokens(cfg: LayerCfg, cache: LayerCache, b: int, prev_len: int,
                  kv_new: np.ndarray, logit_new: np.ndarray) -> None:
    """Append n raw tokens (positions prev_len .. prev_len+n-1) of request b.

    Each token is rotated at its own position. Tokens within the last W positions of the new
    length are written to the window cache. A token that completes a group (position+1 a
    multiple of r) folds the group into compressed entry (position+1)/r - 1."""
    kv_new = np.asarray(kv_new, dtype=np.float32).reshape(-1, cfg.head_dim)
    logit_new = np.asarray(logit_new, dtype=np.float32).reshape(-1)
    n = kv_new.shape[0]
    new_len = prev_len + n
    while len(cache.residue) <= b:
        cache.residue.append([])
    res = cache.residue[b]
    if len(res) != prev_len % cfg.ratio or any(p != prev_len - len(res) + i for i, (p, _, _) in enumerate(res)):
        raise ValueError("residue does not match prev_len")
    for t in range(n):
        pos = prev_len + t
        if cfg.window > 0 and pos >= new_len - cfg.window:
            x = rope_apply(kv_new[t].astype(np.float64), pos, cfg.rope_dim, cfg.base)
            write_window_token(cfg, cache, b, pos, x.astype(np.float32))
        res.append((pos, kv_new[t].copy(), np.float32(logit_new[t])))
        if (pos + 1) % cfg.ratio == 0:
            positions = np.array([p for p, _, _ in res], dtype=np.int64)
            raw = np.stack([k for _, k, _ in res]).astype(np.float64)
            x_rot = rope_apply(raw, positions, cfg.rope_dim, cfg.base)
            lg = np.array([l for _, _, l in res], dtype=np.float64)
            c = compress_group(x_rot, lg)
            write_comp_entry(cfg, cache, b, (pos + 1) // cfg.ratio - 1, c.astype(np.float32))
            res.clear()


# ------------------------------------------------------------------------------------------------
# SWA bounded replay ([CZ] §A "Proč je obnova sliding-window cache drahá": after a prefix-cache hit
# only the last window is run through the model again, and at its start the dependence on older
# positions is cut; §B "Polovina vrstev nemusí číst celý prompt" names the switch that enables it).
# The model's recompute of the window's K=V vectors lies outside this path; the cache side is:
# reading: the caller supplies the recomputed raw tokens and compressor logits of the last
# n_w = min(W, L) positions; each is rotated at its own position and written to the window cache;
# the tokens of the unfinished group [floor(L/r) r, L) that lie in the window become the residue
# (tokens of that group before L - n_w, possible only when r - 1 > W, keep whatever residue state
# they had: the cut); compressed entries are not touched (they come from the prefix cache).
# ------------------------------------------------------------------------------------------------

def window_replay(cfg: LayerCfg, cache: LayerCache, b: int, seq_len: int, kv_win: np.ndarray,
                  logit_win: np.ndarray) -> None:
    """Rewrite request b's window and residue from the raw tokens of positions L-n_w .. L-1.

    kv_win: [n_w, D] fp32 raw (un-rotated) tokens, row i at position L - n_w + i; logit_win: [n_w]."""
    n_w = min(cfg.window, seq_len)
    kv_win = np.asarray(kv_win, dtype=np.float32).reshape(-1, cfg.head_dim)[:n_w]
    logit_win = np.asarray(logit_win, dtype=np.float32).reshape(-1)[:n_w]
    g0 = (seq_len // cfg.ratio) * cfg.ratio  # first position of the unfinished group
    while len(cache.residue) <= b:
        cache.residue.append([])
    kept = [e for e in cache.residue[b] if g0 <= e[0] < seq_len - n_w]
    res = list(kept)
    for i in range(n_w):
        pos = seq_len - n_w + i
        x = rope_apply(kv_win[i].astype(np.float64), pos, cfg.rope_dim, cfg.base)
        write_window_token(cfg, cache, b, pos, x.astype(np.float32))
        if pos >= g0:
            res.append((pos, kv_win[i].copy(), np.float32(logit_win[i])))
    cache.residue[b] = sorted(res, key=lambda e: e[0])


# ------------------------------------------------------------------------------------------------
# Step 2: sparse MQA indexer and top-k ([HR] §A: sparse attention over the top-k compressed
# tokens; [CZ] §C: "Sparse MQA logits" scores the candidate positions).
# reading: the score of candidate j is the head-average of the MQA attention logits of the
# decode query against compressed entry j: s_j = sm_scale * (1/H) * sum_h q~_h . k_j.
# ------------------------------------------------------------------------------------------------

def num_compressed(seq_len: int, ratio: int) -> int:
    """Completed compressed entries for a context of seq_len tokens (the residue excluded)."""
    return seq_len // ratio


def indexer_scores(cfg: LayerCfg, cache: LayerCache, b: int, q_raw: np.ndarray, seq_len: int,
                   chunk: int = 16384) -> np.ndarray:
    """fp64 scores s_j for j < floor(L/r); q_raw is the un-rotated query [H, D]."""
    n_c = num_compressed(seq_len, cfg.ratio)
    qr = rope_apply(np.asarray(q_raw, dtype=np.float64), seq_len - 1, cfg.rope_dim, cfg.base)
    out = np.empty(n_c, dtype=np.float64)
    for j0 in range(0, n_c, chunk):
        j1 = min(n_c, j0 + chunk)
        k = decode_comp_entries(cfg, cache, b, np.arange(j0, j1))
        out[j0:j1] = cfg.scale * np.mean(qr @ k.T, axis=0)
    return out


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """The min(k, N) largest scores, ties to the lower index, returned in ascending index order.

    reading: the decision is taken on the fp32 scores (the precision of the CUDA path)."""
    s32 = np.asarray(scores, dtype=np.float32).astype(np.float64)
    n = s32.shape[0]
    order = np.lexsort((np.arange(n), -s32))
    return np.sort(order[: min(k, n)]).astype(np.int64)


# ------------------------------------------------------------------------------------------------
# Step 3: joint attention over the selected compressed entries and the window ([HR] §A).
# reading: one softmax over the union of the selected entries and the window tokens
# [max(0, L-W), L), no de-duplication of window tokens covered by a selected entry; the key and
# the value are the same vector; the output's rotary dims get the inverse rotation R(-(L-1)).
# ------------------------------------------------------------------------------------------------

def attention(cfg: LayerCfg, cache: LayerCache, b: int, q_raw: np.ndarray, seq_len: int,
              entries) -> np.ndarray:
    """fp64 output [H, D] of one request; ``entries`` are the compressed entries attended."""
    entries = np.asarray(entries, dtype=np.int64)
    qr = rope_apply(np.asarray(q_raw, dtype=np.float64), seq_len - 1, cfg.rope_dim, cfg.base)
    parts = []
    if entries.size:
        parts.append(decode_comp_entries(cfg, cache, b, entries))
    n_w = min(cfg.window, seq_len)
    if n_w > 0:
        parts.append(decode_window_tokens(cfg, cache, b, np.arange(seq_len - n_w, seq_len)))
    if not parts:
        return np.zeros((cfg.num_heads, cfg.head_dim), dtype=np.float64)
    x = np.concatenate(parts, axis=0)
    logits = cfg.scale * (qr @ x.T)
    p = np.exp(logits - np.max(logits, axis=1, keepdims=True))
    p = p / np.sum(p, axis=1, keepdims=True)
    o = p @ x
    return rope_apply(o, seq_len - 1, cfg.rope_dim, cfg.base, inverse=True)


def decode_layer(cfg: LayerCfg, cache: LayerCache, b: int, q_raw: np.ndarray, seq_len: int,
                 top_k):
    """One request of one layer: scores + selection (None for a dense layer) + attention.

    Returns (selected entries, fp64 scores or None, fp64 output [H, D])."""
    n_c = num_compressed(seq_len, cfg.ratio)
    if top_k is None:
        sel = np.arange(n_c, dtype=np.int64)
        scores = None
    else:
        scores = indexer_scores(cfg, cache, b, q_raw, seq_len)
        sel = topk_select(scores, top_k)
    return sel, scores, attention(cfg, cache, b, q_raw, seq_len, sel)


# ------------------------------------------------------------------------------------------------
# Multi-head indexer ([CZ] §C: "Sparse MQA logits" scores only the candidate positions).
# reading (the second indexer form): the indexer has its own H_I heads of width d_I and its own
# compressed key per entry. Per token the caller supplies an index key (position encoding, if
# any, already applied: the projections that make index keys and queries lie outside this path);
# the index keys of a group are folded with the same softmax weights of the same logits as the
# K=V tokens ([HR] §A) and stored as FP8 with one fp32 scale per entry (the window's FP8 rule).
# The decode step supplies one index query per head and one weight per head; the score of
# candidate j is s_j = sum_h w_h * max(0, q^_h . k_j), where q^_h is head h's index query stored
# by the same FP8 rule (one fp32 scale per head: the indexer runs in FP8 end to end, like the
# pages' FP8/FP4 caches) and k_j the decoded entry. No softmax scale (the weights carry it); top-k
# as for the head-averaged score.
# ------------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class IndexCfg:
    """index_heads: H_I; index_dim: d_I (index key and query width)."""
    index_heads: int
    index_dim: int


@dataclass
class IndexCache:
    """The index-key plane of a layer's compressed pool (same blocks, rows and table).

    codes: uint8 [comp_blocks, 256/r, d_I] e4m3; scales: float32 [comp_blocks, 256/r];
    residue: per request, the index keys of the unfinished group as (position, key f32 [d_I],
    logit f32)."""
    codes: np.ndarray
    scales: np.ndarray
    residue: list = field(default_factory=list)


def index_append_tokens(cfg: LayerCfg, icache: IndexCache, comp_table: np.ndarray, b: int,
                        prev_len: int, k_new: np.ndarray, logit_new: np.ndarray) -> None:
    """Append n index keys (positions prev_len .. prev_len+n-1) of request b; a key that
    completes a group folds the group (compress_group, no rotation) into entry (pos+1)/r - 1,
    stored with quantize_fp8_token."""
    d_i = icache.codes.shape[-1]
    k_new = np.asarray(k_new, dtype=np.float32).reshape(-1, d_i)
    logit_new = np.asarray(logit_new, dtype=np.float32).reshape(-1)
    while len(icache.residue) <= b:
        icache.residue.append([])
    res = icache.residue[b]
    if len(res) != prev_len % cfg.ratio:
        raise ValueError("index residue does not match prev_len")
    flat_c = icache.codes.reshape(-1, d_i)
    flat_s = icache.scales.reshape(-1)
    for t in range(k_new.shape[0]):
        pos = prev_len + t
        res.append((pos, k_new[t].copy(), np.float32(logit_new[t])))
        if (pos + 1) % cfg.ratio == 0:
            keys = np.stack([k for _, k, _ in res]).astype(np.float64)
            lg = np.array([l for _, _, l in res], dtype=np.float64)
            c = compress_group(keys, lg)
            row = int(comp_entry_rows(comp_table[b], [(pos + 1) // cfg.ratio - 1], cfg.ratio)[0])
            codes, s = quantize_fp8_token(c.astype(np.float32))
            flat_c[row] = codes
            flat_s[row] = s
            res.clear()


def decode_index_entries(cfg: LayerCfg, icache: IndexCache, comp_table: np.ndarray, b: int,
                         entries) -> np.ndarray:
    """fp64 index keys [n, d_I] of the given entries of request b."""
    rows = comp_entry_rows(comp_table[b], entries, cfg.ratio)
    d_i = icache.codes.shape[-1]
    return dequant_fp8_token(icache.codes.reshape(-1, d_i)[rows], 1.0) * \
        icache.scales.reshape(-1)[rows].astype(np.float64)[:, None]


def index_query_fp8(q_index: np.ndarray) -> np.ndarray:
    """The index query as scored: each head stored by quantize_fp8_token (scale amax/448, e4m3
    codes), decoded to fp64. q_index: [H_I, d_I]."""
    q = np.asarray(q_index, dtype=np.float32)
    out = np.empty(q.shape, dtype=np.float64)
    for h in range(q.shape[0]):
        codes, s = quantize_fp8_token(q[h])
        out[h] = dequant_fp8_token(codes, s)
    return out


def mh_indexer_scores(cfg: LayerCfg, icache: IndexCache, comp_table: np.ndarray, b: int,
                      q_index: np.ndarray, weights: np.ndarray, seq_len: int,
                      chunk: int = 16384) -> np.ndarray:
    """fp64 scores s_j = sum_h w_h max(0, q^_h . k_j) for j < floor(L/r).

    q_index: [H_I, d_I] fp32; weights: [H_I] fp32."""
    n_c = num_compressed(seq_len, cfg.ratio)
    qh = index_query_fp8(q_index)
    w = np.asarray(weights, dtype=np.float32).astype(np.float64)
    out = np.empty(n_c, dtype=np.float64)
    for j0 in range(0, n_c, chunk):
        j1 = min(n_c, j0 + chunk)
        k = decode_index_entries(cfg, icache, comp_table, b, np.arange(j0, j1))
        out[j0:j1] = np.maximum(k @ qh.T, 0.0) @ w
    return out
