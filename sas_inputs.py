"""Seeded synthetic inputs for gated block-sparse attention (SAS).

This module is the one piece shared by the CPU oracle and the CUDA path: it
draws input tensors and nothing else. It holds none of the operator's
arithmetic (no pooling, gate projection, normalisation, gate rotary embedding,
selection or attention).

Random values come from a counter-based generator so that any slice of a
tensor can be drawn on its own, on any device, with bit-identical results:

* counter n (element index within a named tensor) and a key derived from
  (seed, stream) are mixed with the "lowbias32" integer hash published by
  C. Wellons (hash-prospector: x ^= x>>16; x *= 0x7feb352d; x ^= x>>15;
  x *= 0x846ca68b; x ^= x>>16), giving two 32-bit words;
* their four 16-bit halves are summed (Irwin-Hall with n = 4), centred and
  scaled to unit variance in fp32 with one rounding. The result is an
  approximately normal value in [-3.47, 3.47] (excess kurtosis -0.3).

The numpy path (CPU) uses native uint32 wrap-around; the torch path (any
device) does the same 32-bit arithmetic in int64 with 16-bit split
multiplies, so no intermediate overflows. Both are exact integer arithmetic
followed by one IEEE fp32 multiply, so they agree bit for bit.

The backbone's own rotary embedding (base 1e6, rotate-half, over the head
dim) turns the pre-rotary Q/K into the attention's Q/K. That is the host
model's position encoding, not part of the gated sparse operator; it is done
here once, in fp64 with a table built by numpy, and rounded to the storage
dtype, so both sides read the same attention inputs.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

_M32 = 0xFFFFFFFF
_VAR_SUM4 = (65536.0 * 65536.0 - 1.0) / 3.0          # variance of a sum of four U{0..65535}
_SCALE = np.float32(1.0 / math.sqrt(_VAR_SUM4))
_CENTRE = 2 * 65535                                    # mean of that sum

# one stream id per named tensor, so tensors drawn with one seed never overlap
STREAMS = {
    "q_nope": 1, "k_nope": 2, "v": 3, "dout": 4, "wq": 5, "wk": 6,
    "k_cache": 7, "v_cache": 8, "gate_key_cache": 9, "cur_pool": 10,
    "dec_q_nope": 11, "sel_keys": 12, "sel_logg": 13, "qnorm_w": 14, "knorm_w": 15,
}


def _key(seed: int, stream: int) -> tuple[int, int]:
    k = (seed * 0x9E3779B9 + stream * 0x85EBCA6B + 0x27D4EB2F) & _M32
    k1 = _lowbias32_int(k)
    k2 = _lowbias32_int(k1 ^ 0x68E31DA4)
    return k1, k2


def _lowbias32_int(x: int) -> int:
    x ^= x >> 16
    x = (x * 0x7FEB352D) & _M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & _M32
    x ^= x >> 16
    return x


def _lowbias32_np(x: np.ndarray) -> np.ndarray:
    x = x ^ (x >> np.uint32(16))
    x = x * np.uint32(0x7FEB352D)
    x = x ^ (x >> np.uint32(15))
    x = x * np.uint32(0x846CA68B)
    x = x ^ (x >> np.uint32(16))
    return x


def _mul32_t(x: torch.Tensor, c: int) -> torch.Tensor:
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _lowbias32_t(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32_t(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32_t(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def normal_np(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """fp32 approximately-normal values for counters start .. start+count-1 (numpy, CPU)."""
    k1, k2 = _key(seed, stream)
    n = np.arange(start, start + count, dtype=np.uint64)
    lo = (n & np.uint64(_M32)).astype(np.uint32)
    hi = (n >> np.uint64(32)).astype(np.uint32)
    h1 = _lowbias32_np(lo ^ _lowbias32_np(hi ^ np.uint32(k1)))
    h2 = _lowbias32_np(h1 ^ np.uint32(k2))
    s = ((h1 & np.uint32(0xFFFF)).astype(np.int64) + (h1 >> np.uint32(16)).astype(np.int64)
         + (h2 & np.uint32(0xFFFF)).astype(np.int64) + (h2 >> np.uint32(16)).astype(np.int64))
    return (s - _CENTRE).astype(np.float32) * _SCALE


def normal_torch(seed: int, stream: int, start: int, count: int, device) -> torch.Tensor:
    """Same values as normal_np, computed with torch integer ops on `device`."""
    k1, k2 = _key(seed, stream)
    n = torch.arange(start, start + count, dtype=torch.int64, device=device)
    lo = n & _M32
    hi = n >> 32
    h1 = _lowbias32_t(lo ^ _lowbias32_t(hi ^ k1))
    h2 = _lowbias32_t(h1 ^ k2)
    s = (h1 & 0xFFFF) + (h1 >> 16) + (h2 & 0xFFFF) + (h2 >> 16)
    scale = torch.tensor(float(_SCALE), dtype=torch.float32, device=device)
    return (s - _CENTRE).to(torch.float32) * scale


def draw(seed: int, name: str, shape, *, dtype=torch.float32, device="cpu", offset: int = 0,
         chunk: int = 1 << 25, scale: float | None = None) -> torch.Tensor:
    """Tensor of `shape` whose flat element e holds counter offset+e of stream `name`.

    `scale` (applied in fp32, one rounding) gives N(0,1)*scale; the result is then
    rounded once to `dtype`. Large tensors are drawn in chunks on `device`.
    """
    stream = STREAMS[name]
    numel = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(numel, dtype=dtype, device=device)
    dev = torch.device(device)
    sc = None if scale is None else torch.tensor(np.float32(scale), dtype=torch.float32, device=dev)
    for s in range(0, numel, chunk):
        c = min(chunk, numel - s)
        if dev.type == "cpu":
            x = torch.from_numpy(normal_np(seed, stream, offset + s, c))
        else:
            x = normal_torch(seed, stream, offset + s, c, dev)
        if sc is not None:
            x = x * sc
        out[s:s + c] = x.to(dtype)
    return out.view(*shape)


# ----------------------------------------------------------------------------------------------
# backbone rotary embedding for the attention inputs (not part of the gated operator)
# ----------------------------------------------------------------------------------------------

def backbone_rope_table(positions: np.ndarray, head_dim: int, base: float = 1e6):
    """fp64 cos/sin [n, head_dim/2] for rotate-half rotary embedding at `positions`."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * i / head_dim)
    ang = np.outer(positions.astype(np.float64), inv_freq)
    return np.cos(ang), np.sin(ang)


def backbone_rotate(x: torch.Tensor, positions: np.ndarray, dtype, base: float = 1e6,
                    chunk_tokens: int = 8192) -> torch.Tensor:
    """Rotate x [n, H, d] (fp32 values) at per-token positions; fp64 math, one rounding to dtype."""
    n, H, d = x.shape
    out = torch.empty((n, H, d), dtype=dtype, device=x.device)
    half = d // 2
    for s in range(0, n, chunk_tokens):
        e = min(n, s + chunk_tokens)
        c, sn = backbone_rope_table(positions[s:e], d, base)
        c = torch.from_numpy(c).to(x.device)[:, None, :]
        sn = torch.from_numpy(sn).to(x.device)[:, None, :]
        xs = x[s:e].to(torch.float64)
        x1, x2 = xs[..., :half], xs[..., half:]
        r1 = x1 * c - x2 * sn
        r2 = x2 * c + x1 * sn
        out[s:e] = torch.cat([r1, r2], dim=-1).to(dtype)
    return out


# ----------------------------------------------------------------------------------------------
# problem descriptions and per-workload input sets
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class Shape:
    lengths: list            # per-sequence token counts
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    topk: int
    gate_hidden: int
    dtype: str               # "bf16" or "fp32"
    seed: int
    rms_eps: float = 1e-6
    gate_rope_base: float = 1e6
    attn_rope_base: float = 1e6
    gate_heads: int | None = None   # gate (selection) heads: None/Hkv per KV group, Hq per query head

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def sel_heads(self) -> int:
        return self.gate_heads or self.num_kv_heads

    @property
    def sel_group(self) -> int:
        """query heads per gate head"""
        return self.num_q_heads // self.sel_heads

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.lengths))

    @property
    def max_blocks(self) -> int:
        return (self.max_seqlen + self.block - 1) // self.block

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    def positions(self) -> np.ndarray:
        """in-sequence position of every packed token"""
        return np.concatenate([np.arange(L, dtype=np.int64) for L in self.lengths])

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def draw_lengths(seed: int, count: int, lo: int, hi: int) -> list:
    """Sequence lengths uniform on {lo..hi} (numpy PCG64, seeded)."""
    g = np.random.Generator(np.random.PCG64(seed))
    return [int(x) for x in g.integers(lo, hi + 1, size=count)]


# The workloads. Each is named for what it is; sizes follow the Qwen3 attention shapes.
def workload(name: str) -> Shape:
    if name == "tiny-fp32-T1024":
        return Shape([1024], 2, 1, 64, 16, 4, 32, "fp32", seed=0)
    if name in ("qwen3-4b-prefill-32k", "qwen3-4b-train-32k"):
        return Shape([32768], 32, 8, 128, 64, 31, 128, "bf16",
                     seed=1 if name.endswith("prefill-32k") else 2)
    if name == "qwen3-4b-train-16k":      # same layer, half length: profiling captures
        return Shape([16384], 32, 8, 128, 64, 31, 128, "bf16", seed=5)
    if name == "qwen3-14b-train-16k":     # the 14B layer shape on one 16k sequence: captures
        return Shape([16384], 40, 8, 128, 64, 63, 128, "bf16", seed=7)
    if name == "qwen3-14b-varlen-4seq":
        return Shape(draw_lengths(4, 4, 8192, 65536), 40, 8, 128, 64, 63, 128, "bf16", seed=4)
    raise KeyError(name)


def norm_weight(seed: int, name: str, h: int, device) -> torch.Tensor:
    """A learnable RMSNorm weight as a trained gate would hold it: 1 + 0.25 z, z ~ N(0,1),
    fp32 (one rounding). Not all ones, so the weight's place in the gate is exercised."""
    z = draw(seed, name, (h,), device=device)
    return z * torch.tensor(np.float32(0.25), device=z.device) + 1.0


def prefill_inputs(shape: Shape, device="cpu", *, with_dout: bool = False,
                   sequence: int | None = None) -> dict:
    """Pre-rotary and rotated Q/K, V, gate weights (and dO) for a packed prefill problem.

    Values: N(0,1) for Q/K/V/dO; gate weights N(0,1)/sqrt(fan_in); RMSNorm weights
    1 + 0.25 N(0,1). Everything is rounded once to the problem dtype (gate weights
    included); norm weights stay fp32.
    `sequence` = b draws only sequence b's tokens (the same values as in the packed draw)
    and returns them as a one-sequence problem (see `sequence_shape`).
    """
    Hq, Hkv, d, h = shape.num_q_heads, shape.num_kv_heads, shape.head_dim, shape.gate_hidden
    Hs, Gs = shape.sel_heads, shape.sel_group
    dt, s = shape.torch_dtype, shape.seed
    if sequence is None:
        T, t0, pos, cu = shape.total_tokens, 0, shape.positions(), shape.cu_seqlens
    else:
        T, t0 = shape.lengths[sequence], int(shape.cu_seqlens[sequence])
        pos = np.arange(T, dtype=np.int64)
        cu = np.array([0, T], dtype=np.int32)
    q_nope = draw(s, "q_nope", (T, Hq, d), device=device, offset=t0 * Hq * d)
    k_nope = draw(s, "k_nope", (T, Hkv, d), device=device, offset=t0 * Hkv * d)
    out = {
        "q_nope": q_nope.to(dt),
        "k_nope": k_nope.to(dt),
        "v": draw(s, "v", (T, Hkv, d), dtype=dt, device=device, offset=t0 * Hkv * d),
        "wq": draw(s, "wq", (Hs, h, Gs * d), dtype=dt, device=device, scale=1.0 / math.sqrt(Gs * d)),
        "wk": draw(s, "wk", (Hkv, h, 3 * d), dtype=dt, device=device, scale=1.0 / math.sqrt(3 * d)),
        "qnorm_w": norm_weight(s, "qnorm_w", h, device),
        "knorm_w": norm_weight(s, "knorm_w", h, device),
        "cu_seqlens": torch.from_numpy(cu).to(device),
    }
    # the attention reads rotated Q/K; rotate the already-rounded pre-rotary values
    out["q"] = backbone_rotate(out["q_nope"].float(), pos, dt, shape.attn_rope_base)
    out["k"] = backbone_rotate(out["k_nope"].float(), pos, dt, shape.attn_rope_base)
    del q_nope, k_nope
    if with_dout:
        out["dout"] = draw(s, "dout", (T, Hq, d), dtype=dt, device=device, offset=t0 * Hq * d)
    return out


def sequence_shape(shape: Shape, b: int) -> Shape:
    """Sequence b of a packed problem as a one-sequence problem (prefill_inputs(sequence=b))."""
    return dataclasses.replace(shape, lengths=[shape.lengths[b]])


def random_selection(shape: Shape, seed: int | None = None):
    """A valid selection input for the attention alone, drawn independently of any gate.

    Per (token, gate head -- the kv head, or the query head with one gate per query head):
    min(K, c_t) distinct historical blocks chosen uniformly
    (c_t = in-sequence block of the token), ascending, then the current block,
    then -1 padding. Log-gates are -(1 + 2|z|), z ~ N(0,1); padding slots hold 0.
    Returns int32 idx [T, Hs, K+1] and fp32 logg [T, Hs, K+1] (numpy).
    """
    seed = shape.seed if seed is None else seed
    g = np.random.Generator(np.random.PCG64(seed * 7919 + 13))
    T, Hkv, B, K = shape.total_tokens, shape.sel_heads, shape.block, shape.topk
    idx = np.full((T, Hkv, K + 1), -1, dtype=np.int32)
    base = 0
    for L in shape.lengths:
        nb = (L + B - 1) // B
        for c in range(nb):
            t0, t1 = base + c * B, base + min(L, (c + 1) * B)
            rows = (t1 - t0) * Hkv
            n = min(K, c)
            if n > 0:
                if n == c:
                    pick = np.broadcast_to(np.arange(c, dtype=np.int32), (rows, c))
                else:
                    r = g.random((rows, c))
                    pick = np.sort(np.argpartition(r, n - 1, axis=1)[:, :n], axis=1).astype(np.int32)
                idx[t0:t1, :, :n] = pick.reshape(t1 - t0, Hkv, n)
            idx[t0:t1, :, n] = c
        base += L
    z = normal_np(shape.seed, STREAMS["sel_logg"], 0, T * Hkv * (K + 1)).reshape(T, Hkv, K + 1)
    logg = (-(1.0 + 2.0 * np.abs(z.astype(np.float64)))).astype(np.float32)
    logg[idx < 0] = 0.0
    return idx, logg


# ----------------------------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class DecodeShape:
    lengths: list            # context length per sequence, the new token included
    capacity: int            # cache capacity in tokens (Lmax)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    topk: int
    gate_hidden: int
    seed: int
    dtype: str = "bf16"
    rms_eps: float = 1e-6
    gate_rope_base: float = 1e6
    attn_rope_base: float = 1e6
    gate_heads: int | None = None   # gate (selection) heads: None/Hkv per KV group, Hq per query head

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def sel_heads(self) -> int:
        return self.gate_heads or self.num_kv_heads

    @property
    def sel_group(self) -> int:
        return self.num_q_heads // self.sel_heads

    @property
    def max_blocks(self) -> int:
        return (self.capacity + self.block - 1) // self.block

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def decode_workload(name: str) -> DecodeShape:
    if name == "qwen3-8b-decode-b64":
        lengths = draw_lengths(3, 64, 16384, 131072)
        return DecodeShape(lengths, 131072, 32, 8, 128, 64, 31, 128, seed=3)
    if name == "qwen3-8b-decode-b16-32k":  # a few GB of cache: profiling captures
        lengths = draw_lengths(6, 16, 8192, 32768)
        return DecodeShape(lengths, 32768, 32, 8, 128, 64, 31, 128, seed=6)
    raise KeyError(name)


def decode_inputs(shape: DecodeShape, device="cpu", *, batch_rows=None) -> dict:
    """Inputs of one decode step (caches as given, as a server would hold them).

    k_cache/v_cache [b, Hkv, capacity, d]: rotated keys and values ~N(0,1).
    gate_key_cache [b, Hkv, NBmax, h]: cached gate keys ~N(0,1) (bf16), read for
    the complete blocks only. cur_pool [b, Hkv, 3, d] fp32: a running pool state
    (max, min, sum) of the current block drawn as max = 1+|z1|, min = -1-|z2|,
    sum = sqrt(n) z3 with n the current block's token count.
    `batch_rows` restricts the draw to some sequences (same values as the full draw).
    """
    Hq, Hkv, d, h, G, C, NBm = (shape.num_q_heads, shape.num_kv_heads, shape.head_dim,
                               shape.gate_hidden, shape.group, shape.capacity, shape.max_blocks)
    dt, s, B = shape.torch_dtype, shape.seed, shape.block
    rows = list(range(shape.batch)) if batch_rows is None else list(batch_rows)
    nb = len(rows)

    def per_seq(name, inner, dtype=dt):
        t = torch.empty((nb,) + inner, dtype=dtype, device=device)
        n_inner = int(np.prod(inner))
        for i, b in enumerate(rows):
            t[i] = draw(s, name, inner, dtype=dtype, device=device, offset=b * n_inner)
        return t

    q_nope = per_seq("dec_q_nope", (Hq, d), torch.float32)
    lengths = np.array([shape.lengths[b] for b in rows], dtype=np.int64)
    pos = lengths - 1
    q = torch.empty((nb, Hq, d), dtype=dt, device=device)
    for i in range(nb):
        q[i] = backbone_rotate(q_nope[i:i + 1].to(dt).float(), pos[i:i + 1], dt,
                               shape.attn_rope_base)[0]
    z = per_seq("cur_pool", (Hkv, 3, d), torch.float32)
    n_cur = torch.tensor(lengths - (pos // B) * B, dtype=torch.float32, device=device)
    cur_pool = torch.empty_like(z)
    cur_pool[:, :, 0] = 1.0 + z[:, :, 0].abs()
    cur_pool[:, :, 1] = -1.0 - z[:, :, 1].abs()
    cur_pool[:, :, 2] = z[:, :, 2] * n_cur.sqrt()[:, None, None]
    return {
        "lengths": torch.tensor(lengths, dtype=torch.int32, device=device),
        "q_nope": q_nope.to(dt),
        "q": q,
        "k_cache": per_seq("k_cache", (Hkv, C, d)),
        "v_cache": per_seq("v_cache", (Hkv, C, d)),
        "gate_key_cache": per_seq("gate_key_cache", (Hkv, NBm, h), torch.bfloat16),
        "cur_pool": cur_pool,
        "wq": draw(s, "wq", (shape.sel_heads, h, shape.sel_group * d), dtype=dt, device=device,
                   scale=1.0 / math.sqrt(shape.sel_group * d)),
        "wk": draw(s, "wk", (Hkv, h, 3 * d), dtype=dt, device=device, scale=1.0 / math.sqrt(3 * d)),
        "qnorm_w": norm_weight(s, "qnorm_w", h, device),
        "knorm_w": norm_weight(s, "knorm_w", h, device),
    }
