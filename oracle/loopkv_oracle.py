"""Plain CPU oracle for the LoopKV decode path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
CPU-baseline / reference legs of the benchmark may import this module.  The
product path (the CUDA library and its Python binding) never calls it and
shares no code with it.

What it computes, following LoopKV: Loop-Aware KV Cache Compression for
Serving Looped Transformers (Abstract):
  * every (loop, layer) cell is stored 4-bit, 2-bit, or reuses the final
    loop's cell of the same layer;
  * a 4-bit code is stored as two 2-bit planes (top and bottom bits); a
    decode step reads the top plane of every value and the bottom plane only
    for tokens that the cell's own query weights heavily enough.

The pages leave the quantiser and the threshold rule open; this oracle takes
the readings the library documents:
  * asymmetric b-bit quantisation, keys per channel over 32-token groups
    aligned at positions 0, 32, 64, ..., values per token over 32-channel
    groups; scale and minimum rounded to bf16 (round to nearest even);
  * quantiser arithmetic in fp32, one correctly rounded operation at a time,
    because its result is an integer code that both sides must agree on;
  * key tokens of an unfinished group stay exact (bf16) until the group fills;
  * a value's high-plane-only reconstruction is the bucket midpoint
    ``min + scale * (4 * hi + 1.5)``;
  * a token takes the low plane when its softmax weight, rounded to fp32, is
    at least tau (tau = 0 selects every token, tau = +inf none);
  * grouped queries (several query heads per KV head): a token's low plane
    is fetched when any head of the group selects it and then serves every
    head of the group;
  * a reuse cell of a loop before the last may attend, besides the final
    loop's stored tokens, the current token exactly as its own loop computed
    it (that token's K/V exist in the loop but are stored nowhere): one more
    softmax entry with exact key and value and no low plane;
  * attention itself is evaluated in fp64.

Byte layout (the oracle's own reading of the record format, used only to
compare the library's packed bytes): per (physical block, head) record of
``block_size`` (16) tokens,
  4-bit: [K hi plane][K lo plane][K meta][V hi plane][V meta][V lo plane]
  2-bit: [K plane][K meta][V plane][V meta]
  bf16 : [K rows][V rows]
A plane row is one token, channel c at byte c // 4, bits 2 * (c % 4) and up.
The K planes and the V lo plane store the 16 rows one after another
(row-major); the V hi plane (4-bit) and the V plane (2-bit) store the same
bytes transposed (column-major): byte 16 * (c // 4) + t is row t's byte c // 4.
K meta holds (scale, min) bf16 pairs of half the channels of the 32-token
group: channels [0, D/2) in the group's even block, [D/2, D) in the odd one.
V meta holds (scale, min) per token row and 32-channel group.
"""

from __future__ import annotations

import numpy as np

GROUP = 32          # quantisation group (tokens for keys, channels for values)
BLOCK = 16          # tokens per paged block

BITS = {"q4": 4, "q2": 2}


# ---------------------------------------------------------------------------
# bf16 helpers
# ---------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    x = np.asarray(x, dtype=np.float32)
    shape = x.shape
    u = np.ascontiguousarray(x).reshape(-1).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).reshape(shape)


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of bf16-exact fp32 values."""
    x = np.asarray(x, dtype=np.float32)
    u = np.ascontiguousarray(x).reshape(-1).view(np.uint32).reshape(x.shape)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("value is not bf16-exact")
    return (u >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Quantiser
# ---------------------------------------------------------------------------

def quantize_group(x, bits: int):
    """Asymmetric ``bits``-bit quantisation of the last axis (one group).

    Returns (codes uint8[..., G], scale fp32[...], minimum fp32[...]); scale
    and minimum are bf16-exact.  Steps, each a single fp32 operation:
      mn_b = bf16(min x);  s_b = bf16((max x - mn_b) / (2^b - 1));
      code = clamp(rint_half_even((x - mn_b) / s_b), 0, 2^b - 1), 0 if s_b = 0.
    """
    x = np.asarray(x, dtype=np.float32)
    levels = np.float32(2 ** bits - 1)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    mn_b = bf16_round(mn)
    s_b = bf16_round((mx - mn_b) / levels)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x - mn_b[..., None]) / s_b[..., None]
    codes = np.where(s_b[..., None] == 0, np.float32(0),
                     np.clip(np.rint(t), np.float32(0), levels))
    return codes.astype(np.uint8), s_b.astype(np.float32), mn_b.astype(np.float32)


class QuantKeys:
    """Keys of one (sequence, head): complete 32-token groups quantised per
    channel, the tail of an unfinished group kept exact."""

    def __init__(self, k: np.ndarray, bits: int):
        k = np.asarray(k, dtype=np.float32)
        n, d = k.shape
        ng = n // GROUP
        self.bits, self.n, self.d = bits, n, d
        grouped = k[: ng * GROUP].reshape(ng, GROUP, d).transpose(0, 2, 1)  # [g, ch, tok]
        codes, s, mn = quantize_group(grouped, bits)
        self.codes = codes.transpose(0, 2, 1).reshape(ng * GROUP, d)       # [tok, ch]
        self.scale = s            # [g, ch]
        self.minv = mn            # [g, ch]
        self.residual = k[ng * GROUP:].copy()                              # [n % 32, ch]

    def dequant(self) -> np.ndarray:
        ng = self.codes.shape[0] // GROUP
        out = np.empty((self.n, self.d), dtype=np.float64)
        if ng:
            c = self.codes.reshape(ng, GROUP, self.d).astype(np.float64)
            s = self.scale.astype(np.float64)[:, None, :]
            m = self.minv.astype(np.float64)[:, None, :]
            out[: ng * GROUP] = (m + s * c).reshape(ng * GROUP, self.d)
        out[ng * GROUP:] = self.residual
        return out


class QuantValues:
    """Values of one (sequence, head), quantised per token over 32-channel groups."""

    def __init__(self, v: np.ndarray, bits: int):
        v = np.asarray(v, dtype=np.float32)
        n, d = v.shape
        self.bits, self.n, self.d = bits, n, d
        codes, s, mn = quantize_group(v.reshape(n, d // GROUP, GROUP), bits)
        self.codes = codes.reshape(n, d)     # [tok, ch]
        self.scale = s                       # [tok, d/32]
        self.minv = mn                       # [tok, d/32]

    def _expand(self, a):
        return np.repeat(a.astype(np.float64), GROUP, axis=1)

    def dequant_full(self) -> np.ndarray:
        return self._expand(self.minv) + self._expand(self.scale) * self.codes.astype(np.float64)

    def dequant_high(self) -> np.ndarray:
        """High-plane-only reconstruction of a 4-bit value: bucket midpoint."""
        if self.bits != 4:
            raise ValueError("high-plane reconstruction is defined for 4-bit cells")
        hi = (self.codes >> 2).astype(np.float64)
        return self._expand(self.minv) + self._expand(self.scale) * (4.0 * hi + 1.5)


# ---------------------------------------------------------------------------
# Attention of one (cell, sequence, head)
# ---------------------------------------------------------------------------

def softmax_weights(q, k_hat, sm_scale: float):
    """fp64 logits and softmax weights of one query over n keys."""
    s = float(sm_scale) * (np.asarray(k_hat, np.float64) @ np.asarray(q, np.float64))
    m = s.max()
    e = np.exp(s - m)
    return s, e / e.sum()


def select_low_plane(p, tau: float, unit: int = 1) -> np.ndarray:
    """Tokens whose fp32 softmax weight is at least tau.

    ``unit`` > 1 is a coarser granularity of the same rule, offered as a
    variant (16: a paged block, 32: a key group): every
    token of the aligned unit [u*unit, (u+1)*unit) takes its low plane when
    the unit's largest fp32 weight is at least tau.
    """
    tok = np.asarray(p, np.float64).astype(np.float32) >= np.float32(tau)
    if unit == 1 or tok.size == 0:
        return tok
    if unit not in (16, 32):
        raise ValueError("selection unit must be 1, 16 or 32")
    n = tok.size
    units = -(-n // unit)
    padded = np.zeros(units * unit, dtype=bool)
    padded[:n] = tok
    any_in_unit = padded.reshape(units, unit).any(axis=1)
    return np.repeat(any_in_unit, unit)[:n]


def attend(q, k_hat, v_full, v_high, tau: float, sm_scale: float, unit: int = 1, k_cur=None, v_cur=None):
    """Decode attention of one query (``unit``: selection granularity, see
    select_low_plane).

    ``v_high`` is None for cells without a low plane (2-bit, bf16); then every
    token uses ``v_full`` and nothing is selected.

    ``k_cur``, ``v_cur`` (optional, exact rows [D]) add one token after the n
    stored ones: the current token as its own loop computed it, which a reuse
    cell has not stored anywhere (it reads the final loop's cell, where that
    token does not exist yet).  It takes part in the softmax with its exact
    key and value and has no low plane; the selection rule applies to the
    stored tokens with their weights in that softmax.

    Returns (o fp64[D], selected bool[n], p fp64[n], or [n + 1] with the
    current token's weight last).
    """
    k_hat = np.asarray(k_hat, np.float64)
    n, d = k_hat.shape
    cur = k_cur is not None
    if n == 0 and not cur:
        return np.zeros(d), np.zeros(0, dtype=bool), np.zeros(0)
    keys = np.vstack([k_hat, np.asarray(k_cur, np.float64)[None]]) if cur else k_hat
    _, p = softmax_weights(q, keys, sm_scale)
    ps = p[:n]
    if v_high is None:
        sel = np.zeros(n, dtype=bool)
        v_hat = np.asarray(v_full, np.float64).reshape(n, d)
    else:
        sel = select_low_plane(ps, tau, unit)
        v_hat = np.where(sel[:, None], v_full, v_high).reshape(n, d)
    o = ps @ v_hat
    if cur:
        o = o + p[n] * np.asarray(v_cur, np.float64)
    return o, sel, p


def attend_grouped(queries, k_hat, v_full, v_high, tau: float, sm_scale: float, unit: int = 1,
                   k_cur=None, v_cur=None):
    """Decode attention of the G query heads that share one KV head.

    Grouped-query form of the low-plane rule (the survey's selection
    variants; the pages speak of one query per head): the KV head's low plane
    of a token is fetched when any query head of the group selects it (its own
    fp32 weight, or its unit's largest one, reaches tau), and a fetched row
    serves every head of the group.  So each head's values are the full 4-bit
    values on the union of the heads' selections and the high-plane midpoints
    elsewhere, while each head keeps its own softmax weights.  ``k_cur``,
    ``v_cur``: one exact current token of the KV head, as in attend.  Returns
    (o fp64[G, D], selected bool[n], p fp64[G, n] or [G, n + 1]).
    """
    queries = np.asarray(queries, np.float32)
    g = queries.shape[0]
    k_hat = np.asarray(k_hat, np.float64)
    n, d = k_hat.shape
    cur = k_cur is not None
    if n == 0 and not cur:
        return np.zeros((g, d)), np.zeros(0, dtype=bool), np.zeros((g, 0))
    keys = np.vstack([k_hat, np.asarray(k_cur, np.float64)[None]]) if cur else k_hat
    p = np.stack([softmax_weights(qh, keys, sm_scale)[1] for qh in queries])
    ps = p[:, :n]
    sel = np.zeros(n, dtype=bool)
    if v_high is None:
        v_hat = np.asarray(v_full, np.float64).reshape(n, d)
    else:
        for h in range(g):
            sel |= select_low_plane(ps[h], tau, unit)
        v_hat = np.where(sel[:, None], v_full, v_high).reshape(n, d)
    o = ps @ v_hat
    if cur:
        o = o + p[:, n:] * np.asarray(v_cur, np.float64)[None]
    return o, sel, p


class StoredSequence:
    """One (stored cell, sequence, head): the quantised (or exact) K and V."""

    def __init__(self, kind: str, k, v):
        self.kind = kind
        k = np.asarray(k, dtype=np.float32)
        v = np.asarray(v, dtype=np.float32)
        self.n = k.shape[0]
        if kind == "bf16":
            self.k_exact, self.v_exact = k.copy(), v.copy()
        elif kind in BITS:
            self.qk = QuantKeys(k, BITS[kind])
            self.qv = QuantValues(v, BITS[kind])
        else:
            raise ValueError(kind)

    def attend(self, q, tau: float, sm_scale: float, unit: int = 1, k_cur=None, v_cur=None):
        """Attention of one query over every stored token (and the exact
        current token k_cur, v_cur when given; see attend)."""
        if self.kind == "bf16":
            return attend(q, self.k_exact, self.v_exact, None, tau, sm_scale, k_cur=k_cur, v_cur=v_cur)
        k_hat = self.qk.dequant()
        v_full = self.qv.dequant_full()
        v_high = self.qv.dequant_high() if self.kind == "q4" else None
        return attend(q, k_hat, v_full, v_high, tau, sm_scale, unit, k_cur=k_cur, v_cur=v_cur)

    def attend_grouped(self, queries, tau: float, sm_scale: float, unit: int = 1, k_cur=None, v_cur=None):
        """Attention of the G query heads sharing this KV head (see
        attend_grouped)."""
        if self.kind == "bf16":
            return attend_grouped(queries, self.k_exact, self.v_exact, None, tau, sm_scale, k_cur=k_cur,
                                  v_cur=v_cur)
        v_high = self.qv.dequant_high() if self.kind == "q4" else None
        return attend_grouped(queries, self.qk.dequant(), self.qv.dequant_full(), v_high, tau, sm_scale, unit,
                              k_cur=k_cur, v_cur=v_cur)


def resolve_source(plan, cell: int, num_layers: int) -> int:
    """A reuse cell reads the final loop's cell of the same layer."""
    if plan[cell] != "reuse":
        return cell
    num_loops = len(plan) // num_layers
    src = (num_loops - 1) * num_layers + cell % num_layers
    if plan[src] == "reuse":
        raise ValueError("the final loop cannot reuse")
    return src


def decode_cell(plan, num_layers: int, cell: int, stored: dict, q, seq_lens,
                tau: float, sm_scale: float, pairs=None, current=None):
    """Decode attention of one cell for the (b, h) pairs given.

    ``stored[(src_cell, b, h)]`` is the StoredSequence of a stored cell;
    ``q`` is fp32[B, H, D]; ``current`` (optional) maps (b, h) to the exact
    (k, v) rows of the current token, attended after the stored tokens (a
    reuse cell's own K/V of the token being decoded); returns
    {(b, h): (o, selected, p)}.
    """
    src = resolve_source(plan, cell, num_layers)
    out = {}
    for (b, h) in pairs:
        seq = stored[(src, b, h)]
        if int(seq_lens[b]) != seq.n:
            raise ValueError("sequence length does not match the stored sequence")
        kc, vc = (None, None) if current is None else current[(b, h)]
        out[(b, h)] = seq.attend(np.asarray(q[b, h], np.float32), tau, sm_scale, k_cur=kc, v_cur=vc)
    return out


# ---------------------------------------------------------------------------
# Byte layout of a stored cell (the oracle's own reading of the record format)
# ---------------------------------------------------------------------------

def record_sections(kind: str, d: int, block: int = BLOCK):
    """[(name, offset, size)] of one (block, head) record."""
    plane = block * d // 4                 # 2 bits per element
    kmeta = (d // 2) * 4                   # (scale, min) bf16 for half the channels
    vmeta = block * (d // GROUP) * 4       # (scale, min) bf16 per token and channel group
    if kind == "q4":
        sizes = [("k_hi", plane), ("k_lo", plane), ("k_meta", kmeta),
                 ("v_hi", plane), ("v_meta", vmeta), ("v_lo", plane)]
    elif kind == "q2":
        sizes = [("k", plane), ("k_meta", kmeta), ("v", plane), ("v_meta", vmeta)]
    elif kind == "bf16":
        sizes = [("k", block * d * 2), ("v", block * d * 2)]
    else:
        raise ValueError(kind)
    out, off = [], 0
    for name, size in sizes:
        out.append((name, off, size))
        off += size
    return out


def record_bytes(kind: str, d: int, block: int = BLOCK) -> int:
    name, off, size = record_sections(kind, d, block)[-1]
    return off + size


def pack_plane(codes2) -> np.ndarray:
    """2-bit codes uint8[rows, D] -> plane bytes uint8[rows, D/4]."""
    c = np.asarray(codes2, dtype=np.uint8)
    if np.any(c > 3):
        raise ValueError("plane codes must be 2-bit")
    rows, d = c.shape
    c4 = c.reshape(rows, d // 4, 4).astype(np.uint16)
    return (c4[..., 0] | (c4[..., 1] << 2) | (c4[..., 2] << 4) | (c4[..., 3] << 6)).astype(np.uint8)


def pack_plane_columns(codes2, block: int = BLOCK) -> np.ndarray:
    """2-bit codes uint8[block, D] of one block -> column-major plane bytes
    uint8[D/4 * block]: the row-major plane transposed, so that byte
    block * j + t is row t's byte j (channels 4j .. 4j + 3)."""
    rows = pack_plane(codes2)                       # [block, D/4]
    if rows.shape[0] != block:
        raise ValueError("a column-major plane holds exactly one block of rows")
    return np.ascontiguousarray(rows.T).reshape(-1)


def _meta_bytes(scale, minv) -> np.ndarray:
    """(scale, min) bf16 pairs, little-endian, scale first -> uint8[..., 4]."""
    s = bf16_bits(scale).astype(np.uint32)
    m = bf16_bits(minv).astype(np.uint32)
    word = (s | (m << np.uint32(16))).astype("<u4")
    return word.view(np.uint8).reshape(word.shape + (4,))


def sequence_records(kind: str, k, v, block: int = BLOCK):
    """Expected records of one (cell, sequence, head) after its first n tokens
    were appended to a zero-filled arena.

    Returns (records uint8[nblocks, rec], residual fp32[n % 32, D] or None).
    """
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    n, d = k.shape
    nblocks = -(-n // block)
    secs = {name: (off, size) for name, off, size in record_sections(kind, d, block)}
    rec = np.zeros((nblocks, record_bytes(kind, d, block)), dtype=np.uint8)
    row = d // 4

    def put(blk, name, r, data):
        off, _ = secs[name]
        flat = np.asarray(data, np.uint8).ravel()
        rec[blk, off + r * flat.size: off + (r + 1) * flat.size] = flat

    if kind == "bf16":
        kb = bf16_bits(k).view(np.uint8).reshape(n, 2 * d)
        vb = bf16_bits(v).view(np.uint8).reshape(n, 2 * d)
        for t in range(n):
            put(t // block, "k", t % block, kb[t])
            put(t // block, "v", t % block, vb[t])
        return rec, None

    bits = BITS[kind]
    qk, qv = QuantKeys(k, bits), QuantValues(v, bits)
    # values: every token; the high (2-bit: only) plane column-major
    vmeta = _meta_bytes(qv.scale, qv.minv)          # [n, d/32, 4]
    hi_codes = (qv.codes >> 2) if kind == "q4" else qv.codes
    v_lo = pack_plane(qv.codes & 3) if kind == "q4" else None
    for t in range(n):
        blk, r = t // block, t % block
        if v_lo is not None:
            put(blk, "v_lo", r, v_lo[t])
        put(blk, "v_meta", r, vmeta[t])
    off, size = secs["v_hi" if kind == "q4" else "v"]
    for blk in range(nblocks):
        rows = np.zeros((block, d), dtype=np.uint8)          # tokens past n: zero bytes
        part = hi_codes[blk * block: (blk + 1) * block]
        rows[: part.shape[0]] = part
        rec[blk, off: off + size] = pack_plane_columns(rows, block)
    # keys: complete groups only
    ng = n // GROUP
    if kind == "q4":
        k_hi, k_lo = pack_plane(qk.codes >> 2), pack_plane(qk.codes & 3)
    else:
        k_hi, k_lo = pack_plane(qk.codes), None
    for t in range(ng * GROUP):
        blk, r = t // block, t % block
        put(blk, "k_hi" if kind == "q4" else "k", r, k_hi[t])
        if k_lo is not None:
            put(blk, "k_lo", r, k_lo[t])
    kmeta = _meta_bytes(qk.scale, qk.minv)          # [ng, d, 4]
    half = d // 2
    blocks_per_group = GROUP // block
    for g in range(ng):
        for part in range(blocks_per_group):
            chans = slice(part * d // blocks_per_group, (part + 1) * d // blocks_per_group)
            off, size = secs["k_meta"]
            data = kmeta[g, chans].ravel()
            rec[g * blocks_per_group + part, off: off + data.size] = data
    assert half * 4 == secs["k_meta"][1]
    return rec, qk.residual


def unpack_plane(plane_bytes, d: int) -> np.ndarray:
    """Inverse of pack_plane (used by tests to read records back)."""
    b = np.asarray(plane_bytes, np.uint8)
    rows = b.shape[0]
    out = np.empty((rows, d), dtype=np.uint8)
    for i in range(4):
        out[:, i::4] = (b >> (2 * i)) & 3
    return out
