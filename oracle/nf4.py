"""Oracle for NF4 blockwise quantisation and double quantisation (CPU, NumPy).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Notation (page "QLoRA Explained", sections "Store a weight in 4 bits ..."
through "Shrink the scale factors too ..."):

* W is flattened row-major and cut into blocks of 64 consecutive weights.
* a_b = max |w| over block b is the block's scale ("the largest value,
  ignoring sign").
* x = w / a_b maps the block onto [-1, 1]; the stored 4-bit value is the
  index of the closest of 16 table rows; reading back is row * scale.
* Double quantisation re-quantises the fp32 scales to 8 bits in groups of
  256, one 32-bit constant per group.

fp32 arithmetic is IEEE round-to-nearest-even, written out step by step
(NumPy float32 scalar/array operations are correctly rounded); every
rounding the method performs is named RN32 / RNbf16 in the comments.
"""

from __future__ import annotations

import math
import statistics

import numpy as np

BLOCKSIZE = 64       # "QLoRA quantises in blocks of 64" (section "Why the groups are small")
DQ_BLOCKSIZE = 256   # "grouped, 256 at a time" (section "Shrink the scale factors too")


# ---------------------------------------------------------------------------
# The 16-row tables
# ---------------------------------------------------------------------------

def uniform_table() -> np.ndarray:
    """The strawman table: 16 values evenly spaced from -1 to 1, step 2/15.

    Page "QLoRA Explained", section "The table, and the number that
    stretches it" (first paragraph).  Used only to reproduce the page's
    worked example; NF4 replaces it.
    """
    return np.array([-1.0 + 2.0 * i / 15.0 for i in range(16)], dtype=np.float32)


def nf4_table() -> np.ndarray:
    """The NF4 table: 16 normal quantiles normalised to [-1, 1], one exact 0.

    Page "QLoRA Explained", sections "Put the rows where the weights are"
    and "That is NF4": rows sit at quantiles of a standard bell curve,
    computed once and baked in; one entry is exactly 0; finer near 0.

    Reading (the page gives neither the construction nor the numbers, and
    "16 equal piles, value from the middle of each" yields a symmetric table
    with no zero, contradicting the exact-zero sentence): split the 16 rows
    into 8 positive levels, the exact 0 and 7 negative levels.

      delta = (1/30 + 1/32) / 2
      positive side: probabilities p evenly spaced from 1 - delta down to 1/2
                     with 9 points; drop the last (1/2, which is the zero);
                     value = Phi^-1(p)
      negative side: the same with 8 points, drop the last; value = -Phi^-1(p)
      sort {negatives, 0, positives}; divide by the largest magnitude
      (Phi^-1(1 - delta), so the ends are exactly -1 and +1); round to fp32.

    Phi^-1 is Python's statistics.NormalDist().inv_cdf (fp64).
    """
    nd = statistics.NormalDist()
    delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    top = 1.0 - delta

    def probs(count: int) -> list[float]:
        # `count` evenly spaced points from `top` down to 0.5, last one dropped
        return [top + (0.5 - top) * i / (count - 1) for i in range(count - 1)]

    pos = [nd.inv_cdf(p) for p in probs(9)]      # 8 positive levels
    neg = [-nd.inv_cdf(p) for p in probs(8)]     # 7 negative levels
    levels = sorted(neg + [0.0] + pos)
    scale = max(abs(v) for v in levels)
    return np.array([v / scale for v in levels], dtype=np.float32)


def fp4_table() -> np.ndarray:
    """The FP4 table, by code: a 4-bit float with 1 sign, 2 exponent and 1
    mantissa bit, scaled so its largest magnitude is 1.

    Page "QLoRA Explained", config walk-through: besides NF4 the library
    offers "a small floating-point layout" at the same memory cost; section
    "That is NF4" names the two fields an ordinary float is made of (exponent
    and mantissa).  Reading: the layout is the E2M1 float (sign bit 3,
    exponent bits 2-1 with bias 1, mantissa bit 0; no infinities or NaNs):

      e == 0:  value = (-1)^s * m / 2              (subnormal: 0 or 0.5)
      e >  0:  value = (-1)^s * 2^(e-1) * (1 + m/2)

    giving magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Dividing by the largest, 6,
    maps the table onto [-1, 1] as the absmax scaling needs; RN32 of each
    quotient.  Code 8 is -0.
    """
    vals = []
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = m / 2.0 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
        vals.append(-(mag / 6.0) if s else mag / 6.0)
    return np.array(vals, dtype=np.float32)


def distinct_values(table: np.ndarray):
    """The table's distinct values ascending, each with the code that stores
    it: the lowest code holding the value (+0 rather than -0 for FP4)."""
    t = np.asarray(table, dtype=np.float32)
    vals, codes = [], []
    for c in range(t.size):
        if not any(float(t[c]) == v for v in vals):
            vals.append(float(t[c]))
            codes.append(c)
    order = np.argsort(vals, kind="stable")
    return (np.array(vals, dtype=np.float32)[order], np.array(codes, dtype=np.uint8)[order])


def thresholds(table: np.ndarray) -> np.ndarray:
    """Decision thresholds for "store the index of the closest row".

    Page "QLoRA Explained", section "The table, and the number that stretches
    it", step 3 ("Round to a row ... Closest is ...").

    Reading for ties (the page is silent in general, but its own example in
    "The two failures ..." sends 0, exactly between -0.0667 and +0.0667, to
    +0.0667): a value exactly halfway goes to the HIGHER row.

    With the distinct values ascending, q_0 < ... < q_{v-1}, x is
    closest-or-tied-up to q_{j+1} rather than q_j exactly when
    x >= m_j = (q_j + q_{j+1}) / 2.  m_j is exact in fp64 (both q are fp32).
    For an fp32 x, x >= m_j  <=>  x >= T_j where T_j is the smallest fp32
    that is >= m_j.  Returns the v - 1 T_j as fp32 (15 for NF4, 14 for FP4,
    whose +0 and -0 are one value).
    """
    q = distinct_values(table)[0].astype(np.float64)
    out = np.empty(q.size - 1, dtype=np.float32)
    for j in range(q.size - 1):
        m = (q[j] + q[j + 1]) / 2.0                  # exact in fp64
        t = np.float32(m)                            # RN32(m)
        if float(t) < m:                             # round up if RN went down
            t = np.nextafter(t, np.float32(np.inf))
        out[j] = t
    return out


# ---------------------------------------------------------------------------
# Quantise: blocks, absmax, normalise, nearest code, pack
# ---------------------------------------------------------------------------

def _blocks(W: np.ndarray, blocksize: int) -> np.ndarray:
    """Flatten row-major and cut into [n/blocksize, blocksize] (exact widen to fp32).

    Page "QLoRA Explained", section "Why the groups are small": one scale per
    64 consecutive weights.  Reading: blocks are consecutive in the row-major
    flattening and the column count must be a multiple of the block size, so
    that no block straddles two rows.
    """
    W = np.asarray(W)
    if W.ndim != 2:
        raise ValueError("weight must be a 2-D matrix")
    if W.shape[1] % blocksize != 0:
        raise ValueError("columns must be a multiple of the block size")
    w = W.astype(np.float32).reshape(-1)            # bf16/fp32 -> fp32 is exact
    if not np.all(np.isfinite(w)):
        # Reading: the pages never meet NaN/Inf weights; reject them.
        raise ValueError("non-finite weight")
    return w.reshape(-1, blocksize)


def block_absmax(W: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """a_b = max |w| over each block (exact).  Section "The table, and the
    number that stretches it", step 1 ("the largest of them, ignoring sign")."""
    return np.abs(_blocks(W, blocksize)).max(axis=1).astype(np.float32)


def normalise(W: np.ndarray, absmax: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """x = RN32(w / a_b), IEEE fp32 division.  Step 1 of the worked example
    ("Divide every weight in the group by it").

    Reading: a block whose absmax is 0 holds only zeros; its x are all 0.
    """
    blk = _blocks(W, blocksize)
    a = np.asarray(absmax, dtype=np.float32)[:, None]
    safe = np.where(a == 0, np.float32(1), a).astype(np.float32)
    x = (blk / safe).astype(np.float32)             # RN32(w / a_b)
    return np.where(a == 0, np.float32(0), x).astype(np.float32)


def nearest_code(x: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Code of the closest table value, ties to the higher value (see
    thresholds): the k-th smallest distinct value with k = #{ j : x >= T_j },
    stored under the code distinct_values gives it (for NF4, whose values
    ascend with the code, code = k)."""
    T = thresholds(table)
    codes = distinct_values(table)[1]
    x = np.asarray(x, dtype=np.float32)
    return codes[np.searchsorted(T, x, side="right")].astype(np.uint8)


def quantize(W: np.ndarray, table: np.ndarray | None = None,
             blocksize: int = BLOCKSIZE) -> tuple[np.ndarray, np.ndarray]:
    """Blockwise quantisation: returns (codes uint8[n], absmax fp32[n/64]).

    Page "QLoRA Explained", section "The table, and the number that stretches
    it", steps 1-3, with the NF4 table of section "That is NF4" (or any
    other 16-row table, e.g. the uniform one for the worked example).
    """
    if table is None:
        table = nf4_table()
    a = block_absmax(W, blocksize)
    x = normalise(W, a, blocksize)
    codes = nearest_code(x, table).reshape(-1)
    return codes, a


def pack(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte.

    Reading (the pages only say a code is 4 bits): element 2j goes to the
    HIGH nibble and element 2j+1 to the LOW nibble of byte j.
    """
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if c.size % 2:
        raise ValueError("odd number of codes")
    if c.size and c.max() > 15:
        raise ValueError("code out of range")
    return ((c[0::2] << 4) | c[1::2]).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack."""
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0x0F
    return out


# ---------------------------------------------------------------------------
# Double quantisation of the absmax constants
# ---------------------------------------------------------------------------

def dq_mean(absmax: np.ndarray) -> np.float32:
    """Per-tensor mean offset mu = RN32( RN64(exact sum) / n ).

    The pages say only "one 32-bit constant per group" for the second level
    (section "Shrink the scale factors too").  Reading: that per-group
    constant is the scale, and the mean offset subtracted before the 8-bit
    step is ONE fp32 per tensor (O(1) storage, so the page's closed form
    4 + 8/64 + 32/16384 bits is unchanged up to 32/n).  The sum is the exact
    real sum rounded once to fp64 (math.fsum), divided by n in fp64, then
    rounded to fp32.
    """
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    if a.size == 0:
        raise ValueError("empty absmax")
    s = math.fsum(float(v) for v in a)               # correctly rounded exact sum
    return np.float32(s / a.size)                    # fp64 divide, then RN32


def e4m3_values() -> np.ndarray:
    """The 127 non-negative finite values of the 8-bit float E4M3 (sign bit,
    4 exponent bits with bias 7, 3 mantissa bits; exponent field 15 with
    mantissa 7 is NaN), by code 0..126, exact in fp64:
      e == 0:  m / 8 * 2^-6           (subnormal)
      e >  0:  (1 + m / 8) * 2^(e - 7)"""
    out = []
    for code in range(127):
        e, m = code >> 3, code & 7
        out.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out, dtype=np.float64)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """E4M3 code (uint8) of each fp32 value: the nearest finite value, a tie
    to the even code, magnitudes above 448 saturated to 448; the sign bit is
    kept, so a negative value that rounds to zero is -0 (code 0x80)."""
    v = e4m3_values()
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), v[-1])
    hi = np.clip(np.searchsorted(v, a, side="left"), 0, v.size - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - v[lo], v[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """fp64 value of E4M3 codes (NaN codes 0x7F / 0xFF give NaN)."""
    c = np.asarray(code, dtype=np.uint8)
    mag = c & 0x7F
    v = np.append(e4m3_values(), np.nan)[mag]
    return np.where(c & 0x80, -v, v)


def double_quantize(absmax: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE, fmt: str = "int8"):
    """8-bit quantisation of the block scales in groups of 256.

    Page "QLoRA Explained", section "Shrink the scale factors too": each scale
    is stored in 8 bits, grouped 256 at a time with one 32-bit constant per
    group.  Reading (the 8-bit format is not named; the same page's scale-and-
    round recipe is the 8-bit integer one): symmetric linear int8 with an
    absmax per group, after subtracting the per-tensor mean:

      d   = RN32(a - mu)
      s_g = max |d| over the group (a last partial group uses its own elements)
      c   = round_half_even( RN32( RN32(d / s_g) * 127 ) ) in [-127, 127]
      s_g == 0  ->  c = 0

    Returns (qabsmax int8[n], dq_scale fp32[ceil(n/256)], mu fp32).

    fmt = "fp8": the 8-bit float variant (the pages name no 8-bit format; the
    original method's second level is an 8-bit float).  Reading: the same d,
    s_g and t = RN32(d / s_g), then the E4M3 code of 256 * t (exact scaling;
    E4M3's largest value 448 is never reached), round to nearest, ties to the
    even code; the code bytes are returned in the int8 array.
    """
    if fmt not in ("int8", "fp8"):
        raise ValueError("fmt must be int8 or fp8")
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    mu = dq_mean(a)
    d = (a - mu).astype(np.float32)                              # RN32(a - mu)
    ngroups = (a.size + dq_blocksize - 1) // dq_blocksize
    scale = np.zeros(ngroups, dtype=np.float32)
    q = np.zeros(a.size, dtype=np.int8)
    for g in range(ngroups):
        dg = d[g * dq_blocksize:(g + 1) * dq_blocksize]
        sg = np.float32(np.abs(dg).max())
        scale[g] = sg
        if sg == 0:
            continue
        t = (dg / sg).astype(np.float32)                         # RN32(d / s_g)
        if fmt == "fp8":
            u = (t * np.float32(256)).astype(np.float32)         # exact
            q[g * dq_blocksize:(g + 1) * dq_blocksize] = e4m3_encode(u).view(np.int8)
            continue
        t = (t * np.float32(127)).astype(np.float32)             # RN32(. * 127)
        c = np.rint(t)                                           # half to even
        q[g * dq_blocksize:(g + 1) * dq_blocksize] = np.clip(c, -127, 127).astype(np.int8)
    return q, scale, mu


def dq_absmax(qabsmax: np.ndarray, dq_scale: np.ndarray, mu,
              dq_blocksize: int = DQ_BLOCKSIZE, fmt: str = "int8") -> np.ndarray:
    """Recovered block scale a^ = RN32( RN32( RN32(c / 127) * s_g ) + mu ),
    or with fmt = "fp8" RN32( RN32( (e4m3(c) / 256) * s_g ) + mu ) (the
    division by 256 is exact)."""
    s = np.repeat(np.asarray(dq_scale, dtype=np.float32), dq_blocksize)[: np.asarray(qabsmax).size]
    if fmt == "fp8":
        t = (e4m3_decode(np.asarray(qabsmax).view(np.uint8)) / 256.0).astype(np.float32)
    else:
        c = np.asarray(qabsmax, dtype=np.int8).astype(np.float32)
        t = (c / np.float32(127)).astype(np.float32)             # RN32(c / 127)
    t = (t * s).astype(np.float32)                               # RN32(. * s_g)
    return (t + np.float32(mu)).astype(np.float32)               # RN32(. + mu)


# ---------------------------------------------------------------------------
# Dequantise
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """RNbf16: fp32 -> bf16 round-to-nearest-even; returns the bf16 values as fp32.

    bf16 keeps the top 16 bits of the fp32 pattern.  Rounding adds half of the
    dropped part, with ties going to an even kept part.  Finite inputs only.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep = u >> 16
    rest = u & 0xFFFF
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & 1) == 1))
    r = ((keep + up.astype(np.uint64)) << 16).astype(np.uint32)
    return r.view(np.float32)


def dequantize(packed: np.ndarray, absmax_hat: np.ndarray, shape,
               table: np.ndarray | None = None, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """w' = RNbf16( RN32( q[code] * a^ ) ), returned as fp32 holding bf16 values.

    Page "QLoRA Explained", step 4 of the worked example ("Look up the row ...
    multiply by the scale") and section "That is NF4" / the config walk-through
    (the expansion target is bf16).  a^ is the block's absmax (no double
    quantisation) or dq_absmax(...) (with it).
    """
    if table is None:
        table = nf4_table()
    codes = unpack(packed)
    rows, cols = shape
    if codes.size != rows * cols:
        raise ValueError("shape does not match packed size")
    vals = np.asarray(table, dtype=np.float32)[codes].reshape(-1, blocksize)
    a = np.asarray(absmax_hat, dtype=np.float32)[:, None]
    w = (vals * a).astype(np.float32)                            # RN32(q * a^)
    return round_bf16(w).reshape(rows, cols)


# ---------------------------------------------------------------------------
# Storage accounting
# ---------------------------------------------------------------------------

def stored_bits_per_param(n: int, double_quant: bool = True,
                          blocksize: int = BLOCKSIZE,
                          dq_blocksize: int = DQ_BLOCKSIZE) -> float:
    """Bits stored per weight for an n-weight matrix.

    Page "QLoRA Explained", section "Shrink the scale factors too": 4 bits of
    code, plus 32/64 for fp32 scales, or with double quantisation 8/64 for the
    8-bit scales plus 32 per group of 256 scales; plus (reading above) one fp32
    mean per tensor.
    """
    nblocks = n // blocksize
    if not double_quant:
        return (4 * n + 32 * nblocks) / n
    ngroups = (nblocks + dq_blocksize - 1) // dq_blocksize
    return (4 * n + 8 * nblocks + 32 * ngroups + 32) / n
