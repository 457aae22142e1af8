"""NF4 storage with double quantization: the plain, slow CPU definition.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by tests and by
the CPU-baseline legs of the benchmark, never by the product path.

Precision: floating point that decides an integer (a code, an int8 scale) is
done in fp32, as the kernels do; the second-level mean uses an exactly rounded
fp64 sum.  numpy float32 arithmetic is IEEE single with round-to-nearest-even
and no fused multiply-add, so each step below is one correctly rounded
operation.

Readings of the pages taken here (each also listed in the design notes):
  * level table: the snippet's quantile construction evaluated in fp64, then
    rounded once to fp32 (the snippet itself runs in fp32 torch);
  * blocks of 64 run along d_in inside one row of the row-major [d_out, d_in]
    weight, i.e. over the flattened order, as the snippet's [4096, 64] rows do;
  * an all-zero block gets scale 0 and every code = the zero level;
  * ties between two levels go to the lower index (argmin's first minimum);
  * double quantization, per group of 256 consecutive block scales: subtract
    the group mean (fp64 sum, divided, rounded to fp32), then symmetric int8
    absmax (step = max|d|/127, code = round-half-even(d/step) in [-127, 127]);
    the group's step and mean are stored as fp32;
  * packing: byte j of a row holds element 2j in its low nibble and element
    2j+1 in its high nibble;
  * dequantization: s_hat = fl32(fl32(q * step) + mean), then
    w_hat = bf16_rne(fl32(level[code] * s_hat)).
"""

import math
import statistics

import numpy as np

BLOCK = 64          # weights per absmax block  [QLoRA glossary, "Come funziona QLoRA", NF4]
DQ_GROUP = 256      # block scales per second-level group  [QLoRA glossary, "Doppia quantizzazione"]
DQ_QMAX = 127       # symmetric signed 8-bit codes  [Módulo 4: QLoRA, 4.3 b)]


# ---------------------------------------------------------------- bf16 helpers

def bf16_bits_to_f32(bits):
    """Widen bf16 bit patterns (uint16) to float32 exactly (append 16 zero bits)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32)
    return (b << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def f32_to_bf16_bits(x):
    """Round float32 to bf16 with round-to-nearest-even, returning uint16 bits.

    The upper 16 bits of the float32 are kept; the discarded lower half is
    rounded to nearest, ties to the even kept pattern.  NaN maps to a quiet NaN.
    Inputs here are finite; the NaN branch only keeps the function total.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    keep = u >> np.uint64(16)
    low = u & np.uint64(0xFFFF)
    round_up = (low > 0x8000) | ((low == 0x8000) & ((keep & np.uint64(1)) == 1))
    out = (keep + round_up.astype(np.uint64)) & np.uint64(0xFFFF)
    nan = np.isnan(f)
    out = np.where(nan, np.uint64(0x7FC0), out)
    return out.astype(np.uint16)


# ---------------------------------------------------------------- level tables

def nf4_levels_f64():
    """The 16 NF4 levels in fp64.  [QLoRA glossary, NF4 snippet]

    Eight positive levels are the standard-normal quantiles at the first 8 of
    9 evenly spaced probabilities from 0.9677083 down to 0.5; seven negative
    levels are the negated quantiles at the first 7 of 8 such probabilities;
    an exact zero is added; the 16 values are sorted and divided by the largest.
    The inverse normal CDF is Python's ``statistics.NormalDist.inv_cdf``.
    """
    normal = statistics.NormalDist(0.0, 1.0)
    p_pos = np.linspace(0.9677083, 0.5, 9)[:-1]
    p_neg = np.linspace(0.9677083, 0.5, 8)[:-1]
    positive = [normal.inv_cdf(float(p)) for p in p_pos]
    negative = [-normal.inv_cdf(float(p)) for p in p_neg]
    levels = sorted(negative + [0.0] + positive)
    top = max(levels)
    return np.array([v / top for v in levels], dtype=np.float64)


def nf4_levels():
    """The NF4 table as stored and used: fp64 levels rounded once to fp32."""
    return nf4_levels_f64().astype(np.float32)


def int4_levels():
    """Sixteen evenly spaced levels on [-1, 1], the snippet's comparison table.
    [QLoRA glossary, NF4 snippet]"""
    return np.linspace(-1.0, 1.0, 16).astype(np.float32)


def zero_code(levels):
    """Index of the exact zero level (7 for NF4)."""
    idx = np.nonzero(np.asarray(levels) == 0.0)[0]
    return int(idx[0]) if len(idx) else int(np.argmin(np.abs(levels)))


# ---------------------------------------------------------------- first level

def encode_blocks(w32, levels, chunk=8192):
    """Blockwise absmax scaling and nearest-level codes.

    [QLoRA glossary, "Come funziona QLoRA" (one absmax scale per block of 64)
    and the NF4 snippet (normalize by the block absmax, take the index of the
    nearest level, restore as level times absmax)]

    w32: float32 [nblocks, 64].  Returns (codes uint8 [nblocks, 64],
    absmax float32 [nblocks]).  x = fl32(w / absmax); code = first index i
    minimising fl32(|fl32(x - level_i)|).  A block whose absmax is 0 gets all
    codes equal to the zero level.
    """
    w32 = np.asarray(w32, dtype=np.float32)
    levels = np.asarray(levels, dtype=np.float32)
    nb = w32.shape[0]
    absmax = np.max(np.abs(w32), axis=1).astype(np.float32)
    codes = np.empty(w32.shape, dtype=np.uint8)
    zc = zero_code(levels)
    for s in range(0, nb, chunk):
        e = min(nb, s + chunk)
        a = absmax[s:e, None]
        safe = np.where(a == 0, np.float32(1), a).astype(np.float32)
        x = (w32[s:e] / safe).astype(np.float32)
        dist = np.abs(x[..., None] - levels[None, None, :])
        c = np.argmin(dist, axis=-1).astype(np.uint8)
        c[(a == 0)[:, 0]] = zc
        codes[s:e] = c
    return codes, absmax


def decode_blocks_f32(codes, absmax, levels):
    """Restore float32 weights as level[code] * absmax (the snippet's restore)."""
    levels = np.asarray(levels, dtype=np.float32)
    return (levels[codes] * np.asarray(absmax, np.float32)[:, None]).astype(np.float32)


def blockwise_mse(w32, levels):
    """Mean squared reconstruction error of one table on fp32 weight blocks,
    the quantity the NF4 snippet prints for "NF4" and "INT4".
    [QLoRA glossary, NF4 snippet]"""
    codes, absmax = encode_blocks(w32, levels)
    restored = decode_blocks_f32(codes, absmax, levels)
    err = restored.astype(np.float64) - np.asarray(w32, np.float64)
    return float(np.mean(err * err))


# ---------------------------------------------------------------- packing

def pack_codes(codes_nk):
    """[N, K] 4-bit codes -> [N, K/2] bytes; element 2j in the low nibble.
    [Módulo 4: QLoRA, 4.2 (4 bits = 0.5 byte per weight)]"""
    c = np.asarray(codes_nk, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# ---------------------------------------------------------------- second level

def double_quant(absmax):
    """Quantize the fp32 block scales to int8 in groups of 256.

    [QLoRA glossary, "Doppia quantizzazione" (per-block scales quantized to 8
    bits in blocks of 256); Módulo 4: QLoRA, 4.3 b) (the scale constants are
    quantized a second time, to 8 bits)]

    Per group of c consecutive scales (c = 256, the last group holds the rest):
    mean = fl32(S / c) with S the exactly rounded fp64 sum; d_i = fl32(s_i - mean);
    step = fl32(max|d_i| / 127); q_i = clamp(rint_half_even(fl32(d_i / step)),
    -127, 127), and q = 0 when step = 0.
    Returns (q int8 [nblk], step float32 [ngroups], mean float32 [ngroups]).
    """
    s = np.asarray(absmax, dtype=np.float32)
    nblk = s.shape[0]
    ng = (nblk + DQ_GROUP - 1) // DQ_GROUP
    q = np.zeros(nblk, dtype=np.int8)
    step = np.zeros(ng, dtype=np.float32)
    mean = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        grp = s[g * DQ_GROUP:(g + 1) * DQ_GROUP]
        c = grp.shape[0]
        total = math.fsum(float(v) for v in grp)
        m = np.float32(total / c)
        d = (grp - m).astype(np.float32)
        cmax = np.float32(np.max(np.abs(d)))
        st = np.float32(cmax / np.float32(DQ_QMAX))
        if st == 0:
            qi = np.zeros(c, dtype=np.float32)
        else:
            qi = np.rint((d / st).astype(np.float32))
            qi = np.clip(qi, -DQ_QMAX, DQ_QMAX)
        q[g * DQ_GROUP:g * DQ_GROUP + c] = qi.astype(np.int8)
        step[g] = st
        mean[g] = m
    return q, step, mean


def restore_scales(q, step, mean):
    """s_hat = fl32(fl32(q * step) + mean), two separately rounded fp32 steps."""
    q = np.asarray(q, dtype=np.int8)
    g = np.arange(q.shape[0]) // DQ_GROUP
    prod = (q.astype(np.float32) * np.asarray(step, np.float32)[g]).astype(np.float32)
    return (prod + np.asarray(mean, np.float32)[g]).astype(np.float32)


# ---------------------------------------------------------------- whole weight

def quantize(w_bits, n_out, k_in):
    """bf16 W [n_out, k_in] (uint16 bits) -> NF4 storage with double quantization.

    Returns a dict: codes (uint8 [n_out, k_in/2] packed), qscale (int8 [nblk]),
    step (float32 [ngroups]), mean (float32 [ngroups]) and the fp32 absmax
    [nblk] the first level produced (kept for checks; not part of storage).
    """
    assert k_in % BLOCK == 0
    w32 = bf16_bits_to_f32(np.asarray(w_bits).reshape(n_out, k_in))
    blocks = w32.reshape(-1, BLOCK)
    codes, absmax = encode_blocks(blocks, nf4_levels())
    q, step, mean = double_quant(absmax)
    return {
        "codes": pack_codes(codes.reshape(n_out, k_in)),
        "qscale": q,
        "step": step,
        "mean": mean,
        "absmax": absmax,
    }


def dequantize(codes_packed, qscale, step, mean, n_out, k_in):
    """NF4 storage -> bf16 W_hat bits [n_out, k_in].
    [QLoRA glossary, "Come funziona QLoRA" (dequantized to bfloat16 just
    before the matmul); NF4 snippet (restore = level[code] * scale)]"""
    codes = unpack_codes(np.asarray(codes_packed).reshape(n_out, k_in // 2))
    shat = restore_scales(qscale, step, mean)
    lv = nf4_levels()
    prod = (lv[codes.reshape(-1, BLOCK)] * shat[:, None]).astype(np.float32)
    return f32_to_bf16_bits(prod).reshape(n_out, k_in)


def storage_bits_per_param(n_out, k_in, with_mean=True):
    """Bits of scale storage per weight (codes excluded): int8 per block of 64
    plus fp32 step (and fp32 mean) per group of 256 blocks."""
    nblk = n_out * k_in // BLOCK
    ng = (nblk + DQ_GROUP - 1) // DQ_GROUP
    bits = nblk * 8 + ng * 32 * (2 if with_mean else 1)
    return bits / (n_out * k_in)
