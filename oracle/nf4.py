"""Block-wise 4-bit quantisation with double-quantised scales (oracle).

Test infrastructure only; see the package docstring.

The pages state the encoding in this order ("QLoRA技术从入门到精通",
section 3(1) 基座模型初始化量化):

1. split the weight tensor into blocks of 64 (or 256) values;
2. per block, scale = absmax of the block;
3. divide the block by its scale, which maps it into [-1, 1];
4. map each value to the nearest of the 16 levels of the NF4 table and store
   the index 0..15;
5. double quantisation: gather the fp32 block scales and quantise them again
   to 8 bits;
6. keep only the 4-bit indices and the 8-bit scale metadata.

Dequantisation is grid[idx] * scale (same page, section 3(2) 前向传播).
"LoRA 与 QLoRA：用一块 GPU 微调大模型" (section "量化", parts "分块缩放",
"NF4", "存储和计算") gives the same steps, the block of 64, the exact zero in
the NF4 levels and the 4.13 bits per weight after double quantisation.
"QLoRA 量化微调" section 7.1 works one value through the same pipeline with
the 16-level uniform grid.

Readings where the pages are silent (each listed in the design notes):

* NF4 levels: the pages say "split N(0,1) into equal-probability intervals
  and take each interval's median", dense near 0, sparse in the tails, with an
  exact 0.  Sixteen intervals over the whole line would give no zero, so the
  table is built per half: 8 equal-probability intervals of [0, inf) and 7 of
  (-inf, 0], the median of each, each half divided by its own extreme so the
  end levels are exactly -1 and +1, plus the exact 0.
* Nearest level: exact nearest in real arithmetic; a value exactly halfway
  between two levels takes the lower index.
* A block whose scale is 0 maps every value to x = 0.
* Index packing: element 2j in the low nibble of byte j, element 2j+1 in the
  high nibble.
* Double quantisation: symmetric int8 codes in [-127, 127] of the block
  scales centred on their global mean, one fp32 factor absmax/127 per group
  of 256 consecutive scales, round half to even.  The mean is taken on a
  fixed-point grid so that it does not depend on summation order (see
  ``fixed_point_mean``).
"""

import math

import numpy as np

from .bf16 import round_to_bf16

F32 = np.float32
F64 = np.float64


# ---------------------------------------------------------------- tables --

def _std_normal_cdf(z):
    """Phi(z) in fp64 from the complementary error function."""
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def _std_normal_quantile(p):
    """Phi^{-1}(p) in fp64 by bisection on Phi (no approximation formula)."""
    lo, hi = -12.0, 12.0
    for _ in range(400):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if _std_normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def nf4_raw_quantiles():
    """Medians of the equal-probability intervals, before normalisation.

    Returns (negative, positive): 7 values for (-inf, 0] (mass 1/14 each,
    median at p = 1/2 - (j - 1/2)/14) and 8 values for [0, inf) (mass 1/16
    each, median at p = 1/2 + (j - 1/2)/16), j = 1, 2, ..., in fp64.
    """
    neg = [_std_normal_quantile(0.5 - (j - 0.5) / 14.0) for j in range(1, 8)]
    pos = [_std_normal_quantile(0.5 + (j - 0.5) / 16.0) for j in range(1, 9)]
    return np.array(neg, dtype=F64), np.array(pos, dtype=F64)


def nf4_levels():
    """The 16 NF4 levels, ascending, as fp32.

    Each half is divided by its own extreme (normalisation to [-1, 1],
    "QLoRA技术从入门到精通" section 3(1) step 归一化), the exact 0 is added,
    and every value is rounded once from fp64 to fp32.
    """
    neg, pos = nf4_raw_quantiles()
    neg = neg / (-neg[-1])
    pos = pos / pos[-1]
    levels = np.concatenate([neg[::-1], [0.0], pos])
    return levels.astype(F32)


def uniform_levels():
    """The 16-level uniform grid of "QLoRA 量化微调" section 7.1:
    level k = -1 + k * 2/15, computed in fp64 and rounded to fp32."""
    return np.array([-1.0 + k * 2.0 / 15.0 for k in range(16)], dtype=F64).astype(F32)


# ------------------------------------------------------------ quantiser --

def nearest_level(x, levels):
    """Index of the nearest level to each fp32 value x; ties -> lower index.

    For ascending levels q_0 < ... < q_15 the nearest level to x is q_j with
    j = #{k : x > (q_k + q_{k+1}) / 2}.  The midpoints are exact in fp64 (the
    sum of two fp32 values is exact in fp64 and halving is exact), and the
    comparison of an fp32 x with them is exact, so the decision is the exact
    nearest-level decision.  A value equal to a midpoint is not counted,
    which gives the lower index.
    """
    x64 = np.asarray(x, dtype=F32).astype(F64)
    q = np.asarray(levels, dtype=F32).astype(F64)
    assert q.shape == (16,) and np.all(np.diff(q) > 0)
    idx = np.zeros(x64.shape, dtype=np.uint8)
    for k in range(15):
        mid = (q[k] + q[k + 1]) * 0.5
        idx += (x64 > mid).astype(np.uint8)
    return idx


def block_absmax(w, blocksize):
    """scale_b = max |w| over block b of the flattened tensor (fp32, exact).

    Block b covers flattened elements [b*blocksize, (b+1)*blocksize); the
    last block may be partial.
    """
    w = np.asarray(w, dtype=F32).ravel()
    n = w.size
    nb = -(-n // blocksize)
    padded = np.zeros(nb * blocksize, dtype=F32)
    padded[:n] = np.abs(w)
    return padded.reshape(nb, blocksize).max(axis=1)


def pack_nibbles(idx):
    """byte j = idx[2j] | idx[2j+1] << 4 (an odd tail gets a zero high nibble)."""
    idx = np.asarray(idx, dtype=np.uint8).ravel()
    if idx.size % 2:
        idx = np.concatenate([idx, np.zeros(1, dtype=np.uint8)])
    return (idx[0::2] | (idx[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(codes, n):
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    out = np.empty(codes.size * 2, dtype=np.uint8)
    out[0::2] = codes & 0x0F
    out[1::2] = codes >> 4
    return out[:n]


# --------------------------------------------------- double quantisation --

MEAN_FRAC_BITS = 32


def fixed_point_mean(scales):
    """Mean of the block scales, independent of summation order.

    E is the binary exponent of the largest scale (max = m * 2**E with
    m in [0.5, 1)).  Each scale is truncated to the grid 2**(E - 32):
    t_b = floor(s_b * 2**(32 - E)), an integer below 2**32.  The integers are
    summed exactly, S = sum t_b, and mu = fp32( fp64(S) * 2**(E - 32) / nb )
    with each fp64 operation rounded to nearest.  All scales zero -> mu = 0.
    """
    s = np.asarray(scales, dtype=F32).ravel()
    nb = s.size
    smax = float(s.max()) if nb else 0.0
    if smax == 0.0:
        return F32(0.0)
    e = math.frexp(smax)[1]
    t = np.floor(s.astype(F64) * (2.0 ** (MEAN_FRAC_BITS - e))).astype(np.int64)
    total = sum(int(v) for v in t) if nb < 4096 else int(t.sum(dtype=np.int64))
    mu = (float(total) * (2.0 ** (e - MEAN_FRAC_BITS))) / float(nb)
    return F32(mu)


def double_quantize(scales, dq_blocksize=256):
    """Second-level quantisation of the fp32 block scales to int8.

    mu    = fixed_point_mean(scales)
    c_b   = fp32(s_b - mu)
    a_g   = max |c_b| over group g (dq_blocksize consecutive scales; the last
            group may be partial)
    f_g   = fp32(a_g / 127)
    q_b   = clamp(rint_half_even(fp32(c_b / f_g)), -127, 127), or 0 if f_g = 0
    """
    s = np.asarray(scales, dtype=F32).ravel()
    nb = s.size
    ng = -(-nb // dq_blocksize)
    mu = fixed_point_mean(s)
    c = (s - mu).astype(F32)
    padded = np.zeros(ng * dq_blocksize, dtype=F32)
    padded[:nb] = np.abs(c)
    a = padded.reshape(ng, dq_blocksize).max(axis=1)
    f = (a / F32(127.0)).astype(F32)
    f_el = np.repeat(f, dq_blocksize)[:nb]
    ratio = np.zeros(nb, dtype=F32)
    np.divide(c, f_el, out=ratio, where=f_el > 0)
    q = np.where(f_el > 0, np.clip(np.rint(ratio), -127, 127), 0).astype(np.int8)
    return q, f, mu


def dequantize_scales(scale_codes, factors, mean, dq_blocksize=256):
    """s_hat_b = fp32( fp32(q_b * f_g) + mu ): multiply, round, add, round."""
    q = np.asarray(scale_codes, dtype=np.int8).ravel()
    f_el = np.repeat(np.asarray(factors, dtype=F32), dq_blocksize)[:q.size]
    prod = (q.astype(F32) * f_el).astype(F32)
    return (prod + F32(mean)).astype(F32)


# ------------------------------------------------------------ pipeline --

def quantize(w, blocksize=64, dq_blocksize=256, levels=None):
    """Quantise a weight tensor (any shape, flattened row-major).

    Returns a dict with the packed ``codes`` (uint8), the fp32 block
    ``absmax``, the 4-bit ``idx`` (uint8, one per element) and either the
    double-quantised scales (``scale_codes`` int8, ``factors`` fp32 per
    group, ``mean`` fp32) or, with dq_blocksize = 0, ``factors`` = absmax.
    """
    if levels is None:
        levels = nf4_levels()
    w = np.asarray(w, dtype=F32).ravel()
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    n = w.size
    s = block_absmax(w, blocksize)
    s_el = np.repeat(s, blocksize)[:n]
    x = np.zeros(n, dtype=F32)
    np.divide(w, s_el, out=x, where=s_el > 0)
    idx = nearest_level(x, levels)
    out = dict(n=n, blocksize=blocksize, dq_blocksize=dq_blocksize,
               levels=np.asarray(levels, dtype=F32), idx=idx,
               codes=pack_nibbles(idx), absmax=s)
    if dq_blocksize:
        q, f, mu = double_quantize(s, dq_blocksize)
        out.update(scale_codes=q, factors=f, mean=mu)
    else:
        out.update(scale_codes=None, factors=s.copy(), mean=None)
    return out


def block_scales(qt):
    """The scale each block is dequantised with (s_hat, or absmax without DQ)."""
    if qt["dq_blocksize"]:
        return dequantize_scales(qt["scale_codes"], qt["factors"], qt["mean"],
                                 qt["dq_blocksize"])
    return np.asarray(qt["factors"], dtype=F32)


def dequantize(qt):
    """w_hat = fp32(level[idx] * s_hat_b) for every element (flattened)."""
    n = qt["n"]
    idx = unpack_nibbles(qt["codes"], n)
    sh = np.repeat(block_scales(qt), qt["blocksize"])[:n]
    return (qt["levels"][idx] * sh).astype(F32)


def compute_weight(qt):
    """The weight the products use: the dequantised weight rounded to bf16.

    The pages restore the 4-bit weights to bf16 (or fp16) right before the
    matrix product and drop them afterwards ("QLoRA技术从入门到精通", 3(2)
    前向传播, 按需解压; "LoRA 与 QLoRA：用一块 GPU 微调大模型", 量化 part
    "存储和计算"), with bf16 as the compute dtype ("LoRA 与 QLoRA：把大模型微调
    拆成可负担的工程", 8).  Flattened, like ``dequantize``.
    """
    return round_to_bf16(dequantize(qt))


def storage_bits(n, blocksize=64, dq_blocksize=256):
    """Bytes of each stored array and the bits per weight they add up to."""
    nb = -(-n // blocksize)
    sizes = {"codes": -(-n // 2)}
    if dq_blocksize:
        ng = -(-nb // dq_blocksize)
        sizes.update(scale_codes=nb, factors=4 * ng, mean=4)
    else:
        sizes.update(scale_codes=0, factors=4 * nb, mean=0)
    total = sum(sizes.values())
    sizes["bits_per_weight"] = 8.0 * total / n
    return sizes
