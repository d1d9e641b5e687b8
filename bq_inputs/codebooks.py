"""Codebook tables passed by the caller to quantize / dequantize.

These are INPUTS of the method: the library takes the codebook as a
caller-passed float table, and none of the pages prints the table values.  The
tables below are built from the published definitions named on each function
and are used, as the same float32 array, by both the CUDA path and the oracle.
All three are sorted ascending, which the library requires of a codebook.
"""
import numpy as np


def nf4():
    """4-bit NormalFloat (Dettmers et al., "QLoRA", 2023, NormalFloat section).

    Levels are quantiles of N(0, 1) chosen so that each level carries equal
    probability mass, with an exact zero: 8 positive levels and 7 negative
    ones.  Each half is the normal quantile function evaluated on equally
    spaced probabilities from an outermost value p_max down to (but excluding)
    one half.  p_max is the mean of the outermost bin centres of a 15-bin and a
    16-bin equal-probability grid, 1 - (1/(2*15) + 1/(2*16)) / 2, which keeps
    the extreme levels finite.  The table is normalised so the largest
    magnitude is 1.
    """
    from scipy.stats import norm

    p_max = 1.0 - (1.0 / 30.0 + 1.0 / 32.0) / 2.0
    pos = norm.ppf(np.linspace(p_max, 0.5, 9)[:-1])        # 8 positive levels
    neg = -norm.ppf(np.linspace(p_max, 0.5, 8)[:-1])       # 7 negative levels
    levels = np.sort(np.concatenate([pos, [0.0], neg]))
    levels = levels / np.abs(levels).max()
    return levels.astype(np.float32)


def fp4():
    """4-bit float, E2M1 (OCP Microscaling formats v1.0, FP4 E2M1 element).

    Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit, i.e. sixteen
    entries including -0 and +0, divided by 6 so the largest is 1.  Sorted
    ascending, -0 (index 7) sits just before +0 (index 8).
    """
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]) / 6.0
    neg = -mags[::-1]                                       # -1 ... -0
    return np.concatenate([neg, mags]).astype(np.float32)


def dynamic8():
    """Signed dynamic tree quantization, 8 bits (Dettmers et al., "8-bit
    Optimizers via Block-wise Quantization", 2022, dynamic tree section).

    After the sign bit, a run of zero bits gives a decimal exponent e and the
    remaining bits a linear fraction in [0.1, 1].  With 7 bits after the sign,
    exponent e in 0..6 leaves 6 - e fraction bits, i.e. 2^(6-e) fraction
    values, taken as the centres of 2^(6-e) equal bins of [0.1, 1] and scaled
    by 10^-e.  That gives 127 magnitudes per sign; with 0 and 1.0 the table has
    256 entries.
    """
    vals = [0.0, 1.0]
    for e in range(7):
        k = 2 ** (6 - e)
        edges = np.linspace(0.1, 1.0, k + 1)
        centres = (edges[:-1] + edges[1:]) / 2.0
        vals.extend((10.0 ** -e) * centres)
        vals.extend(-(10.0 ** -e) * centres)
    table = np.sort(np.asarray(vals, np.float64)).astype(np.float32)
    assert table.size == 256
    return table


TABLES = {"nf4": nf4, "fp4": fp4, "dyn8": dynamic8}


def get(name):
    """Return the named table as a float32 numpy array."""
    return TABLES[name]()
