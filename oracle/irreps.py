"""Irreps strings, path enumeration and the ir_mul layout (oracle side).

Sobek: Streaming Equivariant Tensor Product Convolutions, section 2:
eq. 3 (a feature field is a direct sum of blocks x_{l,sigma} with C channels and
2l+1 components), eq. 4 (flattened width C_x = sum C(2l+1)), eq. 5 (selection rule
|l_in - l_sh| <= l_out <= l_in + l_sh and sigma_out = sigma_in * sigma_sh), eqs. 9-10
(n_pi = C_in * C_out weights per uvw path, N_w = sum n_pi), eq. 7 (uvu ties the
output multiplicity to the input one, n_pi = C_in).

Layout (section 4, "ir_mul"): a node row is the concatenation of its irrep blocks; a
block with C channels of order l occupies (2l+1)*C consecutive floats stored as
[2l+1][C] (channels contiguous).  Component index k = 0..2l corresponds to the real
SH order m = k - l.

Path order (the weight layout depends on it): for each input block, for each SH order
l_sh = 0..lmax, for each output block, in that nesting, every combination that
satisfies eq. 5 is a path.  Its weights occupy one contiguous slice of a weight row:
[C_in][C_out] for uvw (index u*C_out + w), [C_in] for uvu.
"""

import re
from dataclasses import dataclass

_TOKEN = re.compile(r"^\s*(?:(\d+)\s*x\s*)?(\d+)\s*([eo])\s*$")


@dataclass(frozen=True)
class Block:
    mul: int
    l: int
    parity: int  # +1 even ("e"), -1 odd ("o")
    offset: int  # first float of the block inside a node row

    @property
    def dim(self):
        return 2 * self.l + 1

    @property
    def size(self):
        return self.mul * self.dim


def parse(s):
    """Parse "64x0e+64x1o" into a list of Blocks with ir_mul offsets."""
    blocks = []
    off = 0
    if not s or not s.strip():
        raise ValueError("empty irreps string")
    for tok in s.split("+"):
        m = _TOKEN.match(tok)
        if not m:
            raise ValueError(f"bad irreps token {tok!r}")
        mul = int(m.group(1)) if m.group(1) else 1
        l = int(m.group(2))
        p = 1 if m.group(3) == "e" else -1
        if mul <= 0:
            raise ValueError("multiplicity must be positive")
        b = Block(mul, l, p, off)
        blocks.append(b)
        off += b.size
    return blocks


def width(blocks):
    """Flattened feature dimension, eq. 4."""
    return sum(b.size for b in blocks)


def sh_blocks(lmax):
    """The angular input Y: one copy of every order 0..lmax, parity (-1)^l."""
    out = []
    off = 0
    for l in range(lmax + 1):
        b = Block(1, l, 1 if l % 2 == 0 else -1, off)
        out.append(b)
        off += b.size
    return out


@dataclass(frozen=True)
class Path:
    index: int
    block_in: int
    l_sh: int
    block_out: int
    l_in: int
    l_out: int
    c_in: int
    c_out: int
    w_offset: int  # first weight column of this path
    w_count: int   # n_pi (eq. 9), or C_in for uvu (eq. 7)


def selection_rule(l_in, p_in, l_sh, p_sh, l_out, p_out):
    """Eq. 5: the CG selection rule with parity."""
    return abs(l_in - l_sh) <= l_out <= l_in + l_sh and p_out == p_in * p_sh


def paths(blocks_in, lmax, blocks_out, mode):
    """Enumerate the valid paths in the fixed order described in the module doc."""
    if mode not in ("uvw", "uvu"):
        raise ValueError("mode must be 'uvw' or 'uvu'")
    out = []
    off = 0
    for bi, a in enumerate(blocks_in):
        for l_sh in range(lmax + 1):
            p_sh = 1 if l_sh % 2 == 0 else -1
            for bo, c in enumerate(blocks_out):
                if not selection_rule(a.l, a.parity, l_sh, p_sh, c.l, c.parity):
                    continue
                if mode == "uvu":
                    if c.mul != a.mul:
                        raise ValueError("uvu path needs C_out == C_in (eq. 7)")
                    n = a.mul
                else:
                    n = a.mul * c.mul
                out.append(Path(len(out), bi, l_sh, bo, a.l, c.l, a.mul, c.mul, off, n))
                off += n
    return out


def num_weights(path_list):
    """N_w, eq. 10."""
    return sum(p.w_count for p in path_list)
