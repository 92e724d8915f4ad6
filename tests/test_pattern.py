"""Layer-pattern diagnostics from an overlap matrix: the library's exact dynamic program against
a brute-force enumeration of every pattern, both pinned to closed forms."""

import numpy as np
import pytest

import oracle.pattern_oracle as P
from sparse_attention_token_04_b200 import binding as B


def _block_matrix(sizes, inside=0.9, across=0.2):
    n = sum(sizes)
    o = np.full((n, n), across)
    start = 0
    for s in sizes:
        o[start:start + s, start:start + s] = inside
        start += s
    np.fill_diagonal(o, 1.0)
    return o


def test_brute_force_pins():
    # all-ones overlap: every pattern keeps every layer's selection
    ones = np.ones((7, 7))
    v, pats = P.best_pattern(ones, 3)
    assert v == 7.0 and len(pats) == 15  # C(6, 2) patterns, all optimal
    # every layer Full keeps 1 per layer
    r = np.random.default_rng(0).random((6, 6))
    assert P.best_pattern(r, 6) == (6.0, ["FFFFFF"])
    # blocks of layers agreeing internally: one Full layer at the start of every block
    o = _block_matrix([3, 2, 4])
    v, pats = P.best_pattern(o, 3)
    assert pats == ["FSSFSFSSS"] and v == pytest.approx(3 + 6 * 0.9)
    assert P.blocks(o, 0.5) == [0, 0, 0, 1, 1, 2, 2, 2, 2]


@pytest.mark.parametrize("n,seed", [(5, 1), (9, 2), (12, 3)])
def test_dp_matches_brute_force(n, seed):
    rng = np.random.default_rng(seed)
    o = rng.random((n, n))
    o = (o + o.T) / 2
    np.fill_diagonal(o, 1.0)
    for n_full in range(1, n + 1):
        best, pats = P.best_pattern(o, n_full)
        pat, kept = B.dsa_pattern_from_overlap(o, n_full)
        assert pat.count("F") == n_full and pat[0] == "F"
        assert kept * n == pytest.approx(best, abs=1e-9)
        assert P.kept_overlap(o, pat) == pytest.approx(best, abs=1e-9)


def test_blocks_and_pattern_on_block_structure():
    o = _block_matrix([3, 3, 12, 6, 2])
    nb, blk = B.dsa_overlap_blocks(o, 0.5)
    assert nb == 5 and blk == P.blocks(o, 0.5)
    pat, kept = B.dsa_pattern_from_overlap(o, 5)
    assert pat == "FSSFSSFSSSSSSSSSSSFSSSSSFS"
    uniform = ("F" + "S" * 4) * 5 + "S"  # the same number of Full layers, evenly spaced
    assert len(uniform) == len(o) and uniform.count("F") == 5
    assert kept * len(o) > P.kept_overlap(o, uniform) + 1.0  # the block starts keep far more


def test_pattern_rejects_bad_arguments():
    with pytest.raises(B.DsaError):
        B.dsa_pattern_from_overlap(np.eye(4), 0)
    with pytest.raises(B.DsaError):
        B.dsa_pattern_from_overlap(np.eye(4), 5)
