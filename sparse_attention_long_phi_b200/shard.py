"""Sharding one sequence's work by GQA group across ranks (host side).

The selection is per group (page 2, 重要性分数计算: the importance scores are
summed over the heads of a group and every head of the group attends the same
blocks) and the three branches read only their group's keys and values, so the
operator splits by group with no exchange: a rank takes a contiguous range of
groups, runs the operator on the matching heads, and the outputs concatenate
along the head axis.  This module only slices and reassembles tensors; the
operator itself runs unchanged on each slice.
"""
from __future__ import annotations


def group_range(G: int, rank: int, world: int) -> tuple[int, int]:
    """The contiguous groups [g0, g1) of `rank` among `world` ranks (sizes differ by at most one)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if world > G:
        raise ValueError(f"{world} ranks for {G} groups: every rank needs a group")
    base, extra = divmod(G, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def slice_groups(c: dict, x: dict, g0: int, g1: int) -> tuple[dict, dict]:
    """Config and inputs of groups [g0, g1): q/gates/dout by their heads, k/v by group.
    Tensors are torch tensors or numpy arrays laid out [B,T,H,*] / [B,T,G,*]; the
    slices are made contiguous.  The linear phi's parameters are shared by all groups."""
    Hg = c["H"] // c["G"]
    cs = dict(c, H=Hg * (g1 - g0), G=g1 - g0)
    heads = slice(g0 * Hg, g1 * Hg)

    def contig(t):
        return t.contiguous() if hasattr(t, "contiguous") else t.copy()

    xs = {}
    for key, t in x.items():
        if key in ("q", "gates", "dout"):
            xs[key] = contig(t[:, :, heads])
        elif key in ("k", "v"):
            xs[key] = contig(t[:, :, g0:g1])
        else:
            xs[key] = t
    return cs, xs
