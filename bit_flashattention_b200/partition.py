"""Head-group partition of one attention call across ranks (one process per GPU).

In the HiFA4-style forward every (batch b, kv head g) group -- kv head g with its
G = Hq / Hkv query heads -- is independent of every other: its quantisation (Smooth-QK
scales are per kv head and channel), its tile loop and its outputs touch no other
group.  So a call over B * Hkv groups splits across ranks without any exchange: rank r of
W takes a contiguous range of the groups in (b, g) order, quantises and attends only those
heads and writes its slice of O, m and l.  No collective is on the data path; gathering
the slices is needed only by a consumer that wants the whole O on one rank.
"""


def group_range(B: int, Hkv: int, world: int, rank: int):
    """[u0, u1) of the groups u = b * Hkv + g that `rank` of `world` takes: contiguous,
    in order, sizes differing by at most one (the first B*Hkv % world ranks take one more)."""
    if not (0 <= rank < world) or B <= 0 or Hkv <= 0:
        raise ValueError("bad partition arguments")
    n = B * Hkv
    base, extra = divmod(n, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def group_slices(u0: int, u1: int, Hkv: int):
    """The range [u0, u1) as per-batch head slices (b, g0, g1): kv heads g0..g1-1 of batch
    b, i.e. query heads g0*G .. g1*G-1."""
    out = []
    u = u0
    while u < u1:
        b, g0 = divmod(u, Hkv)
        g1 = min(Hkv, g0 + (u1 - u))
        out.append((b, g0, g1))
        u += g1 - g0
    return out


def call_blocks(slices, Hkv: int):
    """Merge per-batch slices into as few attention calls as possible: runs of whole
    batches become one block (b0, b1, 0, Hkv); a partial batch stays (b, b + 1, g0, g1)."""
    out = []
    for b, g0, g1 in slices:
        whole = g0 == 0 and g1 == Hkv
        if whole and out and out[-1][2] == 0 and out[-1][3] == Hkv and out[-1][1] == b:
            out[-1] = (out[-1][0], b + 1, 0, Hkv)
        else:
            out.append((b, b + 1, g0, g1))
    return out
