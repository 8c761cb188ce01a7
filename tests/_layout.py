"""Pure index permutations between the CUDA library's 4-bit tensor layout and the oracle's
plain layouts (no arithmetic).  Library layout (see include/hifa4.h):
  rows (Q, K)  scales [B, H, N/128, d/64, 512], byte (r%32)*16 + (r//32)*4 + s
  V^T          scales [B, H, N/64, ceil(d/128), 512], same atom with r = channel % 128
"""
import numpy as np


def rows_scales_to_plain(atoms, B, H, N, d):
    a = np.asarray(atoms, np.uint8).reshape(B, H, N // 128, d // 64, 32, 4, 4)      # r0, r1, s
    a = a.transpose(0, 1, 2, 5, 4, 3, 6)                                            # B H nt r1 r0 kc s
    return np.ascontiguousarray(a).reshape(B, H, N, d // 16)


def rows_scales_from_plain(plain, B, H, N, d):
    p = np.asarray(plain, np.uint8).reshape(B, H, N // 128, 4, 32, d // 64, 4)       # nt r1 r0 kc s
    p = p.transpose(0, 1, 2, 5, 4, 3, 6)                                            # B H nt kc r0 r1 s
    return np.ascontiguousarray(p).reshape(-1)


def vt_scales_to_plain(atoms, B, H, N, d):
    nav = (d + 127) // 128
    a = np.asarray(atoms, np.uint8).reshape(B, H, N // 64, nav, 32, 4, 4)           # nc a r0 r1 s
    a = a.transpose(0, 1, 3, 5, 4, 2, 6)                                            # B H a r1 r0 nc s
    return np.ascontiguousarray(a).reshape(B, H, nav * 128, N // 16)[:, :, :d]


def vt_scales_from_plain(plain, B, H, N, d):
    nav = (d + 127) // 128
    full = np.zeros((B, H, nav * 128, N // 16), np.uint8)
    full[:, :, :d] = plain
    p = full.reshape(B, H, nav, 4, 32, N // 64, 4)                                  # a r1 r0 nc s
    p = p.transpose(0, 1, 5, 2, 4, 3, 6)                                            # B H nc a r0 r1 s
    return np.ascontiguousarray(p).reshape(-1)
