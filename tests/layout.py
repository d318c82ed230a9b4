"""Test helpers: read the CUDA path's workspace regions back into logical arrays.

The tile layouts are the documented ones of include/da2.h (tensor-core K-major core-matrix
tiles and 512-byte scale-factor atoms); this is index arithmetic only, no method math.
"""
from __future__ import annotations

import numpy as np


def kmajor_index(rows: int, rowbytes: int) -> np.ndarray:
    r = np.arange(rows)[:, None]
    b = np.arange(rowbytes)[None, :]
    return (r // 8) * (rowbytes * 8) + (b // 16) * 128 + (r % 8) * 16 + (b % 16)


def untile_kmajor(flat: np.ndarray, nblk: int, rows: int, rowbytes: int) -> np.ndarray:
    """[nblk * rows * rowbytes] bytes -> [nblk, rows, rowbytes] logical bytes."""
    t = flat.reshape(nblk, rows * rowbytes)
    return t[:, kmajor_index(rows, rowbytes)]


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] 4-bit codes, element 2i in the low nibble of byte i."""
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


def sf_index(natoms: int, rows: int = 128) -> np.ndarray:
    r = np.arange(rows)[:, None]
    k = np.arange(natoms * 4)[None, :]
    return (k // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + (k % 4)


def untile_sf(flat: np.ndarray, nblk: int, natoms: int) -> np.ndarray:
    """[nblk * natoms * 512] -> [nblk, 128, natoms*4] (row, group) scale bytes."""
    t = flat.reshape(nblk, natoms * 512)
    return t[:, sf_index(natoms)]


class WsReader:
    """Reads regions of a workspace (torch uint8 tensor on the GPU) for heads bh0..bh1."""

    def __init__(self, ws, views: dict, d: int):
        self.ws, self.v, self.d = ws, views, d

    def _bytes(self, region: str, bh0: int, bh1: int, per_bh: int) -> np.ndarray:
        off = self.v[region]
        return self.ws[off + bh0 * per_bh: off + bh1 * per_bh].cpu().numpy()

    def f32(self, region, bh0, bh1, per_bh_elems):
        return self._bytes(region, bh0, bh1, per_bh_elems * 4).view(np.float32)

    def qk8(self, which, bh0, bh1):
        v, d = self.v, self.d
        raw = self._bytes(which + "8", bh0, bh1, v["N"] * v["tile8_qk"])
        return untile_kmajor(raw, (bh1 - bh0) * v["N"], v["bs"], d).reshape(
            bh1 - bh0, v["N"], v["bs"], d)

    def qk4(self, which, bh0, bh1):
        v, d = self.v, self.d
        raw = self._bytes(which + "4", bh0, bh1, v["N"] * v["tile4_qk"])
        t = untile_kmajor(raw, (bh1 - bh0) * v["N"], v["bs"], d // 2)
        codes = unpack_nibbles(t).reshape(bh1 - bh0, v["N"], v["bs"], d)
        sfraw = self._bytes("sf" + which + "4", bh0, bh1, v["N"] * v["sf_qk"])
        sf = untile_sf(sfraw, (bh1 - bh0) * v["N"], d // 64).reshape(bh1 - bh0, v["N"], 128, d // 16)
        return codes, sf

    def v8(self, bh0, bh1):
        v, d = self.v, self.d
        raw = self._bytes("v8", bh0, bh1, v["N"] * v["tile8_v"])
        t = untile_kmajor(raw, (bh1 - bh0) * v["N"], d, v["bs"])   # [.., d, bs]
        return np.swapaxes(t.reshape(bh1 - bh0, v["N"], d, v["bs"]), 2, 3)

    def v4(self, bh0, bh1):
        v, d = self.v, self.d
        raw = self._bytes("v4", bh0, bh1, v["N"] * v["tile4_v"])
        t = untile_kmajor(raw, (bh1 - bh0) * v["N"], d, v["kv4"] // 2)
        codes = unpack_nibbles(t).reshape(bh1 - bh0, v["N"], d, v["kv4"])
        sfraw = self._bytes("sfv4", bh0, bh1, v["N"] * v["sf_v"])
        sf = untile_sf(sfraw, (bh1 - bh0) * v["N"], v["kv4"] // 64).reshape(
            bh1 - bh0, v["N"], 128, v["kv4"] // 16)
        return codes, sf            # codes [.., d, kv4] (channel, slot), sf [.., 128, kv4/16]

    def tags(self, bh0, bh1):
        N = self.v["N"]
        return self._bytes("tags", bh0, bh1, N * N).reshape(bh1 - bh0, N, N)

    def lists(self, bh0, bh1):
        v = self.v
        n4 = v.get("n4max", v["n4"])                # the FP4 list's length (adaptive budget)
        n8s, n4s = max(v["n8"], 1), max(n4, 1)
        l8 = self._bytes("list8", bh0, bh1, v["N"] * n8s * 2).view(np.int16).reshape(bh1 - bh0, v["N"], n8s)
        l4 = self._bytes("list4", bh0, bh1, v["N"] * n4s * 2).view(np.int16).reshape(bh1 - bh0, v["N"], n4s)
        return l8[..., : v["n8"]].astype(np.int64), l4[..., :n4].astype(np.int64)

    def listm(self, bh0, bh1):
        v = self.v
        nms = max(v["nm"], 1)
        lm = self._bytes("listm", bh0, bh1, v["N"] * nms * 2).view(np.int16).reshape(bh1 - bh0, v["N"], nms)
        return lm[..., : v["nm"]].astype(np.int64)

    def scores(self, bh0, bh1):
        N = self.v["N"]
        return self.f32("scores", bh0, bh1, N * N).reshape(bh1 - bh0, N, N)
