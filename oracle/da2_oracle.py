"""CPU oracle of the DraftAttention2 hot path -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s cpu_baseline / reference leg
use this module. It shares no code with the CUDA library.

Sources (cited by page title and section):
  [DA2]  "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
         Attention" (arXiv 2609.32628), Abstract.
  [DA1]  "DraftAttention: Fast Video Diffusion via Low-Resolution Attention Guidance"
         (arXiv 2505.14708), Abstract.
  [NEWS] News article on DraftAttention (szmaozhuayin.com), method overview steps 1-4 and
         the theoretical-analysis paragraph.
  [MX]   OCP Microscaling Formats (MX) Specification v1.0, a public standard outside the
         pages: the MXFP8 element (E4M3) and shared-scale (E8M0, 32 elements) formats used
         by the block-scaled FP8 variant, which only this oracle implements.

Only this oracle implements the bf16 top tier either: a class above FP8 whose blocks run
both products on the bf16 input values with P rounded to bf16 (`bf16_round`).

The pages print no equations; where a step is left open the plainest reading is taken
and listed in the repository's design notes. Every step below is a separate function
returning its own arrays so that each can be compared with the CUDA path on its own.

Numerics. Floating point is fp64 except where a step is defined in fp32 so that the
CUDA path can reproduce it bit for bit: the pooled averages (an fp32 running sum in slot
order, then an IEEE fp32 divide), the operand scales and the operand quantisers (IEEE
fp32 multiplies/divides, then round-to-nearest-even onto the E4M3 / E2M1 grids).

Parity pins: every function is pinned by `tests/test_oracle_*.py` against closed forms,
library routines or brute force. The error-decomposition formula is a reading (the pages
print none); its terms are pinned by torch and by closed forms, see `error_decomposition`.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

F32 = np.float32
E4M3_MAX = 448.0        # largest finite E4M3 value (OCP FP8, bias 7, no infinities)
E2M1_MAX = 6.0          # largest E2M1 value
TAG_SKIP, TAG_FP4, TAG_FP8, TAG_MIX, TAG_BF16 = 0, 1, 2, 3, 4


# ----------------------------------------------------------------------------------------
# Geometry: windows, blocks, budgets
# ----------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Geometry:
    B: int
    H: int
    d: int
    F: int
    Hf: int
    Wf: int
    ph: int
    pw: int
    ny: int
    nx: int
    N: int        # blocks (windows) per (b, h)
    bs: int       # tokens per block, ph * pw
    T: int        # valid tokens
    Tp: int       # padded tokens N * bs
    n8: int       # FP8 blocks per query block
    n4: int       # FP4 blocks per query block
    sm_scale: float
    nm: int = 0   # mixed blocks per query block (E4M3 scores, E2M1 P V)
    n4max: int = 0  # FP4 list length with the adaptive budget (n4 when it is off)
    tau: float = 0.0  # adaptive budget threshold on the draft score (0: off)
    n16: int = 0  # bf16 blocks per query block (the tier above FP8; oracle only)


def budget_counts(N: int, pct_fp8: int, pct_fp4: int) -> tuple[int, int]:
    """Blocks kept at FP8 and FP4 per query block: integer percent, rounded half up.

    [DA2] Abstract: the ranking runs under configurable budgets. Reading: the budgets are
    percentages of the N KV blocks; n8 = floor((p8 N + 50)/100), nk = floor(((p8+p4) N
    + 50)/100), n4 = nk - n8.
    """
    n8 = (pct_fp8 * N + 50) // 100
    nk = ((pct_fp8 + pct_fp4) * N + 50) // 100
    return n8, nk - n8


def budget_counts3(N: int, pct_fp8: int, pct_mix: int, pct_fp4: int) -> tuple[int, int, int]:
    """Blocks kept at FP8, mixed and FP4 per query block: the three classes take the
    ranking's top blocks in that order, each cumulative cut rounded half up as in
    `budget_counts` (with pct_mix = 0 the FP8 and FP4 counts are those of `budget_counts`).

    [DA2] Abstract: the shared ranking gives higher precision to the more important
    blocks and lower precision to the rest under configurable budgets; the mixed class
    (8-bit scores, 4-bit probabilities and values) is a precision between the two.
    """
    c8 = (pct_fp8 * N + 50) // 100
    c8m = ((pct_fp8 + pct_mix) * N + 50) // 100
    ck = ((pct_fp8 + pct_mix + pct_fp4) * N + 50) // 100
    return c8, c8m - c8, ck - c8m


def budget_counts_tiers(N: int, pct_bf16: int, pct_fp8: int, pct_mix: int,
                       pct_fp4: int) -> tuple[int, int, int, int]:
    """Blocks kept at bf16, FP8, mixed and FP4 per query block: the four classes take the
    ranking's top blocks in that order, each cumulative cut rounded half up as in
    `budget_counts` (with pct_bf16 = 0 the last three are those of `budget_counts3`).

    [DA2] Abstract: higher precision for the more important blocks, lower precision for
    the rest. Reading: bf16 (the input precision) is the highest, so its class comes first.
    """
    c16 = (pct_bf16 * N + 50) // 100
    n8, nm, n4 = budget_counts3(N, pct_bf16 + pct_fp8, pct_mix, pct_fp4)
    return c16, n8 - c16, nm, n4


def geometry(w) -> Geometry:
    ny, nx = -(-w.Hf // w.ph), -(-w.Wf // w.pw)
    N = w.F * ny * nx
    bs = w.ph * w.pw
    pm = getattr(w, "pct_mix", 0)
    p16 = getattr(w, "pct_bf16", 0)
    n16, n8, nm, n4 = budget_counts_tiers(N, p16, w.pct_fp8, pm, w.pct_fp4)
    tau = float(np.float32(getattr(w, "adapt_tau", 0.0)))      # a configuration value in fp32
    n4max = budget_counts_tiers(N, p16, w.pct_fp8, pm, w.pct_fp4_max)[3] if tau > 0 else n4
    sm = getattr(w, "sm_scale", 0.0) or 1.0 / math.sqrt(w.d)
    return Geometry(w.B, w.H, w.d, w.F, w.Hf, w.Wf, w.ph, w.pw, ny, nx, N, bs,
                    w.F * w.Hf * w.Wf, N * bs, n8, n4, sm, nm, n4max, tau, n16)


def token_block_slot(g: Geometry):
    """Block n and slot s of every token t (frame-major t = f Hf Wf + y Wf + x).

    [DA1] Abstract and [NEWS] step 4: tokens are reordered so that each pooled region is
    one contiguous block. Block n = f ny nx + (y // ph) nx + (x // pw); slot
    s = (y % ph) pw + (x % pw).
    """
    t = np.arange(g.T)
    f, rem = np.divmod(t, g.Hf * g.Wf)
    y, x = np.divmod(rem, g.Wf)
    blk = f * g.ny * g.nx + (y // g.ph) * g.nx + (x // g.pw)
    slot = (y % g.ph) * g.pw + (x % g.pw)
    return blk, slot


def block_valid(g: Geometry) -> np.ndarray:
    """[N, bs] bool: slot holds a real token (edge windows are padded)."""
    blk, slot = token_block_slot(g)
    valid = np.zeros((g.N, g.bs), dtype=bool)
    valid[blk, slot] = True
    return valid


def block_counts(g: Geometry) -> np.ndarray:
    return block_valid(g).sum(axis=1)


def permute(x: np.ndarray, g: Geometry) -> np.ndarray:
    """[B, H, T, d] -> [B, H, N, bs, d]; padded slots hold zeros."""
    blk, slot = token_block_slot(g)
    out = np.zeros(x.shape[:2] + (g.N, g.bs) + x.shape[3:], dtype=x.dtype)
    out[:, :, blk, slot] = x
    return out


def inverse_permute(xp: np.ndarray, g: Geometry) -> np.ndarray:
    """[B, H, N, bs, d] -> [B, H, T, d]: restore the original token order ([DA1] Abstract)."""
    blk, slot = token_block_slot(g)
    return xp[:, :, blk, slot]


# ----------------------------------------------------------------------------------------
# Pooling ([DA2] Abstract: spatial 2D average- and max-pooled queries and keys;
#          [NEWS] step 1: per-frame spatial downsampling into draft Q/K)
# ----------------------------------------------------------------------------------------
def pool(xp: np.ndarray, valid: np.ndarray):
    """Average and max of each window over its valid tokens, per channel.

    avg: fp32 running sum over the valid slots in increasing slot order, then an IEEE
    fp32 divide by the number of valid tokens. max: exact. Both fp32 [B, H, N, d].
    """
    x = xp.astype(F32)
    B, H, N, bs, d = x.shape
    acc = np.zeros((B, H, N, d), dtype=F32)
    for s in range(bs):
        take = valid[:, s][None, None, :, None]
        acc = np.where(take, (acc + x[:, :, :, s, :]).astype(F32), acc)
    cnt = valid.sum(axis=1).astype(F32)
    avg = (acc / cnt[None, None, :, None]).astype(F32)
    xm = np.where(valid[None, None, :, :, None], x, F32(-np.inf))
    mx = xm.max(axis=3).astype(F32)
    return avg, mx


# ----------------------------------------------------------------------------------------
# Quantisers: E4M3 (OCP FP8, bias 7, max 448, no inf) and E2M1 (values 0, .5, 1, 1.5, 2,
# 3, 4, 6), round to nearest with ties to even, saturating to the largest finite value.
# ----------------------------------------------------------------------------------------
def e4m3_round(y) -> np.ndarray:
    """Nearest E4M3 value (fp64), ties to even mantissa, saturating at +-448."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, e = np.frexp(a)                                  # a = m 2^e, m in [0.5, 1)
    quantum = np.where(a >= 2.0 ** -6, np.ldexp(1.0, e - 4), 2.0 ** -9)
    r = np.minimum(np.rint(a / quantum) * quantum, E4M3_MAX)
    return np.copysign(r, y)


def e4m3_code(y) -> np.ndarray:
    """E4M3 byte of the nearest value: sign | exponent field (4 bits) | mantissa (3 bits)."""
    v = e4m3_round(y)
    a = np.abs(v)
    _, e = np.frexp(a)
    normal = a >= 2.0 ** -6
    ef = np.where(normal, e - 1 + 7, 0)
    man = np.where(normal, np.rint(np.ldexp(a, -(e - 1)) * 8 - 8), np.rint(a / 2.0 ** -9))
    code = (ef.astype(np.int64) << 3) | man.astype(np.int64)
    code = code | (np.signbit(v).astype(np.int64) << 7)
    return code.astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    man = c & 7
    mag = np.where(ef == 0, man * 2.0 ** -9, np.ldexp(1.0 + man / 8.0, ef - 7))
    return s * mag


_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_round(y) -> np.ndarray:
    """Nearest E2M1 value (fp64), ties to even mantissa, saturating at +-6."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    quantum = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    r = np.minimum(np.rint(a / quantum) * quantum, E2M1_MAX)
    return np.copysign(r, y)


def bf16_round(y) -> np.ndarray:
    """Nearest bfloat16 value (fp64), ties to even mantissa: 8 significant bits (1 implicit
    + 7 stored), normal exponents down to 2^-126 and subnormal steps of 2^-133 below; values
    that round past the largest finite bf16 (about 3.39e38) become infinite."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, e = np.frexp(a)                                  # a = m 2^e, m in [0.5, 1)
    quantum = np.where(a >= 2.0 ** -126, np.ldexp(1.0, e - 8), 2.0 ** -133)
    r = np.rint(a / quantum) * quantum
    r = np.where(r > (2.0 - 2.0 ** -7) * 2.0 ** 127, np.inf, r)
    return np.copysign(r, y)


def e2m1_code(y) -> np.ndarray:
    """4-bit E2M1 code (sign bit 3, then 2 exponent bits, 1 mantissa bit)."""
    v = e2m1_round(y)
    idx = np.searchsorted(_E2M1_GRID, np.abs(v))
    return (idx | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.int64)
    return np.where(c & 8, -1.0, 1.0) * _E2M1_GRID[c & 7]


# ----------------------------------------------------------------------------------------
# Operand quantisation ([DA2] Abstract: fused operand preparation producing the 8-bit and
# 4-bit copies used by the mixed-precision kernel). Formats: FP8 E4M3 with an fp32 outer
# scale; NVFP4-style E2M1 with one E4M3 scale per 16 consecutive elements along the
# contraction axis and the same fp32 outer scale.
# ----------------------------------------------------------------------------------------
def outer_scale(amax):
    """(s, inv) per group: s = amax/448 (dequantisation), inv = 448/amax (quantisation),
    both IEEE fp32; s = inv = 1 where amax == 0."""
    amax = np.asarray(amax, dtype=F32)
    safe = np.where(amax > 0, amax, F32(1))
    s = np.where(amax > 0, (safe / F32(E4M3_MAX)).astype(F32), F32(1)).astype(F32)
    inv = np.where(amax > 0, (F32(E4M3_MAX) / safe).astype(F32), F32(1)).astype(F32)
    return s, inv


def fp4_groups(y: np.ndarray):
    """y fp32 [..., K] (K % 16 == 0), already divided by its outer scale.

    Group scale sigma = E4M3(amax16 / 6) (IEEE fp32 divide, then RNE); codes =
    E2M1(y * (1/sigma)) with 1/sigma an IEEE fp32 reciprocal; a group whose sigma is 0
    is all zero codes. Returns (codes uint8 [..., K], sigma codes uint8 [..., K/16]).
    """
    y = y.astype(F32)
    sh = y.shape
    yg = y.reshape(sh[:-1] + (sh[-1] // 16, 16))
    amax16 = np.abs(yg).max(axis=-1).astype(F32)
    sig_code = e4m3_code((amax16 / F32(E2M1_MAX)).astype(F32))
    sig = e4m3_decode(sig_code).astype(F32)
    rcp = np.where(sig > 0, (F32(1) / np.where(sig > 0, sig, F32(1))).astype(F32), F32(0))
    z = (yg * rcp[..., None]).astype(F32)
    codes = np.where(sig[..., None] > 0, e2m1_code(z), np.uint8(0)).astype(np.uint8)
    return codes.reshape(sh), sig_code


def fp4_dequant(codes, sig_code) -> np.ndarray:
    """Values sigma * e2m1 (fp64), without the outer scale."""
    v = e2m1_decode(codes)
    sh = v.shape
    vg = v.reshape(sh[:-1] + (sh[-1] // 16, 16)) * e4m3_decode(sig_code)[..., None]
    return vg.reshape(sh)


def quantise_qk(xp: np.ndarray, valid: np.ndarray):
    """Q or K, per (b, h, block) outer scale from the block amax.

    xp: [B, H, N, bs, d] (padded slots zero). Returns dict with
      s    fp32 [B,H,N]       dequantisation scale amax/448
      q8   uint8 [B,H,N,bs,d] E4M3 codes of x * (448/amax)
      q4   uint8 [B,H,N,bs,d] E2M1 codes (one per element, unpacked)
      sf4  uint8 [B,H,N,bs,d/16] E4M3 group scales along d
    """
    x = xp.astype(F32)
    amax = np.abs(x).max(axis=(3, 4)).astype(F32)
    s, inv = outer_scale(amax)
    y = (x * inv[..., None, None]).astype(F32)
    q8 = e4m3_code(y)
    q4, sf4 = fp4_groups(y)
    return dict(s=s, q8=q8, q4=q4, sf4=sf4)


def v_channel_amax(v: np.ndarray) -> np.ndarray:
    """amax of V over all tokens, per (b, h, channel): fp32 [B, H, d]."""
    return np.abs(v.astype(F32)).max(axis=2).astype(F32)


def quantise_v(vp: np.ndarray, amax_c: np.ndarray):
    """V, per (b, h, channel) outer scale (it must factor out of the P V sum over tokens).

    Groups of 16 run along tokens (the P V contraction axis) within a block.
    Returns s fp32 [B,H,d], q8 uint8 [B,H,N,bs,d], q4 uint8 [B,H,N,bs,d],
    sf4 uint8 [B,H,N,d,bs/16] (group scales of channel c over slots 16g..16g+15).
    """
    x = vp.astype(F32)
    s, inv = outer_scale(amax_c)
    y = (x * inv[:, :, None, None, :]).astype(F32)
    q8 = e4m3_code(y)
    yt = np.swapaxes(y, 3, 4)                        # [B,H,N,d,bs]
    q4t, sf4 = fp4_groups(yt)
    return dict(s=s, q8=q8, q4=np.swapaxes(q4t, 3, 4).copy(), sf4=sf4)


def dequant_qk(qd, precision: int) -> np.ndarray:
    """fp64 [B,H,N,bs,d] values of a quantised Q or K copy (8 or 4 bits)."""
    s = qd["s"].astype(np.float64)[..., None, None]
    if precision == 8:
        return s * e4m3_decode(qd["q8"])
    return s * fp4_dequant(qd["q4"], qd["sf4"])


def dequant_v(vd, precision: int) -> np.ndarray:
    s = vd["s"].astype(np.float64)[:, :, None, None, :]
    if precision == 8:
        return s * e4m3_decode(vd["q8"])
    vt = fp4_dequant(np.swapaxes(vd["q4"], 3, 4), vd["sf4"])
    return s * np.swapaxes(vt, 3, 4)


# ----------------------------------------------------------------------------------------
# Block-scaled FP8, oracle only (no CUDA kernel takes this form): MXFP8 as the OCP
# Microscaling Formats (MX) Specification v1.0 defines it -- 32 consecutive elements along
# the contraction axis share one E8M0 scale 2^e (e in [-127, 127]) and each element is an
# E4M3 value of x / 2^e. [DA2] Abstract fixes 8-bit computation for the important blocks,
# not the scale granularity; this variant puts the scale per 32 elements instead of per
# block (Q, K) or per head channel (V), so no pre-pass over the head is needed for V.
# ----------------------------------------------------------------------------------------
MX_BLOCK = 32
E4M3_EMAX = 8           # exponent of E4M3's largest normal binade (448 = 1.75 * 2^8)


def e8m0_scale_exp(amax) -> np.ndarray:
    """Shared exponent of an MX block: floor(log2 amax) - 8, clamped to the E8M0 range
    [-127, 127]; a block whose amax is 0 takes -127 (its elements are then all 0)."""
    a = np.asarray(amax, dtype=np.float64)
    safe = np.where(a > 0, a, 1.0)
    _, fe = np.frexp(safe)                              # safe = m 2^fe, m in [0.5, 1)
    e = np.where(a > 0, fe - 1 - E4M3_EMAX, -127)
    return np.clip(e, -127, 127).astype(np.int64)


def quantise_mx8(x, axis: int = -1):
    """MXFP8 of x along `axis` (its length a multiple of 32).

    Returns (codes uint8, same shape as x: E4M3 bytes of x / 2^e, round to nearest even,
    saturating at +-448; exps int64, shape of x with `axis` divided by 32)."""
    x = np.moveaxis(np.asarray(x, dtype=np.float64), axis, -1)
    sh = x.shape
    xb = x.reshape(sh[:-1] + (sh[-1] // MX_BLOCK, MX_BLOCK))
    e = e8m0_scale_exp(np.abs(xb).max(axis=-1))
    codes = e4m3_code(np.ldexp(xb, -e[..., None])).reshape(sh)
    return np.moveaxis(codes, -1, axis), np.moveaxis(e, -1, axis)


def dequant_mx8(codes, exps, axis: int = -1) -> np.ndarray:
    """fp64 values 2^e * E4M3(code) of an MXFP8 copy blocked along `axis`."""
    c = np.moveaxis(np.asarray(codes), axis, -1)
    e = np.moveaxis(np.asarray(exps), axis, -1)
    sh = c.shape
    v = e4m3_decode(c).reshape(sh[:-1] + (sh[-1] // MX_BLOCK, MX_BLOCK))
    v = np.ldexp(v, e[..., None]).reshape(sh)
    return np.moveaxis(v, -1, axis)


def quantise_mx_operands(qp, kp, vp):
    """MXFP8 copies of the permuted Q, K, V [B,H,N,bs,d]: Q and K blocked along the
    channels of each token (the Q K^T contraction axis), V along the tokens of each key
    block per channel (the P V contraction axis). Returns dicts {q8, e} per operand."""
    q8, qe = quantise_mx8(qp.astype(F32), axis=-1)
    k8, ke = quantise_mx8(kp.astype(F32), axis=-1)
    v8, ve = quantise_mx8(vp.astype(F32), axis=-2)
    return dict(q8=q8, e=qe), dict(q8=k8, e=ke), dict(q8=v8, e=ve)


# ----------------------------------------------------------------------------------------
# Draft maps and ranking ([DA2] Abstract: low-resolution draft attention map from avg- and
# max-pooled Q/K estimates block importance; a shared ranking gives high precision, low
# precision or skip under budgets. [DA1] Abstract / [NEWS] step 2: the draft map is the
# attention of the pooled queries over the pooled keys.)
# ----------------------------------------------------------------------------------------
def draft_scores(qavg, kavg, qmax, kmax, counts, sm_scale, mass_correction=True):
    """Block-importance score fp64 [B, H, N(query block), N(key block)].

    Each map is a row softmax over key blocks of sm_scale * <pooled q_i, pooled k_j>
    plus ln(c_j) (c_j valid tokens of key block j, so a map estimates the attention MASS
    of block j rather than that of one average token). score = (P_avg + P_max) / 2.
    """
    lc = np.log(counts.astype(np.float64)) if mass_correction else np.zeros(len(counts))

    def one(qp, kp):
        lg = sm_scale * np.einsum("bhid,bhjd->bhij", qp.astype(np.float64),
                                  kp.astype(np.float64)) + lc[None, None, None, :]
        lg = lg - lg.max(axis=-1, keepdims=True)
        e = np.exp(lg)
        return e / e.sum(axis=-1, keepdims=True)

    return 0.5 * (one(qavg, kavg) + one(qmax, kmax))


def rank_classes(scores, n8: int, nm: int, n4: int, n16: int = 0):
    """Shared ranking of each row into the precision classes: order (score desc, block
    index asc); the first n16 blocks are bf16, the next n8 FP8, the next nm mixed, the next
    n4 FP4, the rest skipped.

    Returns tags uint8 [..., N, N] (0 skip, 1 FP4, 2 FP8, 3 mixed, 4 bf16) and the ascending
    block lists of each kept class: list16 [..., N, n16], list8 [..., N, n8], listm
    [..., N, nm], list4 [..., N, n4].
    """
    sc = np.asarray(scores)
    lead = sc.shape[:-1]
    N = sc.shape[-1]
    flat = sc.reshape(-1, N)
    j = np.arange(N)
    tags = np.zeros(flat.shape, dtype=np.uint8)
    c8, c8m = n16 + n8, n16 + n8 + nm
    cuts = ((TAG_BF16, 0, n16), (TAG_FP8, n16, c8), (TAG_MIX, c8, c8m), (TAG_FP4, c8m, c8m + n4))
    lists = {t: np.zeros((flat.shape[0], b - a), dtype=np.int64) for t, a, b in cuts}
    for r in range(flat.shape[0]):
        order = np.lexsort((j, -flat[r]))
        for t, a, b in cuts:
            tags[r, order[a:b]] = t
            lists[t][r] = np.sort(order[a:b])
    return dict(tags=tags.reshape(lead + (N,)),
                list16=lists[TAG_BF16].reshape(lead + (n16,)),
                list8=lists[TAG_FP8].reshape(lead + (n8,)),
                listm=lists[TAG_MIX].reshape(lead + (nm,)),
                list4=lists[TAG_FP4].reshape(lead + (n4,)))


def rank_adaptive(scores, n8: int, nm: int, n4: int, n4max: int, tau: float, n16: int = 0):
    """The shared ranking with an error-bound-driven FP4 budget per row.

    [DA2] Abstract: the analysis separates the sparsification error from the
    attention-weighted quantisation error and establishes when recovering skipped
    interactions with low-bit computation tightens the output-error bound. Reading: a
    skipped block j adds about its attention mass w_j times the output's deviation to the
    sparsification term; kept at FP4 it adds w_j times FP4's much smaller relative error to
    the quantisation term, so recovering it tightens the bound by an amount proportional to
    w_j. Per row the blocks ranked after the fixed budgets therefore join the FP4 class, in
    rank order, while their draft score (the estimated block mass) is at least tau, until
    the row holds n4max FP4 blocks. list4 keeps ascending block order and is padded to n4max
    entries with -1 (no block); count4 holds each row's FP4 count.
    """
    r = rank_classes(scores, n8, nm, n4, n16)
    sc = np.asarray(scores)
    lead = sc.shape[:-1]
    N = sc.shape[-1]
    flat = sc.reshape(-1, N)
    tags = r["tags"].reshape(-1, N).copy()
    l4 = np.full((flat.shape[0], n4max), -1, dtype=np.int64)
    cnt = np.zeros(flat.shape[0], dtype=np.int64)
    j = np.arange(N)
    ck, ckmax = n16 + n8 + nm + n4, min(n16 + n8 + nm + n4max, N)
    base4 = r["list4"].reshape(flat.shape[0], n4)
    for row in range(flat.shape[0]):
        order = np.lexsort((j, -flat[row]))
        extra = [b for b in order[ck:ckmax] if flat[row, b] >= tau]
        # the candidates are in descending score order: the recovered ones form a prefix
        assert extra == list(order[ck:ck + len(extra)])
        tags[row, extra] = TAG_FP4
        kept = np.sort(np.concatenate([base4[row], np.array(extra, dtype=np.int64)]))
        l4[row, :len(kept)] = kept
        cnt[row] = len(kept)
    return dict(tags=tags.reshape(lead + (N,)), list16=r["list16"], list8=r["list8"],
                listm=r["listm"], list4=l4.reshape(lead + (n4max,)), count4=cnt.reshape(lead))


def rank(scores, n8: int, n4: int):
    """The two-class ranking (no mixed blocks): tags, list8 and list4 of `rank_classes`."""
    r = rank_classes(scores, n8, 0, n4)
    return r["tags"], r["list8"], r["list4"]


# ----------------------------------------------------------------------------------------
# P quantisation inside the attention ([DA2] Abstract: both matmuls of a block run at its
# precision). p = exp(S - m) <= 1 with m the running row max.
# ----------------------------------------------------------------------------------------
def quant_p(p: np.ndarray, precision: int) -> np.ndarray:
    """Quantised probabilities (fp64). bf16 (precision 16): bf16(p). FP8: E4M3(448 p)/448.
    FP4: y = 448 p, groups of 16 consecutive keys, sigma = E4M3(amax16/6), value
    sigma*E2M1(y/sigma)/448."""
    if precision == 16:
        return bf16_round(p)
    y = p * E4M3_MAX
    if precision == 8:
        return e4m3_round(y) / E4M3_MAX
    sh = y.shape
    yg = y.reshape(sh[:-1] + (sh[-1] // 16, 16))
    sig = e4m3_round(np.abs(yg).max(axis=-1) / E2M1_MAX)
    safe = np.where(sig > 0, sig, 1.0)
    z = np.where(sig[..., None] > 0, e2m1_round(yg / safe[..., None]) * sig[..., None], 0.0)
    return z.reshape(sh) / E4M3_MAX


def quant_p_mx(p: np.ndarray, precision: int) -> np.ndarray:
    """Probabilities for the block-scaled variant: FP8 as MXFP8 over 32 consecutive keys
    of a row (fp64 values 2^e E4M3(p / 2^e)); FP4 as `quant_p`."""
    if precision != 8:
        return quant_p(p, precision)
    codes, e = quantise_mx8(p, axis=-1)
    return dequant_mx8(codes, e, axis=-1)


# ----------------------------------------------------------------------------------------
# Mixed-precision block-sparse attention ([DA2] Abstract: one kernel with precision-
# specific phases that share data movement, softmax statistics and output accumulation)
# ----------------------------------------------------------------------------------------
@dataclass
class Operands:
    """fp64 operand values per precision: q8/q4/k8/k4/v8/v4 [B,H,N,bs,d], and q16/k16/v16
    (the bf16 input values) where the bf16 tier runs."""
    q: dict
    k: dict
    v: dict


def operands_quantised(qd, kd, vd) -> Operands:
    return Operands({8: dequant_qk(qd, 8), 4: dequant_qk(qd, 4)},
                    {8: dequant_qk(kd, 8), 4: dequant_qk(kd, 4)},
                    {8: dequant_v(vd, 8), 4: dequant_v(vd, 4)})


def operands_mx(qd, kd, vd, qmx, kmx, vmx) -> Operands:
    """8-bit operands from the MXFP8 copies, 4-bit from the NVFP4-style copies."""
    return Operands({8: dequant_mx8(qmx["q8"], qmx["e"], -1), 4: dequant_qk(qd, 4)},
                    {8: dequant_mx8(kmx["q8"], kmx["e"], -1), 4: dequant_qk(kd, 4)},
                    {8: dequant_mx8(vmx["q8"], vmx["e"], -2), 4: dequant_v(vd, 4)})


def operands_exact(qp, kp, vp) -> Operands:
    q, k, v = (x.astype(np.float64) for x in (qp, kp, vp))
    return Operands({16: q, 8: q, 4: q}, {16: k, 8: k, 4: k}, {16: v, 8: v, 4: v})


def with_bf16(ops: Operands, qp, kp, vp) -> Operands:
    """`ops` plus the bf16 tier's operands: the permuted input values themselves (the
    inputs are bf16, so the tier needs no quantiser)."""
    return Operands({**ops.q, 16: qp.astype(np.float64)}, {**ops.k, 16: kp.astype(np.float64)},
                    {**ops.v, 16: vp.astype(np.float64)})


def attention(ops: Operands, valid, list8, list4, sm_scale, quantise_p=True,
              return_parts=False, blocks=None, listm=None, pquant=quant_p, list16=None):
    """Block-sparse attention with one online softmax over all phases.

    For each (b, h, query block i): the bf16 phase (when list16 is given) visits list16[i]
    (bf16 operands, P rounded to bf16), then the FP8 phase visits list8[i] in ascending
    block index,
    then the mixed phase visits listm[i] (scores from the E4M3 copies of Q and K, P
    quantised as for FP4 and multiplied with the E2M1 copy of V), then the FP4 phase visits
    list4[i]; each visited block j updates the running row max
    m, rescales the running sum l and accumulator by exp(m_old - m_new), adds
    sum(exp(S - m_new)) to l (unquantised) and adds P~ V to the accumulator, with P~ the
    block's quantised probabilities taken against the running max. Padded key slots are
    masked (-inf); skipped blocks contribute nothing. Output O = acc / l, fp64
    [B, H, N, bs, d]; rows with no kept block are 0.

    With return_parts, also returns per (b,h,i) lists of (j, alpha_j, sum p~, sum p~ v)
    for the error decomposition. `blocks`, a list of (b, h, i), restricts the computation
    to those query blocks (the others stay 0). `pquant(p, precision)` quantises the
    probabilities (`quant_p_mx` for the block-scaled variant).
    """
    B, H, N, bs, d = ops.q[8].shape
    out = np.zeros((B, H, N, bs, d))
    parts = {} if return_parts else None
    todo = blocks if blocks is not None else [(b, h, i) for b in range(B) for h in range(H)
                                              for i in range(N)]
    for b, h, i in todo:
                m = np.full(bs, -np.inf)
                l = np.zeros(bs)
                acc = np.zeros((bs, d))
                rec = []
                phases = [(16, 16, list16[b, h, i])] if list16 is not None else []
                phases.append((8, 8, list8[b, h, i]))
                if listm is not None:
                    phases.append((8, 4, listm[b, h, i]))
                phases.append((4, 4, list4[b, h, i]))
                for prec, pprec, lst in phases:       # score precision, P V precision
                    qi = ops.q[prec][b, h, i]
                    for j in lst:
                        if j < 0:                     # padding of an adaptive FP4 list
                            continue
                        S = sm_scale * (qi @ ops.k[prec][b, h, j].T)
                        S[:, ~valid[j]] = -np.inf
                        m_new = np.maximum(m, S.max(axis=1))
                        fin = np.isfinite(m_new)
                        alpha = np.where(np.isfinite(m), np.exp(m - np.where(fin, m_new, 0.0)), 0.0)
                        p = np.exp(S - np.where(fin, m_new, 0.0)[:, None])
                        p[~np.isfinite(S)] = 0.0
                        pq = pquant(p, pprec) if quantise_p else p
                        pv = pq @ ops.v[pprec][b, h, j]
                        l = alpha * l + p.sum(axis=1)
                        acc = alpha[:, None] * acc + pv
                        if return_parts:
                            for r in rec:
                                r[1] *= alpha
                            rec.append([j, np.ones(bs), pq.sum(axis=1), pv])
                        m = m_new
                safe = np.where(l > 0, l, 1.0)
                out[b, h, i] = np.where(l[:, None] > 0, acc / safe[:, None], 0.0)
                if return_parts:
                    parts[(b, h, i)] = (rec, l)
    return (out, parts) if return_parts else out


def dense_attention(q, k, v, sm_scale, key_mask=None):
    """Textbook softmax attention in fp64 on [B,H,T,d] (key_mask [..., Tq, Tk] bool keeps)."""
    S = sm_scale * np.einsum("bhqd,bhkd->bhqk", q.astype(np.float64), k.astype(np.float64))
    if key_mask is not None:
        S = np.where(key_mask, S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=-1, keepdims=True)
    return np.einsum("bhqk,bhkd->bhqd", P, v.astype(np.float64))


# ----------------------------------------------------------------------------------------
# Error decomposition ([DA2] Abstract: the analysis separates the sparsification error
# from an attention-weighted quantisation error). The formula is not printed on the pages;
# the reading below is pinned term by term (the skipped mass and E_sp by torch's softmax
# and SDPA, E_q by a closed form for constant scores and by the bound it must satisfy).
# Reading: per query row, with O dense, O_S the exact attention over the
# kept blocks, O~ the mixed result,
#   E_sp = ||O_S - O|| = m_skip ||o_skip - O_S||   (m_skip: softmax mass of skipped blocks)
#   E_q  = sum_b w_b ||o~_b - o_b|| + sum_b |w~_b - w_b| ||o~_b||
# where w_b / o_b are block b's share of the kept mass and its block-normalised output,
# and w~_b / o~_b the same quantities from the mixed computation (O~ = sum_b w~_b o~_b).
# Then ||O~ - O|| <= E_sp + E_q.
# ----------------------------------------------------------------------------------------
def error_decomposition(q, k, v, valid, list8, list4, ops_q: Operands, sm_scale, g: Geometry):
    """Per-row (E_tot, E_sp, E_q, m_skip) arrays [B,H,N,bs] plus (O, O_S, O~)."""
    qp, kp, vp = (permute(x, g).astype(np.float64) for x in (q, k, v))
    ops_x = operands_exact(qp, kp, vp)
    B, H, N, bs, d = qp.shape
    kept = np.zeros((B, H, N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                kept[b, h, i, list8[b, h, i]] = True
                l4 = list4[b, h, i]
                kept[b, h, i, l4[l4 >= 0]] = True          # -1 pads an adaptive FP4 list
    all8 = np.broadcast_to(np.arange(N), (B, H, N, N))
    none = np.zeros((B, H, N, 0), dtype=np.int64)
    O = attention(ops_x, valid, all8, none, sm_scale, quantise_p=False)
    OS, parts_x = attention(ops_x, valid, list8, list4, sm_scale, quantise_p=False,
                            return_parts=True)
    Ot, parts_q = attention(ops_q, valid, list8, list4, sm_scale, quantise_p=True,
                            return_parts=True)
    E_tot = np.linalg.norm(Ot - O, axis=-1)
    E_sp = np.linalg.norm(OS - O, axis=-1)
    E_q = np.zeros((B, H, N, bs))
    m_skip = np.zeros((B, H, N, bs))
    for key, (rec_x, l_x) in parts_x.items():
        rec_q, l_q = parts_q[key]
        b, h, i = key
        for (jx, ax, sx, pvx), (jq, aq, sq, pvq) in zip(rec_x, rec_q):
            assert jx == jq
            w = ax * sx / np.where(l_x > 0, l_x, 1.0)
            o = pvx / np.where(sx > 0, sx, 1.0)[:, None]
            wt = aq * sq / np.where(l_q > 0, l_q, 1.0)
            ot = pvq / np.where(sq > 0, sq, 1.0)[:, None]
            E_q[b, h, i] += w * np.linalg.norm(ot - o, axis=-1) + \
                np.abs(wt - w) * np.linalg.norm(ot, axis=-1)
    # skipped mass from the dense softmax
    for b in range(B):
        for h in range(H):
            for i in range(N):
                S = sm_scale * np.einsum("rd,jsd->rjs", qp[b, h, i], kp[b, h])
                S[:, ~valid] = -np.inf
                S = S - S.max(axis=(1, 2), keepdims=True)
                P = np.exp(S)
                tot = P.sum(axis=(1, 2))
                skip = P[:, ~kept[b, h, i]].sum(axis=(1, 2))
                m_skip[b, h, i] = skip / tot
    return dict(E_tot=E_tot, E_sp=E_sp, E_q=E_q, m_skip=m_skip, O=O, OS=OS, Ot=Ot)


# ----------------------------------------------------------------------------------------
# The whole path
# ----------------------------------------------------------------------------------------
def _np(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().float().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=F32)


def prepare(w, q, k, v):
    """Pooling, permutation and operand quantisation for inputs [B,H,T,d] (bf16 values)."""
    g = geometry(w)
    q, k, v = _np(q), _np(k), _np(v)
    valid = block_valid(g)
    qp, kp, vp = permute(q, g), permute(k, g), permute(v, g)
    qavg, qmax = pool(qp, valid)
    kavg, kmax = pool(kp, valid)
    vamax = v_channel_amax(v)
    return dict(g=g, valid=valid, counts=valid.sum(1), qp=qp, kp=kp, vp=vp,
                qavg=qavg, qmax=qmax, kavg=kavg, kmax=kmax, vamax=vamax,
                Q=quantise_qk(qp, valid), K=quantise_qk(kp, valid), V=quantise_v(vp, vamax))


def draft_select(prep, mass_correction=True):
    g = prep["g"]
    sc = draft_scores(prep["qavg"], prep["kavg"], prep["qmax"], prep["kmax"],
                      prep["counts"], g.sm_scale, mass_correction)
    if g.tau > 0:
        r = rank_adaptive(sc, g.n8, g.nm, g.n4, g.n4max, g.tau, g.n16)
    else:
        r = rank_classes(sc, g.n8, g.nm, g.n4, g.n16)
    return dict(scores=sc, **r)


def run(w, q, k, v, quantised=True, lists=None, fp8="scaled"):
    """Whole hot path. Returns dict with every intermediate and `out` fp64 [B,H,T,d].

    `lists` = (list8, list4) or (list8, list4, listm) overrides the oracle's own selection
    (used to compare the attention step on the CUDA path's selection when rankings differ
    at near-ties). fp8="mx" runs the 8-bit class in the block-scaled MXFP8 form (Q, K, V
    and P), which only the oracle implements; so does the bf16 tier (a workload with
    pct_bf16 > 0).
    """
    prep = prepare(w, q, k, v)
    g = prep["g"]
    sel = draft_select(prep)
    if lists is None:
        l8, l4, lm = sel["list8"], sel["list4"], sel["listm"]
    else:
        l8, l4 = lists[0], lists[1]
        lm = lists[2] if len(lists) > 2 else None
    l16 = sel["list16"] if g.n16 > 0 else None
    if fp8 not in ("scaled", "mx"):
        raise ValueError(f"fp8 must be 'scaled' or 'mx', not {fp8!r}")
    pquant = quant_p
    if quantised and fp8 == "mx":
        ops = operands_mx(prep["Q"], prep["K"], prep["V"],
                          *quantise_mx_operands(prep["qp"], prep["kp"], prep["vp"]))
        pquant = quant_p_mx
    elif quantised:
        ops = operands_quantised(prep["Q"], prep["K"], prep["V"])
    else:
        ops = operands_exact(prep["qp"], prep["kp"], prep["vp"])
    if l16 is not None:
        ops = with_bf16(ops, prep["qp"], prep["kp"], prep["vp"])
    o = attention(ops, prep["valid"], l8, l4, g.sm_scale, quantise_p=quantised,
                  listm=lm if (lm is not None and lm.shape[-1] > 0) else None, pquant=pquant,
                  list16=l16)
    return dict(prep=prep, sel=sel, out_blocks=o, out=inverse_permute(o, g))
