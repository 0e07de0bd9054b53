"""Properties every NVFP4 quantization must have, checked from the definitions
alone (not from the oracle's code): used by the oracle pin tests and, at full
size, by the GPU chain test where the input of a quantization is the GPU's own
GEMM output.

For block values y (x itself, or the RHT output) and a stored result (codes,
canonical E4M3 block scales sb, global scale s_g):
  * s_g = RN(amax / 2688) with amax = max |y| (1 when amax = 0)  ("NVFP4"
    section of the Microscaling page; configuration: amax / (6 * 448));
  * sb = E4M3 nearest-even of RN(RN(block_amax / 6) / s_g) saturated at 448,
    the cast done by torch's float8_e4m3fn (a library routine); with Four Over Six sb may
    instead be the block_amax / 4 candidate, and then the chosen candidate
    has the lower binary64 squared error wherever the two errors differ by
    more than a binary32 evaluation of them can blur (the choice itself sums
    in binary32, so closer pairs are left to the pinned summation order);
  * every code is the nearest value of the pages' E2M1 list (FP4 page, "Bit
    layout of FP4 E2M1") to q = RN(y * r), r = RN(1 / RN(sb * s_g)), found by
    brute force over the list, ties to the even code, saturated at 6, with
    the sign of q; a block with sb = 0 stores zero codes.
"""
import numpy as np
import torch

from conftest import golden_rows


def e2m1_magnitudes():
    rows = {r[0]: r[1:] for r in golden_rows("e2m1_codepoints.txt")}
    return np.array([float(v) for v in rows["nonnegative"]], np.float64)


def e4m3_code(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_value(c):
    return torch.from_numpy(np.ascontiguousarray(c, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def nearest_e2m1_code(q, mags):
    """Brute force over the listed magnitudes: the nearest one to |q| (ties
    to the even code index), with the sign bit of q."""
    a = np.abs(q).astype(np.float64)
    d = np.abs(a[..., None] - mags)
    dmin = d.min(-1, keepdims=True)
    cand = d == dmin
    idx = cand.argmax(-1)                                 # lowest index at the minimum
    tie = cand.sum(-1) > 1                                # two neighbours equally close
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)   # ties go to the even code
    return (idx | (np.signbit(q).astype(np.int64) << 3)).astype(np.uint8)


def unpack_codes(codes):
    """[R, K/2] packed bytes -> [R, K] nibbles (element 2j in the low nibble)."""
    c = np.asarray(codes, np.uint8)
    out = np.empty((c.shape[0], c.shape[1] * 2), np.uint8)
    out[:, 0::2] = c & 15
    out[:, 1::2] = c >> 4
    return out


def check_nvfp4(y, codes, sf, s_g, block_2d=False, four_over_six=False, amax=None, rows_per_chunk=2048,
                what="nvfp4", check_sg=True):
    """Assert the properties above for y [R, K] (float32) against codes
    [R, K/2], canonical sf [R, K/16] and s_g.  amax: the amax the
    quantization used, when it was given rather than computed from y;
    check_sg=False: s_g was given as such (the block scales and codes are
    still checked under it).  Returns the number of blocks where Four Over
    Six kept the /4 candidate."""
    y = np.asarray(y, np.float32)
    R, K = y.shape
    mags = e2m1_magnitudes()
    sg = np.float32(s_g)
    if amax is None:
        amax = np.float32(np.abs(y).max()) if y.size else np.float32(0)
    want_sg = np.float32(1.0) if amax == 0 else np.float32(np.float32(amax) / np.float32(2688.0))
    assert not check_sg or sg == want_sg, f"{what}: s_g {sg!r} != {want_sg!r}"
    step = max(16, rows_per_chunk // 16 * 16)
    picked4 = 0
    for r0 in range(0, R, step):
        r1 = min(R, r0 + step)
        yb = y[r0:r1].reshape(r1 - r0, K // 16, 16)
        sb = np.asarray(sf[r0:r1], np.uint8)
        bamax = np.abs(yb).max(-1)
        if block_2d:
            t = bamax.reshape((r1 - r0) // 16, 16, K // 16).max(1)
            bamax = np.repeat(t, 16, axis=0)
        cands = {}
        for div in ((6.0, 4.0) if four_over_six else (6.0,)):
            t = (bamax / np.float32(div)) / sg
            cands[div] = e4m3_code(np.minimum(t, np.float32(448.0)))   # saturating at the E4M3 maximum
        ok = sb == cands[6.0]
        if four_over_six:
            ok |= sb == cands[4.0]
        bad = np.argwhere(~ok)
        assert bad.size == 0, f"{what}: block scale not a candidate at {bad[:5].tolist()}"
        den = e4m3_value(sb) * sg
        with np.errstate(all="ignore"):   # sb = 0 blocks: r = inf, their codes are checked as zero
            r = np.float32(1.0) / den
            q = (yb * r[..., None]).astype(np.float32)
        want = nearest_e2m1_code(q, mags)
        want[sb == 0] = 0
        got = unpack_codes(codes[r0:r1]).reshape(r1 - r0, K // 16, 16)
        bad = np.argwhere(got != want)
        assert bad.size == 0, (f"{what}: {len(bad)} codes are not the nearest E2M1 value; first at "
                               f"{bad[:5].tolist()}: got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")
        if four_over_six:
            errs, slack = {}, {}
            for div, c in cands.items():
                dv = e4m3_value(c) * sg
                with np.errstate(all="ignore"):
                    rc = np.float32(1.0) / dv
                    qc = (yb * rc[..., None]).astype(np.float32)
                cc = nearest_e2m1_code(qc, mags)
                cc[c == 0] = 0
                val = np.where(cc & 8, -1.0, 1.0) * mags[cc & 7] * dv[..., None].astype(np.float64)
                d = yb.astype(np.float64) - val
                errs[div] = (d ** 2).sum(-1)
                # how far a binary32 evaluation of the same sum can stray: each
                # difference carries about 2^-24 (|y| + 2 |val|) of rounding, each
                # square and each of the four levels of adds 2^-24 relative
                slack[div] = 2.0 ** -21 * (np.abs(d) * (np.abs(yb) + 2 * np.abs(val)) + d ** 2).sum(-1)
            e6, e4 = errs[6.0], errs[4.0]
            clear = np.abs(e6 - e4) > slack[6.0] + slack[4.0] + 1e-30
            want_sb = np.where(e4 < e6, cands[4.0], cands[6.0])
            bad = np.argwhere(clear & (sb != want_sb))
            assert bad.size == 0, f"{what}: Four Over Six kept the higher-error scale at {bad[:5].tolist()}"
            picked4 += int((clear & (e4 < e6)).sum())
    return picked4


def decode_nvfp4(codes, sf, s_g):
    """Binary64 values of an NVFP4 tensor (codes [R, K/2], canonical sf
    [R, K/16], s_g): element x block scale x global scale, from the pages'
    E2M1 list and torch's E4M3 decode (exact)."""
    mags = e2m1_magnitudes()
    c = unpack_codes(codes)
    v = np.where(c & 8, -1.0, 1.0) * mags[c & 7]
    sc = np.repeat(e4m3_value(sf).astype(np.float64), 16, axis=1)
    return v * sc * np.float64(np.float32(s_g))
