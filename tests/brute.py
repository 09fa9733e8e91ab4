"""Pure-Python brute force of the whole method on tiny inputs.

Written independently of the C oracle (plain Python floats and loops, no
shared helpers) so that index or bookkeeping mistakes in either one show up
as a disagreement.  Only usable for N <= a few hundred tokens and small d.
Inputs are nested lists x[n][h][c] of floats (already upcast from bf16/f32).
"""
import math
import struct
from fractions import Fraction


def f32(x: float) -> float:
    """Round a Python float (double) to the nearest fp32 value."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def bf16(x: float) -> float:
    """Round an fp32 value to bf16 (nearest, ties to even)."""
    (u,) = struct.unpack("<I", struct.pack("<f", x))
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return struct.unpack("<f", struct.pack("<I", u))[0]


def fma(x: float, y: float, z: float) -> float:
    """x*y + z with a single rounding (exact rational arithmetic, then one
    correctly rounded conversion back to double)."""
    return float(Fraction(x) * Fraction(y) + Fraction(z))


def fsum_fma(a, b):
    """Dot product accumulated with one rounding per fused multiply-add."""
    acc = 0.0
    for x, y in zip(a, b):
        acc = fma(x, y, acc)
    return acc


def block_ranges(N, blk):
    return [(s, min(N, s + blk)) for s in range(0, N, blk)]


def pool(x, h, N, blk, d):
    out = []
    for s, e in block_ranges(N, blk):
        row = []
        for c in range(d):
            acc = 0.0
            for n in range(s, e):
                acc += x[n][h][c]
            row.append(f32(acc / (e - s)))
        out.append(row)
    return out


def run(q, k, v, N, H, d, p):
    """Returns (keep[h][i][b] bools, out[h][n][c], lse[h][n])."""
    Bq, Bk = p["q_block"], p["k_block"]
    qr, kr = block_ranges(N, Bq), block_ranges(N, Bk)
    nQB, nKB = len(qr), len(kr)
    keep_all, out_all, lse_all = [], [], []
    for h in range(H):
        qb, kb, vb = pool(q, h, N, Bq, d), pool(k, h, N, Bk, d), pool(v, h, N, Bk, d)
        keep_h, extras_h = [], []
        for i in range(nQB):
            S = [f32(fsum_fma(qb[i], kb[j]) / math.sqrt(d)) for j in range(nKB)]
            sel = [False] * nKB
            if p["method"] == "sol":
                tau = p["tau"]
                if tau == -math.inf:
                    sel = [True] * nKB
                elif tau != math.inf:
                    mu = 0.0
                    for s in S:
                        mu += s
                    mu /= nKB
                    var = 0.0
                    for s in S:
                        var += (s - mu) * (s - mu)
                    sig = math.sqrt(var / nKB)
                    t = f32(mu + tau * sig)
                    if sig > 0:
                        sel = [s > t for s in S]
            else:
                kk = min(max(int(math.floor(p["keep_percent"] * nKB / 100.0 + 0.5)), 1), nKB)
                order = sorted(range(nKB), key=lambda j: (-S[j], j))
                for j in order[:kk]:
                    sel[j] = True
            # forced blocks
            for j in range(min(p["sink_blocks"], nKB)):
                sel[j] = True
            if p["prefix_len"] > 0:
                for j in range(nKB):
                    if kr[j][0] < p["prefix_len"]:
                        sel[j] = True
            if p["keep_diag"]:
                s0, e0 = qr[i]
                for j in range(nKB):
                    if kr[j][0] < e0 and kr[j][1] > s0:
                        sel[j] = True
            keep_h.append(sel)
            # extra tokens
            ex = []
            E = p.get("extra_tokens", 0)
            if E > 0:
                qt = [bf16(x) if p["dtype"] == "bf16" else x for x in qb[i]]
                cands = []
                for j in range(nKB):
                    if sel[j]:
                        continue
                    for n in range(*kr[j]):
                        kvec = [k[n][h][c] for c in range(d)]
                        cands.append((-f32(fsum_fma(qt, kvec) / math.sqrt(d)), n))
                cands.sort()
                ex = sorted(n for _, n in cands[:E])
            extras_h.append(ex)
        keep_all.append(keep_h)
        out_h, lse_h = [], []
        for n in range(N):
            i = n // Bq
            qv = [q[n][h][c] for c in range(d)]
            terms = []          # (logit, value vector)
            if p["dense_rows"][0] <= n < p["dense_rows"][1]:
                for m in range(N):
                    terms.append((fsum_fma(qv, [k[m][h][c] for c in range(d)]) / math.sqrt(d),
                                  [v[m][h][c] for c in range(d)]))
            else:
                sel, ex = keep_h[i], set(extras_h[i])
                for j in range(nKB):
                    toks = range(*kr[j])
                    if sel[j]:
                        for m in toks:
                            terms.append((fsum_fma(qv, [k[m][h][c] for c in range(d)]) / math.sqrt(d),
                                          [v[m][h][c] for c in range(d)]))
                        continue
                    for m in toks:
                        if m in ex:
                            terms.append((fsum_fma(qv, [k[m][h][c] for c in range(d)]) / math.sqrt(d),
                                          [v[m][h][c] for c in range(d)]))
                    if not p["centroid"]:
                        continue
                    rest = [m for m in toks if m not in ex]
                    if not rest:
                        continue
                    if len(rest) == len(toks):
                        kc, vc = kb[j], vb[j]
                    else:
                        kc, vc = [], []
                        for c in range(d):
                            a = 0.0
                            b = 0.0
                            for m in rest:
                                a += k[m][h][c]
                                b += v[m][h][c]
                            kc.append(f32(a / len(rest)))
                            vc.append(f32(b / len(rest)))
                    terms.append((fsum_fma(qv, kc) / math.sqrt(d) + math.log(len(rest)), vc))
            mx = max(t[0] for t in terms)
            den = 0.0
            acc = [0.0] * d
            for lg, vec in terms:
                w = math.exp(lg - mx)
                den += w
                for c in range(d):
                    acc[c] += w * vec[c]
            out_h.append([a / den for a in acc])
            lse_h.append(mx + math.log(den))
        out_all.append(out_h)
        lse_all.append(lse_h)
    return keep_all, out_all, lse_all
