"""Loop-only restatement of the VSA forward path, for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

It follows the same reading of the pages as ``vsa_oracle`` (cubes of 4x4x4
tokens, mean pooling, coarse attention with 1/sqrt(d), top-k on coarse logits
with ties to the lower index, exact attention over the selected cubes, gated
combine) but is built differently so that a slip in one does not hide in the
other: plain Python floats and loops, no NumPy arithmetic, no BLAS, and the
token-to-slot map is found by walking the tokens in grid order and ranking
each one inside its cube, instead of walking the cubes.

Cost grows as N^2 d; keep N at a few hundred tokens.
"""

from __future__ import annotations

import math


def _slot_of_token(grid, cube):
    """Map token n -> (cube index, slot inside the cube); also per-cube counts."""
    T, H, W = grid
    ct, cy, cx = cube
    Cy, Cx = -(-H // cy), -(-W // cx)
    Ct = -(-T // ct)
    C = Ct * Cy * Cx
    slot = {}
    counts = [0] * C
    # Rank of a token inside its cube = number of in-grid tokens of the same
    # cube whose local (t, y, x) offset comes first in row-major order.
    for t in range(T):
        for y in range(H):
            for x in range(W):
                c = ((t // ct) * Cy + y // cy) * Cx + x // cx
                lt, ly, lx = t % ct, y % cy, x % cx
                rank = 0
                for a in range(ct):
                    for b in range(cy):
                        for e in range(cx):
                            if (a, b, e) >= (lt, ly, lx):
                                continue
                            tt = (t // ct) * ct + a
                            yy = (y // cy) * cy + b
                            xx = (x // cx) * cx + e
                            if tt < T and yy < H and xx < W:
                                rank += 1
                slot[(t * H + y) * W + x] = (c, rank)
                counts[c] += 1
    return slot, counts, C


def vsa_forward_loops(q, k, v, grid, topk, g_f=None, g_c=None, cube=(4, 4, 4)):
    """q, k, v: nested lists [B][Hh][N][d] of floats.

    Returns dict(counts, slot, S_c, sel, O_c, O_f_tokens, out) where
    ``O_f_tokens`` and ``out`` are in token order [B][Hh][N][d].
    """
    slot, counts, C = _slot_of_token(grid, cube)
    B, Hh, N, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    members = [[] for _ in range(C)]  # tokens of each cube, in slot order
    for n in range(N):
        c, r = slot[n]
        members[c].append((r, n))
    members = [[n for _, n in sorted(m)] for m in members]

    scale = 1.0 / math.sqrt(d)
    S_c_all, sel_all, O_c_all, O_f_all, out_all = [], [], [], [], []
    for b in range(B):
        S_c_b, sel_b, O_c_b, O_f_b, out_b = [], [], [], [], []
        for h in range(Hh):
            def mean(x, c):
                acc = [0.0] * d
                for n in members[c]:
                    for e in range(d):
                        acc[e] += x[b][h][n][e]
                return [a / len(members[c]) for a in acc]

            qb = [mean(q, c) for c in range(C)]
            kb = [mean(k, c) for c in range(C)]
            vb = [mean(v, c) for c in range(C)]
            S = [[sum(qb[i][e] * kb[j][e] for e in range(d)) * scale
                  for j in range(C)] for i in range(C)]
            O_c = []
            for i in range(C):
                mx = max(S[i])
                w = [math.exp(s - mx) for s in S[i]]
                z = sum(w)
                O_c.append([sum(w[j] * vb[j][e] for j in range(C)) / z
                            for e in range(d)])
            sel = []
            for i in range(C):
                ranked = sorted(range(C), key=lambda j: (-S[i][j], j))
                sel.append(sorted(ranked[:topk]))
            O_f = [None] * N
            out = [None] * N
            for i in range(C):
                keys = [n for j in sel[i] for n in members[j]]
                for n in members[i]:
                    logits = [sum(q[b][h][n][e] * k[b][h][t][e] for e in range(d)) * scale
                              for t in keys]
                    mx = max(logits)
                    w = [math.exp(s - mx) for s in logits]
                    z = sum(w)
                    o = [sum(w[a] * v[b][h][keys[a]][e] for a in range(len(keys))) / z
                         for e in range(d)]
                    O_f[n] = o
                    if g_f is None and g_c is None:
                        out[n] = list(o)
                    else:
                        gf, gc = g_f[b][h][n], g_c[b][h][n]
                        out[n] = [gf * o[e] + gc * O_c[i][e] for e in range(d)]
            S_c_b.append(S)
            sel_b.append(sel)
            O_c_b.append(O_c)
            O_f_b.append(O_f)
            out_b.append(out)
        S_c_all.append(S_c_b)
        sel_all.append(sel_b)
        O_c_all.append(O_c_b)
        O_f_all.append(O_f_b)
        out_all.append(out_b)
    return dict(counts=counts, slot=slot, S_c=S_c_all, sel=sel_all, O_c=O_c_all,
                O_f_tokens=O_f_all, out=out_all)
