"""Host-side model of the fragment arithmetic of the tiled backward passes
(csrc/backward_tc.cu: bwd_target_tc_kernel, bwd_source_tc_kernel).

The kernels feed `mma.sync` m16n8k16 (bf16) and m16n8k8 (tf32) from registers
and from `ldmatrix` loads of staged rows, and reuse accumulator fragments as A
operands with their k index permuted (acc_as_a).  This model replays each
lane's fragment registers exactly as the kernels index them (heads of 8
channels, rows [D][C] with the head's channels at 8 h), multiplies the
matrices the fragments encode (the PTX fragment layouts of those shapes),
scatters the products back to lanes, and checks the epilogues' dq, Delta, dk
and dL/dh' against the direct formulas on random data (float64, no rounding).
A wrong lane, row, channel, component or k permutation in the index
arithmetic shows here.  It runs two heads, not sixteen: the formulas only
offset by the head.  Both stage shapes are modelled: 16 union rows per stage
up to lmax 2 (key / query fragments by ldmatrix.x4) and 8 rows at lmax 3
(ldmatrix.x2), where the source pass also runs as two sweeps, one for dk and
one for dL/dh'.  No GPU is involved.
"""
import numpy as np
import pytest

H, DK = 2, 16                  # heads modelled, key dimension
C = 8 * H


def stage_rows(L):
    """union rows per stage: two n8 tiles, one at lmax 3"""
    return 8 if L >= 3 else 16


# ----------------------------------------------------------------- PTX fragment layouts
def mma_tf32(acc, a, b0, b1):
    """acc += A B, m16n8k8: a[lane] = (A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]),
    b0 = B[t][g], b1 = B[t+4][g]; acc[lane] = (D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1])."""
    A = np.zeros((16, 8))
    B = np.zeros((8, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        A[g, t], A[g + 8, t], A[g, t + 4], A[g + 8, t + 4] = a[lane]
        B[t, g], B[t + 4, g] = b0[lane], b1[lane]
    Dm = A @ B
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        acc[lane] += (Dm[g, 2 * t], Dm[g, 2 * t + 1], Dm[g + 8, 2 * t], Dm[g + 8, 2 * t + 1])


def mma_bf16(acc, a, b0, b1):
    """acc += A B, m16n8k16: a[lane] = four pairs (A[g][2t..], A[g+8][2t..], A[g][2t+8..],
    A[g+8][2t+8..]), b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]."""
    A = np.zeros((16, 16))
    B = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        A[g, 2 * t:2 * t + 2], A[g + 8, 2 * t:2 * t + 2] = a[lane][0], a[lane][1]
        A[g, 2 * t + 8:2 * t + 10], A[g + 8, 2 * t + 8:2 * t + 10] = a[lane][2], a[lane][3]
        B[2 * t:2 * t + 2, g], B[2 * t + 8:2 * t + 10, g] = b0[lane], b1[lane]
    Dm = A @ B
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        acc[lane] += (Dm[g, 2 * t], Dm[g, 2 * t + 1], Dm[g + 8, 2 * t], Dm[g + 8, 2 * t + 1])


def ldmatrix(row_words, address, nmat):
    """ldmatrix.x{nmat}: lanes 8i..8i+7 address the rows of matrix i; lane T receives from
    matrix i the 32-bit word T % 4 of row T / 4.  row_words(addr) gives a row's 4 words."""
    mats = [[row_words(address(8 * i + r)) for r in range(8)] for i in range(nmat)]
    return [[mats[i][T >> 2][T & 3] for i in range(nmat)] for T in range(32)]


def acc_as_a(c):
    """The kernels' reuse of an n8 accumulator as a tf32 A fragment, k order (0,2,4,6,1,3,5,7)."""
    return [(x[0], x[2], x[1], x[3]) for x in c]


# ----------------------------------------------------------------- data
def _data(L, seed):
    D = (L + 1) ** 2
    RS = stage_rows(L)
    rng = np.random.default_rng(seed)
    n = 64
    d = dict(D=D, n=n, RS=RS,
             q=rng.standard_normal((n, H, DK)), k=rng.standard_normal((n, H, DK)),
             hp=rng.standard_normal((n, D, C)), dm=rng.standard_normal((n, D, C)),
             lse=rng.standard_normal((n, H)) + 3.0, delta=rng.standard_normal((n, H)),
             qs=np.log2(np.e) / 4.0)
    tile = list(range(16))                       # the tile's 16 atoms
    U = 37                                       # a ragged union: three stages, the last partial
    uni = sorted(rng.choice(np.arange(16, n), U, replace=False).tolist())
    nst = -(-U // RS)
    d.update(tile=tile, uni=uni + [uni[0]] * (nst * RS - U), nst=nst,
             mask=np.pad(rng.random((16, U)) < 0.6, ((0, 0), (0, nst * RS - U))))
    return d


def _bf16_pairs(v):
    return [v[0:2], v[2:4], v[4:6], v[6:8]]


# ----------------------------------------------------------------- target pass
def _target_model(d):
    D, q, k, hp, dm, lse, qs = d["D"], d["q"], d["k"], d["hp"], d["dm"], d["lse"], d["qs"]
    RS = d["RS"]
    dq = np.zeros((16, H, DK))
    dl_out = np.zeros((16, H))
    for h in range(H):
        qa, dma = [], [[None] * 32 for _ in range(D)]
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            a0, a1 = d["tile"][g], d["tile"][g + 8]
            qa.append((q[a0, h, 2 * t:2 * t + 2], q[a1, h, 2 * t:2 * t + 2],
                       q[a0, h, 2 * t + 8:2 * t + 10], q[a1, h, 2 * t + 8:2 * t + 10]))
            for c in range(D):
                o = h * 8 + t
                dma[c][lane] = (dm[a0, c, o], dm[a1, c, o], dm[a0, c, o + 4], dm[a1, c, o + 4])
        accA = [np.zeros((32, 4)) for _ in range(2)]
        accB = [np.zeros((32, 4)) for _ in range(2)]
        dl = np.zeros((32, 2))
        for st in range(d["nst"]):
            rows = d["uni"][st * RS:(st + 1) * RS]
            # stage_frags<RS>: row (lane & 7) + 8 (lane >> 4), half (lane >> 3) & 1;
            # ldmatrix.x4 for 16 rows, .x2 (lanes 0-15 address) for 8
            kf = ldmatrix(lambda a: _bf16_pairs(k[rows[a[0]], h, 8 * a[1]:8 * a[1] + 8]),
                          lambda l: ((l & 7) + 8 * (l >> 4), (l >> 3) & 1), RS // 4)
            for nt in range(RS // 8):
                s = np.zeros((32, 4))
                mma_bf16(s, qa, [kf[l][2 * nt] for l in range(32)], [kf[l][2 * nt + 1] for l in range(32)])
                P = np.zeros((32, 4))
                for lane in range(32):
                    g, t = lane >> 2, lane & 3
                    c0 = st * RS + 8 * nt + 2 * t
                    ls0, ls1 = lse[d["tile"][g], h], lse[d["tile"][g + 8], h]
                    P[lane] = (2 ** (s[lane, 0] * qs - ls0) if d["mask"][g, c0] else 0.0,
                               2 ** (s[lane, 1] * qs - ls0) if d["mask"][g, c0 + 1] else 0.0,
                               2 ** (s[lane, 2] * qs - ls1) if d["mask"][g + 8, c0] else 0.0,
                               2 ** (s[lane, 3] * qs - ls1) if d["mask"][g + 8, c0 + 1] else 0.0)
                # dalpha: B from the staged h' rows, ldmatrix.x4 over two components
                hrow = lambda a: list(hp[rows[8 * nt + a[0]], a[1], h * 8 + 4 * a[2]:h * 8 + 4 * a[2] + 4])
                dp, dp2 = np.zeros((32, 4)), np.zeros((32, 4))
                for c in range(0, D - 1, 2):
                    r = ldmatrix(hrow, lambda l: (l & 7, c + (l >> 4), (l >> 3) & 1), 4)
                    mma_tf32(dp, dma[c], [r[l][0] for l in range(32)], [r[l][1] for l in range(32)])
                    mma_tf32(dp2, dma[c + 1], [r[l][2] for l in range(32)], [r[l][3] for l in range(32)])
                if D % 2:
                    r = ldmatrix(hrow, lambda l: (l & 7, D - 1, (l >> 3) & 1), 2)
                    mma_tf32(dp, dma[D - 1], [r[l][0] for l in range(32)], [r[l][1] for l in range(32)])
                dp += dp2
                E = P * dp
                dl[:, 0] += E[:, 0] + E[:, 1]
                dl[:, 1] += E[:, 2] + E[:, 3]
                ea, pa = acc_as_a(E), acc_as_a(P)
                for nd in range(2):
                    b0 = [k[rows[8 * nt + 2 * (l & 3)], h, 8 * nd + (l >> 2)] for l in range(32)]
                    b1 = [k[rows[8 * nt + 2 * (l & 3) + 1], h, 8 * nd + (l >> 2)] for l in range(32)]
                    mma_tf32(accA[nd], ea, b0, b1)
                    mma_tf32(accB[nd], pa, b0, b1)
        dlr = dl.reshape(8, 4, 2).sum(axis=1)    # the quad reduction over t
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            for half in range(2):
                r = g + 8 * half
                for nd in range(2):
                    for e in range(2):
                        dq[r, h, 8 * nd + 2 * t + e] = (accA[nd][lane, 2 * half + e]
                                                        - dlr[g, half] * accB[nd][lane, 2 * half + e]) * 0.25
                dl_out[r, h] = dlr[g, half]
    return dq, dl_out


def _alpha_dalpha(d, i, j):
    s = (d["q"][i] * d["k"][j]).sum(-1)
    a = 2.0 ** (s * d["qs"] - d["lse"][i])
    head = np.arange(C) // 8
    da = np.array([(d["dm"][i][:, head == hh] * d["hp"][j][:, head == hh]).sum() for hh in range(H)])
    return a, da


@pytest.mark.parametrize("L", [1, 2, 3])
def test_target_pass_fragments(L):
    d = _data(L, seed=10 + L)
    dq, dl = _target_model(d)
    assert d["mask"].any(axis=1).all()           # every target has union neighbours
    for r, i in enumerate(d["tile"]):
        terms = [(_alpha_dalpha(d, i, j), j) for u, j in enumerate(d["uni"]) if d["mask"][r, u]]
        delta = sum(a * da for (a, da), _ in terms)
        ref_dq = sum(((a * (da - delta))[:, None] * d["k"][j]) for (a, da), j in terms) * 0.25
        assert np.allclose(dl[r], delta, rtol=1e-12, atol=1e-12)
        assert np.allclose(dq[r], ref_dq, rtol=1e-10, atol=1e-10)


# ----------------------------------------------------------------- source pass
def _source_model(d, dk_sweep=True, dh_sweep=True):
    """The source pass; at lmax 3 the kernel runs it twice, once with only the
    dk sweep's work (h' fragments, dalpha, ds, dk) and once with only the
    dL/dh' sweep's (the hi/lo weights against dm)."""
    D, q, k, hp, dm, lse, delta, qs = (d["D"], d["q"], d["k"], d["hp"], d["dm"], d["lse"],
                                       d["delta"], d["qs"])
    RS = d["RS"]
    dk = np.zeros((16, H, DK))
    dh = np.zeros((16, D, C))
    for h in range(H):
        ka, ha = [], [[None] * 32 for _ in range(D)]
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            a0, a1 = d["tile"][g], d["tile"][g + 8]
            ka.append((k[a0, h, 2 * t:2 * t + 2], k[a1, h, 2 * t:2 * t + 2],
                       k[a0, h, 2 * t + 8:2 * t + 10], k[a1, h, 2 * t + 8:2 * t + 10]))
            for c in range(D):
                o = h * 8 + t
                ha[c][lane] = (hp[a0, c, o], hp[a1, c, o], hp[a0, c, o + 4], hp[a1, c, o + 4])
        dka = [np.zeros((32, 4)) for _ in range(2)]
        dha = [np.zeros((32, 4)) for _ in range(D)]
        for st in range(d["nst"]):
            rows = d["uni"][st * RS:(st + 1) * RS]
            qf = ldmatrix(lambda a: _bf16_pairs(q[rows[a[0]], h, 8 * a[1]:8 * a[1] + 8]),
                          lambda l: ((l & 7) + 8 * (l >> 4), (l >> 3) & 1), RS // 4)
            for nt in range(RS // 8):
                s = np.zeros((32, 4))
                mma_bf16(s, ka, [qf[l][2 * nt] for l in range(32)], [qf[l][2 * nt + 1] for l in range(32)])
                drow = lambda a: list(dm[rows[8 * nt + a[0]], a[1], h * 8 + 4 * a[2]:h * 8 + 4 * a[2] + 4])
                dp, dp2 = np.zeros((32, 4)), np.zeros((32, 4))
                if dk_sweep:
                    for c in range(0, D - 1, 2):
                        r = ldmatrix(drow, lambda l: (l & 7, c + (l >> 4), (l >> 3) & 1), 4)
                        mma_tf32(dp, ha[c], [r[l][0] for l in range(32)], [r[l][1] for l in range(32)])
                        mma_tf32(dp2, ha[c + 1], [r[l][2] for l in range(32)], [r[l][3] for l in range(32)])
                    if D % 2:
                        r = ldmatrix(drow, lambda l: (l & 7, D - 1, (l >> 3) & 1), 2)
                        mma_tf32(dp, ha[D - 1], [r[l][0] for l in range(32)], [r[l][1] for l in range(32)])
                    dp += dp2
                P, ds = np.zeros((32, 4)), np.zeros((32, 4))
                for lane in range(32):
                    g, t = lane >> 2, lane & 3
                    ca, cb = rows[8 * nt + 2 * t], rows[8 * nt + 2 * t + 1]
                    u0 = st * RS + 8 * nt + 2 * t
                    P[lane] = (2 ** (s[lane, 0] * qs - lse[ca, h]) if d["mask"][g, u0] else 0.0,
                               2 ** (s[lane, 1] * qs - lse[cb, h]) if d["mask"][g, u0 + 1] else 0.0,
                               2 ** (s[lane, 2] * qs - lse[ca, h]) if d["mask"][g + 8, u0] else 0.0,
                               2 ** (s[lane, 3] * qs - lse[cb, h]) if d["mask"][g + 8, u0 + 1] else 0.0)
                    ds[lane] = (P[lane, 0] * (dp[lane, 0] - delta[ca, h]), P[lane, 1] * (dp[lane, 1] - delta[cb, h]),
                                P[lane, 2] * (dp[lane, 2] - delta[ca, h]), P[lane, 3] * (dp[lane, 3] - delta[cb, h]))
                dsa, pa = acc_as_a(ds), acc_as_a(P)
                if dk_sweep:
                    for nd in range(2):
                        b0 = [q[rows[8 * nt + 2 * (l & 3)], h, 8 * nd + (l >> 2)] for l in range(32)]
                        b1 = [q[rows[8 * nt + 2 * (l & 3) + 1], h, 8 * nd + (l >> 2)] for l in range(32)]
                        mma_tf32(dka[nd], dsa, b0, b1)
                if dh_sweep:
                    for c in range(D):
                        b0 = [dm[rows[8 * nt + 2 * (l & 3)], c, h * 8 + (l >> 2)] for l in range(32)]
                        b1 = [dm[rows[8 * nt + 2 * (l & 3) + 1], c, h * 8 + (l >> 2)] for l in range(32)]
                        mma_tf32(dha[c], pa, b0, b1)
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            for half in range(2):
                r = g + 8 * half
                for nd in range(2):
                    for e in range(2):
                        dk[r, h, 8 * nd + 2 * t + e] = dka[nd][lane, 2 * half + e] * 0.25
                for c in range(D):
                    for e in range(2):
                        dh[r, c, h * 8 + 2 * t + e] = dha[c][lane, 2 * half + e]
    return dk, dh


@pytest.mark.parametrize("L", [1, 2, 3])
def test_source_pass_fragments(L):
    d = _data(L, seed=20 + L)
    if L >= 3:   # two sweeps: dk from the first, dL/dh' from the second
        dk, _ = _source_model(d, dk_sweep=True, dh_sweep=False)
        _, dh = _source_model(d, dk_sweep=False, dh_sweep=True)
    else:
        dk, dh = _source_model(d)
    head = np.arange(C) // 8
    for r, j in enumerate(d["tile"]):
        ref_dk = np.zeros((H, DK))
        ref_dh = np.zeros((d["D"], C))
        for u, i in enumerate(d["uni"]):
            if not d["mask"][r, u]:
                continue
            s = (d["q"][i] * d["k"][j]).sum(-1)
            a = 2.0 ** (s * d["qs"] - d["lse"][i])
            da = np.array([(d["dm"][i][:, head == hh] * d["hp"][j][:, head == hh]).sum() for hh in range(H)])
            ref_dk += (a * (da - d["delta"][i]))[:, None] * d["q"][i] * 0.25
            ref_dh += a[head][None, :] * d["dm"][i]
        assert np.allclose(dk[r], ref_dk, rtol=1e-10, atol=1e-10)
        assert np.allclose(dh[r], ref_dh, rtol=1e-10, atol=1e-10)
