"""Host check of the single-token kernel's copy plan (no GPU).

The kernel keeps each CTA's share of the K selected experts in shared memory,
filled by 1-D bulk copies.  ``qe_fused_plan_probe`` runs, on the host, the
same functions the kernel uses to lay out its shared memory, to list its
copies and to address its reads.  This test checks, for whole grids of CTAs
and several shapes:

* every copy is 16-byte aligned at both ends, a positive multiple of 16
  bytes, inside its source segment, inside its own shared-memory slot, and
  overlaps no other copy; each mbarrier is armed with exactly the bytes of
  the copies that complete on it;
* every read the kernel makes lies inside one copy, on the mbarrier the
  kernel waits for before that read, and maps back through that copy to
  exactly the global element it is meant to read (computed here from the
  packed layout of the public header);
* the CTAs' row ranges partition the gate/up rows and the output rows.
"""
import ctypes

import numpy as np
import pytest

B200_SMS = 148
B200_OPTIN = 232448  # 227 KiB of shared memory per block

SHAPES = [
    # H, E, K, I, bits of the K experts
    (4096, 512, 4, 1024, (4, 4, 4, 4)),
    (4096, 512, 4, 1024, (2, 4, 2, 4)),
    (256, 16, 2, 64, (4, 4)),
    (256, 16, 2, 64, (2, 2)),
    (768, 37, 3, 192, (4, 2, 4)),
    (2048, 64, 4, 512, (2, 4, 4, 2)),
    (320, 37, 3, 192, (4, 2, 2)),
    (512, 16, 4, 128, (2, 2, 4, 4)),
    (64, 8, 8, 64, (4, 2, 4, 2, 4, 2, 4, 2)),
    (1024, 64, 16, 64, (4,) * 8 + (2,) * 8),
    (64, 1024, 1, 64, (4,)),
]


def seg_layout(H, I, bits, k, rng):
    """Fake device addresses of expert k's nine segments: 16-byte aligned,
    not 256-byte aligned, with gaps between them."""
    lens = [I * H * bits // 8, I * H * bits // 8, H * I * bits // 8,
            I * H // 32, I * H // 32, I * H // 32, I * H // 32, H * I // 32, H * I // 32]
    addr, out = 0x7F0000000000 + k * 0x100000000, []
    for n in lens:
        addr += 16 * int(rng.integers(1, 64))
        out.append((addr, n))
        addr += n
    return out


def probe(lib, H, E, K, I, bits, segs, cta, sms=B200_SMS, optin=B200_OPTIN):
    geom = (ctypes.c_int * 64)()
    maxc, maxr = 4096, 1 << 19
    copies = (ctypes.c_longlong * (4 * maxc))()
    reads = (ctypes.c_longlong * (6 * maxr))()
    bits_a = (ctypes.c_int * K)(*bits)
    seg_a = (ctypes.c_uint64 * (9 * K))(*[a for s in segs for a, _ in s])
    rc = lib.qe_fused_plan_probe(H, E, K, I, sms, optin, cta, bits_a, seg_a, geom, copies, maxc, reads, maxr)
    assert rc == 0, rc
    g = list(geom)
    nc, nr = g[21], g[22]
    cp = np.frombuffer(copies, dtype=np.int64)[: 4 * nc].reshape(nc, 4)
    rd = np.frombuffer(reads, dtype=np.int64)[: 6 * nr].reshape(nr, 6)
    names = ["grid", "nq", "nrg", "np_max", "no_max", "gu_row", "gu_sc", "gu_bytes", "d_row", "d_sc", "d_bytes",
             "nbar", "off_xn", "off_cand", "off_misc", "off_bar", "off_gred", "off_ycomb", "off_gu", "off_down",
             "smem_bytes"]
    d = dict(zip(names, g))
    d["armed"] = g[24:24 + d["nbar"]]
    return d, cp, rd


@pytest.fixture(scope="module")
def plib():
    import quantized_expert_matvec_b200 as q
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qe_fused_plan_probe.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{s[0]}x{s[1]}k{s[2]}i{s[3]}-{''.join(map(str, s[4]))}"
                                               for s in SHAPES])
def test_plan_copies_and_reads(plib, shape):
    H, E, K, I, bits = shape
    rng = np.random.default_rng(H + 7 * I + K)
    segs = [seg_layout(H, I, bits[k], k, rng) for k in range(K)]
    G = B200_SMS
    ctas = range(G) if H * I <= 2048 * 512 else [0, 1, 2, 66, 67, 68, 146, 147]
    r_cover, o_cover = np.zeros(I, int), np.zeros(H, int)
    for c in range(G):
        r_cover[c * I // G:(c + 1) * I // G] += 1
        o_cover[c * H // G:(c + 1) * H // G] += 1
    assert (r_cover == 1).all() and (o_cover == 1).all()
    for cta in ctas:
        g, cp, rd = probe(plib, H, E, K, I, bits, segs, cta)
        assert g["smem_bytes"] <= B200_OPTIN
        assert g["nq"] * g["nrg"] <= 16 and g["nq"] * 32 * 32 >= H
        assert g["off_cand"] + 16 * 16 * K <= g["off_gred"]  # the top-K candidates have their own region
        assert g["nrg"] * g["nq"] <= 16 and g["gu_bytes"] >= 4 * I  # h_k is staged in expert k's slot
        r_lo, np_ = cta * I // G, (cta + 1) * I // G - cta * I // G
        o_lo, no = cta * H // G, (cta + 1) * H // G - cta * H // G
        assert np_ <= g["np_max"] and no <= g["no_max"]
        # ---- copies
        spans = []
        armed = np.zeros(g["nbar"], dtype=np.int64)
        for dst, src, nb, bar in cp:
            assert dst % 16 == 0 and src % 16 == 0 and nb % 16 == 0 and nb > 0
            assert 0 <= bar < g["nbar"]
            inside = [(a, n) for s in segs for a, n in s if a <= src and src + nb <= a + n]
            assert len(inside) == 1, (hex(src), nb)
            if bar < K:
                assert g["off_gu"] <= dst and dst + nb <= g["off_down"]
            else:
                assert g["off_down"] <= dst and dst + nb <= g["smem_bytes"]
            armed[bar] += nb
            spans.append((dst, dst + nb))
        assert list(armed) == list(g["armed"]), "an mbarrier is armed with other bytes than its copies bring"
        spans.sort()
        for (a0, a1), (b0, _) in zip(spans, spans[1:]):
            assert a1 <= b0, "copies overlap in shared memory"
        # every copy's bytes are counted on exactly one barrier, which the
        # kernel arms with their sum (recomputed here per barrier)
        expect_copies = K * ((6 if np_ else 0) + (3 if no else 0))
        assert len(cp) == expect_copies
        # ---- reads (vectorised): the copy holding each read, by shared-memory offset
        order = np.argsort(cp[:, 0])
        cd, cs, cn, cb_ = (cp[order, i] for i in range(4))
        kind, k, a, b, off, nb = (rd[:, i] for i in range(6))
        hit = np.searchsorted(cd, off, side="right") - 1
        assert (hit >= 0).all()
        assert (off + nb <= cd[hit] + cn[hit]).all(), "a read leaves the copy that holds its start"
        got, bar = cs[hit] + (off - cd[hit]), cb_[hit]
        seg = np.array([[a_ for a_, _ in segs[kk]] for kk in range(K)], dtype=np.int64)  # [K][9]
        bk = np.array(bits, dtype=np.int64)[k]
        cwb = np.where(bk == 4, 16, 8)
        want = np.zeros_like(off)
        want_bar = np.zeros_like(off)
        m0 = kind == 0  # gate/up word: a = 2j + m, b = chunk
        j, m = a // 2, a % 2
        want[m0] = (seg[k, 0] + m * (seg[k, 1] - seg[k, 0]) + (r_lo + j) * (H * bk // 8) + b * cwb)[m0]
        want_bar[m0] = k[m0]
        assert (nb[m0] == cwb[m0]).all()
        m1 = kind == 1  # gate/up scale or bias: a = 4j + s, b = group
        j, sidx = a // 4, a % 4
        want[m1] = (seg[k, 3 + np.minimum(sidx, 3)] + (r_lo + j) * (H // 32) + 2 * b)[m1]
        want_bar[m1] = k[m1]  # scale/bias runs: on the expert's gate/up mbarrier
        m2 = kind == 2  # down word: a = owned row, b = chunk
        want[m2] = (seg[k, 2] + (o_lo + a) * (I * bk // 8) + b * cwb)[m2]
        want_bar[m2] = (K + k)[m2]
        assert (nb[m2] == cwb[m2]).all()
        m3 = kind == 3  # down scale or bias: a = 2i + s, b = group
        i, sidx = a // 2, a % 2
        want[m3] = (seg[k, 7 + np.minimum(sidx, 1)] + (o_lo + i) * (I // 32) + 2 * b)[m3]
        want_bar[m3] = (K + k)[m3]
        assert (m0 | m1 | m2 | m3).all()
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, rd[bad[:5]]
        assert (bar == want_bar).all()
        n_expect = K * (np_ * 2 * (H // 32) + np_ * 4 * (H // 64) + no * (I // 32) + no * 2 * (I // 64))
        assert len(rd) == n_expect


def test_plan_rejects_shapes_beyond_the_kernel(plib):
    geom = (ctypes.c_int * 64)()
    cp = (ctypes.c_longlong * 4)()
    rd = (ctypes.c_longlong * 6)()
    bits = (ctypes.c_int * 16)(*([4] * 16))
    seg = (ctypes.c_uint64 * (9 * 16))()
    for H, E, K, I in ((8192, 64, 4, 256), (4096, 512, 4, 2048), (4096, 512, 16, 1024), (4096, 1200, 4, 1024)):
        rc = plib.qe_fused_plan_probe(H, E, K, I, B200_SMS, B200_OPTIN, 0, bits, seg, geom, cp, 1, rd, 1)
        assert rc == -2, (H, E, K, I, rc)
