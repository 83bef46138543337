"""The arena image written by archead_pack_image decodes back to the canonical
components.  The decoder below is written from the layout description in
quantized_output_head_b200/csrc/layout.h (fragment order of m16n8k16, offset
binary codes, INT5 nibble and fifth-bit planes), independently of the packer.
No GPU."""
import os

import numpy as np
import pytest

import archead_inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qoh():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_archead_build", os.path.join(ROOT, "quantized_output_head_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import quantized_output_head_b200 as m
    return m


# nibble position of fragment register a0..a3 inside a packed word
NIB_POS = (0, 2, 1, 3)


def _ru(x, m):
    return (x + m - 1) // m * m


def decode_image(img, V, d, r_c, r_r, g, g_B):
    Vp, rcp, rrp = _ru(V, 16), _ru(r_c, 64), _ru(r_r, 32)
    n_mt, n_res, n_L, n_A, n_grp = Vp // 16, d // 64, rcp // 64, rrp // 32, d // g
    seg = dict(res=n_res * 512, Lnib=n_L * 512, Lhi=n_L * 128, A=n_A * 512, sres=n_grp * 32, sL=32, sA=32)
    off, o = {}, 0
    for k, n in seg.items():
        off[k] = o
        o += n
    mblk = o
    blocks = img[: n_mt * mblk].reshape(n_mt, mblk)
    lane = np.arange(32)
    gr, cc = lane >> 2, lane & 3
    mt = np.arange(n_mt)

    def frag_cols(n_chunks, chunk_k, steps):
        # column of the low element of pair p, for [chunk, lane, step, p]
        ch = np.arange(n_chunks)[:, None, None, None]
        s = np.arange(steps)[None, None, :, None]
        p = np.arange(4)[None, None, None, :]
        return ch * chunk_k + 16 * s + 2 * cc[None, :, None, None] + 8 * (p >> 1)

    def frag_rows():
        p = np.arange(4)
        return 16 * mt[:, None, None] + gr[None, :, None] + 8 * (p[None, None, :] & 1)   # [mt, lane, p]

    out = {}
    # SC4 residual
    w = blocks[:, off["res"]: off["res"] + seg["res"]].copy().view("<u4").reshape(n_mt, n_res, 32, 4)
    q = np.zeros((Vp, d), np.int64)
    rows = frag_rows()[:, None, :, None, :]                         # [mt, 1, lane, 1, p]
    cols = frag_cols(n_res, 64, 4)[None]                           # [1, ch, lane, s, p]
    for p in range(4):
        q_ = NIB_POS[p]
        lo = (w >> (4 * q_)) & 15
        hi = (w >> (4 * q_ + 16)) & 15
        r = np.broadcast_to(rows[..., p], lo.shape)
        c = np.broadcast_to(cols[..., p], lo.shape)
        q[r, c] = lo.astype(np.int64) - 8
        q[r, c + 1] = hi.astype(np.int64) - 8
    out["q"] = q[:V]
    # INT5 core factor
    Lc = np.zeros((Vp, rcp), np.int64)
    if n_L:
        w = blocks[:, off["Lnib"]: off["Lnib"] + seg["Lnib"]].copy().view("<u4").reshape(n_mt, n_L, 32, 4)
        hb = blocks[:, off["Lhi"]: off["Lhi"] + seg["Lhi"]].copy().view("<u4").reshape(n_mt, n_L, 32)
        cols = frag_cols(n_L, 64, 4)[None]
        s_idx = np.arange(4)[None, None, None, :]
        for p in range(4):
            q_ = NIB_POS[p]
            lo = ((w >> (4 * q_)) & 15) | (((hb[..., None] >> (4 * s_idx + q_)) & 1) << 4)
            hi = ((w >> (4 * q_ + 16)) & 15) | (((hb[..., None] >> (4 * s_idx + q_ + 16)) & 1) << 4)
            r = np.broadcast_to(rows[..., p], lo.shape)
            c = np.broadcast_to(cols[..., p], lo.shape)
            Lc[r, c] = lo.astype(np.int64) - 16
            Lc[r, c + 1] = hi.astype(np.int64) - 16
    out["L"] = Lc[:V, :r_c]
    # INT8 correction factor: [mt, chunk, lane, step, half, 4 bytes]
    Ac = np.zeros((Vp, rrp), np.int64)
    if n_A:
        b = blocks[:, off["A"]: off["A"] + seg["A"]].reshape(n_mt, n_A, 32, 2, 2, 4).astype(np.int64) - 128
        ch = np.arange(n_A)[:, None, None, None]
        s = np.arange(2)[None, None, :, None]
        h = np.arange(2)[None, None, None, :]
        c = (ch * 32 + 16 * s + 2 * cc[None, :, None, None] + 8 * h)[None]          # [1, ch, lane, s, h]
        r0 = (16 * mt[:, None] + gr[None, :])[:, None, :, None, None]               # [mt, 1, lane, 1, 1]
        shp = b.shape[:5]
        R0, C0 = np.broadcast_to(r0, shp), np.broadcast_to(c, shp)
        Ac[R0, C0] = b[..., 0]
        Ac[R0, C0 + 1] = b[..., 1]
        Ac[R0 + 8, C0] = b[..., 2]
        Ac[R0 + 8, C0 + 1] = b[..., 3]
    out["A"] = Ac[:V, :r_r]
    # scales
    sres = blocks[:, off["sres"]: off["sres"] + seg["sres"]].copy().view("<u2").reshape(n_mt, n_grp, 8, 2)
    s_res = np.zeros((Vp, n_grp), np.uint16)
    for half in range(2):
        rr = 16 * mt[:, None, None] + np.arange(8)[None, None, :] + 8 * half
        s_res[np.broadcast_to(rr, sres.shape[:3]), np.broadcast_to(np.arange(n_grp)[None, :, None], sres.shape[:3])] = \
            sres[..., half]
    out["s_res"] = s_res[:V]
    for key in ("sL", "sA"):
        sv = blocks[:, off[key]: off[key] + 32].copy().view("<u2").reshape(n_mt, 8, 2)
        full = np.zeros(Vp, np.uint16)
        full[(16 * mt[:, None] + np.arange(8)[None, :]).ravel()] = sv[..., 0].ravel()
        full[(16 * mt[:, None] + np.arange(8)[None, :] + 8).ravel()] = sv[..., 1].ravel()
        out["s_L" if key == "sL" else "s_A"] = full[:V]
    # shared region
    a = _ru(n_mt * mblk, 256)
    out["R"] = img[a: a + r_c * d].view(np.int8).reshape(r_c, d)
    a += _ru(rcp * d, 256)
    out["s_R"] = img[a: a + 2 * r_c].copy().view("<u2")
    a += _ru(rcp * 2, 256)
    out["B"] = img[a: a + r_r * d].view(np.int8).reshape(r_r, d)
    a += _ru(rrp * d, 256)
    ngB = d // g_B
    out["s_B"] = img[a: a + 2 * r_r * ngB].copy().view("<u2").reshape(r_r, ngB)
    # padding rows hold code 0 and scale 0
    out["_pad_ok"] = bool(np.all(q[V:] == 0) and np.all(Lc[V:] == 0) and np.all(s_res[V:] == 0))
    return out


@pytest.mark.parametrize("shape", [
    (1024, 256, 32, 8, 64, 64),
    (1000, 320, 100, 40, 16, 10),
    (33, 128, 0, 0, 128, 1),
    (48, 64, 64, 32, 64, 64),
])
def test_image_decodes_to_components(qoh, shape):
    comps = gen.random_components(gen.HeadShape(*shape), seed=sum(shape))
    img = qoh.archead_pack_image(*shape, comps)
    assert img.size == qoh.archead_arena_bytes(*shape)
    dec = decode_image(img, *shape)
    for k in ("q", "L", "A", "R", "B"):
        np.testing.assert_array_equal(dec[k], comps[k].astype(np.int64), err_msg=k)
    absent = {"s_L"} if shape[2] == 0 else set()
    absent |= {"s_A"} if shape[3] == 0 else set()
    for k in ("s_res", "s_L", "s_A", "s_R", "s_B"):
        if comps[k].size and k not in absent:
            np.testing.assert_array_equal(dec[k], comps[k], err_msg=k)
    assert dec["_pad_ok"]


def test_image_size_at_qwen_shape_is_payload(qoh):
    # every per-row byte of the Qwen-shaped head is payload: 16 rows x 2500 B per m-tile
    V, d, r_c, r_r, g, g_B = 151936, 4096, 512, 64, 128, 128
    per_row = 5 * r_c // 8 + 2 + d // 2 + 2 * d // g + r_r + 2
    assert per_row == 2500
    assert qoh.archead_arena_bytes(V, d, r_c, r_r, g, g_B) >= V * per_row
