"""Reads a packed weight back in row order, for comparison with the oracle.

Independent of the library's code: the index maps below follow the layout as
include/sq.h documents it.  Row layout: the arrays are row-major already.
Tiled layout (group size 128): rows padded to 16 and channels to 128; tile
t = rb * tpr + g; lane L = 4 * (row % 8) + (channel % 128) / 32 of the tile;
codes: 64 bytes per lane, four groups of words {r0 w=2m, r1 w=2m, r0 w=2m+1,
r1 w=2m+1}; sign / mask: two words per lane (row r0, row r1), channel j of the
lane's 32 at bit 8*(j%4) + j/4; scales: 16 per tile (one per row).
"""
import numpy as np
import torch

import decode_matvec_sq_b200 as sq


def _tiled_code_offsets(rows: np.ndarray, K128: int) -> np.ndarray:
    tpr = K128 // 128
    r = rows.astype(np.int64)[:, None]
    c = np.arange(K128, dtype=np.int64)[None, :]
    t = (r >> 4) * tpr + (c >> 7)
    rr, cc = r & 15, c & 127
    lane = (rr & 7) * 4 + (cc >> 5)
    j = cc & 31
    w = j >> 2
    return (t * 32 + lane) * 64 + (w >> 1) * 16 + ((w & 1) * 2 + (rr >> 3)) * 4 + (j & 3)


def _tiled_word_index(rows: np.ndarray, nwords: int) -> np.ndarray:
    tpr = nwords // 4
    r = rows.astype(np.int64)[:, None]
    word = np.arange(nwords, dtype=np.int64)[None, :]
    t = (r >> 4) * tpr + (word >> 2)
    rr = r & 15
    return (t * 32 + (rr & 7) * 4 + (word & 3)) * 2 + (rr >> 3)


def _to_row_bit_order(words: np.ndarray) -> np.ndarray:
    """Tiled bit order (channel j at bit 8*(j%4) + j/4) -> bit j = channel j."""
    w = words.astype(np.uint32)
    out = np.zeros_like(w)
    for j in range(32):
        out |= ((w >> np.uint32(8 * (j % 4) + j // 4)) & np.uint32(1)) << np.uint32(j)
    return out


def _gather(flat: torch.Tensor, index: np.ndarray) -> np.ndarray:
    ix = torch.from_numpy(index.reshape(-1)).to(flat.device)
    return flat[ix].cpu().numpy().reshape(index.shape)


def unpack(pw: "sq.PackedWeight", rows=None) -> dict:
    """Row-order arrays of the given rows (default: all N rows, plus the pad
    rows of the tiled layout under key 'pad_rows'):
      sign, mask: uint32 [n][words] (bit j of word w = channel 32w + j)
      alpha [n] float32, q [n][Kp] int8, s [n][groups] float32."""
    if rows is None:
        rows = np.arange(pw.N)
    rows = np.asarray(rows, dtype=np.int64)
    if pw.layout == sq.SQ_LAYOUT_ROWS:
        sl = torch.as_tensor(rows, device=pw.buf.device)
        out = {
            "sign": pw.sign_bits()[sl].cpu().numpy().view(np.uint32),
            "mask": None if not pw.with_mask else pw.mask_bits()[sl].cpu().numpy().view(np.uint32),
            "alpha": pw.alpha()[sl].cpu().numpy(),
            "q": pw.res_q()[sl].cpu().numpy(),
            "s": pw.res_scale()[sl].cpu().numpy(),
        }
        return out
    K128 = pw.view.res_stride
    nwords = pw.view.sign_stride
    code_flat = pw.res_q().reshape(-1)
    sign_flat = pw.sign_bits().reshape(-1)
    scale_flat = pw.res_scale().reshape(-1)
    alpha_all = pw._arr("alpha", torch.float32, (pw.rows,))
    wi = _tiled_word_index(rows, nwords)
    keep = None
    if pw.layout == sq.SQ_LAYOUT_TILES_SPARSE:
        q, nbytes_ok = _unpack_sparse_codes(pw, rows, K128)
        keep = _to_row_bit_order(_gather(pw.keep_bits().reshape(-1), wi).view(np.uint32))
    else:
        q = _gather(code_flat, _tiled_code_offsets(rows, K128))
    sign = _to_row_bit_order(_gather(sign_flat, wi).view(np.uint32))
    mask = None
    if pw.with_mask:
        mask = _to_row_bit_order(_gather(pw.mask_bits().reshape(-1), wi).view(np.uint32))
    tpr = K128 // 128
    si = ((rows[:, None] >> 4) * tpr + np.arange(tpr)[None, :]) * 16 + (rows[:, None] & 15)
    s = _gather(scale_flat, si)
    alpha = _gather(alpha_all, rows)
    out = {"sign": sign, "mask": mask, "alpha": alpha, "q": q, "s": s}
    if pw.layout == sq.SQ_LAYOUT_TILES_ASYM:
        out["z"] = _gather(pw.res_zero().reshape(-1), si)
    if keep is not None:
        out["keep"] = keep
        out["res_bytes_ok"] = nbytes_ok
    return out


def _unpack_sparse_codes(pw, rows: np.ndarray, K128: int):
    """Codes [n][K128] of the given rows from SQ_LAYOUT_TILES_SPARSE, as
    include/sq.h describes it: tile t's slot at byte 2048*t holds its kept
    codes packed lane by lane (lane L = 4*(row%8) + (channel%128)/32), within
    a lane row r0's 32 channels then row r1's in ascending channel order; the
    keep words are in the sign-bit layout.  Also whether res_bytes[t] is the
    packed size rounded up to 16 for every tile read."""
    tpr = K128 // 128
    rb = np.unique(rows >> 4)
    tiles = (rb[:, None] * tpr + np.arange(tpr)[None, :]).reshape(-1)           # [nt]
    keep_flat = pw.keep_bits().reshape(-1)
    lanes = np.arange(32)
    kw = _gather(keep_flat, (tiles[:, None, None] * 32 + lanes[None, :, None]) * 2
                 + np.arange(2)[None, None, :]).view(np.uint32)                  # [nt][32][2]
    j = np.arange(32)
    bitpos = (8 * (j % 4) + j // 4).astype(np.uint32)
    kept = ((kw[:, :, :, None] >> bitpos[None, None, None, :]) & 1).astype(np.int64)  # [nt][32][2][32]
    kept = kept.reshape(len(tiles), 32, 64)                                       # stream order
    counts = kept.sum(axis=2)                                                     # [nt][32]
    start = np.cumsum(counts, axis=1) - counts                                    # exclusive
    byte_ix = start[:, :, None] + np.cumsum(kept, axis=2) - 1                    # [nt][32][64]
    packed = _gather(pw.res_q().reshape(-1),
                     tiles[:, None] * 2048 + np.arange(2048)[None, :])           # [nt][2048]
    vals = np.take_along_axis(packed, np.clip(byte_ix.reshape(len(tiles), 2048), 0, 2047), axis=1)
    vals = np.where(kept.astype(bool), vals.reshape(len(tiles), 32, 64), 0).astype(np.int8)
    res_bytes = pw.res_bytes().cpu().numpy()[tiles]
    nbytes_ok = bool(np.all(res_bytes == (counts.sum(axis=1) + 15) // 16 * 16))
    # lane L, stream position R*32 + j -> row 8R + L//4, channel 32*(L%4) + j of the tile
    blk = np.zeros((len(tiles), 16, 128), np.int8)
    L = lanes[:, None, None]
    R = np.arange(2)[None, :, None]
    jj = j[None, None, :]
    rr = (8 * R + L // 4) + 0 * jj                                                # [32][2][32]
    cc = (32 * (L % 4) + jj) + 0 * R
    blk[:, rr.reshape(-1), cc.reshape(-1)] = vals.reshape(len(tiles), 64 * 32)
    tile_pos = {int(t): i for i, t in enumerate(tiles)}
    q = np.zeros((len(rows), K128), np.int8)
    for n, r in enumerate(rows):
        for g in range(tpr):
            q[n, 128 * g:128 * g + 128] = blk[tile_pos[int((r >> 4) * tpr + g)], r & 15]
    return q, nbytes_ok


def pad_rows_are_zero(pw: "sq.PackedWeight") -> bool:
    """The tiled layout's rows N..roundup(N,16) hold only zeros."""
    if not pw.tiled or pw.rows == pw.N:
        return True
    u = unpack(pw, rows=np.arange(pw.N, pw.rows))
    parts = [u["sign"], u["alpha"], u["q"], u["s"]] + ([u["mask"]] if pw.with_mask else []) + \
        ([u["keep"]] if "keep" in u else []) + ([u["z"]] if "z" in u else [])
    return all(not np.asarray(a).view(np.uint8).any() for a in parts)


def unpack_nvfp4(m: "sq.Nvfp4Matrix", rows=None) -> dict:
    """An NVFP4 matrix read back as one E2M1 code per byte [rows][K256] and
    one UE4M3 scale per 16-channel block [rows][K256/16], from the layout of
    include/sq.h: codes two a byte, the lower channel in the low nibble;
    scales in 512-byte chunks (rb, c), byte 16 i + 4 w + s = row
    128 rb + 32 w + i, block 4 c + s.  rows=None: every padded row."""
    v = m.view
    if rows is None:
        rows = np.arange(v.rows_pad)
    rows = np.asarray(rows, dtype=np.int64)
    cb = m.codes()[torch.as_tensor(rows, device=m.buf.device)].cpu().numpy()
    codes = np.empty((len(rows), 2 * v.code_stride), np.uint8)
    codes[:, 0::2] = cb & 15
    codes[:, 1::2] = cb >> 4
    nb = 2 * v.code_stride // 16
    b = np.arange(nb, dtype=np.int64)[None, :]
    r = rows[:, None]
    off = ((r >> 7) * v.sf_chunks + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3)
    scales = _gather(m.scales(), off)
    return {"codes": codes, "scales": scales}
