"""Test-side reader of the packed blob, written from the layout documented in mx.h.

It turns the raw bytes back into the oracle's canonical form (perm, codes8,
scales8, codes4, zeros4, scales4) so the two can be compared element by element.
It imports nothing from the CUDA library besides the layout numbers.
"""
import numpy as np


def unpack(blob: np.ndarray, L) -> dict:
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    N, K, g, n8 = L.N, L.K, L.group, L.n8
    n4, G, t8, t4, kbs = N - n8, K // g, L.t8, L.t4, K // 128
    slots = (t8 + t4) * 128

    hdr = b[:24].view(np.uint32)
    rowmap = b[L.off_rowmap:L.off_rowmap + 4 * slots].view(np.int32)
    rm8, rm4 = rowmap[:t8 * 128], rowmap[t8 * 128:]

    # 8-bit codes: [t8][kb][128 rows][8 chunks stored at c ^ (r % 8)][16]
    raw8 = b[L.off_codes8:L.off_codes8 + t8 * kbs * 128 * 128].reshape(t8, kbs, 128, 8, 16)
    r = np.arange(128)
    c = np.arange(8)
    phys = c[None, :] ^ (r[:, None] % 8)                    # [128, 8] stored position of chunk c
    logical = raw8[:, :, r[:, None], phys, :]                 # [t8, kb, 128, 8, 16]
    codes8 = logical.transpose(0, 2, 1, 3, 4).reshape(t8 * 128, K).view(np.int8)
    sc8 = b[L.off_scales8:L.off_scales8 + t8 * G * 128 * 2].view(np.uint16).reshape(t8, G, 128)
    scales8 = sc8.transpose(0, 2, 1).reshape(t8 * 128, G)

    # 4-bit codes: [t4][kb][128 rows][16 words]; word w, byte j: low nibble k=8w+j, high k=8w+4+j
    raw4 = b[L.off_codes4:L.off_codes4 + t4 * kbs * 128 * 64].reshape(t4, kbs, 128, 16, 4)
    lo = raw4 & 0x0F
    hi = raw4 >> 4
    k8 = np.concatenate([lo, hi], axis=-1)                    # [.., 16 words, 8 codes] in k order
    codes4 = k8.transpose(0, 2, 1, 3, 4).reshape(t4 * 128, K)
    sc4 = b[L.off_scales4:L.off_scales4 + t4 * G * 128 * 2].view(np.uint16).reshape(t4, G, 128)
    scales4 = sc4.transpose(0, 2, 1).reshape(t4 * 128, G)
    z4 = b[L.off_zeros4:L.off_zeros4 + t4 * G * 128].reshape(t4, G, 128)
    zeros4 = z4.transpose(0, 2, 1).reshape(t4 * 128, G)

    return dict(
        header=hdr.tolist(), rowmap=rowmap.copy(),
        perm=np.concatenate([rm8[:n8], rm4[:n4]]).astype(np.int32),
        pad8=rm8[n8:].copy(), pad4=rm4[n4:].copy(),
        codes8=codes8[:n8], scales8=scales8[:n8],
        codes4=codes4[:n4], zeros4=zeros4[:n4], scales4=scales4[:n4],
        pad_codes8=codes8[n8:], pad_scales8=scales8[n8:],
        pad_codes4=codes4[n4:], pad_zeros4=zeros4[n4:], pad_scales4=scales4[n4:],
    )
