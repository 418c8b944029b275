"""Byte layout of the compressed paged KV cache (one 16-token page per KV head).

Oracle module (test infrastructure only). The pages give no byte format (the
llama.cpp fork's own formats are not shown), so this layout is a reading,
chosen so that a GPU warp can turn the bytes straight into tensor-core
operands (key codes and sign bits: the A operand of a 16-token tile, one token
per row; value codes: the A operand of the transposed value tile; the norms of
tokens g and g + 8 share one 32-bit word). It is written out here from its definition, bit by bit.

Block for one (page, KV head), head_dim d = 128, m = 128 sketch rows, with
b_k-bit key codes and b_v-bit value codes:

    offset 0                 K codes   256*b_k bytes = 32 lane chunks of 8*b_k bytes
    offset 256*b_k           sign bits 256 bytes     = 32 lane chunks of 8 bytes
    offset 256*(b_k+1)       V codes   256*b_v bytes = 32 lane chunks of 8*b_v bytes
    offset 256*(b_k+b_v+1)   norms     96 bytes: ||k|| fp16[16], gamma fp16[16], ||v|| fp16[16];
                             token tau sits at entry 2*(tau & 7) + (tau >> 3) of each array

Words are 32-bit little endian; bit x of word w of a section is bit (x mod 8)
of byte 4w + x // 8.

Key codes and sign bits of token tau in 0..15, coordinate (or sketch row) i:
    g = tau & 7, th = tau >> 3 (token half), kt = i >> 5, sub = (i >> 4) & 1,
    t = (i >> 2) & 3, q = i & 3, lane = 4g + t, j = 2 kt + sub (0..7).
    Lane chunk words: 2*b_k per lane (K) / 2 per lane (signs), token half th
    first owns words [th*b_k, th*b_k + b_k) (K) / word th (signs).
    Sign bit: bit 8q + j of the token-half word.
    K code bit p (p = 0 is the least significant) of nibble q of "selector" j:
      b=2: word j>>2, bit 16*(j&1) + 4q + 2*((j>>1)&1) + p
      b=3: j<6: word j>>1, bit 16*(j&1) + 4q + p;
           j>=6: word p, bit 4*(4*(j-6)+q) + 3
      b=4: word j>>1, bit 16*(j&1) + 4q + p

Value codes of token tau, coordinate i:
    mt = i >> 4, hf = (i >> 3) & 1, r = i & 7, tg = tau >> 3, t = (tau >> 1) & 3,
    e = tau & 1, lane = 4r + t, s = 2 mt + tg (0..15), n = 2 hf + e (0..3).
    Lane chunk words: 2*b_v per lane. V code bit p of nibble n of selector s:
      b=2: word s>>2, bit 16*(s&1) + 4n + 2*((s>>1)&1) + p
      b=3: G = s>>3, s' = s&7; s'<6: word 3G + (s'>>1), bit 16*(s'&1) + 4n + p;
           s'>=6: word 3G + p, bit 4*(4*(s'-6)+n) + 3
      b=4: word s>>1, bit 16*(s&1) + 4n + p

Codes are stored as the ascending centroid index (0 = most negative centroid).

q8_0 keys (b_k = 8; see q8.py) use the same block frame with other key sections:

    offset 0                 K values  2048 bytes  = 32 lane chunks of 64 int8
    offset 2048              K scales  128 bytes: fp16 [16 tokens x 4 blocks of 32 coordinates]
    offset 2176              V codes   256*b_v bytes (as above)
    offset 2176 + 256*b_v    norms     32 bytes: ||v|| fp16[16], token tau at entry 2*(tau & 7) + (tau >> 3)

    int8 value of token tau, coordinate i (g, th, kt, sub, t, q, lane as for codes):
        byte 64*lane + 32*th + 8*kt + 4*sub + q
    scale of token tau, block kt = i >> 5: fp16 entry 8*(tau & 7) + 4*(tau >> 3) + kt
"""

from functools import lru_cache

import numpy as np

PAGE = 16
D = 128


def section_offsets(bk: int, bv: int):
    if bk == 8:                                   # q8_0 keys: values, scales
        return {"k": 0, "sign": 2048, "v": 2176, "norm": 2176 + 256 * bv}
    return {"k": 0, "sign": 256 * bk, "v": 256 * (bk + 1), "norm": 256 * (bk + bv + 1)}


def block_bytes(bk: int, bv: int) -> int:
    """Bytes of one (page, KV head) block: 16 tokens x (16 b_k + 16 + 4 + 16 b_v + 2);
    q8_0 keys: 16 tokens x (128 + 8 + 16 b_v + 2)."""
    if bk == 8:
        return 2176 + 256 * bv + 32
    return 256 * (bk + bv + 1) + 96


def _code_bit(b: int, j: int, q: int, p: int):
    """(word, bit) of code bit p for nibble q of selector j inside one group of b words."""
    if b == 2:
        return j >> 2, 16 * (j & 1) + 4 * q + 2 * ((j >> 1) & 1) + p
    if b == 3:
        if j < 6:
            return j >> 1, 16 * (j & 1) + 4 * q + p
        return p, 4 * (4 * (j - 6) + q) + 3
    if b == 4:
        return j >> 1, 16 * (j & 1) + 4 * q + p
    raise ValueError("bits must be 2, 3 or 4")


@lru_cache(maxsize=None)
def k_bit_index(bk: int) -> np.ndarray:
    """[16, 128, bk] absolute bit index (within the block) of every key-code bit."""
    out = np.zeros((PAGE, D, bk), dtype=np.int64)
    for tau in range(PAGE):
        g, th = tau & 7, tau >> 3
        for i in range(D):
            kt, sub, t, q = i >> 5, (i >> 4) & 1, (i >> 2) & 3, i & 3
            lane, j = 4 * g + t, 2 * kt + sub
            base = lane * 2 * bk + th * bk
            for p in range(bk):
                w, bit = _code_bit(bk, j, q, p)
                out[tau, i, p] = 32 * (base + w) + bit
    return out


@lru_cache(maxsize=None)
def sign_bit_index(bk: int) -> np.ndarray:
    """[16, 128] absolute bit index of every QJL sign bit."""
    off = 8 * section_offsets(bk, 2)["sign"]
    out = np.zeros((PAGE, D), dtype=np.int64)
    for tau in range(PAGE):
        g, th = tau & 7, tau >> 3
        for r in range(D):
            kt, sub, t, q = r >> 5, (r >> 4) & 1, (r >> 2) & 3, r & 3
            lane, j = 4 * g + t, 2 * kt + sub
            out[tau, r] = off + 32 * (lane * 2 + th) + 8 * q + j
    return out


def _v_code_bit(b: int, s: int, n: int, p: int):
    if b == 3:
        grp, s2 = s >> 3, s & 7
        w, bit = _code_bit(3, s2, n, p)
        return 3 * grp + w, bit
    return _code_bit(b, s, n, p)


@lru_cache(maxsize=None)
def v_bit_index(bk: int, bv: int) -> np.ndarray:
    """[16, 128, bv] absolute bit index of every value-code bit."""
    off = 8 * section_offsets(bk, bv)["v"]
    out = np.zeros((PAGE, D, bv), dtype=np.int64)
    for tau in range(PAGE):
        tg, t, e = tau >> 3, (tau >> 1) & 3, tau & 1
        for i in range(D):
            mt, hf, r = i >> 4, (i >> 3) & 1, i & 7
            lane, s, n = 4 * r + t, 2 * mt + tg, 2 * hf + e
            base = lane * 2 * bv
            for p in range(bv):
                w, bit = _v_code_bit(bv, s, n, p)
                out[tau, i, p] = off + 32 * (base + w) + bit
    return out


def _set_bits(block: np.ndarray, idx: np.ndarray, values: np.ndarray):
    idx = idx.ravel()
    values = values.ravel().astype(bool)
    byte = idx // 8
    mask = (1 << (idx % 8)).astype(np.uint8)
    np.bitwise_and.at(block, byte, ~mask)
    np.bitwise_or.at(block, byte[values], mask[values])


def _get_bits(block: np.ndarray, idx: np.ndarray) -> np.ndarray:
    return (block[idx // 8] >> (idx % 8).astype(np.uint8)) & 1


def norm_slot(tau: int) -> int:
    """Entry of token tau in each 16-entry fp16 norm array."""
    return 2 * (tau & 7) + (tau >> 3)


def write_token(block, tau, bk, bv, k_codes, sign_bits, v_codes, k_norm16, gamma16, v_norm16):
    """Store one token's fields into a block (uint8 view), leaving other tokens' bits alone."""
    kb = k_bit_index(bk)[tau]                      # [128, bk]
    kval = (np.asarray(k_codes)[:, None] >> np.arange(bk)) & 1
    _set_bits(block, kb, kval)
    _set_bits(block, sign_bit_index(bk)[tau], np.asarray(sign_bits))
    vb = v_bit_index(bk, bv)[tau]
    vval = (np.asarray(v_codes)[:, None] >> np.arange(bv)) & 1
    _set_bits(block, vb, vval)
    no = section_offsets(bk, bv)["norm"]
    e = norm_slot(tau)
    for arr_off, val in ((0, k_norm16), (32, gamma16), (64, v_norm16)):
        h = np.array([val], dtype=np.float16).view(np.uint8)
        block[no + arr_off + 2 * e: no + arr_off + 2 * e + 2] = h


def read_page(block, bk, bv):
    """Unpack all 16 tokens of a block: k_codes, sign_bits, v_codes [16,128] and fp16 norms [16]."""
    block = np.asarray(block, dtype=np.uint8)
    kb = k_bit_index(bk)
    k_codes = np.sum(_get_bits(block, kb).astype(np.int64) << np.arange(bk), axis=-1)
    sign_bits = _get_bits(block, sign_bit_index(bk)).astype(np.int64)
    vb = v_bit_index(bk, bv)
    v_codes = np.sum(_get_bits(block, vb).astype(np.int64) << np.arange(bv), axis=-1)
    no = section_offsets(bk, bv)["norm"]
    norms = block[no:no + 96].view(np.float16).astype(np.float64).reshape(3, PAGE)
    order = [norm_slot(tau) for tau in range(PAGE)]
    return k_codes, sign_bits, v_codes, norms[0][order], norms[1][order], norms[2][order]


# ------------------------------------------------------------------ q8_0 keys
@lru_cache(maxsize=None)
def q8_byte_index() -> np.ndarray:
    """[16, 128] byte of every int8 key value."""
    out = np.zeros((PAGE, D), dtype=np.int64)
    for tau in range(PAGE):
        g, th = tau & 7, tau >> 3
        for i in range(D):
            kt, sub, t, q = i >> 5, (i >> 4) & 1, (i >> 2) & 3, i & 3
            out[tau, i] = 64 * (4 * g + t) + 32 * th + 8 * kt + 4 * sub + q
    return out


def q8_scale_entry(tau: int, kt: int) -> int:
    """fp16 entry (within the scale section) of token tau's block kt."""
    return 8 * (tau & 7) + 4 * (tau >> 3) + kt


def write_token_q8(block, tau, bv, values, scales16, v_codes, v_norm16):
    """Store one token of a q8_0-key block (uint8 view), leaving other tokens alone."""
    idx = q8_byte_index()[tau]
    block[idx] = (np.asarray(values, dtype=np.int64) & 0xFF).astype(np.uint8)
    off = section_offsets(8, bv)
    for kt in range(4):
        e = off["sign"] + 2 * q8_scale_entry(tau, kt)
        block[e:e + 2] = np.array([scales16[kt]], dtype=np.float16).view(np.uint8)
    vb = v_bit_index(8, bv)[tau]
    vval = (np.asarray(v_codes)[:, None] >> np.arange(bv)) & 1
    _set_bits(block, vb, vval)
    e = off["norm"] + 2 * norm_slot(tau)
    block[e:e + 2] = np.array([v_norm16], dtype=np.float16).view(np.uint8)


def read_page_q8(block, bv):
    """Unpack a q8_0-key block: values [16,128], scales16 [16,4], v_codes [16,128], v_norm [16]."""
    block = np.asarray(block, dtype=np.uint8)
    values = block[q8_byte_index()].view(np.int8).astype(np.int64)
    off = section_offsets(8, bv)
    sc = block[off["sign"]:off["sign"] + 128].view(np.float16).astype(np.float64)
    scales = np.array([[sc[q8_scale_entry(tau, kt)] for kt in range(4)] for tau in range(PAGE)])
    vb = v_bit_index(8, bv)
    v_codes = np.sum(_get_bits(block, vb).astype(np.int64) << np.arange(bv), axis=-1)
    nv = block[off["norm"]:off["norm"] + 32].view(np.float16).astype(np.float64)
    v_norm = np.array([nv[norm_slot(tau)] for tau in range(PAGE)])
    return values, scales, v_codes, v_norm
