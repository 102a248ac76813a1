"""CPU models of the index maps of the GPU kernels (regression pins): the fused
decode kernel's fragment mapping, shared-memory plan, copies and table lookups,
and the tensor-core decoders.

Each model restates, in numpy and exact arithmetic, how a kernel's threads
place data -- which packed bytes a thread decodes, where it stores them, which
MMA fragment registers they feed (PTX m16n8k16 layout) -- and checks the
result against the plain definition.  The GPU tests check the compiled
kernels against the oracle; these pin the index arithmetic itself.
"""
import numpy as np
import pytest

from oracle import nf4

CB = nf4.codebook_f64()


def _mma(acc, A, B):
    """One m16n8k16: A[lane] = 4 pairs (a0..a3), B[lane] = 2 pairs; acc[lane] += 4 outputs."""
    Am = np.zeros((16, 16))
    Bm = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        a0, a1, a2, a3 = A[lane]
        b0, b1 = B[lane]
        Am[g, 2 * t:2 * t + 2] = a0
        Am[g + 8, 2 * t:2 * t + 2] = a1
        Am[g, 2 * t + 8:2 * t + 10] = a2
        Am[g + 8, 2 * t + 8:2 * t + 10] = a3
        Bm[2 * t:2 * t + 2, g] = b0
        Bm[2 * t + 8:2 * t + 10, g] = b1
    D = Am @ Bm
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        acc[lane] += [D[g, 2 * t], D[g, 2 * t + 1], D[g + 8, 2 * t], D[g + 8, 2 * t + 1]]


def _pair(byte):
    """An NF4 byte as (element 2i, element 2i+1): the high nibble first."""
    return CB[byte >> 4], CB[byte & 15]


def _layer_rows(seed, rows, K):
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    absmax = rng.random((rows, K // 64)) + 0.5
    # the definition, through the oracle's own unpacking (independent of _pair)
    W = CB[nf4.unpack_codes(packed).reshape(rows, K)] * np.repeat(absmax, 64, axis=1)
    return packed, absmax, W


@pytest.mark.parametrize("K", [128, 192, 2880])
def test_decode_block_fragment_mapping(K):
    """csrc/decode.cu block_mma: in each 64-element k-block thread (g, t) holds
    packed bytes [8t, 8t+8) of rows g and g+8 (elements 16t .. 16t+15) and the
    16 matching x values of token column g; MMA j takes bytes 2j and 2j+1 and
    x words 2j, 2j+1; the four MMAs of a block go into a zeroed partial that
    the block's fp32 absmax of each row scales afterwards."""
    packed, absmax, W = _layer_rows(1, 16, K)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, K))
    KB = K // 64
    acc = np.zeros((32, 4))
    for kb in range(KB):
        d = np.zeros((32, 4))
        for j in range(4):
            A = [None] * 32
            B = [None] * 32
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                r0 = packed[g, kb * 32 + 8 * t: kb * 32 + 8 * t + 8]
                r1 = packed[g + 8, kb * 32 + 8 * t: kb * 32 + 8 * t + 8]
                xs = x[g, kb * 64 + 16 * t: kb * 64 + 16 * t + 16]
                A[lane] = (_pair(r0[2 * j]), _pair(r1[2 * j]), _pair(r0[2 * j + 1]), _pair(r1[2 * j + 1]))
                B[lane] = ((xs[4 * j], xs[4 * j + 1]), (xs[4 * j + 2], xs[4 * j + 3]))
            _mma(d, A, B)
        for lane in range(32):
            g = lane >> 2
            acc[lane] += d[lane] * np.array([absmax[g, kb], absmax[g, kb], absmax[g + 8, kb], absmax[g + 8, kb]])
    got = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        got[g, 2 * t], got[g, 2 * t + 1], got[g + 8, 2 * t], got[g + 8, 2 * t + 1] = acc[lane]
    ref = W @ x.T
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


# ---- csrc/decode.cu: the fused kernel's shared-memory plan and copies -------------
SMEM_LIMIT = 227 * 1024 - 1024   # opt-in dynamic shared memory minus the kernel's reserve


def _al(v, a):
    return (v + a - 1) // a * a


def _copy_stride(K):
    return 2 * K + 32


def _am_stride(KB):
    b = 16 * KB
    return b + (144 - b % 128) % 128


def _gu_stage(H):
    return 8 * _copy_stride(H) + 8 * _am_stride(H // 64)


def _dn_block(I):
    return 4 * _copy_stride(I) + 4 * _am_stride(I // 64)


def _plan(M, k, E, H, I, r):
    KB, KBI = H // 64, I // 64
    spw = -(-((KB + 1) // 2) // 8)
    gu, dn = _gu_stage(H), _dn_block(I)
    dpe = max(1, min(gu // dn, 4, 48 // KBI))
    ppw = -(-(dpe * KBI) // 16)
    slot = _al(max(gu, dpe * dn), 128)
    S = M * k
    o = 256 * 256  # the byte -> bf16x2 table, the partial sums in its entries' upper halves
    for n in (S * 4, S * 4, E * 4, S * 4, S * 8 * 4):
        o = _al(o + n, 16)
    if r:
        o = _al(o + S * r * 4, 16)
    fixed = _al(o, 128) + 2 * 32 * 8
    stages = min((SMEM_LIMIT - fixed) // slot, 32) & ~1
    ring = _al(_al(o + (2 * stages + 4) * 8, 16), 128)
    return dict(spw=spw, ppw=ppw, dpe=dpe, slot=slot, stages=stages, ring=ring, total=ring + stages * slot)


def _block_copies(K, row0, dst, am_dst):
    """(lane_c, dst, src byte offset in packed / absmax, bytes, is_absmax) of one staged block of 16 rows."""
    KB = K // 64
    out = []
    for lc in range(8):
        c = lc & 3
        row = row0 + 4 * c
        if lc < 4:
            out.append((dst + c * _copy_stride(K), row * (K // 2), 2 * K, False))
        else:
            out.append((am_dst + c * _am_stride(KB), row * KB * 4, 16 * KB, True))
    return out


def _check_copies(copies, slot, packed_bytes, absmax_bytes):
    written = set()
    for dst, src, n, is_am in copies:
        assert dst % 16 == 0 and src % 16 == 0 and n % 16 == 0 and dst + n <= slot
        assert src + n <= (absmax_bytes if is_am else packed_bytes)
        assert not (set(range(dst, dst + n)) & written), "copies overlap"
        written.update(range(dst, dst + n))
    return written


DECODE_SHAPES = [
    # (M, k, E, H, I, r): the decode rows of the bench and every decode shape the GPU tests run
    (1, 8, 64, 2048, 1024, 0), (4, 8, 64, 2048, 1024, 0), (8, 8, 64, 2048, 1024, 0),
    (1, 4, 32, 2880, 2880, 0), (8, 4, 32, 2880, 2880, 0), (8, 8, 128, 2048, 768, 8), (3, 8, 128, 2048, 768, 8),
    (1, 2, 8, 256, 128, 0), (8, 2, 8, 256, 128, 0), (5, 3, 12, 192, 320, 0), (3, 2, 6, 128, 192, 8),
    (2, 6, 40, 448, 128, 0), (7, 32, 33, 128, 64, 0), (8, 2, 8, 2880, 704, 0), (8, 2, 8, 4096, 128, 0),
    (8, 8, 512, 128, 64, 0), (6, 1, 8, 256, 192, 0), (7, 4, 4, 256, 192, 0), (4, 2, 4, 3072, 3072, 16),
]


@pytest.mark.parametrize("shape", DECODE_SHAPES)
def test_decode_fused_plan_copies_and_reads_stay_in_bounds(shape):
    """Every bulk copy of a stage is 16-byte aligned at both ends, a multiple of
    16 bytes, inside its slot, disjoint from the others and inside the source
    stack; the transaction count equals the bytes copied; every fragment and
    absmax read of the math warps lies in bytes the copies wrote; the plan
    fits the shared memory and holds an even number of stages."""
    M, k, E, H, I, r = shape
    pl = _plan(M, k, E, H, I, r)
    assert pl["total"] <= SMEM_LIMIT and pl["stages"] >= 2 and pl["stages"] % 2 == 0
    assert pl["spw"] <= 4 and pl["ppw"] <= 3 and pl["dpe"] <= 4 and pl["ring"] % 128 == 0 and pl["slot"] % 128 == 0
    KB, KBI = H // 64, I // 64
    cs, am0 = _copy_stride(H), 8 * _copy_stride(H)
    # phase 1: the first and the last item of the last expert
    for rb in (0, I // 16 - 1):
        grow = (E - 1) * 2 * I + rb * 16
        copies = []
        for blk in range(2):
            copies += _block_copies(H, grow + blk * I, blk * 4 * cs, am0 + blk * 4 * _am_stride(KB))
        written = _check_copies(copies, pl["slot"], E * 2 * I * (H // 2), E * 2 * I * KB * 4)
        assert sum(n for _, _, n, _ in copies) == 32 * (H // 2) + 32 * KB * 4
        for g in range(8):
            for t in range(4):
                for T in range(2):
                    rr, cg = 2 * T + (g >> 2), g & 3
                    for kb in range(KB):
                        off = rr * (H // 2) + kb * 32 + 8 * t
                        for base in (cg * cs, (4 + cg) * cs):
                            assert set(range(base + off, base + off + 8)) <= written
                        for ci in (cg, 4 + cg):
                            a = am0 + ci * _am_stride(KB) + (rr * KB + kb) * 4
                            assert set(range(a, a + 4)) <= written
                        # the row read is column 4 (g % 4) + 2T + g / 4 of the item, in its copy
                        assert 4 * cg + rr == 4 * (g & 3) + 2 * T + (g >> 2)
    # phase 2: the last row block of the last experts, every expert count of a stage
    exp, csd, amd = _dn_block(I), _copy_stride(I), 4 * _copy_stride(I)
    for ne in range(1, pl["dpe"] + 1):
        copies = []
        for ei in range(ne):
            row0 = (E - 1 - ei) * H + (H // 16 - 1) * 16
            copies += _block_copies(I, row0, ei * exp, ei * exp + amd)
        written = _check_copies(copies, pl["slot"], E * H * (I // 2), E * H * KBI * 4)
        assert sum(n for _, _, n, _ in copies) == ne * (16 * (I // 2) + 16 * KBI * 4)
        assert ne * KBI <= 16 * pl["ppw"]
        for ei in range(ne):
            for g in range(8):
                for t in range(4):
                    cg, rr = g & 3, g >> 2
                    for kb in range(KBI):
                        off = ei * exp + cg * csd + rr * (I // 2) + kb * 32 + 8 * t
                        for o in (off, off + I):
                            assert set(range(o, o + 8)) <= written
                        for row in (rr, rr + 2):
                            a = ei * exp + amd + cg * _am_stride(KBI) + (row * KBI + kb) * 4
                            assert set(range(a, a + 4)) <= written


def _lut_address(word, byte, lane):
    """csrc/decode.cu block_mma: __byte_perm(word, 4 lane, 0x5504 | byte << 4)."""
    return _byte_perm(word, 4 * lane, 0x5504 | (byte << 4))


def _red_offset(i):
    return ((i >> 3) << 8) + 128 + ((i & 7) << 4)


def test_decode_table_lookup_address_and_partial_sum_slots():
    """The decode table: the byte permute of a packed word puts byte `byte` of
    the word at bits 8-15 above 4 lane, i.e. entry b of lane l at 256 b + 4 l;
    a warp's 32 lookups hit 32 distinct banks whatever the bytes; every address
    lies in the lower half of its 256-byte entry.  The partial sums take the
    upper halves: 2048 float4 slots (phase 1's [group][parity][warp][tile][lane]
    and phase 2's [warp][lane]) inside the 64 KB table, disjoint from the
    entries and from one another, each quarter warp's slots one 128-byte row."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        words = rng.integers(0, 2**32, size=32, dtype=np.uint64)
        for byte in range(4):
            addrs = [_lut_address(int(w), byte, lane) for lane, w in enumerate(words)]
            for lane, (w, a) in enumerate(zip(words, addrs)):
                b = (int(w) >> (8 * byte)) & 255
                assert a == 256 * b + 4 * lane
            assert len({(a // 4) % 32 for a in addrs}) == 32
            assert all(a % 256 < 128 and a < 256 * 256 for a in addrs)
    slots = [_red_offset(i) for i in range(2 * 2 * 8 * 2 * 32)]
    assert all(o % 256 >= 128 and o + 16 <= 256 * 256 for o in slots)
    assert len(set(slots)) == len(slots)
    for q in range(0, len(slots), 8):
        row = slots[q:q + 8]
        assert row == list(range(row[0], row[0] + 128, 16))


@pytest.mark.parametrize("K", [128, 192, 320, 448, 704, 768, 1024, 2048, 2880, 3072, 4096])
def test_decode_fused_fragment_reads_are_conflict_free(K):
    """Copies 32 mod 128 bytes apart: the 8-byte fragment loads of each
    half-warp (MMA rows g = 4h .. 4h+3 -> copies 0-3, one row each; t = 0..3)
    hit 32 distinct banks; the absmax loads of the 8 rows g touch at most two
    addresses per bank."""
    cs, asz = _copy_stride(K), _am_stride(K // 64)
    assert cs % 128 == 32 and asz % 128 == 16
    KB = K // 64
    for kb in range(KB):
        for half in range(2):
            for r2 in (0, 2):
                banks = []
                for g in range(4 * half, 4 * half + 4):
                    for t in range(4):
                        w = ((g & 3) * cs + ((g >> 2) + r2) * (K // 2) + kb * 32 + 8 * t) // 4
                        banks += [w % 32, (w + 1) % 32]
                assert len(set(banks)) == 32
        words = [((g & 3) * asz + ((g >> 2) * KB + kb) * 4) // 4 for g in range(8)]
        per_bank = {}
        for w in words:
            per_bank.setdefault(w % 32, set()).add(w)
        assert max(len(v) for v in per_bank.values()) <= 2


def test_warp_mma_gemm_fragment_mapping():
    """csrc/gemm_mma.cu: lane t owns physical k [8t, 8t+8) of each 32-k chunk --
    one 32-bit word of packed nibbles per row and one 16-byte vector of x -- the
    chunk's two MMAs accumulate unscaled codebook values, folded into the result
    times the row's absmax once per 64-k block."""
    K = 192
    packed, absmax, W = _layer_rows(3, 16, K)
    x = np.random.default_rng(4).standard_normal((8, K))
    acc = np.zeros((32, 4))
    for kb in range(K // 64):
        tmp = np.zeros((32, 4))
        for c in range(2):
            A0, A1, B0, B1 = [], [], [], []
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                b0 = packed[g, kb * 32 + 16 * c + 4 * t: kb * 32 + 16 * c + 4 * t + 4]
                b1 = packed[g + 8, kb * 32 + 16 * c + 4 * t: kb * 32 + 16 * c + 4 * t + 4]
                A0.append((_pair(b0[0]), _pair(b1[0]), _pair(b0[1]), _pair(b1[1])))
                A1.append((_pair(b0[2]), _pair(b1[2]), _pair(b0[3]), _pair(b1[3])))
                kx = kb * 64 + 32 * c + 8 * t
                B0.append(((x[g, kx], x[g, kx + 1]), (x[g, kx + 2], x[g, kx + 3])))
                B1.append(((x[g, kx + 4], x[g, kx + 5]), (x[g, kx + 6], x[g, kx + 7])))
            _mma(tmp, A0, B0)
            _mma(tmp, A1, B1)
        for lane in range(32):
            g = lane >> 2
            acc[lane] += tmp[lane] * [absmax[g, kb], absmax[g, kb], absmax[g + 8, kb], absmax[g + 8, kb]]
    got = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        got[g, 2 * t], got[g, 2 * t + 1], got[g + 8, 2 * t], got[g + 8, 2 * t + 1] = acc[lane]
    ref = W @ x.T
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


@pytest.mark.parametrize("halves,tpr", [(2, 2), (1, 4)])
def test_tensor_core_decoders_fill_the_swizzled_k_major_tile(halves, tpr):
    """csrc/gemm_tc.cu decoders: thread dt decodes row dt / tpr of the tile (half
    = row / 128) and its part dt % tpr of the 64-k block (32 / tpr packed bytes,
    one 32-bit word = 8 elements = one 16-byte chunk), scales by the block's
    absmax and stores chunk c of row ri at byte (ri / 8) * 1024 + (ri % 8) * 128
    + ((c ^ (ri % 8)) * 16) of its half: read back through the same 128-byte
    swizzle, the tile is the block's W rows."""
    rows = 128 * halves
    packed, absmax, W = _layer_rows(5, rows, 64)      # one 64-k block per row
    tile = np.full(rows * 64, np.nan)                   # bf16 slots of the A stage
    nchunks = 8 // tpr
    for dt in range(512):
        r, kq = dt // tpr, dt % tpr
        half, ri = r >> 7, r & 127
        src = packed[r, kq * (32 // tpr): (kq + 1) * (32 // tpr)]
        for c in range(nchunks):
            w = src[4 * c: 4 * c + 4]
            vals = []
            for byte in w:                               # decode4 on the low, then the high half-word
                vals += [v * absmax[r, 0] for v in _pair(byte)]
            chunk = kq * nchunks + c
            base = half * 128 * 64 + (ri >> 3) * 512 + (ri & 7) * 64 + ((chunk ^ (ri & 7)) << 3)
            assert np.isnan(tile[base:base + 8]).all(), "slot written twice"
            tile[base:base + 8] = vals
    assert not np.isnan(tile).any()
    for r in range(rows):
        half, ri = r >> 7, r & 127
        for k in range(64):
            addr = half * 128 * 64 + (ri >> 3) * 512 + (ri & 7) * 64 + (((k // 8) ^ (ri & 7)) << 3) + (k % 8)
            assert tile[addr] == W[r, k]


def _byte_perm(x: int, y: int, s: int) -> int:
    """PTX prmt (default mode): result byte i = byte (selector nibble i & 7) of
    the 8-byte value y:x, or that byte's sign replicated when the nibble's bit 3 is set."""
    src = (x & 0xFFFFFFFF) | ((y & 0xFFFFFFFF) << 32)
    out = 0
    for i in range(4):
        n = (s >> (4 * i)) & 0xF
        b = (src >> (8 * (n & 7))) & 0xFF
        if n & 8:
            b = 0xFF if b & 0x80 else 0x00
        out |= b << (8 * i)
    return out


@pytest.mark.parametrize("table", ["nf4", "fp4", "mxfp4"])
def test_tensor_core_byte_permute_decoder_is_a_table_lookup(table):
    """csrc/gemm_tc.cu decode4 for every 16-bit input: the codebook's bf16
    patterns split into low and high bytes (four entries per word), two
    permutes look up entries 0-7 and 8-15 by the nibbles' low three bits, a
    third keeps the half each nibble's top bit names, two more interleave the
    bytes -> (element 2i, 2i+1) and (2i+2, 2i+3), the high nibble of a byte
    being the lower-index element.  Checked against direct lookup for the NF4
    and the FP4 (e2m1 / 6, with -0 at code 8) tables, and for MXFP4 codes (the
    e2m1 values, element 2i in the LOW nibble: the other final selectors)."""
    from oracle import fp4, mxfp4
    from quantized_moe_expert_nf4_b200 import workloads
    if table == "nf4":
        cb32 = nf4.NF4_CODEBOOK
    elif table == "fp4":
        cb32 = fp4.codebook_f64().astype(np.float32)
    else:
        cb32 = mxfp4.e2m1_table().astype(np.float32)
    sel0, sel1 = (0x5140, 0x7362) if table == "mxfp4" else (0x4051, 0x6273)
    bits = [int(b) for b in workloads.to_bf16_bits(np.asarray(cb32, np.float32))]
    lo = [0, 0, 0, 0]
    hi = [0, 0, 0, 0]
    for j, b in enumerate(bits):
        lo[j >> 2] |= (b & 0xFF) << (8 * (j & 3))
        hi[j >> 2] |= (b >> 8) << (8 * (j & 3))
    for g in range(1 << 16):
        s = g & 0x7777
        pick = ((g >> 1) & 0x4444) | 0x3210
        L = _byte_perm(_byte_perm(lo[0], lo[1], s), _byte_perm(lo[2], lo[3], s), pick)
        Hh = _byte_perm(_byte_perm(hi[0], hi[1], s), _byte_perm(hi[2], hi[3], s), pick)
        w0 = _byte_perm(L, Hh, sel0)
        w1 = _byte_perm(L, Hh, sel1)
        n = [g & 15, (g >> 4) & 15, (g >> 8) & 15, (g >> 12) & 15]
        if table == "mxfp4":   # byte = (element 2i+1 << 4) | element 2i
            assert w0 == bits[n[0]] | (bits[n[1]] << 16), hex(g)
            assert w1 == bits[n[2]] | (bits[n[3]] << 16), hex(g)
        else:                  # byte = (element 2i << 4) | element 2i+1
            assert w0 == bits[n[1]] | (bits[n[0]] << 16), hex(g)
            assert w1 == bits[n[3]] | (bits[n[2]] << 16), hex(g)


@pytest.mark.parametrize("tpr", [2, 4])
def test_tensor_core_mxfp4_decoders_take_their_scale_block(tpr):
    """csrc/gemm_tc.cu MXFP4 decoders: thread part kq of a 64-k block (64 / tpr
    k from 64 kq / tpr) multiplies by scale byte 2 kb + (2 kq) / tpr of its row,
    the one e8m0 block of 32 that holds all of its k; with the e2m1 values and
    2^(x - 127) this rebuilds the oracle's dequantised row."""
    from oracle import mxfp4
    rng = np.random.default_rng(21)
    K = 320
    row = rng.integers(0, 256, K // 2, dtype=np.uint8)
    sc = rng.integers(120, 135, K // 32, dtype=np.uint8)
    want = mxfp4.dequantize_expert(row[None, :], sc[None, :], 1, K)[0]
    got = np.full(K, np.nan)
    e2m1 = mxfp4.e2m1_table()
    for kb in range(K // 64):
        for kq in range(tpr):
            k0 = kb * 64 + kq * (64 // tpr)
            x = int(sc[2 * kb + (2 * kq) // tpr])
            assert all((k0 + j) // 32 == 2 * kb + (2 * kq) // tpr for j in range(64 // tpr))
            for j in range(0, 64 // tpr, 2):
                byte = int(row[(k0 + j) // 2])
                got[k0 + j] = e2m1[byte & 15] * 2.0 ** (x - 127)
                got[k0 + j + 1] = e2m1[byte >> 4] * 2.0 ** (x - 127)
    assert np.array_equal(got, want)


def _quant_cell_table(cb):
    """csrc/quantize.cu quant_cell_table: levels = distinct codebook values
    ascending (each with its lowest code), thresholds = smallest float above
    each exact midpoint, and per cell c of [c/64 - 1, (c+1)/64 - 1] widened by
    1e-5 the one threshold inside it (+inf if none) with the codes below and at
    or above it."""
    vals, codes = [], []
    for c in range(16):
        v = float(cb[c]) + 0.0
        if v not in vals:
            vals.append(v)
            codes.append(c)
    order = np.argsort(vals, kind="stable")
    vals = [vals[i] for i in order]
    codes = [codes[i] for i in order]
    T = []
    for lv in range(len(vals) - 1):
        mid = (vals[lv] + vals[lv + 1]) / 2
        f = np.float32(mid)
        T.append(float(f if float(f) > mid else np.nextafter(f, np.float32(np.inf))))
    cells = []
    for c in range(128):
        lo, hi = c / 64.0 - 1.0 - 1e-5, (c + 1) / 64.0 - 1.0 + 1e-5
        base = sum(1 for t in T if t <= lo)
        inside = [t for t in T if lo < t <= hi]
        assert len(inside) <= 1, "two thresholds in one cell"
        cells.append((inside[0] if inside else np.inf, codes[base], codes[min(base + 1, len(vals) - 1)]))
    return cells


def _kernel_codes(w, a, cells):
    """csrc/quantize.cu code_of for every (w, a): s' = fl32(w * fl32(1/a)) for
    absmax in [2^-125, 2^125], the cell of s', and the exact fl32(w / a) when
    s' lies within 2^-22 of the cell's threshold (or the absmax is outside)."""
    f32 = np.float32
    t_tab = np.array([c[0] for c in cells], f32)
    lo_tab = np.array([c[1] for c in cells])
    hi_tab = np.array([c[2] for c in cells])
    with np.errstate(all="ignore"):
        fast = (a >= f32(2.0 ** -125)) & (a <= f32(2.0 ** 125))
        exact = (w / a).astype(f32)
        s = np.where(fast, (w * (f32(1) / a).astype(f32)).astype(f32), exact)
        c = np.clip(np.floor((s + f32(1)).astype(f32) * f32(64)).astype(np.int64), 0, 127)
        t = t_tab[c]
        near = fast & ~(np.abs((s - t).astype(f32)) > f32(2.0 ** -22))
        s = np.where(near, exact, s)
    return np.where(s >= t, hi_tab[c], lo_tab[c]).astype(np.uint8), int(near.sum())


@pytest.mark.parametrize("table", ["nf4", "fp4"])
def test_quantiser_cell_lookup_and_reciprocal_path_match_the_oracle(table):
    """The quantiser kernel's decision -- one cell lookup, the weight scaled by
    the block's reciprocal unless it lands within 2^-22 of the cell's threshold
    -- equals the oracle's code of fl32(w / a), on random weights, on every
    decision point times random absmax (and 3 floats either side), and on
    |w| = a, zeros and subnormal absmax."""
    from oracle import fp4
    mod = nf4 if table == "nf4" else fp4
    cells = _quant_cell_table(mod.codebook_f64())
    rng = np.random.default_rng(11)
    f32 = np.float32
    n = 200_000
    fallbacks = 0
    for kind in range(3):
        a = (rng.uniform(1, 2, n) * 2.0 ** rng.integers(-40, 40, n)).astype(f32)
        if kind == 0:
            w = (rng.uniform(-1, 1, n) * a).astype(f32)
        elif kind == 1:
            w = (rng.choice(mod.midpoints(), n) * a.astype(np.float64)).astype(f32)
            k = rng.integers(-3, 4, n)
            for step in range(3):
                w = np.where(k > step, np.nextafter(w, f32(np.inf)), w)
                w = np.where(k < -step, np.nextafter(w, f32(-np.inf)), w)
        else:
            tiny = (rng.uniform(1, 2, n) * 2.0 ** rng.integers(-149, -120, n)).astype(f32)
            a = np.where(rng.random(n) < 0.2, tiny, a).astype(f32)
            a = np.where(a == 0, f32(1e-45), a).astype(f32)
            r = rng.random(n)
            w = np.where(r < 0.25, a, np.where(r < 0.5, -a, (rng.uniform(-1, 1, n) * a).astype(f32))).astype(f32)
            w = np.where(rng.random(n) < 0.05, f32(0), w).astype(f32)
        got, nf = _kernel_codes(w, a, cells)
        fallbacks += nf
        with np.errstate(all="ignore"):
            want = mod.code_of_scaled((w / a).astype(f32))
        assert np.array_equal(got, want), kind
    assert fallbacks > 0   # the exact path was exercised


def test_tensor_memory_decoders_fill_the_a_operand_the_mma_reads():
    """csrc/gemm_tc.cu TMEM-operand tile: decoder warp w (lane quadrant w % 4,
    part c = (w - 4) / 4: half c / 2, 32-k part c % 2) takes weight row
    32 (w % 4) + lane of its half, decodes its 32 k (4 words, decode4 on each
    half-word: v[i] = elements 2i, 2i+1) and stores v[0..15] as 16 consecutive
    32-bit columns of its TMEM lane from column A + half*32 + part*16.  The MMA
    of k-step kk of half h reads columns A + h*32 + kk*8 .. +7 of lanes 0..127,
    two bf16 per column, the lower k in the low half: that must be the half's
    rows and k [16 kk, 16 kk + 16) of the 64-k block."""
    packed, absmax, W = _layer_rows(9, 256, 64)
    tmem = {}
    for w in range(4, 20):
        qd, c = w & 3, (w - 4) >> 2
        half, part = c >> 1, c & 1
        for lane in range(32):
            ri = qd * 32 + lane
            r = half * 128 + ri
            src = packed[r, part * 16: part * 16 + 16]          # 16 bytes = this thread's 32 k
            vals = []
            for byte in src:
                vals += [v * absmax[r, 0] for v in _pair(byte)]   # elements in k order
            v = [(vals[2 * i], vals[2 * i + 1]) for i in range(16)]
            for i in range(16):
                key = (ri, half * 32 + part * 16 + i)
                assert key not in tmem, "column written twice"
                tmem[key] = v[i]                                  # (low half, high half)
    for h in range(2):
        for kk in range(4):
            for lane in range(128):
                row = [x for col in range(8) for x in tmem[(lane, h * 32 + kk * 8 + col)]]
                assert row == list(W[h * 128 + lane, kk * 16: kk * 16 + 16]), (h, kk, lane)


@pytest.mark.parametrize("RS", [2, 4, 6, 32])
def test_decode_stage_indices_advance_like_their_definitions(RS):
    """csrc/decode.cu advances ring slots, passes, items and chunks per stage
    instead of dividing: the copy-issuing warp's (s, ph, u, rb, ch, rq), each
    group's (s, ph) over its items jj = gi, gi + 2, ..., and the down loop's
    (s, ph, ch, rbq) must equal j % RS, (j / RS) & 1, (i0 + j) / ipe and
    % ipe, jd % nch and jd / nch of every stage."""
    rng = np.random.default_rng(RS)
    for _ in range(300):
        ipe = int(rng.integers(1, 200))
        i0 = int(rng.integers(0, 5000))
        n_gu = int(rng.integers(0, 40))
        nch = int(rng.integers(1, 9))
        n_dn = nch * int(rng.integers(0, 6))
        # producer
        s = ph = ch = rq = 0
        u, rb = i0 // ipe, i0 % ipe
        for j in range(n_gu + n_dn):
            assert (s, ph) == (j % RS, (j // RS) & 1)
            if j < n_gu:
                assert (u, rb) == ((i0 + j) // ipe, (i0 + j) % ipe)
                rb += 1
                if rb == ipe:
                    rb, u = 0, u + 1
            else:
                jd = j - n_gu
                assert (ch, rq) == (jd % nch, jd // nch)
                ch += 1
                if ch == nch:
                    ch, rq = 0, rq + 1
            s += 1
            if s == RS:
                s, ph = 0, ph ^ 1
        # phase 1: group gi takes items gi, gi + 2, ...
        for gi in range(2):
            s, ph = gi, 0
            for jj in range(gi, n_gu, 2):
                if s >= RS:
                    s, ph = s - RS, ph ^ 1
                assert (s, ph) == (jj % RS, (jj // RS) & 1)
                s += 2
        # phase 2: stage jd is ring stage n_gu + jd
        s, ph, ch, rbq = n_gu % RS, (n_gu // RS) & 1, 0, 0
        for jd in range(n_dn):
            j = n_gu + jd
            assert (s, ph, ch, rbq) == (j % RS, (j // RS) & 1, jd % nch, jd // nch)
            ch1 = 0 if ch + 1 == nch else ch + 1
            s += 1
            if s == RS:
                s, ph = 0, ph ^ 1
            if ch1 == 0:
                rbq += 1
            ch = ch1
