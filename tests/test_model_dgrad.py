"""CPU models of the grouped dgrad kernels (csrc/dgrad.cu and the dgrad
instance of csrc/gemm_tc.cu).

The warp-MMA model follows every thread's transposed decode, its shared-memory
stores and the m16n8k16 fragments (PTX fragment layout) and must reproduce the
oracle's grouped dgrad exactly (no bf16 rounding in the model); the
tensor-core model follows the decoders' writes into the 128-byte-swizzled
K-major A tile and must give exactly W^T once unswizzled, ragged last tile
included.  They model the kernels' index arithmetic; the GPU tests check the
compiled kernels.
"""
import numpy as np

from oracle import backward, nf4

# ---- warp-MMA kernel

CB = nf4.codebook_f64()
LUT = [(CB[b >> 4], CB[b & 15]) for b in range(256)]   # (low half, high half)
kTileK = kTileT = kStep = 64

def mma(acc, A, B):
    Am = np.zeros((16, 16)); Bm = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        a0, a1, a2, a3 = A[lane]; b0, b1 = B[lane]
        Am[g, 2*t:2*t+2] = a0; Am[g+8, 2*t:2*t+2] = a1; Am[g, 2*t+8:2*t+10] = a2; Am[g+8, 2*t+8:2*t+10] = a3
        Bm[2*t:2*t+2, g] = b0; Bm[2*t+8:2*t+10, g] = b1
    D = Am @ Bm
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        acc[lane] += [D[g, 2*t], D[g, 2*t+1], D[g+8, 2*t], D[g+8, 2*t+1]]

def words(row, start):   # 8 consecutive "bf16" values -> 4 pairs
    return [(row[start + 2*m], row[start + 2*m + 1]) for m in range(4)]

def run(E=3, N=128, K=192, counts=(70, 0, 9), seed=0):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    rows = int(offsets[-1])
    dY = rng.standard_normal((rows + 5, N))
    idx = rng.permutation(rows + 5)[:rows]
    ref = backward.grouped_nf4_gemm_dgrad(dY, idx, offsets, packed, absmax, N, K)
    out = np.full((rows, K), np.nan)
    KB = K // 64
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        pk_e = packed[e].reshape(N, K // 2)
        am_e = absmax[e].reshape(N, KB)
        for rb in range(lo, hi, kTileT):
            nrows = min(kTileT, hi - rb)
            rows_s = [idx[rb + i] if i < nrows else -1 for i in range(kTileT)]
            for kt in range(K // kTileK):
                acc = np.zeros((4, 8, 32, 4))   # [warp][nt][lane][4]
                for s in range(N // kStep):
                    ys = np.zeros((kTileT, 64))
                    for r in range(kTileT):
                        if rows_s[r] >= 0: ys[r] = dY[rows_s[r], s*64:(s+1)*64]
                    pk = pk_e[s*64:(s+1)*64, kt*32:(kt+1)*32]
                    am = am_e[s*64:(s+1)*64, kt]
                    wt = np.full((64, 64), np.nan)
                    for tid in range(128):
                        o, q = tid & 7, tid >> 3
                        for j in range(4):
                            n = 8*o + 2*j
                            x = int(pk[n, 2*q]) | (int(pk[n, 2*q+1]) << 8)
                            y = int(pk[n+1, 2*q]) | (int(pk[n+1, 2*q+1]) << 8)
                            ev = (x & 0xF0F0) | ((y >> 4) & 0x0F0F)
                            od = ((x << 4) & 0xF0F0) | (y & 0x0F0F)
                            v = [LUT[ev & 0xff], LUT[od & 0xff], LUT[(ev >> 8) & 0xff], LUT[(od >> 8) & 0xff]]
                            for c in range(4):
                                assert np.isnan(wt[4*q + c, n]) and np.isnan(wt[4*q + c, n+1])
                                wt[4*q + c, n] = v[c][0] * am[n]
                                wt[4*q + c, n+1] = v[c][1] * am[n+1]
                    assert not np.isnan(wt).any()
                    for w in range(4):
                        for ch in range(2):
                            for nt in range(8):
                                A0, A1, B0, B1 = [], [], [], []
                                for lane in range(32):
                                    g, t = lane >> 2, lane & 3
                                    w0 = words(wt[16*w + g], 32*ch + 8*t)
                                    w1 = words(wt[16*w + g + 8], 32*ch + 8*t)
                                    yv = words(ys[nt*8 + g], 32*ch + 8*t)
                                    A0.append((w0[0], w1[0], w0[1], w1[1])); A1.append((w0[2], w1[2], w0[3], w1[3]))
                                    B0.append((yv[0], yv[1])); B1.append((yv[2], yv[3]))
                                mma(acc[w, nt], A0, B0)
                                mma(acc[w, nt], A1, B1)
                for w in range(4):
                    for nt in range(8):
                        for lane in range(32):
                            g, t = lane >> 2, lane & 3
                            k0 = kt*64 + 16*w + g; k1 = k0 + 8
                            for qq in range(2):
                                tok = nt*8 + 2*t + qq
                                if tok >= nrows: continue
                                out[rb + tok, k0] = acc[w, nt, lane, qq]
                                out[rb + tok, k1] = acc[w, nt, lane, 2 + qq]
    assert not np.isnan(out).any()
    err = np.abs(out - ref).max() / np.abs(ref).max()
    print("dgrad emulation max rel err", err)
    assert err < 1e-12


def test_warp_mma_dgrad_model_matches_oracle():
    run()
    run(E=2, N=64, K=64, counts=(0, 3), seed=1)


# ---- tensor-core decoders

kBM, HALVES = 128, 2
kAHalfBytes = kBM * 128

def decode4(g):
    """(elements 2i, 2i+1), (2i+2, 2i+3) from 16 bits: byte0 hi = elem 0, lo = elem 1, byte1 hi = 2, lo = 3."""
    b0, b1 = g & 0xff, (g >> 8) & 0xff
    return (CB[b0 >> 4], CB[b0 & 15]), (CB[b1 >> 4], CB[b1 & 15])

def run_tc(N_w=192, K_w=640, E=2, e=1, seed=0):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, N_w, K_w)) * 0.05).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    pk = packed.reshape(E * N_w, K_w // 2)
    am_all = absmax.reshape(E * N_w, K_w // 64)
    kbw = K_w // 64
    n_tiles = (K_w + 255) // 256
    for n_tile in range(n_tiles):
        r0 = n_tile * 256
        for kb in range(N_w // 64):
            # TMA box {128 B, 64 rows} at x = r0/2, y = e*N_w + kb*64 (zero fill out of range)
            box = np.zeros((64, 128), dtype=np.uint8)
            x0 = r0 // 2
            w = min(128, K_w // 2 - x0)
            box[:, :w] = pk[e * N_w + kb * 64: e * N_w + kb * 64 + 64, x0:x0 + w]
            stage = box.reshape(-1)
            A = np.full(HALVES * kAHalfBytes // 2, np.nan)   # bf16 slots
            written = np.zeros(HALVES * kAHalfBytes, dtype=bool)
            for dt in range(512):
                q = (dt & 7) | (((dt >> 5) & 7) << 3)
                o = ((dt >> 3) & 3) | ((dt >> 8) << 2)
                kcol = r0 + 4 * q
                valid = kcol < K_w
                sc = [am_all[e * N_w + kb * 64 + 8 * o + i, kcol // 64] if valid else 0.0 for i in range(8)]
                col = [[None] * 4 for _ in range(4)]
                for j in range(4):
                    n = 8 * o + 2 * j
                    xx = int(stage[n * 128 + 2 * q]) | (int(stage[n * 128 + 2 * q + 1]) << 8)
                    yy = int(stage[(n + 1) * 128 + 2 * q]) | (int(stage[(n + 1) * 128 + 2 * q + 1]) << 8)
                    ev = (xx & 0xF0F0) | ((yy >> 4) & 0x0F0F)
                    od = ((xx << 4) & 0xF0F0) | (yy & 0x0F0F)
                    v = [None] * 4
                    v[0], v[2] = decode4(ev)
                    v[1], v[3] = decode4(od)
                    for c in range(4):
                        col[c][j] = (v[c][0] * sc[2 * j], v[c][1] * sc[2 * j + 1])
                for c in range(4):
                    kl = 4 * q + c
                    half, ri = kl >> 7, kl & 127
                    base = half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128 + ((o ^ (ri & 7)) << 4)
                    assert not written[base:base + 16].any(), "byte written twice"
                    written[base:base + 16] = True
                    vals = [col[c][j][h] for j in range(4) for h in range(2)]
                    A[base // 2: base // 2 + 8] = vals
            assert written.all()
            # unswizzle: logical element (row kl, K position n) of the K-major SW128 tile
            for kl in range(256):
                half, ri = kl >> 7, kl & 127
                kg = r0 + kl
                for n in range(64):
                    chunk, inner = n // 8, n % 8
                    addr = half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128 + ((chunk ^ (ri & 7)) << 4) + 2 * inner
                    got = A[addr // 2]
                    if kg < K_w:
                        row = e * N_w + kb * 64 + n
                        code = (pk[row, kg // 2] >> 4) if kg % 2 == 0 else (pk[row, kg // 2] & 15)
                        ref = CB[code] * am_all[row, kg // 64]
                        assert got == ref, (n_tile, kb, kl, n, got, ref)
                    else:
                        assert got == 0.0
    print("tc dgrad decoder emulation: A tile == W^T for", n_tiles, "tiles x", N_w // 64, "steps")


def test_tensor_core_dgrad_decoders_write_w_transposed():
    run_tc()
    run_tc(N_w=128, K_w=256, e=0, seed=3)
