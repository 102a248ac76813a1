"""CPU model of the MXFP4 warp-MMA kernel (csrc/mxfp4.cu): its byte table,
e8m0 scale decode and fragment mapping (PTX m16n8k16 layout, contraction order
permuted identically on both operands, one scale fold per 32-element chunk)
reproduce the oracle's grouped MXFP4 GEMM exactly.  It models the kernel's
index arithmetic; the GPU tests check the compiled kernel."""
import numpy as np

from oracle import mxfp4


def _mma(acc, A, B):
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


def test_mxfp4_kernel_model_matches_oracle():
    rng = np.random.default_rng(2)
    N, K = 16, 128   # one warp's 16 weight rows, two K steps
    blocks = rng.integers(0, 256, size=N * K // 2, dtype=np.uint8)
    scales = rng.integers(118, 136, size=N * K // 32, dtype=np.uint8)
    x = rng.standard_normal((8, K))            # one n8 tile of routed rows
    t2 = mxfp4.e2m1_table()
    lut = [(t2[b & 15], t2[b >> 4]) for b in range(256)]
    pk = blocks.reshape(N, K // 2)
    sc = scales.reshape(N, K // 32)
    acc = np.zeros((32, 4))
    for kb in range(K // 64):
        for c in range(2):
            A0, A1, B0, B1 = [], [], [], []
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                word = lambda r: [int(pk[r, kb * 32 + 16 * c + 4 * t + i]) for i in range(4)]
                w0, w1 = word(g), word(g + 8)
                A0.append((lut[w0[0]], lut[w1[0]], lut[w0[1]], lut[w1[1]]))
                A1.append((lut[w0[2]], lut[w1[2]], lut[w0[3]], lut[w1[3]]))
                kx = kb * 64 + 32 * c + 8 * t
                B0.append(((x[g, kx], x[g, kx + 1]), (x[g, kx + 2], x[g, kx + 3])))
                B1.append(((x[g, kx + 4], x[g, kx + 5]), (x[g, kx + 6], x[g, kx + 7])))
            tmp = np.zeros((32, 4))
            _mma(tmp, A0, B0)
            _mma(tmp, A1, B1)
            for lane in range(32):
                g = lane >> 2
                s0 = 2.0 ** (int(sc[g, 2 * kb + c]) - 127)
                s1 = 2.0 ** (int(sc[g + 8, 2 * kb + c]) - 127)
                acc[lane] += tmp[lane] * [s0, s0, s1, s1]
    got = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        got[g, 2 * t], got[g, 2 * t + 1], got[g + 8, 2 * t], got[g + 8, 2 * t + 1] = acc[lane]
    ref = mxfp4.grouped_mxfp4_gemm(x, None, np.array([0, 8]), blocks, scales, N, K).T   # [rows n, routed rows]
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
