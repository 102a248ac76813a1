"""CPU models of the bulk-ring decode kernels (csrc/decode.cu).

These restate, in numpy, the kernels' shared-memory geometry and copy
addressing, their MMA fragment mapping and their mbarrier protocol, and check
them against the global data, the dense product and an exact model of
mbarrier phases under random schedules (no waiter ever lags a barrier by two
phases; no slot is refilled or reused while read).  They model the kernels'
index arithmetic; the GPU tests check the compiled kernels.
"""
import random

import numpy as np
import pytest

from oracle import nf4  # the codebook values of the fragment model

# ---- geometry and addressing

kMaxM, kMath, kMaxStages, kMinStages = 8, 16, 12, 2
kRedLane = 32 * 16
SMEM_LIMIT = 232448 - 1024

def al(v, a): return (v + a - 1) // a * a

def ring_geom(K, h_rows, red_warps):
    KB = K // 64
    g = {}
    g['ps'] = K // 2 + 16
    g['am_rows'] = KB % 4 == 0
    g['sa'] = (KB if KB % 8 == 4 else KB + 4) if g['am_rows'] else KB
    g['am_off'] = 16 * g['ps']
    g['h_off'] = g['am_off'] + al(16 * g['sa'] * 4, 16)
    g['hs'] = 2 * K + 16
    g['red_off'] = g['h_off'] + h_rows * g['hs']
    g['bytes'] = al(g['red_off'] + red_warps * kRedLane, 128)
    return g

def msplit(H):
    nsp = (H // 64 + 1) // 2
    return 16 if nsp <= 16 else (12 if nsp <= 24 else 16)

def make_layout(is_a, M, k, E, r, g, stages):
    S = M * k
    o = 256 * 32 * 4
    o = al(o + S * 4, 16); o = al(o + S * 4, 16); o = al(o + E * 4, 16); o = al(o + S * 4, 16)
    o = al(o + S * kMaxM * 4, 16)
    if is_a and r > 0: o = al(o + S * r * 4, 16)
    o = al(o + (3 * stages if is_a else 2 * stages + 4) * 8, 16)
    if not is_a: o = al(o + stages * 4, 16)
    if not is_a: o += 2 * kMath * kRedLane
    ring = al(o, 128)
    return ring, ring + stages * g['bytes']

def pick(is_a, M, k, E, r, g):
    for s in range(kMaxStages, kMinStages - 1, -1):
        if make_layout(is_a, M, k, E, r, g, s)[1] <= SMEM_LIMIT: return s
    return 0

def copies(g, K, row_a, row_b):
    """(dst_off_in_stage, src_kind, src_byte_off, size) of one stage's weight copies."""
    KB, rowb = K // 64, K // 2
    out = []
    for lane in range(32):
        if lane < 16:
            row = (row_a if lane < 8 else row_b) + (lane & 7)
            out.append((lane * g['ps'], 'pk', row * rowb, rowb))
        elif g['am_rows']:
            i = lane - 16
            row = (row_a if i < 8 else row_b) + (i & 7)
            out.append((g['am_off'] + i * g['sa'] * 4, 'am', row * KB * 4, KB * 4))
        elif lane < 18:
            i = lane - 16
            out.append((g['am_off'] + i * 8 * g['sa'] * 4, 'am', (row_a if i == 0 else row_b) * KB * 4, 8 * KB * 4))
    return out

def wavefronts(addrs, width):
    """Shared-memory wavefronts of one warp access (distinct 4-byte words per bank, lanes with equal
    addresses broadcast); width in bytes per lane."""
    words = set()
    for a in addrs:
        if a is None: continue
        for w in range(width // 4): words.add(a // 4 + w)
    per_bank = {}
    for w in words: per_bank.setdefault(w % 32, set()).add(w)
    return max(len(v) for v in per_bank.values()) if per_bank else 0

def check(name, E, H, I, k, r=0):
    rng = np.random.default_rng(0)
    for M in range(1, 9):
        ga, gb = ring_geom(H, 0, msplit(H)), ring_geom(I, M, 0)
        sa_, sb_ = pick(True, M, k, E, 16, ga), pick(False, M, k, E, 0, gb)
        assert sa_ >= 2 and sb_ >= 2, (name, M, sa_, sb_)
        ra, ta = make_layout(True, M, k, E, r, ga, pick(True, M, k, E, r, ga))
        rb_, tb = make_layout(False, M, k, E, 0, gb, sb_)
        assert ta <= SMEM_LIMIT and tb <= SMEM_LIMIT
        assert ra % 128 == 0 and rb_ % 128 == 0 and ga['bytes'] % 128 == 0 and gb['bytes'] % 128 == 0
    # byte-level emulation for one expert each
    for (K, g, rows_ab, label, hrows) in ((H, ring_geom(H, 0, msplit(H)), lambda rb: (5 * 2 * I + rb * 8, 5 * 2 * I + I + rb * 8), 'A', 0),
                                          (I, ring_geom(I, 8, 0), lambda rb: (3 * H + rb * 16, 3 * H + rb * 16 + 8), 'B', 8)):
        KB, rowb, NSP = K // 64, K // 2, (K // 64 + 1) // 2
        nrows = (6 * 2 * I) if label == 'A' else 4 * H
        pk = rng.integers(0, 256, size=nrows * rowb, dtype=np.uint8)
        am = rng.standard_normal(nrows * KB).astype(np.float32)
        amb = am.view(np.uint8)
        for rb in (0, 1, (I // 8 - 1) if label == 'A' else (H // 16 - 1)):
            row_a, row_b = rows_ab(rb)
            st = np.full(g['bytes'], 0xEE, dtype=np.uint8)
            written = np.zeros(g['bytes'], dtype=bool)
            total = 0
            for dst, kind, src, size in copies(g, K, row_a, row_b):
                assert dst % 16 == 0 and src % 16 == 0 and size % 16 == 0, (name, label, dst, src, size)
                assert dst + size <= (g['h_off'] if label == 'B' else g['red_off'])
                assert not written[dst:dst + size].any(), 'overlap'
                written[dst:dst + size] = True
                st[dst:dst + size] = (pk if kind == 'pk' else amb)[src:src + size]
                total += size
            assert total == 16 * rowb + 16 * KB * 4
            if label == 'B':
                for tok in range(8):
                    d = g['h_off'] + tok * g['hs']
                    assert d % 16 == 0 and (2 * I) % 16 == 0 and d + 2 * I <= g['bytes']
            # math-lane reads (k-block-uniform mapping) vs the global rows
            for sp in range(NSP):
                for hh in range(2):
                    kb = 2 * sp + hh
                    if kb >= KB: continue
                    lds_w, lds_a = [], []
                    for lane in range(32):
                        gg, t = lane >> 2, lane & 3
                        for rr, grow in ((gg, row_a + gg), (gg + 8, row_b + gg)):
                            off = rr * g['ps'] + sp * 64 + 32 * hh + 8 * t
                            assert written[off:off + 8].all()
                            assert np.array_equal(st[off:off + 8], pk[grow * rowb + kb * 32 + 8 * t:][:8])
                            aoff = g['am_off'] + (rr * g['sa'] + kb) * 4
                            assert written[aoff:aoff + 4].all()
                            assert st[aoff:aoff + 4].view(np.float32)[0] == am[grow * KB + kb]
                        lds_w.append(gg * g['ps'] + sp * 64 + 32 * hh + 8 * t)
                        lds_a.append(g['am_off'] + (gg * g['sa'] + kb) * 4)
                    assert wavefronts(lds_w, 8) <= 2, (name, label, sp, wavefronts(lds_w, 8))
                    assert wavefronts(lds_a, 4) == 1, (name, label, 'am', wavefronts(lds_a, 4))
                    if label == 'B':
                        for i in range(2):
                            hx = [g['h_off'] + (l >> 2) * g['hs'] + sp * 256 + 32 * (l & 3) + 128 * hh + 16 * i
                                  for l in range(32)]
                            assert wavefronts(hx, 16) <= 4
                            for l, a in enumerate(hx):
                                row_start = g['h_off'] + (l >> 2) * g['hs']
                                assert row_start <= a and a + 16 <= row_start + 2 * I
    print(f"{name}: ok  stagesA/B(M=1)={pick(True,1,k,E,r,ring_geom(H,0,msplit(H)))}/{pick(False,1,k,E,0,ring_geom(I,1,0))}"
          f"  (M=8)={pick(True,8,k,E,r,ring_geom(H,0,msplit(H)))}/{pick(False,8,k,E,0,ring_geom(I,8,0))}"
          f"  stage bytes A={ring_geom(H,0,msplit(H))['bytes']} B(M=1)={ring_geom(I,1,0)['bytes']}")

CONFIGS = [("tiny", 8, 256, 128, 2), ("ragged", 12, 192, 320, 3), ("lora", 6, 128, 192, 2, 8),
           ("zipf", 16, 256, 128, 4), ("dir", 8, 320, 192, 2), ("wide", 40, 448, 128, 6), ("k32", 33, 128, 64, 32),
           ("oddkb", 8, 2880, 704, 2), ("olmoe", 64, 2048, 1024, 8), ("qwen3", 128, 2048, 768, 8),
           ("qwen3_lora", 128, 2048, 768, 8, 8), ("gptoss", 32, 2880, 2880, 4)]


@pytest.mark.parametrize("args", CONFIGS, ids=[c[0] for c in CONFIGS])
def test_ring_geometry_and_addressing(args):
    check(*args)


# ---- fragment mapping
CB = nf4.codebook_f64()

def lut_pair(byte):          # (low half, high half) = (element 2j, element 2j+1)
    return (CB[byte >> 4], CB[byte & 15])

def mma(d, A, B):            # A[lane] = 4 pairs, B[lane] = 2 pairs (each a (lo, hi) tuple)
    Am = np.zeros((16, 16)); Bm = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        (a0, a1, a2, a3), (b0, b1) = A[lane], B[lane]
        Am[g, 2*t:2*t+2] = a0; Am[g+8, 2*t:2*t+2] = a1; Am[g, 2*t+8:2*t+10] = a2; Am[g+8, 2*t+8:2*t+10] = a3
        Bm[2*t:2*t+2, g] = b0; Bm[2*t+8:2*t+10, g] = b1
    D = Am @ Bm
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        d[lane] += np.array([D[g, 2*t], D[g, 2*t+1], D[g+8, 2*t], D[g+8, 2*t+1]])

def span_kb(rows_bytes, am, x, sp, KB):
    """rows_bytes[16][span 64 bytes], am[16][KB], x[8 tokens][K]: returns c[lane][4]."""
    c = np.zeros((32, 4))
    for h in range(2):
        kb = 2 * sp + h
        if kb >= KB: continue
        d = np.zeros((32, 4))
        for j in range(4):
            A, B = [], []
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                # thread's 8 bytes of row r in k-block half h: bytes [32h + 8t, +8) of the span
                by = lambda r, i: rows_bytes[r][32*h + 8*t + i]
                A.append((lut_pair(by(g, 2*j)), lut_pair(by(g+8, 2*j)), lut_pair(by(g, 2*j+1)), lut_pair(by(g+8, 2*j+1))))
                kx = 128*sp + 64*h + 16*t + 4*j     # physical k of x word 2j
                B.append(((x[g][kx], x[g][kx+1]), (x[g][kx+2], x[g][kx+3])))
            mma(d, A, B)
        for lane in range(32):
            g = lane >> 2
            c[lane] += d[lane] * np.array([am[g][kb], am[g][kb], am[g+8][kb], am[g+8][kb]])
    return c


def test_kblock_uniform_span_mapping():
    rng = np.random.default_rng(1)
    for K in (128, 192, 2880):
        KB = K // 64
        NSP = (KB + 1) // 2
        rows = rng.integers(0, 256, size=(16, K // 2))
        am = rng.random((16, KB)) + 0.5
        x = rng.standard_normal((8, K))
        W = np.zeros((16, K))
        for r in range(16):
            for j in range(K // 2):
                W[r, 2*j], W[r, 2*j+1] = CB[rows[r, j] >> 4] * am[r, (2*j)//64], CB[rows[r, j] & 15] * am[r, (2*j+1)//64]
        ref = W @ x.T                      # [16 rows, 8 tokens]
        c = np.zeros((32, 4))
        for sp in range(NSP):
            span = np.zeros((16, 64), dtype=np.int64)
            nb = min(64, K // 2 - 64 * sp)
            span[:, :nb] = rows[:, 64*sp:64*sp+nb]
            xx = np.zeros((8, 128 * NSP)); xx[:, :K] = x
            c += span_kb(span, am, xx, sp, KB)
        got = np.zeros((16, 8))
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            got[g, 2*t], got[g, 2*t+1], got[g+8, 2*t], got[g+8, 2*t+1] = c[lane]
        err = np.abs(got - ref).max() / np.abs(ref).max()
        print(K, "max rel err", err)
        assert err < 1e-12

# ---- barrier protocol

class MBar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0
    def _maybe(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1; self.pending = self.count
    def arrive(self):
        assert self.pending > 0; self.pending -= 1; self._maybe()
    def expect_arrive(self, b):
        self.tx += b; self.arrive()
    def complete(self, b):
        self.tx -= b; self._maybe()
    def ready(self, n):
        # waiting for completion of phase number n with parity n & 1: exact
        # only while the barrier is at phase n or n + 1
        assert self.phase >= n, f"waiter ahead: barrier phase {self.phase}, waiting for {n}"
        assert self.phase - n <= 1, f"parity aliasing: phase {self.phase} waiter {n}"
        return (self.phase & 1) != (n & 1)
    def ready_raw(self, n):
        return (self.phase & 1) != (n & 1)

def wait(bar, n):
    while not bar.ready(n):
        yield

def run(tasks, engine, seed):
    rng = random.Random(seed)
    live = list(tasks)
    steps = 0
    while live or engine.inflight:
        steps += 1
        assert steps < 2_000_000, "deadlock/livelock"
        if engine.inflight and (not live or rng.random() < 0.3):
            engine.land(rng)
            continue
        t = rng.choice(live)
        try:
            next(t)
        except StopIteration:
            live.remove(t)
    return steps

class Engine:
    def __init__(self): self.inflight = []
    def copy(self, bar, nbytes, on_land):
        self.inflight.append((bar, nbytes, on_land))
    def land(self, rng):
        i = rng.randrange(len(self.inflight))
        bar, nb, cb = self.inflight.pop(i)
        cb(); bar.complete(nb)

def kernel_a(n_items, RS, nact, seed):
    eng = Engine()
    full = [MBar(1) for _ in range(RS)]; done = [MBar(nact) for _ in range(RS)]; empty = [MBar(1) for _ in range(RS)]
    stage_item = [None] * RS          # item whose data the stage holds (landed)
    readers = [set() for _ in range(RS)]
    red = [dict() for _ in range(RS)]  # warp -> item of the partial in the slot
    summed = []
    def producer():
        for j in range(n_items):
            s = j % RS
            if j >= RS:
                yield from wait(empty[s], (j // RS) - 1)
            assert not readers[s], f"stage {s} refilled while read by {readers[s]}"
            full[s].expect_arrive(17)
            for c in range(17):
                def cb(s=s, j=j): stage_item[s] = j
                eng.copy(full[s], 1, cb)
            yield
        # drain: bounded waits in the kernel; here the engine lands everything anyway
    def math(w):
        for j in range(n_items):
            s = j % RS
            yield from wait(full[s], j // RS)
            assert stage_item[s] == j
            readers[s].add(w); yield
            assert stage_item[s] == j, "stage overwritten while read"
            readers[s].discard(w)
            assert w not in red[s] or red[s][w] == j - RS and j - RS in summed, "partial overwritten before summed"
            red[s][w] = j
            done[s].arrive(); yield
    def epilogue():
        for j in range(n_items):
            s = j % RS
            yield from wait(done[s], j // RS)
            assert all(red[s].get(w) == j for w in range(nact)), "missing partial"
            summed.append(j)
            empty[s].arrive(); yield
    run([producer(), epilogue()] + [math(w) for w in range(nact)], eng, seed)
    assert summed == list(range(n_items))

def kernel_b(nrb, nU, NSP, RS, nmath, seed):
    eng = Engine()
    T = nrb * nU
    full = [MBar(1) for _ in range(RS)]; empty = [MBar(NSP) for _ in range(RS)]
    rdone = [MBar(nmath) for _ in range(2)]; rfree = [MBar(1) for _ in range(2)]
    stage_w = [None] * RS; stage_h = [None] * RS
    seq = [-1] * RS
    readers = [0] * RS
    red = [dict() for _ in range(2)]
    outs = []
    h_ready = [False]
    def producer():
        def issue_w(j):
            s = j % RS
            seq[s] = j                       # st.release after the empty wait
            full[s].expect_arrive(16 + 2)   # 16 rows + 2 h rows
            for _ in range(16):
                eng.copy(full[s], 1, lambda s=s, j=j: stage_w.__setitem__(s, j))
        def issue_h(j):
            s = j % RS
            assert h_ready[0]
            for _ in range(2):
                eng.copy(full[s], 1, lambda s=s, j=j: stage_h.__setitem__(s, j))
        pre = min(RS, T)
        for j in range(pre):
            issue_w(j); yield
        h_ready[0] = True   # griddepcontrol.wait
        for j in range(pre):
            issue_h(j); yield
        for j in range(pre, T):
            s = j % RS
            yield from wait(empty[s], (j // RS) - 1)
            assert readers[s] == 0
            issue_w(j); issue_h(j); yield
    def math(w):
        for rbi in range(nrb):
            acc = []
            for qp in range(w, nU * NSP, nmath):
                u, sp = divmod(qp, NSP)
                j = rbi * nU + u; s = j % RS
                while True:                    # ld.acquire of seq, then the parity wait
                    if seq[s] == j and full[s].ready(j // RS):
                        break
                    yield
                assert stage_w[s] == j and stage_h[s] == j
                readers[s] += 1; yield
                assert stage_w[s] == j and stage_h[s] == j, "stage overwritten while read"
                readers[s] -= 1
                acc.append((j, sp))
                empty[s].arrive(); yield
            par = rbi & 1
            if rbi >= 2:
                yield from wait(rfree[par], (rbi >> 1) - 1)
            assert w not in red[par] or red[par][w][0] == rbi - 2, "partial overwritten before summed"
            red[par][w] = (rbi, acc)
            rdone[par].arrive(); yield
    def epilogue():
        for rbi in range(nrb):
            par = rbi & 1
            yield from wait(rdone[par], rbi >> 1)
            pairs = []
            for w in range(nmath):
                r, acc = red[par][w]
                assert r == rbi
                pairs += acc
            assert sorted(pairs) == [(rbi * nU + u, sp) for u in range(nU) for sp in range(NSP)]
            outs.append(rbi)
            rfree[par].arrive(); yield
    run([producer(), epilogue()] + [math(w) for w in range(nmath)], eng, seed)
    assert outs == list(range(nrb))


@pytest.mark.parametrize("seed", range(0, 200, 20))
def test_ring_barrier_protocol(seed):
    for s_ in range(seed, seed + 20):
        r = random.Random(s_)
        kernel_a(n_items=r.randint(0, 40), RS=r.randint(2, 12), nact=r.choice([1, 2, 12, 16]), seed=s_)
        kernel_b(nrb=r.randint(1, 4), nU=r.randint(1, 10), NSP=r.choice([1, 2, 3, 6, 8, 23]), RS=r.randint(2, 12),
                 nmath=16, seed=s_)
