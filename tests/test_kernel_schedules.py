"""CPU checks of the arithmetic schedules the CUDA kernels use, restated in
NumPy (no code shared with the library): they must reproduce the oracle's
definitions exactly (bit tricks) or up to fp64 rounding (butterfly order).

* rotate_kernel: the Walsh-Hadamard butterflies split into 3 in-thread index
  bits, 5 lane bits (shuffles) and the warp bits through a shared-memory
  transpose in which each of the 256 positions of a warp's chunk is handled
  by some thread, for every block size 256..8192.
* qgemv_kernel: a code c at bit b*j of a 16-bit half word, given the exponent
  of 2^(23 - b j), is the float 2^(23 - b j) + c exactly.
* qgemm_tc_kernel: a byte permute and a mask put codes c_2i, c_2i+1 of a word
  into a half2 holding M + c (M = 1024 for f16), and (M + c) - (M + zero) is
  c - zero exactly.
* qgemm_mma_kernel: the parked slab layout and the bytes each lane takes form
  the m16n8k16 B fragments of every k-step exactly once, the reads of a tile's
  8 rows are conflict-free, and a byte becomes the pair (M + c_lo, M + c_hi).
"""

import numpy as np
import pytest

import oracle as O


def _rotate_schedule(x, s, W, inverse):
    B = 256 * W
    sg = np.where(s < 0, -1.0, 1.0)
    v = x.astype(np.float64) * (1.0 if inverse else sg)
    v = v.reshape(W, 32, 8).copy()          # element = warp * 256 + lane * 8 + e
    for h in (1, 2, 4):                      # in-thread bits
        for e in range(8):
            if e & h == 0:
                a, b = v[:, :, e].copy(), v[:, :, e + h].copy()
                v[:, :, e], v[:, :, e + h] = a + b, a - b
    for m in (1, 2, 4, 8, 16):               # lane bits (shuffle xor m)
        u = v[:, np.arange(32) ^ m, :]
        upper = (np.arange(32) & m) != 0
        v = np.where(upper[None, :, None], u - v, v + u)
    if W > 1:                                # warp bits: positions looped over the CTA's threads
        sm = v.reshape(W, 256).copy()
        done = np.zeros(256, bool)
        for tid in range(32 * W):
            for pos in range(tid, 256, 32 * W):
                done[pos] = True
                u = sm[:, pos].copy()
                h = 1
                while h < W:
                    for w in range(W):
                        if w & h == 0:
                            a, b = u[w], u[w + h]
                            u[w], u[w + h] = a + b, a - b
                    h <<= 1
                sm[:, pos] = u
        assert done.all()
        v = sm
    v = v.reshape(B) / np.sqrt(B)
    return v * (sg if inverse else 1.0)


@pytest.mark.parametrize("W", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("inverse", [False, True])
def test_rotation_butterfly_schedule(W, inverse):
    rng = np.random.default_rng(W)
    B = 256 * W
    x, s = rng.standard_normal(B), rng.choice([-1, 1], B)
    ref = O.rotate(x[None], s, B, inverse)[0]
    assert np.allclose(_rotate_schedule(x, s, W, inverse), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_decode_code_to_float_is_exact(bits):
    half = 16 // bits
    mask = (1 << bits) - 1
    for j in range(half):
        sh = bits * j
        for c in range(1 << bits):
            other = 0xA5C3 & ~(mask << sh) & 0xFFFF  # neighbouring codes must not leak in
            hw = (c << sh) | other
            u = ((0x4B000000 - (sh << 23)) | (hw & (mask << sh))) & 0xFFFFFFFF
            f = np.array([u], dtype=np.uint32).view(np.float32)[0]
            assert float(f) == 2.0 ** (23 - sh) + c
            assert np.float32(f) - np.float32(2.0 ** (23 - sh)) == c


def _byte_perm(x, y, sel):
    pool = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(pool[(sel >> (4 * k)) & 7] << (8 * k) for k in range(4))


def test_tensor_core_pair_expansion_is_exact():
    rng = np.random.default_rng(0)
    for _ in range(500):
        codes = rng.integers(0, 16, 8)
        w = int(sum(int(c) << (4 * j) for j, c in enumerate(codes)))
        z = int(rng.integers(0, 16))
        for i in range(4):
            v = _byte_perm(w, w >> 4, i | (i << 4) | ((4 + i) << 8) | (i << 12)) & 0x000F000F
            for hv, c in ((v & 0xFFFF, codes[2 * i]), (v >> 16, codes[2 * i + 1])):
                h = np.array([0x6400 | hv], dtype=np.uint16).view(np.float16)[0]  # f16
                assert float(h) == 1024 + c
                assert float(np.float16(h) - np.float16(1024 + z)) == c - z
                hb = np.array([(0x4300 | hv) << 16], dtype=np.uint32).view(np.float32)[0]  # bf16
                assert float(hb) == 128 + c and 128 + z < 256  # both exact in bf16


def test_small_batch_fragment_schedule():
    # qgemm_mma_kernel: lane (q, p) parks the 16-byte piece p of rows 4 i + q of a
    # 256-column slab at words 4 p .. 4 p + 3 of row 4 i + q (rows of 36 words);
    # for k-step s, fragment lane (g, t) of tile nt reads words 2 s, 2 s + 1 of row
    # 8 nt + g and takes byte t of each: codes 2t, 2t+1 and 2t+8, 2t+9 of the
    # step -- the m16n8k16 B fragment of column g; its accumulators are the C
    # entries (g | g + 8, 2t | 2t + 1), which the kernel sums as (token, row
    # 8 nt + 2t | + 1); the byte becomes the pair (M + c_lo, M + c_hi) exactly.
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (16, 256))
    words = np.zeros((16, 32), dtype=np.uint64)
    for c in range(256):
        words[:, c // 8] |= codes[:, c].astype(np.uint64) << np.uint64(4 * (c % 8))
    park = np.zeros((16, 36), dtype=np.uint64)
    for lane in range(32):
        q, p = lane >> 3, lane & 7
        for i in range(4):
            park[4 * i + q, 4 * p:4 * p + 4] = words[4 * i + q, 4 * p:4 * p + 4]
    for s in range(16):
        for nt in range(2):
            B = np.full((16, 8), -1)
            banks = set()
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                R = 8 * nt + g
                w0, w1 = int(park[R, 2 * s]), int(park[R, 2 * s + 1])
                b = [(w0 >> (8 * t)) & 15, (w0 >> (8 * t + 4)) & 15,
                     (w1 >> (8 * t)) & 15, (w1 >> (8 * t + 4)) & 15]
                for kk, v in zip((2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9), b):
                    assert B[kk, g] == -1
                    B[kk, g] = v
                banks.add((R * 36 + 2 * s) % 32)
            # the B fragments of the 32 lanes are the tile's 16 x 8 operand, each
            # entry once; the 8 rows' reads sit in distinct bank pairs
            assert np.array_equal(B, codes[8 * nt:8 * nt + 8, 16 * s:16 * s + 16].T)
            assert len(banks) == 8
    # C layout: (lane, accumulator e) -> (token, column) covers the 16 x 8 tile once
    seen = set()
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        for e, (tok, n) in enumerate(((g, 2 * t), (g, 2 * t + 1), (g + 8, 2 * t), (g + 8, 2 * t + 1))):
            seen.add((tok, n))
    assert seen == {(tok, n) for tok in range(16) for n in range(8)}
    # byte -> pair (M + c_lo, M + c_hi) in f16 (M = 1024) and bf16 (M = 128)
    for x in range(256):
        h = (x & 0x0F) | ((x & 0xF0) << 12)
        lo, hi = np.array([0x6400 | (h & 0xFFFF), 0x6400 | (h >> 16)],
                          dtype=np.uint16).view(np.float16)
        assert float(lo) == 1024 + (x & 15) and float(hi) == 1024 + (x >> 4)
        blo, bhi = (np.array([(0x4300 | (h & 0xFFFF)) << 16, (0x4300 | (h >> 16)) << 16],
                             dtype=np.uint32).view(np.float32))
        assert float(blo) == 128 + (x & 15) and float(bhi) == 128 + (x >> 4)
