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
