"""Host-side arithmetic of bench.py: the byte and flop models the roofline
fractions divide by, and the workload description of the variants."""

import os
import sys

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_hessian_issued_tiles_at_q_proj():
    # 128 x 256 tiles that reach the upper triangle of a 4096 x 4096 H:
    # row tile i keeps column tiles j >= floor(i / 2): 512 - 2 * (0 + ... + 15) = 272
    s = synth.CONFIGS["q_proj"]
    assert bench.hessian_issued_flop(s) == 2.0 * s.n * 272 * 128 * 256
    assert 1.06 < bench.hessian_issued_flop(s) / (s.n * s.k * (s.k + 1)) < 1.07


def test_sweep_byte_model_at_q_proj():
    # 8 r sigma + 4 B sigma + 16 r k + r k + 2 r k with sigma = B nb (nb - 1) / 2
    s = synth.CONFIGS["q_proj"]
    r, k, B = s.r, s.k, s.block_size
    nb = k // B
    sigma = B * nb * (nb - 1) // 2
    assert bench.sweep_model_bytes(s) == 8 * r * sigma + 4 * B * sigma + 16 * r * k + r * k + 2 * r * k
    assert abs(bench.sweep_model_bytes(s) - 2.43e9) < 0.01e9


def test_workload_names_the_variants():
    s = synth.CONFIGS["q_proj"].scaled(act_order=True, sym=True, static_groups=True)
    w = bench.workload_config(s)["workload"]
    assert "int4 sym g128" in w and "act-order" in w and "static-groups" in w
    assert "asym" in bench.workload_config(synth.CONFIGS["q_proj"])["workload"]
