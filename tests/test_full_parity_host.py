"""The counting worker of the full-size parity test, on the CPU: fed the
oracle's own codes it counts nothing; a planted wrong code, scale or bf16
value is counted; and it runs in a spawn-started pool."""

import multiprocessing as mp

import numpy as np

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S

import full_parity as FP
from parity import bf16_bits_rne


def _oracle_outputs(name, r0, r1, ti=0):
    wl = S.WORKLOADS[name]
    x = S.tensor_rows(wl, ti, r0, r1, threads=1)
    ref = O.rotate_quantize(x, block=wl.block, signs=S.signs(wl), bits=wl.bits, group=wl.group,
                            method=FP.oracle_method(wl))
    return wl, ref


def test_oracle_codes_count_nothing():
    wl, ref = _oracle_outputs("c5_tok32768_w11008_b128_signs_int4_g128", 256, 260)
    got = FP.compare_rows(wl.name, 0, 256, 260, ref["codes"], ref["scales"])
    assert got == {"mismatches": 0, "elements": 4 * wl.dim, "far": 0, "scale_bad": 0, "max_scale_rel": 0.0}


def test_planted_errors_are_counted():
    wl, ref = _oracle_outputs("c2_qk_h32_s8192_d128_int8", 0, 64, ti=1)
    codes = ref["codes"].copy()
    v = ref["pre_round"]
    i = np.unravel_index(np.argmax(np.abs(O.half_boundary_distance(v) - 0.5) < 0.3), v.shape)
    codes[i] = np.int8(codes[i] + (1 if codes[i] < 0 else -1))     # off by one, far from a boundary
    scales = ref["scales"].copy()
    scales[3, 0] *= np.float32(1 + 1e-4)
    got = FP.compare_rows(wl.name, 1, 0, 64, codes, scales)
    assert got["mismatches"] == 1 and got["far"] == 1 and got["scale_bad"] == 1


def test_bf16_reconstruction_check():
    wl, ref = _oracle_outputs("c4_kv_h8_t131072_d128_int4_g128", 1000, 1016)
    rec = O.dequant_rotate_inv(ref["codes"], ref["scales"], wl.dim, block=wl.block, bits=wl.bits,
                               group=wl.group)
    bits = bf16_bits_rne(rec)
    got = FP.compare_rows(wl.name, 0, 1000, 1016, ref["codes"], ref["scales"], bits)
    assert got["bf16_bad"] == 0 and got["bf16_exact"] == bits.size
    bad = bits.copy()
    bad[2, 5] ^= np.uint16(0x0004)                                  # four bf16 steps off
    got = FP.compare_rows(wl.name, 0, 1000, 1016, ref["codes"], ref["scales"], bad)
    assert got["bf16_bad"] == 1


def test_runs_in_a_spawned_pool():
    wl, ref = _oracle_outputs("c1_tok256_h4096_b128_int4", 0, 8)
    with mp.get_context("spawn").Pool(2, initializer=FP.init_worker) as p:
        got = p.apply_async(FP.compare_rows, (wl.name, 0, 0, 8, ref["codes"], ref["scales"])).get(timeout=300)
    assert got["mismatches"] == 0 and got["elements"] == 8 * wl.dim
