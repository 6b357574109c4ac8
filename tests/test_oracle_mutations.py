"""The pins catch plausible mistakes in the oracle.

Each case compiles a copy of the oracle's C source with one planted mistake
(on the CPU, in a temporary directory), loads it in place of the real library
for the duration of the case, and checks that at least one of the named pins
fails. The real oracle is restored afterwards.
"""

import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild

import test_oracle_bf16 as tb
import test_oracle_reconcile as trc
import test_oracle_ring as trg
import test_oracle_allreduce as tar
import test_oracle_mx as tmx
import test_oracle_nvfp4 as tnv

SRC = open(obuild.SRC).read()


def _integer_exact():
    trc.test_integer_exact(4, 2, 256, 32)
    trc.test_integer_exact(2, 3, 64, 16)

MUTATIONS = {
    # rounding: half-up instead of half-to-even
    "round_half_up": ("u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;",
                      [tb.test_bf16_rne_matches_exact_rounding_on_edges]),
    # rounding: truncation
    "round_truncate": ("u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0u;",
                       [tb.test_bf16_rne_matches_torch_conversion]),
    # ring: chunks travel the other way round the ring
    "ring_direction": ("int src = (r - 1 + N) % N;\n            int c = ((src - s) % N + N) % N;",
                       "int src = (r + 1) % N;\n            int c = ((src - s) % N + N) % N;",
                       [trg.test_ring_fold_order_golden]),
    # ring: chunk c starts one rank late
    "ring_start": ("int c = ((r - s) % N + N) % N;", "int c = ((r - s + 1) % N + N) % N;",
                   [trg.test_ring_fold_order_golden]),
    # partials: accumulate in double (not the fp32 reading)
    "acc_double": ([("float acc = 0.0f;", "double acc = 0.0;"),
                    ("acc = fmaf(orc_f32(xr[kk]), orc_f32(wr[kk]), acc);",
                     "acc = fma((double)orc_f32(xr[kk]), (double)orc_f32(wr[kk]), acc);")],
                   None, [trc.test_partial_order_fp32_ascending]),
    # partials: the product rounded to fp32 before it is added
    "round_then_add": ("acc = fmaf(orc_f32(xr[kk]), orc_f32(wr[kk]), acc);",
                       "acc = acc + orc_f32(xr[kk]) * orc_f32(wr[kk]);",
                       [trc.test_partial_adds_each_product_with_one_rounding]),
    # partials: k descending
    "k_descending": ("for (int64_t kk = 0; kk < ks; ++kk) {",
                     "for (int64_t kk = ks - 1; kk >= 0; --kk) {",
                     [trc.test_partial_order_fp32_ascending]),
    # partials: subtract instead of add
    "acc_sign": ("acc = fmaf(orc_f32(xr[kk]), orc_f32(wr[kk]), acc);",
                 "acc = fmaf(-orc_f32(xr[kk]), orc_f32(wr[kk]), acc);",
                 [_integer_exact]),
    # partials: a rank reads the wrong slice of x
    "x_slice": ("const uint16_t *xr = j->x + m * j->k + (int64_t)r * ks;",
                "const uint16_t *xr = j->x + m * j->k;",
                [_integer_exact]),
    # residual dropped
    "no_residual": ("out[i] = orc_bf16_rne(orc_f32(residual[i]) + orc_f32(reduced[i]));",
                    "out[i] = reduced[i];",
                    [_integer_exact]),
    # byte model: N in place of N-1
    "bytes_n": ("return 2u * (uint64_t)(n_ranks - 1) * payload",
                "return 2u * (uint64_t)(n_ranks) * payload",
                [trg.test_ring_bytes_pages_worked_example]),
    # all-reduce schemes: the switch hands back every slice, not one
    "sharp_all_slices": ("        slices += 1;          /* the reduced slice r from the switch */",
                         "        slices += (uint64_t)n_ranks;",
                         [tar.test_allreduce_bytes_golden]),
    # all-reduce schemes: the naive reader also counts its own buffer
    "naive_self": ("                for (int c = 0; c < n_ranks; ++c)\n                    slices += 1;  /* every slice of the peer's buffer */",
                   "                for (int c = 0; c < n_ranks; ++c)\n                    slices += 1;  /* every slice of the peer's buffer */\n        slices += (uint64_t)n_ranks;",
                   [tar.test_allreduce_bytes_golden]),
    # MoE combine: the local accumulation is skipped (every slot all-reduced)
    "combine_no_local_acc": ("const int64_t buffers = local_accumulate ? 1 : top_k;",
                             "const int64_t buffers = top_k;",
                             [tar.test_moe_combine_bytes_golden]),
    # NVFP4: E2M1 ties go up instead of to the even index
    "e2m1_half_up": ("    if (d_hi < d_lo || (d_hi == d_lo && (lo & 1)))",
                     "    if (d_hi <= d_lo)",
                     [lambda: [tnv.test_e2m1_midpoints_and_saturation(v, c)
                               for v, c in ((0.25, 0), (1.25, 2), (2.5, 4))]]),
    # NVFP4: no saturation at 6
    "e2m1_no_saturation": ("    if (a >= 6.0)\n        return sign | 7;\n", "    if (a >= 12.0)\n        return sign | 7;\n",
                           [lambda: tnv.test_e2m1_midpoints_and_saturation(6.5, 7)]),
    # NVFP4: the second-level exponent one too large
    "nvfp4_g_plus_one": ("    while (amax / ldexp(1.0, g) > 6.0 * 448.0)\n        ++g;\n    return g;",
                         "    while (amax / ldexp(1.0, g) > 6.0 * 448.0)\n        ++g;\n    return g + 1;",
                         [lambda: tnv.test_global_exponent_rule(0.1)]),
    # MXFP8: element rounding half away from zero instead of to even
    "e4m3_half_up": ("if (rem > 0.5 || (rem == 0.5 && fmod(m, 2.0) == 1.0))",
                     "if (rem >= 0.5)",
                     [tmx.test_e4m3_midpoints_go_to_even_and_saturation]),
    # MXFP8: shared exponent from E4M3's bias instead of its largest exponent
    "mx_exp_off_by_one": ("int s = (e - 1) - 8;", "int s = (e - 1) - 7;",
                          [tmx.test_scale_rule_and_block_max]),
    # MXFP8: no saturation at 448
    "e4m3_no_saturation": ("    if (a >= 448.0)\n        return sign | 0x7E;\n", "",
                           [tmx.test_e4m3_midpoints_go_to_even_and_saturation]),
}


def _build_mutant(name, old, new):
    edits = old if isinstance(old, list) else [(old, new)]
    text = SRC
    for o, n in edits:
        assert text.count(o) >= 1, f"mutation {name}: pattern not found"
        text = text.replace(o, n)
    d = tempfile.mkdtemp(prefix="orc_mut_")
    src = os.path.join(d, "m.c")
    lib = os.path.join(d, "libm.so")
    with open(src, "w") as f:
        f.write(text)
    subprocess.run(["gcc", *[c for c in obuild.CFLAGS if c != "-Werror"], src, "-o", lib, "-lm"],
                   check=True)
    return lib


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pin_catches_mutation(name, monkeypatch):
    old, new, pins = MUTATIONS[name]
    path = _build_mutant(name, old, new)
    real = oracle.lib()
    mutant = ctypes.CDLL(path)
    for fn in ("orc_bf16_rne", "orc_bf16_rne_f64", "orc_f32", "orc_bf16_rne_array",
               "orc_bf16_rne_f64_array", "orc_partials", "orc_ring", "orc_residual",
               "orc_reconcile", "orc_ring_bytes", "orc_allreduce_bytes", "orc_moe_combine_bytes",
               "orc_e4m3_rne", "orc_e2m1_rne", "orc_e2m1_value", "orc_nvfp4_global_exp",
               "orc_nvfp4_quantize", "orc_nvfp4_dequant_bf16",
               "orc_e4m3_value", "orc_mx_quantize", "orc_mx_dequant_bf16"):
        f = getattr(mutant, fn)
        g = getattr(real, fn)
        f.argtypes, f.restype = g.argtypes, g.restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, oracle.OracleError):
            caught += 1
    assert caught, f"no pin caught mutation {name}"
