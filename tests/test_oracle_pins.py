"""The oracle against its pins, plus mutants that the pins must catch (CPU only)."""
import json
import os
import shutil

import pytest

import mla_workloads as W
import oracle
import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.load())


# Mistakes planted in copies of the oracle's C source.  Each replaces one
# exact snippet; every mutant must fail at least one pin.
MUTANTS = {
    "drop_rope_term": ("dot += oracle_bf16_to_f64(qp[d]) * kv_value(p, page, slot, ORACLE_DL + d);",
                       "dot += 0.0;"),
    "exp_sign_flipped": ("Z += exp(scores[j] - M);", "Z += exp(M - scores[j]);"),
    "page_index_from_slot": ("int32_t page = p->page_table[(int64_t)b * p->page_table_stride + j / ORACLE_PAGE];\n        int slot = j % ORACLE_PAGE;\n        double dot",
                             "int32_t page = p->page_table[(int64_t)b * p->page_table_stride + j % ORACLE_PAGE];\n        int slot = j % ORACLE_PAGE;\n        double dot"),
    "mask_off_by_one": ("return p->ctx_lens[b] - p->T + t + 1;", "return p->ctx_lens[b] - p->T + t;"),
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal_exp": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "value_reads_shifted": ("out[d] += w * kv_value(p, page, slot, d);",
                            "out[d] += w * kv_value(p, page, slot, d + 1);"),
    "fp8_scale_dropped": ("* (double)p->kv_scale[p->kv_scale_per_tensor ? 0 : row];", "* 1.0;"),
    "lse_base2": ("*lse = M + log(Z);", "*lse = M + log2(Z);"),
    "sm_scale_dropped": ("scores[j] = p->sm_scale * dot;", "scores[j] = dot;"),
    "merge_unweighted": ("double w = exp(l - L);", "double w = 1.0;"),
    "bf16_shift": ("uint32_t u = (uint32_t)bits << 16;", "uint32_t u = (uint32_t)bits << 15;"),
    "head_token_swapped": ("int h = (int)(row % p->H);\n    int t = (int)((row / p->H) % p->T);",
                           "int t = (int)(row % p->T);\n    int h = (int)((row / p->T) % p->H);"),
    "weights_not_normalised": ("double w = exp(scores[j] - M) / Z;", "double w = exp(scores[j] - M);"),
    "e4m3_encode_truncates": ("double r = nearbyint(n);                /* default rounding: ties to even */",
                              "double r = floor(n);"),
    "e4m3_encode_no_clamp": ("if (a > 448.0) a = 448.0;", ""),
    "quantise_scale_447": ("float scale = amax / 448.0f;", "float scale = amax / 447.0f;"),
    "append_position_shifted": ("int pos = ctx - T + t;", "int pos = ctx - T + t + 1;"),
    "append_drops_rope": ("memcpy(row + ORACLE_DL, k_pe_new", "memset(row + ORACLE_DL, 0, 1); (void)(k_pe_new"),
    "empty_row_lse_zero": ("*lse = -INFINITY;\n        return 0;", "*lse = 0.0;\n        return 0;"),
    "merge_nan_not_checked": ("if (poisoned) {", "if (0) {"),
    "vis_lens_transposed": ("return p->vis_lens[(int64_t)b * p->T + t];", "return p->vis_lens[(int64_t)t * p->B + b];"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_dir):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    msrc = os.path.join(mutant_dir, f"{name}.c")
    mlib = os.path.join(mutant_dir, f"{name}.so")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    oracle.build(src=msrc, out=mlib)
    lib = oracle.load(mlib)
    caught = []
    for pin in oracle_pins.PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"


def test_pages_byte_formula():
    """24 layers x 142,000 positions x 576 FP8 bytes is the printed ~1.96 GB, ~245 MB with DCP8."""
    g = json.load(open(GOLDEN))["mla_payload"]
    total = g["layers"] * g["positions"] * g["fp8_bytes_per_position"]
    assert total == 1_963_008_000
    assert round(total / 1e9, 2) == g["total_gb_printed"]
    assert round(total / g["dcp_ways"] / 1e6) == g["dcp8_mb_printed"]
    # 576 stored values per position: the 512 + 64 reading of the workloads
    assert W.D_QK == g["fp8_bytes_per_position"]
    # one layer of the 142K workload in the per-token-scaled format
    assert g["positions"] * (W.D_QK + 4) == 82_360_000


def test_pages_paging_and_heads():
    g = json.load(open(GOLDEN))
    assert W.PAGE == g["page_size"]["tokens_per_page"]
    hp = g["head_padding"]
    assert hp["total_heads"] // hp["tp"] == hp["heads_per_rank"]
    assert W.CONFIGS["spec_verify_small"].H == hp["heads_per_rank"]
    assert W.CONFIGS["long_ctx_142k"].H == hp["total_heads"]


def test_pages_fp8_capacity_ratio():
    """FP8 halves bytes per position: 1152 bf16 bytes vs 576 (+4 scale) FP8 bytes."""
    g = json.load(open(GOLDEN))["fp8_capacity"]
    printed = g["fp8_tokens"] / g["bf16_tokens"]
    assert round(printed, 2) == g["ratio_printed"]
    ours_per_tensor = (2 * W.D_QK) / W.D_QK
    ours_per_token = (2 * W.D_QK) / (W.D_QK + 4)
    assert abs(ours_per_tensor - printed) < 0.01
    assert abs(ours_per_token - printed) < 0.03


def test_oracle_rejects_bad_page():
    w = oracle_pins._small(W.KV_BF16, T=1, H=1, B=1, ctx=("fixed", 20), seed=1)
    w.page_table[0, 1] = w.num_pages + 5
    with pytest.raises(ValueError):
        oracle.decode_workload(w)


def test_oracle_sampled_rows_equal_full():
    w = oracle_pins._small(W.KV_FP8, T=3, H=4, B=2, seed=2)
    full_o, full_l = oracle.decode_workload(w)
    rows = W.sample_rows(w.B, w.T, w.H, 7)
    so, sl = oracle.decode_workload(w, rows=rows)
    assert (so == full_o[rows.numpy()]).all() and (sl == full_l[rows.numpy()]).all()
