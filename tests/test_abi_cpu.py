"""CPU checks of the C ABI: the library loads, exports every entry point that
include/ssta.h declares, plans sizes that agree with the oracle's geometry, and
rejects malformed calls on the host with the documented status codes."""
import os
import re
import subprocess
import sys

import pytest

import block_sparse_video_ssta_b200 as S
import oracle
import ssta_inputs as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "ssta.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+(ssta_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert set(names) >= {"ssta_plan", "ssta_tile_reorder", "ssta_build_block_mask", "ssta_attention_fwd",
                          "ssta_tile_unorder", "ssta_status_string", "ssta_read_device_status"}
    out = subprocess.run(["nm", "-D", "--defined-only", S.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ssta_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(S.lib, n)


def test_status_strings():
    assert S.ssta_status_string(0) == "SSTA_OK"
    assert S.ssta_status_string(6) == "SSTA_ERR_DEVICE_TIMEOUT"
    assert S.ssta_status_string(99) == "SSTA_ERR_UNKNOWN"


@pytest.mark.parametrize("name", list(si.WORKLOADS))
def test_plan_matches_oracle_geometry(name):
    w = si.get_workload(name)
    p = S.ssta_plan(S.desc_from(w))
    g = oracle.geometry(w)
    assert (p.packed_len, p.num_tiles, p.num_text_tiles, p.num_q_tiles, p.tile_tokens, p.topk) == \
        (g.Lq, g.NT, g.n_text, g.NQ, g.N, g.k)
    W = int(oracle.window_mask(w)[0].sum())
    assert p.window_tiles == W
    # the kv_idx row must hold the longest kept list the oracle can produce
    longest = g.NT + g.n_text if g.n_text else min(g.NT, g.k + W)
    assert p.max_kept == longest
    assert p.workspace_bytes >= 256 and p.attn_workspace_bytes == 256


def test_host_validation_codes():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "abi_validation_cases.py")], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    got = dict(line.split() for line in r.stdout.strip().splitlines())
    got = {k: int(v) for k, v in got.items()}
    OK, INVALID, UNSUP, ALIGN, WS = 0, 1, 2, 3, 4
    expect = {
        "plan_null_desc": INVALID, "plan_null_info": INVALID, "plan_bad_B": INVALID, "plan_bad_T": INVALID,
        "plan_bad_tX": INVALID, "plan_bad_wY": INVALID, "plan_bad_topk": INVALID, "plan_bad_L_text": INVALID,
        "plan_bad_dtype": INVALID, "plan_bad_score_mode": INVALID, "plan_bad_lambda_high": INVALID,
        "plan_bad_lambda_nan": INVALID, "plan_bad_combine": INVALID, "plan_bad_window_mode": INVALID,
        "plan_similarity_ignores_lambda": OK, "plan_all_modes": OK, "plan_importance_workspace_larger": OK,
        "plan_D64": UNSUP, "plan_tile_too_big": UNSUP, "plan_too_many_tiles": UNSUP,
        "plan_neg_scale": INVALID, "reorder_null_out": INVALID, "reorder_misaligned": ALIGN,
        "reorder_text_missing": INVALID, "unorder_null_in": INVALID, "unorder_misaligned_text": ALIGN,
        "mask_no_workspace": WS, "mask_small_workspace": WS, "mask_ws_misaligned": ALIGN, "mask_null_q": INVALID,
        "mask_misaligned_cnt": ALIGN, "attn_bf16_tile_not_128": UNSUP, "attn_no_workspace": WS,
        "attn_small_workspace": WS, "attn_null_q": INVALID, "attn_misaligned_o": ALIGN,
        "bwd_no_workspace": WS, "bwd_small_workspace": WS, "bwd_ws_misaligned": ALIGN, "bwd_null_do": INVALID,
        "bwd_misaligned_dk": ALIGN, "bwd_bad_desc": INVALID, "bwd_bf16_tile_not_128": UNSUP,
        "read_status_null": INVALID, "selftest_timeout_zero": INVALID, "selftest_timeout_huge": INVALID,
        "selftest_no_workspace": WS,
    }
    assert got == expect


def test_binding_refuses_cpu_tensors():
    import torch
    w = si.get_workload("tiny_f32")
    d = S.desc_from(w)
    x = torch.zeros((1, 2, 4, 8, 8, 128))
    with pytest.raises(ValueError, match="CUDA tensor"):
        S.ssta_tile_reorder(d, x)
