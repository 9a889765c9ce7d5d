"""Host-side argument validation of libssta.so, run in a child process with no
visible CUDA device (CUDA_VISIBLE_DEVICES=""), so that a validation bug could
at worst produce a launch error, never a kernel running on bogus pointers.
Prints one line per case: name, returned status."""
import ctypes
import os
import sys

assert os.environ.get("CUDA_VISIBLE_DEVICES") == "", "run only with CUDA_VISIBLE_DEVICES=''"
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import block_sparse_video_ssta_b200 as S  # noqa: E402

lib = S.lib
A = 0x10000   # fake, 256-byte aligned, never dereferenced
P = ctypes.c_void_p


def desc(**kw):
    base = dict(B=1, H=2, D=128, T=4, Y=8, X=8, tT=2, tY=4, tX=4, wT=1, wY=1, wX=1, topk=2, L_text=0,
                dtype=S.SSTA_F32, scale=0.0)
    base.update(kw)
    return S.Desc(**base)


def call(name, *args):
    return getattr(lib, name)(*args)


cases = []
d = desc()
info = S._PlanInfo()
cases.append(("plan_null_desc", call("ssta_plan", None, ctypes.byref(info))))
cases.append(("plan_null_info", call("ssta_plan", ctypes.byref(d), None)))
for field, val, _ in [("B", -1, 1), ("T", 0, 1), ("tX", 0, 1), ("wY", 0, 1), ("topk", -1, 1),
                      ("L_text", -2, 1), ("dtype", 7, 1)]:
    cases.append((f"plan_bad_{field}", call("ssta_plan", ctypes.byref(desc(**{field: val})), ctypes.byref(info))))
cases.append(("plan_D64", call("ssta_plan", ctypes.byref(desc(D=64)), ctypes.byref(info))))
for name, kw in [("score_mode", dict(score_mode=2)), ("lambda_high", dict(score_mode=1, lambda_=1.5)),
                 ("lambda_nan", dict(score_mode=1, lambda_=float("nan"))), ("combine", dict(combine=3)),
                 ("window_mode", dict(window_mode=-1))]:
    cases.append((f"plan_bad_{name}", call("ssta_plan", ctypes.byref(desc(**kw)), ctypes.byref(info))))
# lambda is ignored by the similarity score; modes in range are accepted
cases.append(("plan_similarity_ignores_lambda", call("ssta_plan", ctypes.byref(desc(lambda_=float("nan"))),
                                                     ctypes.byref(info))))
cases.append(("plan_all_modes", call("ssta_plan", ctypes.byref(desc(score_mode=1, lambda_=0.9, combine=1,
                                                                    window_mode=1)), ctypes.byref(info))))
_sim = S._PlanInfo(); _imp = S._PlanInfo()
call("ssta_plan", ctypes.byref(desc()), ctypes.byref(_sim))
call("ssta_plan", ctypes.byref(desc(score_mode=1, lambda_=0.9)), ctypes.byref(_imp))
cases.append(("plan_importance_workspace_larger", 0 if _imp.workspace_bytes > _sim.workspace_bytes else 99))
cases.append(("plan_tile_too_big", call("ssta_plan", ctypes.byref(desc(tT=16, tY=16, tX=32)), ctypes.byref(info))))
cases.append(("plan_too_many_tiles", call("ssta_plan", ctypes.byref(desc(T=64, Y=64, X=64, tT=1, tY=1, tX=1)),
                                         ctypes.byref(info))))
bad_scale = desc()
bad_scale.scale = -1.0
cases.append(("plan_neg_scale", call("ssta_plan", ctypes.byref(bad_scale), ctypes.byref(info))))

cases.append(("reorder_null_out", call("ssta_tile_reorder", ctypes.byref(d), P(A), None, None, None)))
cases.append(("reorder_misaligned", call("ssta_tile_reorder", ctypes.byref(d), P(A + 8), None, P(A), None)))
dt = desc(L_text=5)
cases.append(("reorder_text_missing", call("ssta_tile_reorder", ctypes.byref(dt), P(A), None, P(A), None)))
cases.append(("unorder_null_in", call("ssta_tile_unorder", ctypes.byref(d), None, P(A), None, None)))
cases.append(("unorder_misaligned_text", call("ssta_tile_unorder", ctypes.byref(dt), P(A), P(A), P(A + 4), None)))

cases.append(("mask_no_workspace", call("ssta_build_block_mask", ctypes.byref(d), P(A), P(A), P(A), P(A), None,
                                        None, ctypes.c_size_t(0), None)))
cases.append(("mask_small_workspace", call("ssta_build_block_mask", ctypes.byref(d), P(A), P(A), P(A), P(A), None,
                                           P(A), ctypes.c_size_t(300), None)))
cases.append(("mask_ws_misaligned", call("ssta_build_block_mask", ctypes.byref(d), P(A), P(A), P(A), P(A), None,
                                         P(A + 16), ctypes.c_size_t(1 << 30), None)))
cases.append(("mask_null_q", call("ssta_build_block_mask", ctypes.byref(d), None, P(A), P(A), P(A), None,
                                  P(A), ctypes.c_size_t(1 << 30), None)))
cases.append(("mask_misaligned_cnt", call("ssta_build_block_mask", ctypes.byref(d), P(A), P(A), P(A), P(A + 4), None,
                                          P(A), ctypes.c_size_t(1 << 30), None)))

attn = lambda dd, q=P(A), o=P(A), ws=P(A), wsb=4096: call(
    "ssta_attention_fwd", ctypes.byref(dd), q, P(A), P(A), P(A), P(A), o, P(A), ws, ctypes.c_size_t(wsb), None)
cases.append(("attn_bf16_tile_not_128", attn(desc(dtype=S.SSTA_BF16))))
cases.append(("attn_no_workspace", attn(d, ws=None)))
cases.append(("attn_small_workspace", attn(d, wsb=64)))
cases.append(("attn_null_q", attn(d, q=None)))
cases.append(("attn_misaligned_o", attn(d, o=P(A + 2))))
bwd = lambda dd, ws=P(A), wsb=1 << 30, do=P(A), dk=P(A): call(
    "ssta_attention_bwd", ctypes.byref(dd), P(A), P(A), P(A), P(A), P(A), do, P(A), P(A), P(A), dk, P(A), ws,
    ctypes.c_size_t(wsb), None)
cases.append(("bwd_no_workspace", bwd(d, ws=None)))
cases.append(("bwd_small_workspace", bwd(d, wsb=64)))
cases.append(("bwd_ws_misaligned", bwd(d, ws=P(A + 16))))
cases.append(("bwd_null_do", bwd(d, do=None)))
cases.append(("bwd_misaligned_dk", bwd(d, dk=P(A + 8))))
cases.append(("bwd_bad_desc", bwd(desc(topk=-1))))
cases.append(("bwd_bf16_tile_not_128", bwd(desc(dtype=S.SSTA_BF16))))
cases.append(("read_status_null", call("ssta_read_device_status", None, None, None)))
lib.ssta_selftest_bounded_wait.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p]
cases.append(("selftest_timeout_zero", lib.ssta_selftest_bounded_wait(0, 0, P(A), 4096, None)))
cases.append(("selftest_timeout_huge", lib.ssta_selftest_bounded_wait(3000000, 0, P(A), 4096, None)))
cases.append(("selftest_no_workspace", lib.ssta_selftest_bounded_wait(1000, 0, None, 0, None)))

for name, code in cases:
    print(name, code)
