"""ctypes loader for libtokengate.so with the C signatures of include/tokengate.h.

There is no fallback: if the shared library is missing the import fails with a
message naming the build command.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtokengate.so")

_p = C.c_void_p
_i32 = C.c_int
_i64 = C.c_int64
_f32 = C.c_float
_f64 = C.c_double
_sz = C.c_size_t

# name -> (restype, argtypes); mirrors include/tokengate.h
SIGNATURES = {
    "tg_error_string": (C.c_char_p, [_i32]),
    "tg_last_cuda_error": (_i32, []),
    "tg_device_supported": (_i32, [_i32]),
    "tg_version": (_i32, []),
    "tg_status_clear": (_i32, [_p, _p]),
    "tg_status_read": (_i32, [_p, _p, _p]),
    "tg_set_launch_overlap": (_i32, [_i32]),
    "tg_get_launch_overlap": (_i32, []),
    "tg_set_gather_tma": (_i32, [_i32]),
    "tg_get_gather_tma": (_i32, []),
    "tg_set_scorer_pair": (_i32, [_i32]),
    "tg_get_scorer_pair": (_i32, []),
    "tg_prefetch_l2": (_i32, [_p, _sz, _p]),
    "tg_rope_table": (_i32, [_p, _i32, _i32, _f64, _p]),
    "tg_rope_rows": (_i32, [_p, _i64, _p, _i32, _i32, _p, _i64, _p, _p]),
    "tg_plan_kept": (_i32, [_p, _p, _p, _i32, _p]),
    "tg_gate_score_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "tg_gate_score": (_i32, [_p, _i64, _i64, _i32, _p, _p, _i32, _p, _f32, _p, _p, _i32, _f32,
                             _p, _p, _p, _p, _p, _sz, _p, _p]),
    "tg_gate_score_noalloc": (_i32, [_p, _i64, _i64, _i32, _p, _p, _i32, _p, _f32, _p, _p, _i32,
                                     _f32, _p, _p, _p, _p, _p, _p]),
    "tg_seq_rmsnorm": (_i32, [_p, _p, _p, _i32, _p, _f32, _p, _p, _p]),
    "tg_topk_compact": (_i32, [_p, _p, _p, _p, _p, _p, _i32, _p, _p, _p, _p, _p]),
    "tg_gather_rope": (_i32, [_p, _i64, _i64, _p, _i64, _i32, _p, _i32, _i32, _i32, _p, _i32,
                              _p, _i64, _p, _i64, _p, _p]),
    "tg_kv_compact": (_i32, [_p, _i64, _p, _i64, _i64, _p, _i64, _i32, _p, _p, _i64, _i64, _i64,
                             _p, _p]),
    "tg_gated_attention": (_i32, [_p, _i64, _p, _i64, _p, _i64, _p, _p, _i32, _i32, _i32, _i32,
                                  _p, _p, _p, _f32, _p, _i64, _p, _p, _sz, _p, _p]),
    "tg_gated_attention_workspace_size": (_sz, [_p, _i32, _i32, _i32, _i32]),
    "tg_qkv_rope_cache": (_i32, [_p, _i64, _p, _i64, _i64, _i32, _i32, _i32, _i32, _f32, _p, _p,
                                 _i32, _p, _i64, _p, _p, _i64, _i64, _p, _i64, _p, _sz, _p, _p]),
    "tg_qkv_qknorm_rope_cache": (_i32, [_p, _i64, _p, _i64, _i64, _i32, _i32, _i32, _i32, _f32,
                                        _p, _p, _p, _p, _i32, _p, _i64, _p, _p, _i64, _i64,
                                        _p, _i64, _p, _sz, _p, _p]),
    "tg_gemm_workspace_size": (_sz, []),
    "tg_gated_attention_bias_grad": (_i32, [_p, _i64, _p, _i64, _p, _i64, _p, _i64, _p, _i64,
                                            _p, _p, _p, _i32, _i32, _i32, _i32, _p, _p, _p,
                                            _f32, _p, _p, _p, _p, _sz, _p, _p]),
    "tg_gated_attention_bias_grad_workspace_size": (_sz, [_p, _i32, _i32, _i32, _i32]),
    "tg_gate_score_backward": (_i32, [_p, _i64, _i64, _i32, _p, _p, _i32, _p, _f32, _p, _p, _p,
                                      _i32, _f32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz,
                                      _p, _p]),
    "tg_gate_score_backward_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "tg_swiglu": (_i32, [_p, _i64, _p, _i64, _i64, _i32, _i32, _f32, _p, _i64, _p, _i64, _p,
                         _p]),
    "tg_fold_norm_weight": (_i32, [_p, _i64, _i64, _i32, _p, _p, _i64, _p]),
    "tg_pack_gate_up": (_i32, [_p, _i64, _p, _i64, _i32, _i32, _p, _p, _i64, _p]),
    "tg_out_proj_qkv_next": (_i32, [_p, _i64, _p, _i64, _p, _i64, _p, _i64, _i64, _i32, _i32,
                                     _p, _i64, _i32, _i32, _i32, _f32, _p, _p, _i32, _p, _i64,
                                     _p, _p, _i64, _i64, _p, _sz, _p, _p]),
    "tg_out_proj_qkv_workspace_size": (_sz, [_i64]),
    "tg_linear": (_i32, [_p, _i64, _p, _i64, _p, _i64, _i64, _i32, _i32, _i32, _f32, _p, _i64,
                         _p, _i64, _p, _sz, _p, _p]),
}


def load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python learned_token_pruning_scoring_b200/build.py` (nvcc, sm_100a)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
