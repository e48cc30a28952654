"""ctypes binding of libmla.so: one Python function per C entry point, same names.

Arguments are marshalled only: torch tensors (or raw integer addresses) become
pointers, ``None`` becomes NULL, streams default to torch's current stream.
Every call raises MlaError on a non-OK status. Nothing here computes; every
step of the decode path runs in the library's CUDA kernels.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

MLA_OK = 0
MLA_ERR_INVALID_ARGUMENT = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE = 5

MLA_DEV_BAD_PAGE = 0x1
MLA_DEV_BAD_POSITION = 0x2
MLA_DEV_TIMEOUT = 0x4
MLA_DEV_BAD_PLAN = 0x8
MLA_DEV_RANGE = 0x10

D_C, D_R, D_NOPE, D_V, ROW, PAGE = 512, 64, 128, 128, 576, 64
MAX_Q_LEN = 1024

_STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARGUMENT", 2: "MLA_ERR_UNSUPPORTED",
                 3: "MLA_ERR_WORKSPACE_TOO_SMALL", 4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE"}


class MlaError(RuntimeError):
    def __init__(self, status: int, func: str, msg: str):
        self.status = status
        super().__init__(f"{func}: {_STATUS_NAMES.get(status, status)}: {msg}")


class mla_plan_info_t(ctypes.Structure):
    _fields_ = [("num_items", ctypes.c_int), ("num_ctas", ctypes.c_int),
                ("num_partials", ctypes.c_int), ("num_combine", ctypes.c_int),
                ("plan_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "mla_last_error": (ctypes.c_char_p, []),
    "mla_version": (_I, []),
    "mla_rope_table": (_I, [_P, _I, ctypes.c_double]),
    "mla_cache_append": (_I, [_P, _I, _P, _I, _I, _P, _P, _P, _I, _P, _I, _P, _I, _I, _P, _P]),
    "mla_absorb_q": (_I, [_P, _I, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "mla_plan_bytes": (_SZ, [_I, _I, _I]),
    "mla_decode_plan": (_I, [_P, _I, _I, _I, _I, _I, _P, _SZ, ctypes.POINTER(mla_plan_info_t)]),
    "mla_decode_attention": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _P, _SZ, _P, _P,
                                  _P, _P]),
    "mla_debug_decode_wait": (_I, [ctypes.c_double, _I]),
    "mla_debug_gemm_plan": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "mla_decode_attention_cudacore": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _P, _SZ,
                                           _P, _P, _P, _P]),
    "mla_decode_attention_noalloc": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _P, _P,
                                          _P, _P]),
    "mla_out_absorb": (_I, [_P, _P, _I, _I, _P, _I, _P]),
    "mla_gemm_bf16": (_I, [_P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _P]),
    "mla_gemm_bf16_workspace_bytes": (_SZ, [_I, _I, _I]),
    "mla_gemm_bf16_ws": (_I, [_P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "mla_read_status": (_I, [_P, _P, _I, _P]),
    "mla_check_status": (_I, [_P, _P, _P]),
    "mla_reset_status": (_I, [_P, _P]),
    "mla_plan_used_bytes": (_SZ, [_P]),
    "mla_plan_upload": (_I, [_P, _P, _SZ, _P]),
    "mla_cache_append_fp8": (_I, [_P, _P, _I, _P, _I, _I, _P, _P, _P, _I, _P, _I, _P, _I, _I,
                                  _P, _P]),
    "mla_decode_attention_fp8": (_I, [_P, _P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _P, _SZ,
                                      _P, _P, _P, _P]),
    "mla_append_absorb_q": (_I, [_P, _I, _P, _I, _I, _P, _P, _P, _I, _P, _I, _I, _P, _I, _P, _I,
                                 _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "mla_append_fp8_absorb_q": (_I, [_P, _P, _I, _P, _I, _I, _P, _P, _P, _I, _P, _I, _I, _P,
                                     _I, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "mla_fold_qk_workspace_bytes": (_SZ, [_I]),
    "mla_fold_qk": (_I, [_P, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "mla_fold_o": (_I, [_P, _I, _I, _P, _I, _P, _P]),
    "mla_absorb_q_folded": (_I, [_P, _I, _I, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
}

_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmla.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with mla_latent_kv_32_b200.build.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, name: str):
    if st != MLA_OK:
        raise MlaError(st, name, load().mla_last_error().decode(errors="replace"))


def mla_version() -> int:
    return load().mla_version()


def mla_rope_table(max_pos: int, base: float = 10000.0) -> np.ndarray:
    """Host RoPE table float32 [max_pos, 32, 2] of (cos, sin)."""
    out = np.empty((max_pos, D_R // 2, 2), dtype=np.float32)
    _check(load().mla_rope_table(out.ctypes.data, max_pos, base), "mla_rope_table")
    return out


def mla_cache_append(cache, num_pages, block_table, batch, max_pages, seq_idx, pos, c_kv, ld_c,
                     k_pe, ld_k, rope_table, max_pos, n_tokens, status=None, stream=None):
    _check(load().mla_cache_append(_ptr(cache), num_pages, _ptr(block_table), batch, max_pages,
                                   _ptr(seq_idx), _ptr(pos), _ptr(c_kv), ld_c, _ptr(k_pe), ld_k,
                                   _ptr(rope_table), max_pos, n_tokens, _ptr(status),
                                   _stream(stream)), "mla_cache_append")


def mla_absorb_q(q_nope, ld_qn, q_pe, ld_qp, w_uk, pos, rope_table, max_pos, T, n_h, q_full,
                 status=None, stream=None):
    _check(load().mla_absorb_q(_ptr(q_nope), ld_qn, _ptr(q_pe), ld_qp, _ptr(w_uk), _ptr(pos),
                               _ptr(rope_table), max_pos, T, n_h, _ptr(q_full), _ptr(status),
                               _stream(stream)), "mla_absorb_q")


def mla_plan_bytes(batch: int, q_len: int, num_ctas: int = 0) -> int:
    return int(load().mla_plan_bytes(batch, q_len, num_ctas))


def mla_decode_plan(seq_lens: np.ndarray, batch: int, q_len: int, n_h: int, num_ctas: int = 0,
                    max_split: int = -1):
    """Returns (plan bytes as a uint8 numpy array, mla_plan_info_t)."""
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    nbytes = mla_plan_bytes(batch, q_len, num_ctas)
    plan = np.zeros(max(nbytes, 64), dtype=np.uint8)
    info = mla_plan_info_t()
    _check(load().mla_decode_plan(lens.ctypes.data if batch else None, batch, q_len, n_h,
                                  num_ctas, max_split, plan.ctypes.data, plan.nbytes,
                                  ctypes.byref(info)), "mla_decode_plan")
    return plan, info


def mla_decode_attention(q_full, cache, num_pages, block_table, max_pages, batch, q_len, n_h,
                         scale, plan_host, plan_dev, workspace, workspace_bytes, o_latent,
                         lse=None, status=None, stream=None):
    _check(load().mla_decode_attention(_ptr(q_full), _ptr(cache), num_pages, _ptr(block_table),
                                       max_pages, batch, q_len, n_h, scale, _ptr(plan_host),
                                       _ptr(plan_dev), _ptr(workspace), workspace_bytes,
                                       _ptr(o_latent), _ptr(lse), _ptr(status),
                                       _stream(stream)), "mla_decode_attention")


def mla_debug_decode_wait(wait_cap_seconds: float = 1.0, suppress_arrive: int = 0):
    """Failure-detection switch of the tensor-core decode kernel (include/mla_debug.h)."""
    _check(load().mla_debug_decode_wait(float(wait_cap_seconds), int(suppress_arrive)),
           "mla_debug_decode_wait")


def mla_debug_gemm_plan(M, N, K, batch=1, a_mn=0, c_fp32=0, fp32_part=0, atomic_split=0,
                        sms=148) -> dict:
    """The tensor-core GEMM's tile plan for a problem (include/mla_debug.h)."""
    out = (ctypes.c_int32 * 8)()
    _check(load().mla_debug_gemm_plan(M, N, K, batch, int(a_mn), int(c_fp32), int(fp32_part),
                                      int(atomic_split), sms, out), "mla_debug_gemm_plan")
    keys = ("BN", "accumulators", "ntile", "mtile", "splits", "k_chunks", "part", "part_bytes")
    return dict(zip(keys, list(out)))


def mla_decode_attention_cudacore(q_full, cache, num_pages, block_table, max_pages, batch, q_len,
                                  n_h, scale, plan_host, plan_dev, workspace, workspace_bytes,
                                  o_latent, lse=None, status=None, stream=None):
    """Debug entry point: the same attention on CUDA cores (differential tests)."""
    _check(load().mla_decode_attention_cudacore(_ptr(q_full), _ptr(cache), num_pages,
                                                _ptr(block_table), max_pages, batch, q_len, n_h,
                                                scale, _ptr(plan_host), _ptr(plan_dev),
                                                _ptr(workspace), workspace_bytes, _ptr(o_latent),
                                                _ptr(lse), _ptr(status), _stream(stream)),
           "mla_decode_attention_cudacore")


def mla_decode_attention_noalloc(q_full, cache, num_pages, block_table, max_pages, batch, q_len,
                                 n_h, scale, plan_host, plan_dev, o_latent, lse=None, status=None,
                                 stream=None):
    _check(load().mla_decode_attention_noalloc(_ptr(q_full), _ptr(cache), num_pages,
                                               _ptr(block_table), max_pages, batch, q_len, n_h,
                                               scale, _ptr(plan_host), _ptr(plan_dev),
                                               _ptr(o_latent), _ptr(lse), _ptr(status),
                                               _stream(stream)), "mla_decode_attention_noalloc")


def mla_out_absorb(o_latent, w_uv, T, n_h, u, ld_u, stream=None):
    _check(load().mla_out_absorb(_ptr(o_latent), _ptr(w_uv), T, n_h, _ptr(u), ld_u,
                                 _stream(stream)), "mla_out_absorb")


def mla_gemm_bf16(X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K, stream=None):
    _check(load().mla_gemm_bf16(_ptr(X), ld_x, _ptr(W), ld_w, _ptr(C), ld_c, int(c_fp32), M, N,
                                K, _stream(stream)), "mla_gemm_bf16")


def mla_gemm_bf16_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load().mla_gemm_bf16_workspace_bytes(M, N, K))


def mla_gemm_bf16_ws(X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K, workspace, workspace_bytes,
                     stream=None):
    _check(load().mla_gemm_bf16_ws(_ptr(X), ld_x, _ptr(W), ld_w, _ptr(C), ld_c, int(c_fp32), M,
                                   N, K, _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "mla_gemm_bf16_ws")


def mla_read_status(status, clear: bool = True, stream=None) -> int:
    """Returns the device status bits (raises nothing for set bits)."""
    bits = ctypes.c_uint32(0)
    st = load().mla_read_status(_ptr(status), ctypes.addressof(bits), int(clear), _stream(stream))
    if st not in (MLA_OK, MLA_ERR_DEVICE):
        _check(st, "mla_read_status")
    return int(bits.value)


def mla_check_status(status, stream=None) -> int:
    """Returns the device status bits without clearing them."""
    bits = ctypes.c_uint32(0)
    st = load().mla_check_status(_ptr(status), ctypes.addressof(bits), _stream(stream))
    if st not in (MLA_OK, MLA_ERR_DEVICE):
        _check(st, "mla_check_status")
    return int(bits.value)


def mla_reset_status(status, stream=None):
    _check(load().mla_reset_status(_ptr(status), _stream(stream)), "mla_reset_status")


def mla_plan_used_bytes(plan_host) -> int:
    return int(load().mla_plan_used_bytes(_ptr(plan_host)))


def mla_plan_upload(plan_host, plan_dev, plan_dev_bytes, stream=None):
    _check(load().mla_plan_upload(_ptr(plan_host), _ptr(plan_dev), int(plan_dev_bytes),
                                  _stream(stream)), "mla_plan_upload")


def mla_fold_qk_workspace_bytes(n_h: int) -> int:
    return int(load().mla_fold_qk_workspace_bytes(n_h))


def mla_fold_qk(w_uq, ld_uq, q_in, w_uk, n_h, w_qk, workspace, workspace_bytes, stream=None):
    _check(load().mla_fold_qk(_ptr(w_uq), ld_uq, q_in, _ptr(w_uk), n_h, _ptr(w_qk),
                              _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "mla_fold_qk")


def mla_fold_o(w_o, ld_o, d_model, w_uv, n_h, w_o_folded, stream=None):
    _check(load().mla_fold_o(_ptr(w_o), ld_o, d_model, _ptr(w_uv), n_h, _ptr(w_o_folded),
                             _stream(stream)), "mla_fold_o")


def mla_absorb_q_folded(x, ld_x, k_in, q_pe, ld_qp, w_qk, pos, rope_table, max_pos, T, n_h,
                        q_full, status=None, stream=None):
    _check(load().mla_absorb_q_folded(_ptr(x), ld_x, k_in, _ptr(q_pe), ld_qp, _ptr(w_qk),
                                      _ptr(pos), _ptr(rope_table), max_pos, T, n_h,
                                      _ptr(q_full), _ptr(status), _stream(stream)),
           "mla_absorb_q_folded")


def mla_cache_append_fp8(cache, scales, num_pages, block_table, batch, max_pages, seq_idx, pos,
                         c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, n_tokens, status=None,
                         stream=None):
    _check(load().mla_cache_append_fp8(_ptr(cache), _ptr(scales), num_pages, _ptr(block_table),
                                       batch, max_pages, _ptr(seq_idx), _ptr(pos), _ptr(c_kv),
                                       ld_c, _ptr(k_pe), ld_k, _ptr(rope_table), max_pos, n_tokens,
                                       _ptr(status), _stream(stream)), "mla_cache_append_fp8")


def mla_decode_attention_fp8(q_full, cache, scales, num_pages, block_table, max_pages, batch,
                             q_len, n_h, scale, plan_host, plan_dev, workspace, workspace_bytes,
                             o_latent, lse=None, status=None, stream=None):
    _check(load().mla_decode_attention_fp8(_ptr(q_full), _ptr(cache), _ptr(scales), num_pages,
                                           _ptr(block_table), max_pages, batch, q_len, n_h,
                                           scale, _ptr(plan_host), _ptr(plan_dev),
                                           _ptr(workspace), workspace_bytes, _ptr(o_latent),
                                           _ptr(lse), _ptr(status), _stream(stream)),
           "mla_decode_attention_fp8")


def mla_append_fp8_absorb_q(cache, scales, num_pages, block_table, batch, max_pages, seq_idx,
                            tok_pos, c_kv, ld_c, k_pe, ld_k, n_tokens, q_nope, ld_qn, q_pe, ld_qp,
                            w_uk, q_pos, rope_table, max_pos, T, n_h, q_full, status=None,
                            stream=None):
    _check(load().mla_append_fp8_absorb_q(_ptr(cache), _ptr(scales), num_pages,
                                          _ptr(block_table), batch, max_pages, _ptr(seq_idx),
                                          _ptr(tok_pos), _ptr(c_kv), ld_c, _ptr(k_pe), ld_k,
                                          n_tokens, _ptr(q_nope), ld_qn, _ptr(q_pe), ld_qp,
                                          _ptr(w_uk), _ptr(q_pos), _ptr(rope_table), max_pos, T,
                                          n_h, _ptr(q_full), _ptr(status), _stream(stream)),
           "mla_append_fp8_absorb_q")


def mla_append_absorb_q(cache, num_pages, block_table, batch, max_pages, seq_idx, tok_pos, c_kv,
                        ld_c, k_pe, ld_k, n_tokens, q_nope, ld_qn, q_pe, ld_qp, w_uk, q_pos,
                        rope_table, max_pos, T, n_h, q_full, status=None, stream=None):
    _check(load().mla_append_absorb_q(_ptr(cache), num_pages, _ptr(block_table), batch,
                                      max_pages, _ptr(seq_idx), _ptr(tok_pos), _ptr(c_kv), ld_c,
                                      _ptr(k_pe), ld_k, n_tokens, _ptr(q_nope), ld_qn, _ptr(q_pe),
                                      ld_qp, _ptr(w_uk), _ptr(q_pos), _ptr(rope_table), max_pos,
                                      T, n_h, _ptr(q_full), _ptr(status), _stream(stream)),
           "mla_append_absorb_q")
