"""Python binding of libmla.so (the MLA latent-KV C ABI declared in include/mla.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, checks their dtype/shape/contiguity, and passes raw device
pointers plus the current CUDA stream to the C entry point of the same name.
All compute runs in the library's CUDA kernels.  Importing this module fails
loudly if the library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python mla_latent_kv_40_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

MLA_F32, MLA_BF16 = 0, 1
MLA_CACHE_ROWS, MLA_CACHE_TILED = 0, 1
STATUS = {0: "MLA_OK", -1: "MLA_ERR_INVALID_ARG", -2: "MLA_ERR_UNSUPPORTED", -3: "MLA_ERR_WORKSPACE",
          -4: "MLA_ERR_CUDA", -5: "MLA_ERR_TIMEOUT", -6: "MLA_ERR_BAD_INDEX", -7: "MLA_ERR_STATIC_WS"}
NOALLOC_SCRATCH_BYTES = 16 << 20   # MLA_NOALLOC_SCRATCH_BYTES in include/mla.h


class MlaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code} ({STATUS.get(code, '?')}: {mla_status_string(code)})")
        self.code = code


class mla_dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int), ("d_c", ctypes.c_int), ("d_rope", ctypes.c_int),
                ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int), ("d_model", ctypes.c_int),
                ("block_size", ctypes.c_int), ("ckv_stride", ctypes.c_int), ("kpe_stride", ctypes.c_int),
                ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("dtype", ctypes.c_int), ("cache_layout", ctypes.c_int)]


def make_dims(n_heads, d_c, d_rope, d_nope, d_v, d_model, block_size, dtype, ckv_stride=None,
              kpe_stride=None, rope_base=10000.0, softmax_scale=0.0, rms_eps=1e-6, cache_layout=MLA_CACHE_ROWS) -> mla_dims:
    """Dims of a fused row pool (rows of d_c + d_rope elements) by default, or of a tiled page pool."""
    w = d_c + d_rope
    dt = MLA_BF16 if dtype in ("bf16", torch.bfloat16, MLA_BF16) else MLA_F32
    return mla_dims(n_heads, d_c, d_rope, d_nope, d_v, d_model, block_size,
                    w if ckv_stride is None else ckv_stride, w if kpe_stride is None else kpe_stride,
                    rope_base, softmax_scale, rms_eps, dt, int(cache_layout))


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.POINTER(mla_dims)
_SZ = ctypes.POINTER(ctypes.c_size_t)
_sigs = {
    "mla_append_latent": [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, ctypes.c_size_t, _P, _P],
    "mla_append_workspace_size": [_D, _I, _SZ],
    "mla_absorb_q": [_D, _I, _I, _P, _P, _P, _P, _P, _P],
    "mla_decode_workspace_size": [_D, _I, _I, _I, _SZ],
    "mla_decode": [_D, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P],
    "mla_decode_latent": [_D, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P, _P],
    "mla_decode_attention": [_D, _I, _I, _P, _P, _P, _P, _I, _I, _P, _I, _P, ctypes.c_size_t, _P, _P],
    "mla_decode_combine": [_D, _I, _I, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "mla_prefill_workspace_size": [_D, _I, _I, _I, _SZ],
    "mla_decode_sparse_workspace_size": [_D, _I, _I, _I, _SZ],
    "mla_decode_partial": [_D, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _P, _P, _P, _P, ctypes.c_size_t,
                           _P, _P],
    "mla_merge_workspace_size": [_D, _I, _I, _I, _SZ],
    "mla_decode_step_workspace_size": [_D, _I, _I, _I, _SZ],
    "mla_decode_step": [_D, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P,
                        ctypes.c_size_t, _P, _P],
    "mla_fold_query_weights": [_D, _I, _P, _P, _P, _P],
    "mla_fold_output_weights": [_D, _P, _P, _P, _P],
    "mla_decode_absorbed_workspace_size": [_D, _I, _I, _I, _I, _SZ],
    "mla_decode_absorbed": [_D, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P,
                            ctypes.c_size_t, _P, _P],
    "mla_merge_partials": [_D, _I, _I, _I, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "mla_decode_sparse": [_D, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _I, _P, _P, _P, _P, _P,
                          ctypes.c_size_t, _P, _P],
    "mla_decode_launches": [_D, _I, ctypes.POINTER(ctypes.c_int)],
    "mla_decode_path": [_D, _I, ctypes.POINTER(ctypes.c_int)],
    "mla_cache_pack": [_D, _P, _P, ctypes.c_int64, _P],
    "mla_cache_unpack": [_D, _P, _P, ctypes.c_int64, _P],
    "mla_decode_noalloc": [_D, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P],
    "mla_prefill": [_D, _I, _P, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P],
    "mla_wait_selftest": [ctypes.c_longlong, _P, _P],
}
for _n, _a in _sigs.items():
    getattr(_lib, _n).argtypes = _a
    getattr(_lib, _n).restype = ctypes.c_int
_lib.mla_status_string.argtypes = [_I]
_lib.mla_status_string.restype = ctypes.c_char_p


def mla_status_string(code: int) -> str:
    return _lib.mla_status_string(int(code)).decode()


def _elem_dtype(dims: mla_dims):
    return torch.bfloat16 if dims.dtype == MLA_BF16 else torch.float32


def _ptr(t, dtype=None, name="", optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _dense(t, name):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise MlaError(fn, rc)


def mla_append_workspace_size(dims, T) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_append_workspace_size", _lib.mla_append_workspace_size(ctypes.byref(dims), int(T), ctypes.byref(n)))
    return int(n.value)


def mla_append_latent(dims, h, w_dkv, w_kr, rms_gamma, seq_idx, pos, c_kv, k_pe, block_table, num_seqs,
                      max_blocks_per_seq, num_blocks, dev_status=None, stream=None, workspace=None):
    """workspace: None runs the CUDA-core path; a buffer of mla_append_workspace_size bytes
    lets bf16 shapes run the tensor-core projection."""
    et = _elem_dtype(dims)
    T = 0 if h is None else h.shape[0]
    for n, t in (("h", h), ("w_dkv", w_dkv), ("w_kr", w_kr), ("rms_gamma", rms_gamma), ("seq_idx", seq_idx),
                 ("pos", pos), ("block_table", block_table)):
        _dense(t, n)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.mla_append_latent(ctypes.byref(dims), T, _ptr(h, et, "h"), _ptr(w_dkv, et, "w_dkv"),
                                _ptr(w_kr, et, "w_kr"), _ptr(rms_gamma, et, "rms_gamma", True),
                                _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(pos, torch.int32, "pos"),
                                _ptr(c_kv, et, "c_kv"), _ptr(k_pe, et, "k_pe"),
                                _ptr(block_table, torch.int32, "block_table", True), int(num_seqs),
                                int(max_blocks_per_seq), int(num_blocks), _ptr(workspace, None, "workspace", True),
                                ctypes.c_size_t(ws_bytes), _ptr(dev_status, torch.int32, "dev_status", True),
                                _stream(stream))
    _check("mla_append_latent", rc)


def mla_absorb_q(dims, q_nope, q_pe, w_uk, seqlens, q_out, stream=None):
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    for n, t in (("q_nope", q_nope), ("q_pe", q_pe), ("w_uk", w_uk), ("seqlens", seqlens), ("q_out", q_out)):
        _dense(t, n)
    rc = _lib.mla_absorb_q(ctypes.byref(dims), B, n_q, _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"),
                           _ptr(w_uk, et, "w_uk"), _ptr(seqlens, torch.int32, "seqlens"),
                           _ptr(q_out, et, "q_out"), _stream(stream))
    _check("mla_absorb_q", rc)


def mla_decode_workspace_size(dims, B, n_q, max_seqlen) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_workspace_size",
           _lib.mla_decode_workspace_size(ctypes.byref(dims), int(B), int(n_q), int(max_seqlen), ctypes.byref(n)))
    return int(n.value)


def _decode_common(fn, dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                   max_seqlen, w_uk, w_uv, out, lse, workspace, dev_status, stream):
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    for n, t in (("q_nope", q_nope), ("q_pe", q_pe), ("block_table", block_table), ("seqlens", seqlens),
                 ("w_uk", w_uk), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    args = [ctypes.byref(dims), B, n_q, _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"),
            _ptr(c_kv, et, "c_kv"), _ptr(k_pe, et, "k_pe"), _ptr(block_table, torch.int32, "block_table", True),
            int(max_blocks_per_seq), int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"), int(max_seqlen),
            _ptr(w_uk, et, "w_uk")]
    if fn == "mla_decode":
        args.append(_ptr(w_uv, et, "w_uv"))
    args += [_ptr(out, et, "out"), _ptr(lse, torch.float32, "lse", True), _ptr(workspace, None, "workspace"),
             ctypes.c_size_t(workspace.numel() * workspace.element_size()),
             _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream)]
    _check(fn, getattr(_lib, fn)(*args))


def mla_decode(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens, max_seqlen,
               w_uk, w_uv, out, lse, workspace, dev_status=None, stream=None):
    _decode_common("mla_decode", dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks,
                   seqlens, max_seqlen, w_uk, w_uv, out, lse, workspace, dev_status, stream)


def mla_decode_noalloc(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                       max_seqlen, w_uk, w_uv, out, lse, dev_status=None, stream=None):
    """mla_decode without a workspace argument: the library's static device
    scratch (NOALLOC_SCRATCH_BYTES per GPU) stands in for it.  For callers that
    cannot allocate; calls that overlap on one GPU race on that scratch."""
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    for n, t in (("q_nope", q_nope), ("q_pe", q_pe), ("block_table", block_table), ("seqlens", seqlens),
                 ("w_uk", w_uk), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_decode_noalloc(ctypes.byref(dims), B, n_q, _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"),
                                 _ptr(c_kv, et, "c_kv"), _ptr(k_pe, et, "k_pe"),
                                 _ptr(block_table, torch.int32, "block_table", True), int(max_blocks_per_seq),
                                 int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"), int(max_seqlen),
                                 _ptr(w_uk, et, "w_uk"), _ptr(w_uv, et, "w_uv"), _ptr(out, et, "out"),
                                 _ptr(lse, torch.float32, "lse", True), _ptr(dev_status, torch.int32, "dev_status", True),
                                 _stream(stream))
    _check("mla_decode_noalloc", rc)


def mla_decode_step_workspace_size(dims, B, n_q, max_seqlen) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_step_workspace_size",
           _lib.mla_decode_step_workspace_size(ctypes.byref(dims), int(B), int(n_q), int(max_seqlen), ctypes.byref(n)))
    return int(n.value)


def mla_decode_step(dims, h_new, w_dkv, w_kr, rms_gamma, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq,
                    num_blocks, seqlens, max_seqlen, w_uk, w_uv, out, lse, workspace, dev_status=None, stream=None):
    """Append of the n_q new tokens of every sequence (h_new [B, n_q, D]) and the decode, in one call."""
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    if h_new.shape[0] * (h_new.shape[1] if h_new.dim() == 3 else 1) != B * n_q:
        raise ValueError("h_new must hold B * n_q rows")
    for n, t in (("h_new", h_new), ("w_dkv", w_dkv), ("w_kr", w_kr), ("rms_gamma", rms_gamma), ("q_nope", q_nope),
                 ("q_pe", q_pe), ("block_table", block_table), ("seqlens", seqlens), ("w_uk", w_uk), ("w_uv", w_uv),
                 ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_decode_step(ctypes.byref(dims), B, n_q, _ptr(h_new, et, "h_new"), _ptr(w_dkv, et, "w_dkv"),
                              _ptr(w_kr, et, "w_kr"), _ptr(rms_gamma, et, "rms_gamma", True),
                              _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"), _ptr(c_kv, et, "c_kv"),
                              _ptr(k_pe, et, "k_pe"), _ptr(block_table, torch.int32, "block_table", True),
                              int(max_blocks_per_seq), int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"),
                              int(max_seqlen), _ptr(w_uk, et, "w_uk"), _ptr(w_uv, et, "w_uv"), _ptr(out, et, "out"),
                              _ptr(lse, torch.float32, "lse", True), _ptr(workspace, None, "workspace"),
                              ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                              _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_decode_step", rc)


def mla_decode_partial(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                       max_seqlen, kv_begin, kv_end, w_uk, o_lat, lse, workspace, dev_status=None, stream=None):
    """This device's share of a decode split by key range: o_lat [B, n_q, H, d_c] and lse [B, n_q, H]
    over the keys in [kv_begin, kv_end) (kv_begin a multiple of 64)."""
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    for n, t in (("q_nope", q_nope), ("q_pe", q_pe), ("block_table", block_table), ("seqlens", seqlens),
                 ("w_uk", w_uk), ("o_lat", o_lat), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_decode_partial(ctypes.byref(dims), B, n_q, _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"),
                                 _ptr(c_kv, et, "c_kv"), _ptr(k_pe, et, "k_pe"),
                                 _ptr(block_table, torch.int32, "block_table", True), int(max_blocks_per_seq),
                                 int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"), int(max_seqlen),
                                 int(kv_begin), int(kv_end), _ptr(w_uk, et, "w_uk"), _ptr(o_lat, et, "o_lat"),
                                 _ptr(lse, torch.float32, "lse"), _ptr(workspace, None, "workspace"),
                                 ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                 _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_decode_partial", rc)


def mla_merge_workspace_size(dims, B, n_q, n_parts) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_merge_workspace_size",
           _lib.mla_merge_workspace_size(ctypes.byref(dims), int(B), int(n_q), int(n_parts), ctypes.byref(n)))
    return int(n.value)


def mla_merge_partials(dims, o_lat_parts, lse_parts, w_uv, out, lse, workspace, stream=None):
    """o_lat_parts [N, B, n_q, H, d_c], lse_parts [N, B, n_q, H] -> out [B, n_q, H, d_v] (o_lat when w_uv is None)."""
    et = _elem_dtype(dims)
    N, B, n_q = o_lat_parts.shape[0], o_lat_parts.shape[1], o_lat_parts.shape[2]
    for n, t in (("o_lat_parts", o_lat_parts), ("lse_parts", lse_parts), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_merge_partials(ctypes.byref(dims), int(B), int(n_q), int(N), _ptr(o_lat_parts, et, "o_lat_parts"),
                                 _ptr(lse_parts, torch.float32, "lse_parts"), _ptr(w_uv, et, "w_uv", True),
                                 _ptr(out, et, "out"), _ptr(lse, torch.float32, "lse", True),
                                 _ptr(workspace, None, "workspace"),
                                 ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("mla_merge_partials", rc)


def mla_fold_query_weights(dims, w_uq, w_uk, w_uqk, stream=None):
    """w_uq [d_cq, H, d_nope], w_uk [H, d_c, d_nope] -> w_uqk [H, d_cq, d_c] = W_UQ^(s) W_UK^(s)T."""
    et = _elem_dtype(dims)
    for n, t in (("w_uq", w_uq), ("w_uk", w_uk), ("w_uqk", w_uqk)):
        _dense(t, n)
    _check("mla_fold_query_weights", _lib.mla_fold_query_weights(ctypes.byref(dims), int(w_uq.shape[0]),
                                                                 _ptr(w_uq, et, "w_uq"), _ptr(w_uk, et, "w_uk"),
                                                                 _ptr(w_uqk, et, "w_uqk"), _stream(stream)))


def mla_fold_output_weights(dims, w_uv, w_o, w_uvo, stream=None):
    """w_uv [H, d_c, d_v], w_o [H * d_v, D] -> w_uvo [H, d_c, D] = W_UV^(s) W_O^(s)."""
    et = _elem_dtype(dims)
    for n, t in (("w_uv", w_uv), ("w_o", w_o), ("w_uvo", w_uvo)):
        _dense(t, n)
    _check("mla_fold_output_weights", _lib.mla_fold_output_weights(ctypes.byref(dims), _ptr(w_uv, et, "w_uv"),
                                                                   _ptr(w_o, et, "w_o"), _ptr(w_uvo, et, "w_uvo"),
                                                                   _stream(stream)))


def mla_decode_absorbed_workspace_size(dims, d_cq, B, n_q, max_seqlen) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_absorbed_workspace_size",
           _lib.mla_decode_absorbed_workspace_size(ctypes.byref(dims), int(d_cq), int(B), int(n_q), int(max_seqlen),
                                                   ctypes.byref(n)))
    return int(n.value)


def mla_decode_absorbed(dims, h, w_dq, w_uqk, w_qr, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                        max_seqlen, w_uvo, out, lse, workspace, dev_status=None, stream=None):
    """h [B, n_q, D] -> out [B, n_q, D]: the attention block's decode output with folded weights."""
    et = _elem_dtype(dims)
    B, n_q = h.shape[0], h.shape[1]
    d_cq = w_dq.shape[1]
    for n, t in (("h", h), ("w_dq", w_dq), ("w_uqk", w_uqk), ("w_qr", w_qr), ("block_table", block_table),
                 ("seqlens", seqlens), ("w_uvo", w_uvo), ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_decode_absorbed(ctypes.byref(dims), int(d_cq), B, n_q, _ptr(h, et, "h"), _ptr(w_dq, et, "w_dq"),
                                  _ptr(w_uqk, et, "w_uqk"), _ptr(w_qr, et, "w_qr"), _ptr(c_kv, et, "c_kv"),
                                  _ptr(k_pe, et, "k_pe"), _ptr(block_table, torch.int32, "block_table", True),
                                  int(max_blocks_per_seq), int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"),
                                  int(max_seqlen), _ptr(w_uvo, et, "w_uvo"), _ptr(out, et, "out"),
                                  _ptr(lse, torch.float32, "lse", True), _ptr(workspace, None, "workspace"),
                                  ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                  _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_decode_absorbed", rc)


def mla_decode_sparse_workspace_size(dims, B, n_q, topk) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_sparse_workspace_size",
           _lib.mla_decode_sparse_workspace_size(ctypes.byref(dims), int(B), int(n_q), int(topk), ctypes.byref(n)))
    return int(n.value)


def mla_decode_sparse(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                      max_seqlen, topk_idx, w_uk, w_uv, out, lse, workspace, dev_status=None, stream=None):
    """topk_idx [B, n_q, topk] int32: the token indices each query token attends to (-1 = padding)."""
    et = _elem_dtype(dims)
    B, n_q = q_nope.shape[0], q_nope.shape[1]
    for n, t in (("q_nope", q_nope), ("q_pe", q_pe), ("block_table", block_table), ("seqlens", seqlens),
                 ("topk_idx", topk_idx), ("w_uk", w_uk), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    if topk_idx.dim() != 3 or tuple(topk_idx.shape[:2]) != (B, n_q):
        raise ValueError("topk_idx must be [B, n_q, topk]")
    rc = _lib.mla_decode_sparse(ctypes.byref(dims), B, n_q, _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"),
                                _ptr(c_kv, et, "c_kv"), _ptr(k_pe, et, "k_pe"),
                                _ptr(block_table, torch.int32, "block_table", True), int(max_blocks_per_seq),
                                int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"), int(max_seqlen),
                                _ptr(topk_idx, torch.int32, "topk_idx"), int(topk_idx.shape[2]),
                                _ptr(w_uk, et, "w_uk"), _ptr(w_uv, et, "w_uv"), _ptr(out, et, "out"),
                                _ptr(lse, torch.float32, "lse", True), _ptr(workspace, None, "workspace"),
                                ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_decode_sparse", rc)


def mla_decode_latent(dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens,
                      max_seqlen, w_uk, o_lat, lse, workspace, dev_status=None, stream=None):
    _decode_common("mla_decode_latent", dims, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq,
                   num_blocks, seqlens, max_seqlen, w_uk, None, o_lat, lse, workspace, dev_status, stream)


def mla_decode_attention(dims, q_abs, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks, seqlens, max_seqlen,
                         workspace, dev_status=None, stream=None):
    et = _elem_dtype(dims)
    B, n_q = q_abs.shape[0], q_abs.shape[1]
    for n, t in (("q_abs", q_abs), ("block_table", block_table), ("seqlens", seqlens)):
        _dense(t, n)
    rc = _lib.mla_decode_attention(ctypes.byref(dims), B, n_q, _ptr(q_abs, et, "q_abs"), _ptr(c_kv, et, "c_kv"),
                                   _ptr(k_pe, et, "k_pe"), _ptr(block_table, torch.int32, "block_table", True),
                                   int(max_blocks_per_seq), int(num_blocks), _ptr(seqlens, torch.int32, "seqlens"),
                                   int(max_seqlen), _ptr(workspace, None, "workspace"),
                                   ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                   _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_decode_attention", rc)


def mla_decode_combine(dims, B, n_q, seqlens, max_seqlen, w_uv, out, lse, workspace, stream=None):
    et = _elem_dtype(dims)
    for n, t in (("seqlens", seqlens), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_decode_combine(ctypes.byref(dims), int(B), int(n_q), _ptr(seqlens, torch.int32, "seqlens"),
                                 int(max_seqlen), _ptr(w_uv, et, "w_uv", True), _ptr(out, et, "out"),
                                 _ptr(lse, torch.float32, "lse", True), _ptr(workspace, None, "workspace"),
                                 ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("mla_decode_combine", rc)


def mla_decode_launches(dims, n_q) -> int:
    n = ctypes.c_int(0)
    _check("mla_decode_launches", _lib.mla_decode_launches(ctypes.byref(dims), int(n_q), ctypes.byref(n)))
    return int(n.value)


PATH_CUDA_CORES, PATH_TCGEN05 = 0, 1   # MLA_PATH_* in include/mla.h


def mla_decode_path(dims, n_q) -> int:
    """PATH_TCGEN05 when mla_decode runs the tensor-core kernels for this shape, else PATH_CUDA_CORES."""
    n = ctypes.c_int(-1)
    _check("mla_decode_path", _lib.mla_decode_path(ctypes.byref(dims), int(n_q), ctypes.byref(n)))
    return int(n.value)


def mla_prefill_workspace_size(dims, B, total_tokens, max_seqlen) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_prefill_workspace_size",
           _lib.mla_prefill_workspace_size(ctypes.byref(dims), int(B), int(total_tokens), int(max_seqlen),
                                           ctypes.byref(n)))
    return int(n.value)


def mla_prefill(dims, cu_seqlens, max_seqlen, q_nope, q_pe, c_kv, k_pe, block_table, max_blocks_per_seq, num_blocks,
                w_uk, w_uv, out, lse, workspace, dev_status=None, stream=None):
    et = _elem_dtype(dims)
    B = cu_seqlens.shape[0] - 1
    total = q_nope.shape[0]
    for n, t in (("cu_seqlens", cu_seqlens), ("q_nope", q_nope), ("q_pe", q_pe), ("block_table", block_table),
                 ("w_uk", w_uk), ("w_uv", w_uv), ("out", out), ("lse", lse)):
        _dense(t, n)
    rc = _lib.mla_prefill(ctypes.byref(dims), B, _ptr(cu_seqlens, torch.int32, "cu_seqlens"), int(max_seqlen), total,
                          _ptr(q_nope, et, "q_nope"), _ptr(q_pe, et, "q_pe"), _ptr(c_kv, et, "c_kv"),
                          _ptr(k_pe, et, "k_pe"), _ptr(block_table, torch.int32, "block_table", True),
                          int(max_blocks_per_seq), int(num_blocks), _ptr(w_uk, et, "w_uk"), _ptr(w_uv, et, "w_uv"),
                          _ptr(out, et, "out"), _ptr(lse, torch.float32, "lse", True),
                          _ptr(workspace, None, "workspace"),
                          ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                          _ptr(dev_status, torch.int32, "dev_status", True), _stream(stream))
    _check("mla_prefill", rc)


def mla_cache_pack(dims, rows, tiled, stream=None):
    """Row pool [num_rows, d_c + d_rope] (bf16) -> tiled page pool of the same byte size."""
    _dense(rows, "rows")
    _check("mla_cache_pack", _lib.mla_cache_pack(ctypes.byref(dims), _ptr(rows, torch.bfloat16, "rows"),
                                                 _ptr(tiled, torch.bfloat16, "tiled"), int(rows.shape[0]),
                                                 _stream(stream)))


def mla_cache_unpack(dims, tiled, rows, stream=None):
    """Tiled page pool -> row pool [num_rows, d_c + d_rope] (bf16)."""
    _dense(rows, "rows")
    _check("mla_cache_unpack", _lib.mla_cache_unpack(ctypes.byref(dims), _ptr(tiled, torch.bfloat16, "tiled"),
                                                     _ptr(rows, torch.bfloat16, "rows"), int(rows.shape[0]),
                                                     _stream(stream)))


def mla_wait_selftest(limit_ns, dev_status, stream=None):
    """Bounded device wait on a barrier nothing completes: *dev_status becomes MLA_ERR_TIMEOUT."""
    _check("mla_wait_selftest", _lib.mla_wait_selftest(int(limit_ns), _ptr(dev_status, torch.int32, "dev_status"),
                                                       _stream(stream)))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned uint8 device buffer (torch's caching allocator aligns to 512 B)."""
    t = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t
