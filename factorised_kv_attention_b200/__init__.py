"""Python binding of libkpa (factor-space KPA / TPA attention for B200, sm_100a).

The functions here carry the C names of ``include/kpa.h`` and only marshal
arguments: tensors become device pointers, ``stream=None`` becomes torch's
current CUDA stream, and a non-OK status raises :class:`KpaError`.  Every step
of the computation runs in the CUDA library; there is no CPU path.  Importing
fails loudly when ``libkpa.so`` has not been built (``python
factorised_kv_attention_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python factorised_kv_attention_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

KPA_OK = 0
KPA_ERR_INVALID_ARG = 1
KPA_ERR_UNSUPPORTED = 2
KPA_ERR_WORKSPACE = 3
KPA_ERR_CUDA = 4
KPA_ERR_TIMEOUT = 5
KPA_ERR_DEVICE_CHECK = 6
KPA_F32 = 0
KPA_BF16 = 1
KPA_TOKEN_GROUP = 8


class kpa_config(ctypes.Structure):
    _fields_ = [("h1", ctypes.c_int32), ("h2", ctypes.c_int32), ("d1", ctypes.c_int32),
                ("d2", ctypes.c_int32), ("r_q", ctypes.c_int32), ("r_k", ctypes.c_int32),
                ("r_v", ctypes.c_int32), ("d_model", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("dtype", ctypes.c_int), ("shared_b", ctypes.c_int32), ("order", ctypes.c_int32)]


class KpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.kpa_status_string(status).decode()
        if status == KPA_ERR_CUDA:
            msg += f" (cudaError {_lib.kpa_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


_vp, _i32, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
_cfgp = ctypes.POINTER(kpa_config)
_szp = ctypes.POINTER(ctypes.c_size_t)
_i32p = ctypes.POINTER(ctypes.c_int32)
_SIGS = {
    "kpa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "kpa_last_cuda_error": ([], ctypes.c_int),
    "kpa_cache_bytes_per_token": ([_cfgp, _szp, _szp], ctypes.c_int),
    "kpa_append_factors": ([_cfgp, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
    "kpa_decode_workspace_size": ([_cfgp, _i32, _i32, _i32, _szp], ctypes.c_int),
    "kpa_decode_plan": ([_cfgp, _i32, _i32, _i32, _i32p, _i32p, _i32p], ctypes.c_int),
    "kpa_decode_qf": ([_cfgp, _i32, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _vp, _vp, _sz, _vp],
                      ctypes.c_int),
    "kpa_decode": ([_cfgp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _vp, _vp, _sz, _vp],
                   ctypes.c_int),
    "kpa_decode_split": ([_cfgp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _i32, _vp, _vp,
                          _sz, _vp], ctypes.c_int),
    "kpa_prefill_workspace_size": ([_cfgp, _i32, _i32, _szp], ctypes.c_int),
    "kpa_prefill": ([_cfgp, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _sz, _vp],
                    ctypes.c_int),
    "kpa_prefill_qf": ([_cfgp, _i32, _i32, _vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp,
                        _i32, _f32, _vp, _vp, _sz, _vp], ctypes.c_int),
    "kpa_append_workspace_size": ([_cfgp, _i32, _i32, _szp], ctypes.c_int),
    "kpa_append": ([_cfgp, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp],
                   ctypes.c_int),
    "kpa_read_device_error": ([_vp, ctypes.POINTER(_i32)], ctypes.c_int),
    "kpa_decode_noalloc": ([_cfgp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _vp, _vp],
                           ctypes.c_int),
    "kpa_test_set_decode_hooks": ([_i32, _i32, ctypes.c_uint64], ctypes.c_int),
    "kpa_test_set_decode_engine": ([_i32], ctypes.c_int),
    "kpa_decode_kernel_kind": ([_cfgp, _i32, _i32, _i32, _i32p], ctypes.c_int),
    "kpa_prefill_kernel_kind": ([_cfgp, _i32p], ctypes.c_int),
    "kpa_test_set_prefill_engine": ([_i32], ctypes.c_int),
    "kpa_test_exp2_poly": ([_vp, _vp, ctypes.c_int64, _vp], ctypes.c_int),
    "kpa_append_factors_pos": ([_cfgp, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
    "kpa_decode_lse": ([_cfgp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _vp, _vp, _vp, _sz, _vp],
                       ctypes.c_int),
    "kpa_merge_lse": ([_i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def make_config(shape, dtype: str = "bf16") -> kpa_config:
    """kpa_config from any object with h1, h2, d1, d2, r_k, r_v (and optionally
    r_q, d_model, rope_base, shared_b, order)."""
    return kpa_config(int(shape.h1), int(shape.h2), int(shape.d1), int(shape.d2),
                      int(getattr(shape, "r_q", 0)), int(shape.r_k), int(shape.r_v),
                      int(getattr(shape, "d_model", 0)), float(getattr(shape, "rope_base", 10000.0)),
                      KPA_BF16 if dtype == "bf16" else KPA_F32, int(getattr(shape, "shared_b", 0)),
                      int(getattr(shape, "order", 2)))


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, where):
    if status != KPA_OK:
        raise KpaError(status, where)


def kpa_status_string(status: int) -> str:
    return _lib.kpa_status_string(status).decode()


def kpa_last_cuda_error() -> int:
    return int(_lib.kpa_last_cuda_error())


def kpa_cache_bytes_per_token(cfg: kpa_config):
    k, v = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.kpa_cache_bytes_per_token(ctypes.byref(cfg), ctypes.byref(k), ctypes.byref(v)),
           "kpa_cache_bytes_per_token")
    return k.value, v.value


def kpa_append_factors(cfg, batch, n_tok, k_factors, v_factors, start_pos, capacity, kcache,
                       vcache, stream=None):
    _check(_lib.kpa_append_factors(ctypes.byref(cfg), batch, n_tok, _addr(k_factors),
                                   _addr(v_factors), _addr(start_pos), capacity, _addr(kcache),
                                   _addr(vcache), _stream(stream)), "kpa_append_factors")


def kpa_decode_workspace_size(cfg, batch, max_len, tokens_per_split=0) -> int:
    n = ctypes.c_size_t()
    _check(_lib.kpa_decode_workspace_size(ctypes.byref(cfg), batch, max_len, tokens_per_split,
                                          ctypes.byref(n)), "kpa_decode_workspace_size")
    return n.value


def kpa_decode_plan(cfg, batch, max_len, tokens_per_split=0):
    """(splits per sequence, tokens per split, kernel launches per kpa_decode call)."""
    n, t, l = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.kpa_decode_plan(ctypes.byref(cfg), batch, max_len, tokens_per_split, ctypes.byref(n),
                                ctypes.byref(t), ctypes.byref(l)), "kpa_decode_plan")
    return n.value, t.value, l.value


DECODE_KERNEL_NAMES = {0: "cuda_cores", 1: "mma_sync", 2: "tcgen05"}


def kpa_decode_kernel_kind(cfg, batch, max_len, tokens_per_split=0):
    """Name of the kernel a dense-query decode with these arguments runs."""
    k = ctypes.c_int32()
    _check(_lib.kpa_decode_kernel_kind(ctypes.byref(cfg), batch, max_len, tokens_per_split, ctypes.byref(k)),
           "kpa_decode_kernel_kind")
    return DECODE_KERNEL_NAMES[k.value]


PREFILL_KERNEL_NAMES = {1: "mma_sync", 2: "tcgen05"}


def kpa_prefill_kernel_kind(cfg):
    """Name of the kernel kpa_prefill runs for this config on the calling thread."""
    k = ctypes.c_int32()
    _check(_lib.kpa_prefill_kernel_kind(ctypes.byref(cfg), ctypes.byref(k)), "kpa_prefill_kernel_kind")
    return PREFILL_KERNEL_NAMES[k.value]


def kpa_decode_qf(cfg, batch, q_factors, qf_stride, qf_seq_stride, q_pos, kcache, vcache, capacity, seq_len,
                  max_len, sm_scale, out, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.kpa_decode_qf(ctypes.byref(cfg), batch, _addr(q_factors), qf_stride, qf_seq_stride, _addr(q_pos),
                              _addr(kcache), _addr(vcache), capacity, _addr(seq_len), max_len, sm_scale,
                              _addr(out), _addr(workspace), ws_bytes, _stream(stream)), "kpa_decode_qf")


def kpa_decode(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale, out,
               workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.kpa_decode(ctypes.byref(cfg), batch, _addr(q), _addr(q_pos), _addr(kcache),
                           _addr(vcache), capacity, _addr(seq_len), max_len, sm_scale, _addr(out),
                           _addr(workspace), ws_bytes, _stream(stream)), "kpa_decode")


def kpa_decode_split(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale,
                     tokens_per_split, out, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.kpa_decode_split(ctypes.byref(cfg), batch, _addr(q), _addr(q_pos), _addr(kcache),
                                 _addr(vcache), capacity, _addr(seq_len), max_len, sm_scale,
                                 tokens_per_split, _addr(out), _addr(workspace), ws_bytes,
                                 _stream(stream)), "kpa_decode_split")


def kpa_prefill_workspace_size(cfg, batch, n_tok) -> int:
    n = ctypes.c_size_t()
    _check(_lib.kpa_prefill_workspace_size(ctypes.byref(cfg), batch, n_tok, ctypes.byref(n)),
           "kpa_prefill_workspace_size")
    return n.value


def kpa_prefill_qf(cfg, batch, n_tok, q_factors, qf_stride, qf_seq_stride, qf_tok_stride, start_pos, kcache,
                   vcache, capacity, sm_scale, out, workspace=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kpa_prefill_qf(ctypes.byref(cfg), batch, n_tok, _addr(q_factors), qf_stride, qf_seq_stride,
                               qf_tok_stride, _addr(start_pos), _addr(kcache), _addr(vcache), capacity, sm_scale,
                               _addr(out), _addr(workspace), ws_bytes, _stream(stream)), "kpa_prefill_qf")


def kpa_prefill(cfg, batch, n_tok, q, start_pos, kcache, vcache, capacity, sm_scale, out,
                workspace=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kpa_prefill(ctypes.byref(cfg), batch, n_tok, _addr(q), _addr(start_pos),
                            _addr(kcache), _addr(vcache), capacity, sm_scale, _addr(out),
                            _addr(workspace), ws_bytes, _stream(stream)), "kpa_prefill")


def kpa_append_workspace_size(cfg, batch, n_tok) -> int:
    n = ctypes.c_size_t()
    _check(_lib.kpa_append_workspace_size(ctypes.byref(cfg), batch, n_tok, ctypes.byref(n)),
           "kpa_append_workspace_size")
    return n.value


def kpa_append(cfg, batch, n_tok, x, w, start_pos, capacity, kcache, vcache, q_out, workspace,
               ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kpa_append(ctypes.byref(cfg), batch, n_tok, _addr(x), _addr(w), _addr(start_pos),
                           capacity, _addr(kcache), _addr(vcache), _addr(q_out), _addr(workspace),
                           ws_bytes, _stream(stream)), "kpa_append")


KPA_DECODE_NOALLOC_MAX_BYTES = 16 << 20


def kpa_decode_noalloc(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale,
                       out, stream=None):
    """kpa_decode without a workspace argument, for callers that cannot allocate:
    the library's fixed device scratch array stands in for it (see kpa.h)."""
    _check(_lib.kpa_decode_noalloc(ctypes.byref(cfg), batch, _addr(q), _addr(q_pos), _addr(kcache),
                                   _addr(vcache), capacity, _addr(seq_len), max_len, sm_scale,
                                   _addr(out), _stream(stream)), "kpa_decode_noalloc")


def kpa_test_set_decode_hooks(skip_tile=-1, skip_split=-1, wait_limit_ns=1_000_000_000):
    _check(_lib.kpa_test_set_decode_hooks(skip_tile, skip_split, wait_limit_ns),
           "kpa_test_set_decode_hooks")


def kpa_test_set_decode_engine(engine=0):
    _check(_lib.kpa_test_set_decode_engine(engine), "kpa_test_set_decode_engine")


def kpa_test_set_prefill_engine(engine=0):
    _check(_lib.kpa_test_set_prefill_engine(engine), "kpa_test_set_prefill_engine")


def kpa_append_factors_pos(cfg, batch, n_tok, k_factors, v_factors, start_pos, pos_offset, capacity, kcache,
                           vcache, stream=None):
    """kpa_append_factors with the keys of slot start_pos[b] + t rotated at position
    start_pos[b] + t + pos_offset[b] (a cache holding a range of a longer sequence)."""
    _check(_lib.kpa_append_factors_pos(ctypes.byref(cfg), batch, n_tok, _addr(k_factors), _addr(v_factors),
                                       _addr(start_pos), _addr(pos_offset), capacity, _addr(kcache), _addr(vcache),
                                       _stream(stream)), "kpa_append_factors_pos")


def kpa_decode_lse(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale, out, lse,
                   workspace, ws_bytes=None, stream=None):
    """kpa_decode that also writes each head's log-sum-exp of its scores into lse [batch][h]."""
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.kpa_decode_lse(ctypes.byref(cfg), batch, _addr(q), _addr(q_pos), _addr(kcache), _addr(vcache),
                               capacity, _addr(seq_len), max_len, sm_scale, _addr(out), _addr(lse),
                               _addr(workspace), ws_bytes, _stream(stream)), "kpa_decode_lse")


def kpa_merge_lse(outs, lses, out, lse=None, stream=None):
    """Log-sum-exp merge of normalised partial decodes: outs [n_parts][batch][h][d_h],
    lses [n_parts][batch][h] -> out [batch][h][d_h] (and the merged lse when given)."""
    n_parts, batch, heads, d_h = outs.shape
    _check(_lib.kpa_merge_lse(batch, heads, d_h, n_parts, _addr(outs), _addr(lses), _addr(out), _addr(lse),
                              _stream(stream)), "kpa_merge_lse")


def kpa_test_exp2_poly(x, y, stream=None):
    """y = 2^x (float32 device tensors of the same size) through the prefill's
    polynomial exponential (testing)."""
    if x.numel() != y.numel():
        raise ValueError("x and y differ in size")
    _check(_lib.kpa_test_exp2_poly(_addr(x), _addr(y), x.numel(), _stream(stream)), "kpa_test_exp2_poly")


def kpa_read_device_error(stream=None) -> int:
    code = ctypes.c_int32()
    _check(_lib.kpa_read_device_error(_stream(stream), ctypes.byref(code)), "kpa_read_device_error")
    return code.value


__all__ = [n for n in list(globals()) if n.startswith("kpa_") or n.startswith("KPA_")] + [
    "KpaError", "make_config", "LIB_PATH"]
