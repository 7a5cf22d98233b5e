"""ctypes binding of libxmla (include/xmla.h), same names as the C ABI.

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch tensors on the current CUDA device; the stream defaults to
torch's current stream.  A non-OK status raises XmlaError.  Loading fails
loudly when the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libxmla.so")

XMLA_OK = 0
STATUS_NAMES = {
    0: "XMLA_OK", 1: "XMLA_ERR_INVALID_ARG", 2: "XMLA_ERR_SHAPE", 3: "XMLA_ERR_WORKSPACE",
    4: "XMLA_ERR_CUDA", 5: "XMLA_ERR_DEVICE_OOB", 6: "XMLA_ERR_TIMEOUT", 7: "XMLA_ERR_UNSUPPORTED",
}

# Every symbol include/xmla.h declares.
EXPORTS = [
    "xmla_yarn_default", "xmla_yarn_inv_freq", "xmla_softmax_scale", "xmla_rope_yarn",
    "xmla_cache_append", "xmla_kv_produce", "xmla_decode_workspace_size", "xmla_decode_num_splits",
    "xmla_decode", "xmla_decode_step_from_hidden",
    "xmla_decode_profiled", "xmla_decode_step", "xmla_decode_noalloc",
    "xmla_shard_partial_floats", "xmla_decode_shard_workspace_size", "xmla_decode_shard",
    "xmla_combine_shards",
    "xmla_cache_append_q8", "xmla_decode_q8_workspace_size", "xmla_decode_q8_num_splits",
    "xmla_decode_q8", "xmla_decode_q8_profiled",
    "xmla_selftest_wait_timeout",
    "xmla_status_string",
]


class XmlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({xmla_status_string(status)})")
        self.status = status


class xmla_yarn_cfg(ctypes.Structure):
    _fields_ = [
        ("rope_theta", ctypes.c_double),
        ("factor", ctypes.c_double),
        ("original_max_position_embeddings", ctypes.c_int64),
        ("beta_fast", ctypes.c_double),
        ("beta_slow", ctypes.c_double),
        ("mscale", ctypes.c_double),
        ("mscale_all_dim", ctypes.c_double),
        ("rotary_dim", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libxmla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libxmla.so not built at {LIB_PATH}; run mla_latent_kv_yarn_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_float, ctypes.c_double, ctypes.c_size_t)
        cfgp = ctypes.POINTER(xmla_yarn_cfg)
        L.xmla_yarn_default.argtypes = [cfgp]
        L.xmla_yarn_default.restype = None
        L.xmla_yarn_inv_freq.argtypes = [cfgp, ctypes.POINTER(ctypes.c_double)]
        L.xmla_yarn_inv_freq.restype = ctypes.c_int
        L.xmla_softmax_scale.argtypes = [cfgp, i32]
        L.xmla_softmax_scale.restype = f64
        L.xmla_rope_yarn.argtypes = [cfgp, vp, i64, i32, i64, i64, i32, vp, vp]
        L.xmla_rope_yarn.restype = ctypes.c_int
        L.xmla_cache_append.argtypes = [vp, i64, vp, i32, i32, vp, vp, vp, vp, cfgp, i64, vp, vp]
        L.xmla_cache_append.restype = ctypes.c_int
        L.xmla_kv_produce.argtypes = [vp, vp, vp, i64, cfgp, vp, i64, vp, i32, i32, vp, vp, vp, vp]
        L.xmla_kv_produce.restype = ctypes.c_int
        L.xmla_decode_workspace_size.argtypes = [i32, i32, i64, i32, i32]
        L.xmla_decode_workspace_size.restype = sz
        L.xmla_decode_num_splits.argtypes = [i32, i32, i64, i32, i32]
        L.xmla_decode_num_splits.restype = i32
        L.xmla_decode.argtypes = [cfgp, vp, vp, vp, vp, i64, vp, i32, vp, i32, i32, i64, f32, i32,
                                  vp, sz, vp, vp, vp]
        L.xmla_decode.restype = ctypes.c_int
        L.xmla_decode_profiled.argtypes = L.xmla_decode.argtypes + [vp, vp]
        L.xmla_decode_profiled.restype = ctypes.c_int
        L.xmla_decode_step.argtypes = [cfgp, vp, vp, vp, vp, i64, vp, i32, vp, i32, i32, i64, vp, vp,
                                       vp, vp, i64, f32, i32, vp, sz, vp, vp, vp, vp, vp]
        L.xmla_decode_step.restype = ctypes.c_int
        L.xmla_decode_step_from_hidden.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, i64, vp, i32, vp,
                                                   i32, i32, i64, vp, vp, i64, f32, i32, vp, sz,
                                                   vp, vp, vp, vp, vp]
        L.xmla_decode_step_from_hidden.restype = ctypes.c_int
        L.xmla_decode_noalloc.argtypes = [cfgp, vp, vp, vp, vp, i64, vp, i32, vp, i32, i32, i64, f32,
                                          i32, vp, vp, vp]
        L.xmla_decode_noalloc.restype = ctypes.c_int
        L.xmla_shard_partial_floats.argtypes = [i32, i32]
        L.xmla_shard_partial_floats.restype = sz
        L.xmla_decode_shard_workspace_size.argtypes = [i32, i32, i64, i64, i64, i32, i32]
        L.xmla_decode_shard_workspace_size.restype = sz
        L.xmla_decode_shard.argtypes = [cfgp, vp, vp, vp, i64, vp, i32, vp, i32, i32, i64, f32, i64,
                                        i64, i32, vp, sz, vp, vp, vp]
        L.xmla_decode_shard.restype = ctypes.c_int
        L.xmla_combine_shards.argtypes = [vp, i32, vp, i32, i32, vp, vp]
        L.xmla_combine_shards.restype = ctypes.c_int
        L.xmla_cache_append_q8.argtypes = L.xmla_cache_append.argtypes
        L.xmla_cache_append_q8.restype = ctypes.c_int
        L.xmla_decode_q8_workspace_size.argtypes = [i32, i32, i64, i32, i32]
        L.xmla_decode_q8_workspace_size.restype = sz
        L.xmla_decode_q8_num_splits.argtypes = [i32, i32, i64, i32, i32]
        L.xmla_decode_q8_num_splits.restype = i32
        L.xmla_decode_q8.argtypes = L.xmla_decode.argtypes
        L.xmla_decode_q8.restype = ctypes.c_int
        L.xmla_decode_q8_profiled.argtypes = L.xmla_decode_profiled.argtypes
        L.xmla_decode_q8_profiled.restype = ctypes.c_int
        L.xmla_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
        L.xmla_selftest_wait_timeout.restype = ctypes.c_int
        L.xmla_status_string.argtypes = [ctypes.c_int]
        L.xmla_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != XMLA_OK:
        raise XmlaError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def xmla_status_string(status: int) -> str:
    return lib().xmla_status_string(int(status)).decode()


def xmla_yarn_default() -> xmla_yarn_cfg:
    cfg = xmla_yarn_cfg()
    lib().xmla_yarn_default(ctypes.byref(cfg))
    return cfg


def xmla_yarn_inv_freq(cfg: xmla_yarn_cfg) -> list[float]:
    out = (ctypes.c_double * (cfg.rotary_dim // 2))()
    _check(lib().xmla_yarn_inv_freq(ctypes.byref(cfg), out), "xmla_yarn_inv_freq")
    return list(out)


def xmla_softmax_scale(cfg: xmla_yarn_cfg, qk_head_dim: int = 192) -> float:
    return float(lib().xmla_softmax_scale(ctypes.byref(cfg), int(qk_head_dim)))


def xmla_rope_yarn(cfg: xmla_yarn_cfg, x: torch.Tensor, rows: int, n_heads: int,
                   head_stride_elems: int, row_stride_elems: int, rope_offset_elems: int,
                   positions: torch.Tensor, stream=None) -> None:
    _check(lib().xmla_rope_yarn(ctypes.byref(cfg), _ptr(x), int(rows), int(n_heads),
                                int(head_stride_elems), int(row_stride_elems),
                                int(rope_offset_elems), _ptr(positions), _stream(stream)),
           "xmla_rope_yarn")


def xmla_cache_append(pool: torch.Tensor, num_blocks: int, block_table: torch.Tensor,
                      max_blocks: int, batch: int, seq_ids: torch.Tensor, positions: torch.Tensor,
                      c_kv: torch.Tensor, k_pe: torch.Tensor, rope_cfg: xmla_yarn_cfg | None,
                      T: int, status: torch.Tensor | None = None, stream=None) -> None:
    _check(lib().xmla_cache_append(_ptr(pool), int(num_blocks), _ptr(block_table),
                                   int(max_blocks), int(batch), _ptr(seq_ids), _ptr(positions),
                                   _ptr(c_kv), _ptr(k_pe),
                                   None if rope_cfg is None else ctypes.byref(rope_cfg), int(T),
                                   _ptr(status), _stream(stream)),
           "xmla_cache_append")


def xmla_kv_produce(hidden, W_kva, bias, T, rope_cfg, pool, num_blocks, block_table, max_blocks,
                    batch, seq_ids, positions, status=None, stream=None) -> None:
    """kv_a_proj_with_mqa of T hidden states, RoPE of the rope key, append to the cache."""
    cfg = None if rope_cfg is None else ctypes.byref(rope_cfg)
    _check(lib().xmla_kv_produce(_ptr(hidden), _ptr(W_kva), _ptr(bias), int(T), cfg, _ptr(pool),
                                 int(num_blocks), _ptr(block_table), int(max_blocks), int(batch),
                                 _ptr(seq_ids), _ptr(positions), _ptr(status), _stream(stream)),
           "xmla_kv_produce")


def xmla_decode_workspace_size(batch: int, q_len: int, max_seqlen: int, num_sms: int,
                               num_splits: int = 0) -> int:
    return int(lib().xmla_decode_workspace_size(int(batch), int(q_len), int(max_seqlen),
                                                int(num_sms), int(num_splits)))


def xmla_decode_num_splits(batch: int, q_len: int, max_seqlen: int, num_sms: int,
                           num_splits: int = 0) -> int:
    return int(lib().xmla_decode_num_splits(int(batch), int(q_len), int(max_seqlen),
                                            int(num_sms), int(num_splits)))


def xmla_decode(cfg: xmla_yarn_cfg, q: torch.Tensor, W_UK: torch.Tensor, W_UV: torch.Tensor, pool: torch.Tensor,
                num_blocks: int, block_table: torch.Tensor, max_blocks: int,
                seqlens: torch.Tensor, batch: int, q_len: int, max_seqlen: int,
                softmax_scale: float, num_splits: int, workspace: torch.Tensor,
                workspace_bytes: int, status: torch.Tensor | None, out: torch.Tensor,
                stream=None) -> None:
    _check(lib().xmla_decode(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(pool), int(num_blocks),
                             _ptr(block_table), int(max_blocks), _ptr(seqlens), int(batch),
                             int(q_len), int(max_seqlen), float(softmax_scale), int(num_splits),
                             _ptr(workspace), int(workspace_bytes), _ptr(status), _ptr(out),
                             _stream(stream)),
           "xmla_decode")


def xmla_decode_profiled(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                         q_len, max_seqlen, softmax_scale, num_splits, workspace, workspace_bytes,
                         status, out, stream=None, attn_start=None, attn_stop=None) -> None:
    ev = [None if e is None else (e.cuda_event if hasattr(e, "cuda_event") else int(e))
          for e in (attn_start, attn_stop)]
    _check(lib().xmla_decode_profiled(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(pool), int(num_blocks),
                                      _ptr(block_table), int(max_blocks), _ptr(seqlens), int(batch),
                                      int(q_len), int(max_seqlen), float(softmax_scale),
                                      int(num_splits), _ptr(workspace), int(workspace_bytes),
                                      _ptr(status), _ptr(out), _stream(stream), ev[0], ev[1]),
           "xmla_decode_profiled")


def xmla_decode_step(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                     q_len, max_seqlen, seq_ids, positions, c_kv, k_pe, T, softmax_scale,
                     num_splits, workspace, workspace_bytes, status, out, stream=None,
                     attn_start=None, attn_stop=None) -> None:
    """Append the step's T new rows (k_pe raw, rotated with cfg) and decode."""
    ev = [None if e is None else (e.cuda_event if hasattr(e, "cuda_event") else int(e))
          for e in (attn_start, attn_stop)]
    _check(lib().xmla_decode_step(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(pool),
                                  int(num_blocks), _ptr(block_table), int(max_blocks), _ptr(seqlens),
                                  int(batch), int(q_len), int(max_seqlen), _ptr(seq_ids),
                                  _ptr(positions), _ptr(c_kv), _ptr(k_pe), int(T),
                                  float(softmax_scale), int(num_splits), _ptr(workspace),
                                  int(workspace_bytes), _ptr(status), _ptr(out), _stream(stream),
                                  ev[0], ev[1]),
           "xmla_decode_step")


def xmla_decode_step_from_hidden(cfg, q, W_UK, W_UV, hidden, W_kva, bias, pool, num_blocks,
                                 block_table, max_blocks, seqlens, batch, q_len, max_seqlen,
                                 seq_ids, positions, T, softmax_scale, num_splits, workspace,
                                 workspace_bytes, status, out, stream=None, attn_start=None,
                                 attn_stop=None) -> None:
    """Produce the step's T new cache rows from hidden states, then decode."""
    ev = [None if e is None else (e.cuda_event if hasattr(e, "cuda_event") else int(e))
          for e in (attn_start, attn_stop)]
    _check(lib().xmla_decode_step_from_hidden(
        ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(hidden), _ptr(W_kva), _ptr(bias),
        _ptr(pool), int(num_blocks), _ptr(block_table), int(max_blocks), _ptr(seqlens), int(batch),
        int(q_len), int(max_seqlen), _ptr(seq_ids), _ptr(positions), int(T), float(softmax_scale),
        int(num_splits), _ptr(workspace), int(workspace_bytes), _ptr(status), _ptr(out),
        _stream(stream), ev[0], ev[1]), "xmla_decode_step_from_hidden")


def xmla_decode_noalloc(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens,
                        batch, q_len, max_seqlen, softmax_scale, num_splits, status, out,
                        stream=None) -> None:
    """xmla_decode with the library's fixed device scratch instead of a caller
    workspace (for callers that may not allocate device memory)."""
    _check(lib().xmla_decode_noalloc(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(pool),
                                     int(num_blocks), _ptr(block_table), int(max_blocks),
                                     _ptr(seqlens), int(batch), int(q_len), int(max_seqlen),
                                     float(softmax_scale), int(num_splits), _ptr(status), _ptr(out),
                                     _stream(stream)),
           "xmla_decode_noalloc")


def xmla_shard_partial_floats(batch: int, q_len: int) -> int:
    return int(lib().xmla_shard_partial_floats(int(batch), int(q_len)))


def xmla_decode_shard_workspace_size(batch: int, q_len: int, max_seqlen: int, page_lo: int,
                                     page_hi: int, num_sms: int, num_splits: int = 0) -> int:
    return int(lib().xmla_decode_shard_workspace_size(int(batch), int(q_len), int(max_seqlen),
                                                      int(page_lo), int(page_hi), int(num_sms),
                                                      int(num_splits)))


def xmla_decode_shard(cfg, q, W_UK, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                      q_len, max_seqlen, softmax_scale, page_lo, page_hi, num_splits, workspace,
                      workspace_bytes, status, shard_partial, stream=None) -> None:
    """One rank's part of a sequence-parallel decode over logical pages
    [page_lo, page_hi): its merged partial goes to shard_partial (fp32)."""
    _check(lib().xmla_decode_shard(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(pool),
                                   int(num_blocks), _ptr(block_table), int(max_blocks),
                                   _ptr(seqlens), int(batch), int(q_len), int(max_seqlen),
                                   float(softmax_scale), int(page_lo), int(page_hi),
                                   int(num_splits), _ptr(workspace), int(workspace_bytes),
                                   _ptr(status), _ptr(shard_partial), _stream(stream)),
           "xmla_decode_shard")


def xmla_combine_shards(partials, num_shards, W_UV, batch, q_len, out, stream=None) -> None:
    """Merge of gathered shard partials (rank-major) and the W_UV product."""
    _check(lib().xmla_combine_shards(_ptr(partials), int(num_shards), _ptr(W_UV), int(batch),
                                     int(q_len), _ptr(out), _stream(stream)),
           "xmla_combine_shards")


def xmla_cache_append_q8(pool_q8: torch.Tensor, num_blocks: int, block_table: torch.Tensor,
                         max_blocks: int, batch: int, seq_ids: torch.Tensor,
                         positions: torch.Tensor, c_kv: torch.Tensor, k_pe: torch.Tensor,
                         rope_cfg: xmla_yarn_cfg | None, T: int,
                         status: torch.Tensor | None = None, stream=None) -> None:
    _check(lib().xmla_cache_append_q8(_ptr(pool_q8), int(num_blocks), _ptr(block_table),
                                      int(max_blocks), int(batch), _ptr(seq_ids), _ptr(positions),
                                      _ptr(c_kv), _ptr(k_pe),
                                      None if rope_cfg is None else ctypes.byref(rope_cfg), int(T),
                                      _ptr(status), _stream(stream)),
           "xmla_cache_append_q8")


def xmla_decode_q8_workspace_size(batch: int, q_len: int, max_seqlen: int, num_sms: int,
                                  num_splits: int = 0) -> int:
    return int(lib().xmla_decode_q8_workspace_size(int(batch), int(q_len), int(max_seqlen),
                                                   int(num_sms), int(num_splits)))


def xmla_decode_q8_num_splits(batch: int, q_len: int, max_seqlen: int, num_sms: int,
                              num_splits: int = 0) -> int:
    return int(lib().xmla_decode_q8_num_splits(int(batch), int(q_len), int(max_seqlen),
                                               int(num_sms), int(num_splits)))


def xmla_decode_q8(cfg, q, W_UK, W_UV, pool_q8, num_blocks, block_table, max_blocks, seqlens,
                   batch, q_len, max_seqlen, softmax_scale, num_splits, workspace,
                   workspace_bytes, status, out, stream=None) -> None:
    _check(lib().xmla_decode_q8(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(pool_q8),
                                int(num_blocks), _ptr(block_table), int(max_blocks),
                                _ptr(seqlens), int(batch), int(q_len), int(max_seqlen),
                                float(softmax_scale), int(num_splits), _ptr(workspace),
                                int(workspace_bytes), _ptr(status), _ptr(out), _stream(stream)),
           "xmla_decode_q8")


def xmla_decode_q8_profiled(cfg, q, W_UK, W_UV, pool_q8, num_blocks, block_table, max_blocks,
                            seqlens, batch, q_len, max_seqlen, softmax_scale, num_splits,
                            workspace, workspace_bytes, status, out, stream=None,
                            attn_start=None, attn_stop=None) -> None:
    ev = [None if e is None else (e.cuda_event if hasattr(e, "cuda_event") else int(e))
          for e in (attn_start, attn_stop)]
    _check(lib().xmla_decode_q8_profiled(ctypes.byref(cfg), _ptr(q), _ptr(W_UK), _ptr(W_UV),
                                         _ptr(pool_q8), int(num_blocks), _ptr(block_table),
                                         int(max_blocks), _ptr(seqlens), int(batch), int(q_len),
                                         int(max_seqlen), float(softmax_scale), int(num_splits),
                                         _ptr(workspace), int(workspace_bytes), _ptr(status),
                                         _ptr(out), _stream(stream), ev[0], ev[1]),
           "xmla_decode_q8_profiled")


def xmla_selftest_wait_timeout(status: torch.Tensor, timeout_ns: int, stream=None) -> None:
    _check(lib().xmla_selftest_wait_timeout(_ptr(status), int(timeout_ns), _stream(stream)),
           "xmla_selftest_wait_timeout")
