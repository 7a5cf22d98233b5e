// Host-side interface of the prompt-chunk kernels (prefill.cu): a chunk of at
// least kPrefillMinChunk new tokens per sequence, attended in the non-absorbed
// form with fp16 tensor-core operands.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "append.cuh"
#include "yarn.cuh"

namespace xmla {

// Chunks of at least this many new tokens per sequence take this path.
constexpr int32_t kPrefillMinChunk = 64;

// Workspace tensors (fp16), rows of every sequence padded to s_pad tokens (a
// multiple of 128):
//   qh  [B * q_len, 32, 192]   the queries [q_nope | rope(q_pe)]
//   kx  [B * s_pad, 32, 128]   K_nope = W_UK[h] c_kv[t]
//   vx  [B * s_pad, 32, 128]   V = W_UV[h]^T c_kv[t]
//   kp  [B * s_pad, 64]        the cached rotated rope key
struct PrefillParams {
  const int32_t* block_table;
  const int32_t* seqlens;
  const uint16_t* pool;  // [num_blocks, 64, 576] bf16 bits
  __half* kx;
  __half* vx;
  __half* kp;
  __nv_bfloat16* out;    // [B, q_len, 32, 128]
  int32_t* status;
  int64_t num_blocks;
  int64_t max_seqlen;
  int64_t s_pad;
  uint64_t wait_limit_ns;
  float scale_log2;      // softmax scale * log2 e
  int32_t max_blocks;
  int32_t batch;
  int32_t q_len;
};

// The queries as fp16 rows (RoPE of q_pe at each query's position) and, for a
// decode step, the append of the chunk's cache rows (ap.T > 0).
cudaError_t launch_prefill_prep(const __nv_bfloat16* q, const int32_t* seqlens, __half* qh, int rows,
                                int q_len, const RopeTable& q_tab, const AppendArgs& ap,
                                const RopeTable& k_tab, cudaStream_t st);

// K_nope, V and the rope key of every cached token of every sequence.
// pool_map: the cache rows (576 bf16), box 64 x 64; wuk_map: W_UK as [4096, 512]
// and wuv_map: W_UV as [16384, 128], box 64 x 128 (all 128-byte swizzle).
cudaError_t launch_kv_expand(const CUtensorMap& pool_map, const CUtensorMap& wuk_map,
                             const CUtensorMap& wuv_map, const PrefillParams& p, cudaStream_t st);

// The attention of every query of the chunk, written to p.out.  q_map: qh as
// [rows, 32, 192]; k_map / v_map: kx / vx as [B * s_pad, 32, 128] (3-D, box
// 64 x 1 x 128); kp_map: kp as [B * s_pad, 64] (box 64 x 128); all fp16 with
// the 128-byte swizzle.
cudaError_t launch_prefill_attn(const CUtensorMap& q_map, const CUtensorMap& k_map,
                                const CUtensorMap& kp_map, const CUtensorMap& v_map,
                                const PrefillParams& p, cudaStream_t st);

}  // namespace xmla
