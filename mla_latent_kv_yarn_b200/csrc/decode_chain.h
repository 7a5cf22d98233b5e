// Host-side interface between the kernels of one decode call and the C ABI.
//
// A decode call runs three kernels on one stream, chained with programmatic
// dependent launch (each waits with griddepcontrol.wait for its predecessor
// before reading anything that predecessor may write):
//   q_absorb   (absorb_combine.cu)  q_ext = c * [W_UK^T q_nope | rope(q_pe)]
//   split-K    (mla_decode.cu)      per-split (m, l, O) over the paged cache
//   combine    (absorb_combine.cu)  log-sum-exp merge of the splits, then W_UV
// The decode-step entry fuses the cache append into the first kernel
// (step_prologue_kernel in absorb_combine.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "produce.cuh"
#include "split_kv.h"
#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

constexpr float kLog2e = 1.4426950408889634f;

// Length-aware split plan of a batch, computed on the device by one extra
// block of the first kernel of the call (after its griddepcontrol.wait, from
// the sequence lengths): every (sequence, row group) unit u gets ns_u >= 1 of
// the `ctas` split-K CTAs and its pages are divided evenly over them, with the
// largest share per CTA as small as the CTA count allows.  unit_tab[u] =
// {first CTA, ns_u}; work_tab[k] as in DecodeParams.
constexpr int kMaxPlanCtas = 256;
struct WorkPlanArgs {
  const int32_t* seqlens;
  int64_t max_seqlen;
  int32_t batch;
  int32_t groups;
  int32_t ctas;  // split-K grid size, units < ctas <= kMaxPlanCtas
  int4* work_tab;
  int2* unit_tab;
  // a unit of at most short_pages pages costs short_weight times its pages
  // (the mixed kernel runs one pass per query over a short sequence)
  int32_t short_pages;
  int32_t short_weight;
  // block-table lines (32 entries of 128 B each) every block of the first
  // kernel helps bring into L2, so that the split-K kernel's first block-id
  // reads hit it; 0 = none.  Read by every launch of the first kernel, with
  // or without a plan.
  const int32_t* bt_prefetch;
  int64_t bt_lines;
};

// q_ext[r, h] for rows r = b*q_len + j; qscale = softmax scale * log2 e.
// split: each query row as a hi and a lo bf16 row (the split-K kernel's
// split_q layout).  with_plan: also compute the length-aware plan of `plan`
// (whose block-table prefetch fields are used either way).
// rope_only: only the rope columns (the latent part comes from
// launch_absorb_gemm).
// f16: q_ext holds f16 values (single rows) for the 8-bit cache's kernel.
cudaError_t launch_q_absorb(const __nv_bfloat16* q, const __nv_bfloat16* W_UK,
                            const int32_t* seqlens, __nv_bfloat16* q_ext, int rows, int q_len,
                            int split, float qscale, const RopeTable& tab,
                            const WorkPlanArgs& plan, bool with_plan, bool rope_only,
                            cudaStream_t st, bool f16 = false);

// The new tokens of a decode step, appended by step_prologue_kernel.
struct AppendArgs {
  uint4* pool;
  int64_t num_blocks;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t batch;
  const int32_t* seq_ids;
  const int64_t* positions;
  const uint4* c_kv;
  const uint4* k_pe;
  int64_t T;
  int32_t* status;
  int rotate;
};

// q_absorb and the cache rows of the same step in one launch: ready rows are
// appended (ap), rows from hidden states are produced (pa, nullable); plan and
// with_plan as for launch_q_absorb.
cudaError_t launch_step_prologue(const __nv_bfloat16* q, const __nv_bfloat16* W_UK,
                                 const int32_t* seqlens, __nv_bfloat16* q_ext, int rows,
                                 int q_len, int split, float qscale, const RopeTable& q_tab,
                                 const AppendArgs& ap, const RopeTable& k_tab,
                                 const ProduceArgs* pa, const WorkPlanArgs& plan, bool with_plan,
                                 bool rope_only, cudaStream_t st);

// Merge of the splits and the W_UV product, written to out[rows, 32, 128].
// Split s of a row is o_stride floats (O) and ml_stride (m, l) pairs after
// split 0; 0 means the split-K kernel's layout (rows_per_cta rows apart).
// unit_tab (non-null, split-K layout only): the splits of unit u are the
// unit_tab[u].y work items from unit_tab[u].x on, as the plan above made them.
cudaError_t launch_combine(const float* part_o, const float* part_ml, const __nv_bfloat16* W_UV,
                           __nv_bfloat16* out, int rows, int q_len, int groups, int nsplit,
                           int rows_per_cta, cudaStream_t st, int64_t o_stride = 0,
                           int64_t ml_stride = 0, const int2* unit_tab = nullptr);

// Per-head tensor-core products of a prompt chunk (head_gemm.cu).  Rows r =
// b*q_len + j, R of them.
struct HeadGemmParams {
  int rows;                 // R
  float scale;              // absorb: softmax scale * log2 e
  __nv_bfloat16* q_ext;     // absorb: latent columns of the hi/lo query rows
  __nv_bfloat16* out;       // W_UV: out[R, 32, 128]
  int32_t* status;
  uint64_t wait_limit_ns;
};
// q_lat = q_nope . W_UK[h] for every head, written scaled as hi/lo bf16 into
// q_ext (split query layout).  q_map: the query [R, 32, 192] as a 3-D map, box
// 64 x 1 x 128; wuk_map: W_UK as [4096, 512], box 64 x 128 (both 128-B swizzle).
cudaError_t launch_absorb_gemm(const CUtensorMap& q_map, const CUtensorMap& wuk_map,
                               const HeadGemmParams& p, cudaStream_t st);
// out = (o_hi + o_lo) . W_UV[h] for every head.  ohi/olo_map: [R, 32, 512]
// bf16 as 3-D maps, box 64 x 1 x 128; wuv_map: W_UV as [16384, 128], box 64 x 128.
cudaError_t launch_uv_gemm(const CUtensorMap& ohi_map, const CUtensorMap& olo_map,
                           const CUtensorMap& wuv_map, const HeadGemmParams& p, cudaStream_t st);

// The merged latent output of every (row, head), normalised, as two bf16 parts
// o_hi = bf16(o), o_lo = bf16(o - o_hi), each [rows, 32, 512]; unit_tab as for
// launch_combine.
cudaError_t launch_latent_out(const float* part_o, const float* part_ml, __nv_bfloat16* o_hi,
                              __nv_bfloat16* o_lo, int rows, int q_len, int groups, int nsplit,
                              int rows_per_cta, const int2* unit_tab, cudaStream_t st);

// Merge of the splits into one partial per (row, head) -- (M, L, unnormalised
// O) -- for a sequence-parallel decode; layout in absorb_combine.cu.
cudaError_t launch_merge_splits(const float* part_o, const float* part_ml, float* out, int rows,
                                int q_len, int groups, int nsplit, int rows_per_cta,
                                cudaStream_t st);

// Quantise and append T cache rows to the 8-bit pool ([num_blocks, 64, 608]
// bytes, layout in q8_append.cu); rotate: RoPE the rope key with tab first.
cudaError_t launch_cache_append_q8(uint8_t* pool, int64_t num_blocks, const int32_t* block_table,
                                   int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                                   const int64_t* positions, const __nv_bfloat16* c_kv,
                                   const __nv_bfloat16* k_pe, int32_t* status, int rotate,
                                   const RopeTable& tab, int64_t T, cudaStream_t st);

// Split-K attention over the 8-bit pool ([num_blocks, 64, 608] bytes), 32 rows
// per CTA, f16 q_ext (q_map as for launch_split_kv with 32-row boxes); writes
// the same partials as launch_split_kv.  (The pool pointer is an argument of
// its own: DecodeParams is the bf16 kernel's parameter block, whose code
// generation has proven sensitive to its layout.)
cudaError_t launch_split_kv_q8(const CUtensorMap& q_map, const DecodeParams& dp,
                               const uint8_t* pool_q8, int64_t items, cudaStream_t st);

}  // namespace xmla
