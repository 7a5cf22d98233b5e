// Interface of the split-K attention kernel (mla_decode.cu) to the host code
// that launches it.  Kept apart from the rest of the decode chain so that the
// kernel's translation unit depends on nothing else.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace xmla {

constexpr int kMaxSplits = 1024;

// Sequences of at most this many tokens are attended with the query as a hi
// and a lo bf16 part (see launch_split_kv and launch_split_kv_mixed).
constexpr int64_t kSplitQMaxSeqlen = 4096;

// Arguments of the split-K attention kernel.  Partial results are laid out
// per work item: (sequence b, row group g, split s) in that order, or, with a
// work table, in the order of the table's entries.
struct DecodeParams {
  const int32_t* block_table;
  const int32_t* seqlens;
  float* part_o;   // [items, NR, 512] unnormalised O of each split
  float* part_ml;  // [items, NR, 2] running max m (log2 units) and sum l
  int32_t* status;
  int64_t num_blocks;
  int64_t max_seqlen;
  uint64_t wait_limit_ns;
  int32_t max_blocks;
  int32_t batch;
  int32_t q_len;
  int32_t groups;
  int32_t nsplit;
  // logical pages of every sequence this call attends over: [page_lo, page_hi)
  // clipped to the sequence (0 and INT64_MAX for the whole sequence); the
  // splits partition that range
  int64_t page_lo;
  int64_t page_hi;
  // non-null: a work table written on the device by the first kernel of the
  // call (length-aware plan, batch > 1): entry k = {unit b * groups + g,
  // first logical page, end page, 0} of CTA k, unit -1 for an idle CTA.  The
  // kernel reads it after griddepcontrol.wait; nsplit and page_lo/hi are unused.
  const int4* work_tab;
  // non-null (split_q, one split per unit, no work table): the kernel writes
  // the normalised latent output o = O / l itself as o_hi = bf16(o) and
  // o_lo = bf16(o - o_hi) at [(r * 32 + h) * 512 + d] (r = b * q_len + j)
  // instead of part_o / part_ml
  __nv_bfloat16* o_hi;
  __nv_bfloat16* o_lo;
};

// Split-K attention over `items` work items; nr = rows per CTA (32 or 64);
// split_q (nr 32 only): q_ext holds a hi and a lo bf16 row per query row, 32
// heads of hi then 32 of lo per query.  pool_map: 576-column rows of the cache
// pool, box 64 x 64; q_map: rows of q_ext, box 64 x 64 (both 128-byte swizzled).
cudaError_t launch_split_kv(int nr, bool split_q, const CUtensorMap& pool_map,
                            const CUtensorMap& q_map, const DecodeParams& dp, int64_t items,
                            cudaStream_t st);

// Split-K attention of a batch that may hold short and long sequences, q_ext
// in the split layout (as for split_q): each CTA attends its sequence with the
// hi/lo query (q2_map: box 64 x 64) when it has at most kSplitQMaxSeqlen
// tokens, one pass per query of its nr-row group, else with the hi rows alone
// (q_map: the same rows, box 64 x 32).  Writes the partials
// launch_split_kv(nr, false, ...) writes.
cudaError_t launch_split_kv_mixed(int nr, const CUtensorMap& pool_map, const CUtensorMap& q_map,
                                  const CUtensorMap& q2_map, const DecodeParams& dp,
                                  int64_t items, cudaStream_t st);

}  // namespace xmla
