// C ABI of the decode path: argument checks, the workspace plan, TMA tensor
// maps, and the launch of the kernel chain (decode_chain.h).
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": attention over the cached latent, absorbed form.
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", sections 一 and 二:
//      YaRN RoPE on q_pe; the cache read dominates a long-context decode step.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "decode_chain.h"
#include "prefill.h"

namespace xmla {

// ---------------------------------------------------------------- self-test kernel

__global__ void wait_timeout_selftest_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar_word;
  const uint32_t b = smem_u32(&bar_word);
  mbar_init(b, 1);
  fence_barrier_init();
  // nothing ever arrives on this barrier: the bounded wait must give up
  mbar_wait(b, 0, nullptr, status, limit_ns);
}

// ---------------------------------------------------------------- host plan

// Up to kSplitQMaxSeqlen tokens per sequence, and for every call with more
// than kSplitQMinChunk new tokens (a prefill chunk, whose first queries see
// only a few tokens), the query goes to the QK product as a hi and a lo bf16
// part (the split-K kernel's split_q layout, one query of 32 heads per CTA).
// A short context is dominated by a few tokens and its output is large (|out|
// up to ~4), so the ~2^-9 relative score error of a single bf16 query reaches
// the 1e-2 output bound there; the split costs a shallower page ring, which
// only long decode contexts, dominated by streaming, would notice.  A decode
// call of several sequences whose longest exceeds kSplitQMaxSeqlen may also
// hold short ones: it runs the mixed kernel, which makes that choice per
// sequence on the device (q_ext in the split layout; long sequences use the hi
// rows alone).
constexpr int32_t kSplitQMinChunk = 8;

struct Plan {
  // a prompt chunk of >= kPrefillMinChunk new tokens: the non-absorbed path of
  // prefill.cu (workspace: qh, kx, vx, kp; s_pad token rows per sequence)
  bool prefill;
  int64_t s_pad;
  size_t off_qh, off_kx, off_vx, off_kp, prefill_bytes;
  bool split;   // hi/lo query (split_q) for every sequence
  bool mixed;   // hi/lo query for the sequences of <= kSplitQMaxSeqlen tokens only
  bool gemm;    // a prompt chunk: absorb and W_UV on the tensor cores (head_gemm.cu)
  int nr;       // rows per CTA (32 or 64)
  int groups;   // row groups per sequence
  int nsplit;   // KV splits per (sequence, group) when every sequence has max_seqlen tokens
  bool table;   // splits planned on the device from the actual lengths (WorkPlanArgs)
  int64_t items;
  size_t off_qext, off_o, off_ml, off_wtab, off_utab, off_olat, bytes;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// span_pages: logical pages a call attends over at most (the split count is
// sized for them); 0 = all pages of max_seqlen.  allow_table: a batch of
// several sequences with automatic splits gets the length-aware plan: one
// CTA per SM, the pages of each sequence divided over them in proportion to
// its length by the first kernel of the call.
// q8: the 8-bit cache's kernel (32 rows per CTA, one f16 query row each).
static bool make_plan(int32_t B, int32_t q_len, int64_t max_seqlen, int32_t num_sms,
                      int32_t num_splits, Plan* pl, int64_t span_pages = 0,
                      bool allow_table = true, bool q8 = false, bool allow_prefill = true) {
  if (B < 1 || q_len < 1 || q_len > (q8 ? kQ8MaxQLen : kMaxQLen) || max_seqlen < q_len ||
      max_seqlen > (int64_t)0x7fffffff - kPage || num_sms < 1 || num_splits < 0 || span_pages < 0)
    return false;
  // query rows, and (row, head) pairs, are counted in 32-bit integers by the kernels
  if ((int64_t)B * q_len * kHeads > (int64_t)0x7fffffff) return false;
  Plan P;
  P.split = !q8 && (max_seqlen <= kSplitQMaxSeqlen || q_len > kSplitQMinChunk);
  P.mixed = !q8 && !P.split && B > 1;
  P.nr = q8 || P.split || q_len == 1 ? 32 : 64;
  P.groups = (q_len * 32 + P.nr - 1) / P.nr;
  int64_t max_pages = (max_seqlen + kPage - 1) / kPage;
  if (span_pages > 0 && span_pages < max_pages) max_pages = span_pages;
  int64_t ns;
  if (num_splits > 0) {
    ns = num_splits;
  } else {
    const int64_t units = (int64_t)B * P.groups;
    ns = units >= num_sms ? 1 : num_sms / units;
    const int64_t cap = max_pages >= 2 ? max_pages / 2 : 1;  // at least two pages per split
    if (ns > cap) ns = cap;
  }
  if (ns < 1) ns = 1;
  if (ns > kMaxSplits) return false;
  P.nsplit = (int)ns;
  const int64_t units = (int64_t)B * P.groups;
  P.table = allow_table && num_splits == 0 && span_pages == 0 && B > 1 && units < num_sms &&
            num_sms <= kMaxPlanCtas;
  P.items = P.table ? num_sms : units * P.nsplit;
  if (P.items > 0x7fffffff) return false;
  // q_ext: bf16 rows of 576; split or mixed, each row also has its low half
  const size_t qext = (size_t)B * q_len * kHeads * kDRow * 2 * (P.split || P.mixed ? 2 : 1);
  P.off_qext = 0;
  P.off_o = align_up(qext, 1024);
  P.off_ml = align_up(P.off_o + (size_t)P.items * P.nr * kDLatent * 4, 1024);
  P.off_wtab = align_up(P.off_ml + (size_t)P.items * P.nr * 2 * 4, 1024);
  P.off_utab = align_up(P.off_wtab + (P.table ? (size_t)P.items * 16 : 0), 256);
  // a prompt chunk's merged latent output, hi and lo bf16 [rows, 32, 512] each
  P.gemm = !q8 && allow_table && q_len > kSplitQMinChunk;
  P.off_olat = align_up(P.off_utab + (P.table ? (size_t)units * 8 : 0), 1024);
  const size_t olat = P.gemm ? (size_t)B * q_len * kHeads * kDLatent * 2 : 0;
  P.bytes = align_up(P.off_olat + 2 * olat, 1024);
  // a chunk of >= kPrefillMinChunk tokens runs the non-absorbed path (the
  // absorbed one above stays for a chunk whose cache rows come from hidden
  // states); the workspace covers both
  P.prefill = false;
  P.s_pad = (max_seqlen + 127) / 128 * 128;
  P.prefill_bytes = 0;
  // (the expanded rows' TMA coordinates are int32: past that bound, the absorbed path)
  if (!q8 && allow_table && q_len >= kPrefillMinChunk &&
      (int64_t)B * P.s_pad <= (int64_t)0x7fffffff - 128) {
    P.off_qh = 0;
    P.off_kx = align_up((size_t)B * q_len * kHeads * kDQ * 2, 1024);
    P.off_vx = align_up(P.off_kx + (size_t)B * P.s_pad * kHeads * kDNope * 2, 1024);
    P.off_kp = align_up(P.off_vx + (size_t)B * P.s_pad * kHeads * kDV * 2, 1024);
    P.prefill_bytes = align_up(P.off_kp + (size_t)B * P.s_pad * kDRope * 2, 1024);
    P.prefill = allow_prefill;
    if (P.prefill_bytes > P.bytes) P.bytes = P.prefill_bytes;
  }
  *pl = P;
  return true;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D map over rows of 576 bf16 (1152 B), box = 64 columns x box_rows rows,
// 128-byte swizzle (the layout the tensor-core descriptors above expect).
static bool encode_rows576(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDRow, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDRow * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over a [rows, 32, cols] bf16 tensor (the query, cols 192, or o_lat,
// cols 512), box 64 columns x 1 head x 128 rows, 128-byte swizzle: one box is a
// 128-row K-major tile of one head.
static bool encode_heads3d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)kHeads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * kHeads};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a row-major [rows, cols] bf16 weight, box 64 columns x 128 rows,
// 128-byte swizzle: one box is 128 K rows of 64 N columns (an MN-major tile).
static bool encode_weight(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 maps of the prompt-chunk path: a 3-D [rows, 32, cols] tensor with box
// 64 columns x 1 head x 128 rows, and a 2-D [rows, cols] one with box 64 x 128,
// 128-byte swizzle (K-major 128-row tiles, or MN-major ones read by rows).
static bool encode_f16_3d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)kHeads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * kHeads};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_f16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool device_ok(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev);
  return major == 10 && minor == 0;
}

}  // namespace xmla

using namespace xmla;

extern "C" size_t xmla_decode_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                             int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P) ? P.bytes : 0;
}

extern "C" int32_t xmla_decode_num_splits(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                          int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P) ? P.nsplit : 0;
}

static cudaError_t record_event(void* ev, cudaStream_t st) {
  if (ev == nullptr) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  // inside a graph capture the record must become an event-record node
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal)
             : cudaEventRecord((cudaEvent_t)ev, st);
}

// The decode chain shared by the entries below; `ap` (nullable) adds the
// step's cache append to the first kernel.
static xmla_status run_decode(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                              const void* W_UV, const void* pool, int64_t num_blocks,
                              const int32_t* block_table, int32_t max_blocks,
                              const int32_t* seqlens, int32_t batch, int32_t q_len,
                              int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                              void* workspace, size_t workspace_bytes, int32_t* status_dev,
                              void* out, void* stream, void* attn_start, void* attn_stop,
                              const AppendArgs* ap, const ProduceArgs* pa = nullptr,
                              int64_t page_lo = 0, int64_t page_hi = INT64_MAX,
                              float* shard_partial = nullptr, bool q8 = false) {
  if (q == nullptr || W_UK == nullptr || W_UV == nullptr || pool == nullptr ||
      block_table == nullptr || seqlens == nullptr || workspace == nullptr || out == nullptr)
    return XMLA_ERR_INVALID_ARG;
  if (!yarn_cfg_ok(cfg)) return XMLA_ERR_INVALID_ARG;
  if (cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)pool) & 15u) || (((uintptr_t)workspace) & 255u) || (((uintptr_t)q) & 15u) ||
      (((uintptr_t)W_UK) & 15u) || (((uintptr_t)W_UV) & 15u) || (((uintptr_t)out) & 15u))
    return XMLA_ERR_INVALID_ARG;
  if (page_lo < 0 || page_hi < page_lo) return XMLA_ERR_SHAPE;
  if (num_blocks < 1 || num_blocks * kPage >= 0x7fffffffLL || max_blocks < 1 ||
      (int64_t)max_blocks * kPage < max_seqlen)
    return XMLA_ERR_SHAPE;
  int nsm = 0;
  if (!device_ok(&nsm)) return XMLA_ERR_UNSUPPORTED;
  Plan P;
  const int64_t span = page_hi == INT64_MAX ? 0 : (page_hi > page_lo ? page_hi - page_lo : 1);
  if (q8 && (ap != nullptr || pa != nullptr || shard_partial != nullptr || page_lo != 0 ||
             page_hi != INT64_MAX))
    return XMLA_ERR_INVALID_ARG;
  if (!make_plan(batch, q_len, max_seqlen, nsm, num_splits, &P, span, shard_partial == nullptr,
                 q8, pa == nullptr))
    return XMLA_ERR_SHAPE;
  if (workspace_bytes < P.bytes) return XMLA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = (uint8_t*)workspace;
  if (P.prefill) {
    // a prompt chunk: queries as fp16 rows (and the chunk's append), K_nope / V
    // expanded per head, then the tensor-core attention writing `out`
    const int rows = batch * q_len;
    PrefillParams pp;
    pp.block_table = block_table;
    pp.seqlens = seqlens;
    pp.pool = (const uint16_t*)pool;
    pp.kx = (__half*)(ws + P.off_kx);
    pp.vx = (__half*)(ws + P.off_vx);
    pp.kp = (__half*)(ws + P.off_kp);
    pp.out = (__nv_bfloat16*)out;
    pp.status = status_dev;
    pp.num_blocks = num_blocks;
    pp.max_seqlen = max_seqlen;
    pp.s_pad = P.s_pad;
    pp.wait_limit_ns = kWaitLimitNs;
    pp.scale_log2 = softmax_scale * kLog2e;
    pp.max_blocks = max_blocks;
    pp.batch = batch;
    pp.q_len = q_len;
    __half* qh = (__half*)(ws + P.off_qh);
    const uint64_t krows = (uint64_t)batch * P.s_pad;
    CUtensorMap m_pool, m_wuk, m_wuv, m_q, m_k, m_v, m_kp;
    if (!encode_rows576(&m_pool, pool, (uint64_t)num_blocks * kPage, kPage) ||
        !encode_weight(&m_wuk, W_UK, (uint64_t)kHeads * kDNope, kDLatent) ||
        !encode_weight(&m_wuv, W_UV, (uint64_t)kHeads * kDLatent, kDV) ||
        !encode_f16_3d(&m_q, qh, (uint64_t)rows, kDQ) ||
        !encode_f16_3d(&m_k, pp.kx, krows, kDNope) || !encode_f16_3d(&m_v, pp.vx, krows, kDV) ||
        !encode_f16_2d(&m_kp, pp.kp, krows, kDRope))
      return XMLA_ERR_CUDA;
    const RopeTable tab = make_rope_table(cfg);
    AppendArgs none{};
    if (launch_prefill_prep((const __nv_bfloat16*)q, seqlens, qh, rows, q_len, tab,
                            ap != nullptr ? *ap : none, tab, st) != cudaSuccess ||
        launch_kv_expand(m_pool, m_wuk, m_wuv, pp, st) != cudaSuccess)
      return XMLA_ERR_CUDA;
    if (record_event(attn_start, st) != cudaSuccess) return XMLA_ERR_CUDA;
    if (launch_prefill_attn(m_q, m_k, m_kp, m_v, pp, st) != cudaSuccess) return XMLA_ERR_CUDA;
    return record_event(attn_stop, st) == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
  }
  __nv_bfloat16* q_ext = (__nv_bfloat16*)(ws + P.off_qext);
  const int rows = batch * q_len;

  CUtensorMap tmap_pool, tmap_q;
  if (!q8 && !encode_rows576(&tmap_pool, pool, (uint64_t)num_blocks * kPage, kPage))
    return XMLA_ERR_CUDA;
  // the QK product's B tile: 64 rows (32 heads hi then lo when split, 32 heads of one query
  // at 32 rows per CTA, else 2 queries x 32 heads)
  // mixed: q_ext in the split layout, read as 32-row boxes of hi rows (long
  // sequences, tmap_q) and as 64-row boxes of hi and lo rows (short ones, tmap_q2)
  if (!encode_rows576(&tmap_q, q_ext, (uint64_t)rows * kHeads * (P.split || P.mixed ? 2 : 1),
                      P.mixed ? 32 : P.split || P.nr == 64 ? 64 : 32))
    return XMLA_ERR_CUDA;
  CUtensorMap tmap_q2;
  if (P.mixed && !encode_rows576(&tmap_q2, q_ext, (uint64_t)rows * kHeads * 2, 64))
    return XMLA_ERR_CUDA;
  const int split_arg = P.split || P.mixed ? 1 : 0;

  const float qscale = softmax_scale * kLog2e;
  const RopeTable tab = make_rope_table(cfg);
  WorkPlanArgs plan{};
  if (P.table) {
    plan.seqlens = seqlens;
    plan.max_seqlen = max_seqlen;
    plan.batch = batch;
    plan.groups = P.groups;
    plan.ctas = (int32_t)P.items;
    plan.work_tab = (int4*)(ws + P.off_wtab);
    plan.unit_tab = (int2*)(ws + P.off_utab);
    // a short sequence's CTA runs one pass per query of its row group
    plan.short_pages = P.mixed ? (int32_t)(kSplitQMaxSeqlen / kPage) : 0;
    plan.short_weight = P.nr / 32;
  }
  // the first kernel brings the block table into L2 for the split-K kernel's
  // first block-id reads (after an L2 flush or eviction they would miss)
  plan.bt_prefetch = block_table;
  plan.bt_lines = ((int64_t)batch * max_blocks + 31) / 32;
  // Every kernel of the chain waits (griddepcontrol.wait) for its predecessor
  // before reading anything a kernel of this step may have written, so once
  // the first kernel completes all earlier work on the stream has landed.
  // A prompt chunk runs five kernels: the first does the rope columns of q_ext
  // (and the append, the plan) while the tensor-core absorb fills the latent
  // columns; the latent output goes out as hi/lo bf16 (from the split-K
  // kernel itself when every unit has one split, else from a merge kernel)
  // and the tensor-core W_UV product writes `out`.
  HeadGemmParams gp{};
  CUtensorMap tmap_qin, tmap_wuk, tmap_ohi, tmap_olo, tmap_wuv;
  __nv_bfloat16* o_hi = (__nv_bfloat16*)(ws + P.off_olat);
  __nv_bfloat16* o_lo = o_hi + (size_t)rows * kHeads * kDLatent;
  if (P.gemm) {
    if (!encode_heads3d(&tmap_qin, q, (uint64_t)rows, kDQ) ||
        !encode_weight(&tmap_wuk, W_UK, (uint64_t)kHeads * kDNope, kDLatent) ||
        !encode_heads3d(&tmap_ohi, o_hi, (uint64_t)rows, kDLatent) ||
        !encode_heads3d(&tmap_olo, o_lo, (uint64_t)rows, kDLatent) ||
        !encode_weight(&tmap_wuv, W_UV, (uint64_t)kHeads * kDLatent, kDV))
      return XMLA_ERR_CUDA;
    gp.rows = rows;
    gp.scale = qscale;
    gp.q_ext = q_ext;
    gp.out = (__nv_bfloat16*)out;
    gp.status = status_dev;
    gp.wait_limit_ns = kWaitLimitNs;
  }
  const cudaError_t e0 =
      ap != nullptr
          ? launch_step_prologue((const __nv_bfloat16*)q, (const __nv_bfloat16*)W_UK, seqlens, q_ext,
                                 rows, q_len, split_arg, qscale, tab, *ap, tab, pa, plan, P.table,
                                 P.gemm, st)
          : launch_q_absorb((const __nv_bfloat16*)q, (const __nv_bfloat16*)W_UK, seqlens, q_ext,
                            rows, q_len, split_arg, qscale, tab, plan, P.table, P.gemm, st, q8);
  if (e0 != cudaSuccess) return XMLA_ERR_CUDA;
  if (P.gemm && launch_absorb_gemm(tmap_qin, tmap_wuk, gp, st) != cudaSuccess) return XMLA_ERR_CUDA;

  DecodeParams dp;
  dp.block_table = block_table;
  dp.seqlens = seqlens;
  dp.part_o = (float*)(ws + P.off_o);
  dp.part_ml = (float*)(ws + P.off_ml);
  dp.status = status_dev;
  dp.num_blocks = num_blocks;
  dp.max_seqlen = max_seqlen;
  dp.wait_limit_ns = kWaitLimitNs;
  dp.max_blocks = max_blocks;
  dp.batch = batch;
  dp.q_len = q_len;
  dp.groups = P.groups;
  dp.nsplit = P.nsplit;
  dp.page_lo = page_lo;
  dp.page_hi = page_hi;
  dp.work_tab = P.table ? plan.work_tab : nullptr;
  // a prompt chunk with one split per unit needs no merge: the attention
  // kernel writes the normalised hi/lo latent output the W_UV GEMM reads
  const bool direct = P.gemm && P.split && P.nsplit == 1 && !P.table && shard_partial == nullptr;
  dp.o_hi = direct ? o_hi : nullptr;
  dp.o_lo = direct ? o_lo : nullptr;
  if (record_event(attn_start, st) != cudaSuccess) return XMLA_ERR_CUDA;
  const cudaError_t ea =
      q8      ? launch_split_kv_q8(tmap_q, dp, (const uint8_t*)pool, P.items, st)
      : P.mixed ? launch_split_kv_mixed(P.nr, tmap_pool, tmap_q, tmap_q2, dp, P.items, st)
                : launch_split_kv(P.nr, P.split, tmap_pool, tmap_q, dp, P.items, st);
  if (ea != cudaSuccess) return XMLA_ERR_CUDA;
  if (record_event(attn_stop, st) != cudaSuccess) return XMLA_ERR_CUDA;
  if (shard_partial != nullptr) {
    const cudaError_t em = launch_merge_splits(dp.part_o, dp.part_ml, shard_partial, rows, q_len,
                                               P.groups, P.nsplit, P.nr, st);
    return em == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
  }
  if (P.gemm) {
    if (!direct &&
        launch_latent_out(dp.part_o, dp.part_ml, o_hi, o_lo, rows, q_len, P.groups, P.nsplit, P.nr,
                          P.table ? plan.unit_tab : nullptr, st) != cudaSuccess)
      return XMLA_ERR_CUDA;
    return launch_uv_gemm(tmap_ohi, tmap_olo, tmap_wuv, gp, st) == cudaSuccess ? XMLA_OK
                                                                               : XMLA_ERR_CUDA;
  }
  const cudaError_t e = launch_combine(dp.part_o, dp.part_ml, (const __nv_bfloat16*)W_UV,
                                       (__nv_bfloat16*)out, rows, q_len, P.groups, P.nsplit, P.nr,
                                       st, 0, 0, P.table ? plan.unit_tab : nullptr);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" xmla_status xmla_decode_profiled(const xmla_yarn_cfg* cfg, const void* q,
                                            const void* W_UK, const void* W_UV,
                                            const void* pool, int64_t num_blocks,
                                            const int32_t* block_table, int32_t max_blocks,
                                            const int32_t* seqlens, int32_t batch, int32_t q_len,
                                            int64_t max_seqlen, float softmax_scale,
                                            int32_t num_splits, void* workspace,
                                            size_t workspace_bytes, int32_t* status_dev, void* out,
                                            void* stream, void* attn_start, void* attn_stop) {
  return run_decode(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                    q_len, max_seqlen, softmax_scale, num_splits, workspace, workspace_bytes,
                    status_dev, out, stream, attn_start, attn_stop, nullptr);
}

extern "C" xmla_status xmla_decode_step(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                        const void* W_UV, void* pool, int64_t num_blocks,
                                        const int32_t* block_table, int32_t max_blocks,
                                        const int32_t* seqlens, int32_t batch, int32_t q_len,
                                        int64_t max_seqlen, const int32_t* seq_ids,
                                        const int64_t* positions, const void* c_kv,
                                        const void* k_pe, int64_t T, float softmax_scale,
                                        int32_t num_splits, void* workspace,
                                        size_t workspace_bytes, int32_t* status_dev, void* out,
                                        void* stream, void* attn_start, void* attn_stop) {
  if (T < 0) return XMLA_ERR_SHAPE;
  if (T > 0 && (seq_ids == nullptr || positions == nullptr || c_kv == nullptr || k_pe == nullptr))
    return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)c_kv) | ((uintptr_t)k_pe)) & 15u) return XMLA_ERR_INVALID_ARG;
  AppendArgs ap;
  ap.pool = (uint4*)pool;
  ap.num_blocks = num_blocks;
  ap.block_table = block_table;
  ap.max_blocks = max_blocks;
  ap.batch = batch;
  ap.seq_ids = seq_ids;
  ap.positions = positions;
  ap.c_kv = (const uint4*)c_kv;
  ap.k_pe = (const uint4*)k_pe;
  ap.T = T;
  ap.status = status_dev;
  ap.rotate = 1;
  return run_decode(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                    q_len, max_seqlen, softmax_scale, num_splits, workspace, workspace_bytes,
                    status_dev, out, stream, attn_start, attn_stop, &ap);
}

extern "C" xmla_status xmla_decode_step_from_hidden(
    const xmla_yarn_cfg* cfg, const void* q, const void* W_UK, const void* W_UV,
    const void* hidden, const void* W_kva, const void* bias, void* pool, int64_t num_blocks,
    const int32_t* block_table, int32_t max_blocks, const int32_t* seqlens, int32_t batch,
    int32_t q_len, int64_t max_seqlen, const int32_t* seq_ids, const int64_t* positions,
    int64_t T, float softmax_scale, int32_t num_splits, void* workspace, size_t workspace_bytes,
    int32_t* status_dev, void* out, void* stream, void* attn_start, void* attn_stop) {
  if (T < 0) return XMLA_ERR_SHAPE;
  if (T > 0 && (hidden == nullptr || W_kva == nullptr || seq_ids == nullptr || positions == nullptr))
    return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)hidden) | ((uintptr_t)W_kva)) & 15u || ((uintptr_t)bias) & 1u)
    return XMLA_ERR_INVALID_ARG;
  AppendArgs ap{};  // no ready rows: the producer writes them
  ap.pool = (uint4*)pool;
  ap.num_blocks = num_blocks;
  ap.block_table = block_table;
  ap.max_blocks = max_blocks;
  ap.batch = batch;
  ap.status = status_dev;
  const ProduceArgs pa{(const __nv_bfloat16*)hidden, (const __nv_bfloat16*)W_kva,
                       (const __nv_bfloat16*)bias, T, (uint16_t*)pool, num_blocks, block_table,
                       max_blocks, batch, seq_ids, positions, status_dev, 1};
  return run_decode(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                    q_len, max_seqlen, softmax_scale, num_splits, workspace, workspace_bytes,
                    status_dev, out, stream, attn_start, attn_stop, &ap, &pa);
}

extern "C" xmla_status xmla_decode(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                   const void* W_UV, const void* pool, int64_t num_blocks,
                                   const int32_t* block_table, int32_t max_blocks,
                                   const int32_t* seqlens, int32_t batch, int32_t q_len,
                                   int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                                   void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                   void* out, void* stream) {
  return xmla_decode_profiled(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens,
                              batch, q_len, max_seqlen, softmax_scale, num_splits, workspace,
                              workspace_bytes, status_dev, out, stream, nullptr, nullptr);
}

// ---------------------------------------------------------------- sequence-parallel decode

// ---------------------------------------------------------------- 8-bit latent cache

extern "C" size_t xmla_decode_q8_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                                int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P, 0, true, true) ? P.bytes
                                                                                      : 0;
}

extern "C" int32_t xmla_decode_q8_num_splits(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                             int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P, 0, true, true) ? P.nsplit
                                                                                      : 0;
}

extern "C" xmla_status xmla_cache_append_q8(void* pool_q8, int64_t num_blocks,
                                            const int32_t* block_table, int32_t max_blocks,
                                            int32_t batch, const int32_t* seq_ids,
                                            const int64_t* positions, const void* c_kv,
                                            const void* k_pe, const xmla_yarn_cfg* rope_cfg,
                                            int64_t T, int32_t* status_dev, void* stream) {
  if (T < 0 || num_blocks < 1 || max_blocks < 1 || batch < 1) return XMLA_ERR_SHAPE;
  if (T == 0) return XMLA_OK;
  if (pool_q8 == nullptr || block_table == nullptr || seq_ids == nullptr || positions == nullptr ||
      c_kv == nullptr || k_pe == nullptr)
    return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)pool_q8) | ((uintptr_t)c_kv) | ((uintptr_t)k_pe)) & 15u)
    return XMLA_ERR_INVALID_ARG;
  RopeTable tab = {};
  if (rope_cfg != nullptr) {
    if (!yarn_cfg_ok(rope_cfg)) return XMLA_ERR_INVALID_ARG;
    if (rope_cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
    tab = make_rope_table(rope_cfg);
  }
  const cudaError_t e = launch_cache_append_q8(
      (uint8_t*)pool_q8, num_blocks, block_table, max_blocks, batch, seq_ids, positions,
      (const __nv_bfloat16*)c_kv, (const __nv_bfloat16*)k_pe, status_dev,
      rope_cfg != nullptr ? 1 : 0, tab, T, (cudaStream_t)stream);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" xmla_status xmla_decode_q8_profiled(
    const xmla_yarn_cfg* cfg, const void* q, const void* W_UK, const void* W_UV,
    const void* pool_q8, int64_t num_blocks, const int32_t* block_table, int32_t max_blocks,
    const int32_t* seqlens, int32_t batch, int32_t q_len, int64_t max_seqlen, float softmax_scale,
    int32_t num_splits, void* workspace, size_t workspace_bytes, int32_t* status_dev, void* out,
    void* stream, void* attn_start, void* attn_stop) {
  return run_decode(cfg, q, W_UK, W_UV, pool_q8, num_blocks, block_table, max_blocks, seqlens,
                    batch, q_len, max_seqlen, softmax_scale, num_splits, workspace,
                    workspace_bytes, status_dev, out, stream, attn_start, attn_stop, nullptr,
                    nullptr, 0, INT64_MAX, nullptr, true);
}

extern "C" xmla_status xmla_decode_q8(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                      const void* W_UV, const void* pool_q8, int64_t num_blocks,
                                      const int32_t* block_table, int32_t max_blocks,
                                      const int32_t* seqlens, int32_t batch, int32_t q_len,
                                      int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* status_dev, void* out, void* stream) {
  return xmla_decode_q8_profiled(cfg, q, W_UK, W_UV, pool_q8, num_blocks, block_table,
                                 max_blocks, seqlens, batch, q_len, max_seqlen, softmax_scale,
                                 num_splits, workspace, workspace_bytes, status_dev, out, stream,
                                 nullptr, nullptr);
}

extern "C" size_t xmla_shard_partial_floats(int32_t batch, int32_t q_len) {
  if (batch < 1 || q_len < 1 || q_len > kMaxQLen) return 0;
  return (size_t)batch * q_len * kHeads * (kDLatent + 2);
}

extern "C" size_t xmla_decode_shard_workspace_size(int32_t batch, int32_t q_len,
                                                   int64_t max_seqlen, int64_t page_lo,
                                                   int64_t page_hi, int32_t num_sms,
                                                   int32_t num_splits) {
  if (page_lo < 0 || page_hi < page_lo) return 0;
  Plan P;
  const int64_t span = page_hi > page_lo ? page_hi - page_lo : 1;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P, span) ? P.bytes : 0;
}

extern "C" xmla_status xmla_decode_shard(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                         const void* pool, int64_t num_blocks,
                                         const int32_t* block_table, int32_t max_blocks,
                                         const int32_t* seqlens, int32_t batch, int32_t q_len,
                                         int64_t max_seqlen, float softmax_scale, int64_t page_lo,
                                         int64_t page_hi, int32_t num_splits, void* workspace,
                                         size_t workspace_bytes, int32_t* status_dev,
                                         float* shard_partial, void* stream) {
  if (shard_partial == nullptr) return XMLA_ERR_INVALID_ARG;
  if (((uintptr_t)shard_partial) & 15u) return XMLA_ERR_INVALID_ARG;
  if (page_lo < 0 || page_hi < page_lo) return XMLA_ERR_SHAPE;
  // W_UV and out are not used: the shard ends with its merged partial
  return run_decode(cfg, q, W_UK, W_UK, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                    q_len, max_seqlen, softmax_scale, num_splits, workspace, workspace_bytes,
                    status_dev, shard_partial, stream, nullptr, nullptr, nullptr, nullptr,
                    page_lo, page_hi, shard_partial);
}

extern "C" xmla_status xmla_combine_shards(const float* partials, int32_t num_shards,
                                           const void* W_UV, int32_t batch, int32_t q_len,
                                           void* out, void* stream) {
  if (partials == nullptr || W_UV == nullptr || out == nullptr) return XMLA_ERR_INVALID_ARG;
  if (batch < 1 || q_len < 1 || q_len > kMaxQLen || num_shards < 1 || num_shards > kMaxSplits ||
      (int64_t)batch * q_len * kHeads > (int64_t)0x7fffffff)
    return XMLA_ERR_SHAPE;
  if ((((uintptr_t)partials) | ((uintptr_t)W_UV) | ((uintptr_t)out)) & 15u)
    return XMLA_ERR_INVALID_ARG;
  int nsm = 0;
  if (!device_ok(&nsm)) return XMLA_ERR_UNSUPPORTED;
  const int rows = batch * q_len;
  const int64_t R = (int64_t)rows * kHeads;
  // the gathered partials, read as num_shards splits of one row group holding
  // every (row, head): row r*32 + h of a shard is at r*32 + h
  const cudaError_t e = launch_combine(partials, partials + R * kDLatent,
                                       (const __nv_bfloat16*)W_UV, (__nv_bfloat16*)out, rows, rows,
                                       1, num_shards, (int)R, (cudaStream_t)stream,
                                       R * (kDLatent + 2), R * (kDLatent + 2) / 2);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

// ---------------------------------------------------------------- decode without caller scratch

namespace xmla {

// Fixed device scratch for xmla_decode_noalloc.  It is part of the library's
// module image, so every GPU that loads the library holds it until the
// process exits; its size is the largest workspace that entry point accepts.
constexpr size_t kNoAllocScratchBytes = (size_t)XMLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mutex;

// The array's device address belongs to the CUDA context that loaded the
// library's module: a context destroyed and created again (cudaDeviceReset,
// or the primary context released and retained anew) loads the module again,
// possibly elsewhere.  Addresses are therefore cached per context, keyed on
// the context's unique id (cuCtxGetId), never reused across contexts.
struct NoAllocSlot {
  unsigned long long ctx_id;
  void* addr;
};
static NoAllocSlot g_noalloc_slots[64] = {};
static int g_noalloc_next = 0;

static bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* p1 = nullptr;
    void* p2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p1);
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context.  In host code
// the array's name is only a host-side stand-in, so the real address is asked
// from the runtime (with the context's device current) the first time a
// context is seen, and cached for that context.
static xmla_status noalloc_scratch(void** addr) {
  unsigned long long id = 0;
  if (!current_context_id(&id)) {
    // no context current yet: let the runtime make the device's primary
    // context current (and initialise it), then ask again
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        !current_context_id(&id))
      return XMLA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  for (const NoAllocSlot& s : g_noalloc_slots) {
    if (s.addr != nullptr && s.ctx_id == id) {
      *addr = s.addr;
      return XMLA_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return XMLA_ERR_CUDA;
  g_noalloc_slots[g_noalloc_next] = NoAllocSlot{id, p};
  g_noalloc_next = (g_noalloc_next + 1) % 64;
  *addr = p;
  return XMLA_OK;
}

}  // namespace xmla

extern "C" xmla_status xmla_decode_noalloc(const xmla_yarn_cfg* cfg, const void* q,
                                           const void* W_UK, const void* W_UV, const void* pool,
                                           int64_t num_blocks, const int32_t* block_table,
                                           int32_t max_blocks, const int32_t* seqlens,
                                           int32_t batch, int32_t q_len, int64_t max_seqlen,
                                           float softmax_scale, int32_t num_splits,
                                           int32_t* status_dev, void* out, void* stream) {
  int nsm = 0;
  if (!xmla::device_ok(&nsm)) return XMLA_ERR_UNSUPPORTED;
  const size_t need = xmla_decode_workspace_size(batch, q_len, max_seqlen, nsm, num_splits);
  if (need == 0) return XMLA_ERR_SHAPE;
  if (need > xmla::kNoAllocScratchBytes) return XMLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const xmla_status st = xmla::noalloc_scratch(&scratch);
  if (st != XMLA_OK) return st;
  return xmla_decode(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                     q_len, max_seqlen, softmax_scale, num_splits, scratch,
                     xmla::kNoAllocScratchBytes, status_dev, out, stream);
}

extern "C" xmla_status xmla_selftest_wait_timeout(int32_t* status_dev, uint64_t timeout_ns,
                                                  void* stream) {
  if (status_dev == nullptr) return XMLA_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(status_dev, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" const char* xmla_status_string(xmla_status s) {
  switch (s) {
    case XMLA_OK: return "ok";
    case XMLA_ERR_INVALID_ARG: return "invalid argument";
    case XMLA_ERR_SHAPE: return "unsupported shape";
    case XMLA_ERR_WORKSPACE: return "workspace too small";
    case XMLA_ERR_CUDA: return "CUDA error";
    case XMLA_ERR_DEVICE_OOB: return "device: index out of range";
    case XMLA_ERR_TIMEOUT: return "device: bounded wait timed out";
    case XMLA_ERR_UNSUPPORTED: return "device not supported (needs sm_100a)";
  }
  return "unknown status";
}
