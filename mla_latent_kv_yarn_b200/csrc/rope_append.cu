// YaRN rotary embedding (in place, bf16) and the paged latent-cache append.
//
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 一:
//      rope_scaling yarn (frequency table in yarn.cuh).
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": the cache holds the 512-dim latent and the 64-dim rope key.
#include <cmath>
#include <cstdint>

#include "append.cuh"
#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

// ---------------------------------------------------------------- device: RoPE

// One thread per (vector, pair).  Angle formed in float64 from the exact
// integer position; the rotated pair is rounded once to bf16.
//
// Inputs that the kernel launched just before may write carry no __restrict__
// (here and in the kernels below): such loads are then not taken as invariant
// and cannot be hoisted above the griddepcontrol.wait that orders them.
__global__ void __launch_bounds__(256) rope_yarn_kernel(__nv_bfloat16* x, int64_t rows,
                                                        int32_t n_heads, int64_t head_stride,
                                                        int64_t row_stride, int32_t offset,
                                                        const int64_t* positions,
                                                        const RopeTable tab) {
  pdl_wait();  // inputs may come from the kernel launched just before
  pdl_launch_dependents();
  const int64_t total = rows * (int64_t)n_heads * (kDRope / 2);
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(idx % (kDRope / 2));
    const int64_t rh = idx / (kDRope / 2);
    const int64_t h = rh % n_heads;
    const int64_t r = rh / n_heads;
    __nv_bfloat16* v = x + r * row_stride + h * head_stride + offset;
    double y1, y2;
    rope_pair((double)__bfloat162float(v[i]), (double)__bfloat162float(v[i + kDRope / 2]),
              positions[r], i, tab, &y1, &y2);
    v[i] = __double2bfloat16(y1);
    v[i + kDRope / 2] = __double2bfloat16(y2);
  }
}

// ---------------------------------------------------------------- device: append

// One thread per 16-byte piece of a cache row (append_piece in append.cuh).
__global__ void __launch_bounds__(256) cache_append_kernel(
    uint4* pool, int64_t num_blocks, const int32_t* block_table, int32_t max_blocks,
    int32_t batch, const int32_t* seq_ids, const int64_t* positions, const uint4* c_kv,
    const uint4* k_pe, int64_t T, int32_t* status, int rotate, const RopeTable tab) {
  pdl_wait();  // inputs may come from the kernel launched just before
  pdl_launch_dependents();
  const int64_t total = T * kRowPieces;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x)
    append_piece(idx, pool, num_blocks, block_table, max_blocks, batch, seq_ids, positions, c_kv,
                 k_pe, status, rotate, tab);
}

static int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  if (g > (1 << 20)) g = 1 << 20;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace xmla

using namespace xmla;

extern "C" void xmla_yarn_default(xmla_yarn_cfg* cfg) {
  if (cfg == nullptr) return;
  cfg->rope_theta = 10000.0;
  cfg->factor = 64.0;
  cfg->original_max_position_embeddings = 4096;
  cfg->beta_fast = 32.0;
  cfg->beta_slow = 1.0;
  cfg->mscale = 1.0;
  cfg->mscale_all_dim = 1.0;
  cfg->rotary_dim = kDRope;
}

extern "C" xmla_status xmla_yarn_inv_freq(const xmla_yarn_cfg* cfg, double* inv_freq_out) {
  if (!yarn_cfg_ok(cfg) || inv_freq_out == nullptr) return XMLA_ERR_INVALID_ARG;
  if (cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
  yarn_table(cfg, inv_freq_out);
  return XMLA_OK;
}

extern "C" double xmla_softmax_scale(const xmla_yarn_cfg* cfg, int32_t qk_head_dim) {
  if (cfg == nullptr || qk_head_dim <= 0) return 0.0;
  const double m = mscale_of(cfg->factor, cfg->mscale_all_dim);
  return m * m / std::sqrt((double)qk_head_dim);
}

extern "C" xmla_status xmla_rope_yarn(const xmla_yarn_cfg* cfg, void* x, int64_t rows,
                                      int32_t n_heads, int64_t head_stride_elems,
                                      int64_t row_stride_elems, int32_t rope_offset_elems,
                                      const int64_t* positions, void* stream) {
  if (!yarn_cfg_ok(cfg)) return XMLA_ERR_INVALID_ARG;
  if (cfg->rotary_dim != kDRope || n_heads < 1 || rows < 0) return XMLA_ERR_SHAPE;
  if (rows == 0) return XMLA_OK;
  if (x == nullptr || positions == nullptr || head_stride_elems < 0 || row_stride_elems < 0 ||
      rope_offset_elems < 0)
    return XMLA_ERR_INVALID_ARG;
  const RopeTable tab = make_rope_table(cfg);
  const int64_t work = rows * n_heads * (kDRope / 2);
  const cudaError_t e = launch_pdl(rope_yarn_kernel, dim3(grid_for(work, 256)), dim3(256), 0,
                                   (cudaStream_t)stream, (__nv_bfloat16*)x, rows, n_heads,
                                   head_stride_elems, row_stride_elems, rope_offset_elems,
                                   positions, tab);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" xmla_status xmla_cache_append(void* pool, int64_t num_blocks, const int32_t* block_table,
                                         int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                                         const int64_t* positions, const void* c_kv,
                                         const void* k_pe, const xmla_yarn_cfg* rope_cfg, int64_t T,
                                         int32_t* status_dev, void* stream) {
  if (T < 0 || num_blocks < 1 || max_blocks < 1 || batch < 1) return XMLA_ERR_SHAPE;
  if (T == 0) return XMLA_OK;
  if (pool == nullptr || block_table == nullptr || seq_ids == nullptr || positions == nullptr ||
      c_kv == nullptr || k_pe == nullptr)
    return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)pool) | ((uintptr_t)c_kv) | ((uintptr_t)k_pe)) & 15u)
    return XMLA_ERR_INVALID_ARG;
  RopeTable tab = {};
  if (rope_cfg != nullptr) {
    if (!yarn_cfg_ok(rope_cfg)) return XMLA_ERR_INVALID_ARG;
    if (rope_cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
    tab = make_rope_table(rope_cfg);
  }
  const int64_t work = T * kRowPieces;
  const cudaError_t e = launch_pdl(cache_append_kernel, dim3(grid_for(work, 256)), dim3(256), 0,
                                   (cudaStream_t)stream, (uint4*)pool, num_blocks, block_table,
                                   max_blocks, batch, seq_ids, positions, (const uint4*)c_kv,
                                   (const uint4*)k_pe, T, status_dev, rope_cfg != nullptr ? 1 : 0,
                                   tab);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}
