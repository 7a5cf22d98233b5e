// Standalone producer of cache rows from hidden states (produce.cuh): one CTA
// of 8 warps per block of 4 output columns.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": kv_a_proj_with_mqa feeds the latent cache.
#include <cstdint>

#include "produce.cuh"

namespace xmla {

constexpr int kProdWarps = 8;

__global__ void __launch_bounds__(kProdWarps * 32) kv_produce_kernel(const ProduceArgs a,
                                                                      const RopeTable tab) {
  __shared__ ProduceSmem<kProdWarps> sm;
  pdl_launch_dependents();
  produce_block<kProdWarps>(blockIdx.x, threadIdx.x, a, tab, sm, [] { __syncthreads(); },
                            [] { pdl_wait(); });
}

}  // namespace xmla

using namespace xmla;

extern "C" xmla_status xmla_kv_produce(const void* hidden, const void* W_kva, const void* bias,
                                       int64_t T, const xmla_yarn_cfg* rope_cfg, void* pool,
                                       int64_t num_blocks, const int32_t* block_table,
                                       int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                                       const int64_t* positions, int32_t* status_dev,
                                       void* stream) {
  if (T < 0 || num_blocks < 1 || max_blocks < 1 || batch < 1) return XMLA_ERR_SHAPE;
  if (T == 0) return XMLA_OK;
  if (hidden == nullptr || W_kva == nullptr || pool == nullptr || block_table == nullptr ||
      seq_ids == nullptr || positions == nullptr)
    return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)hidden) | ((uintptr_t)W_kva)) & 15u) return XMLA_ERR_INVALID_ARG;
  if (((uintptr_t)pool) & 1u || ((uintptr_t)bias) & 1u) return XMLA_ERR_INVALID_ARG;
  RopeTable tab = {};
  if (rope_cfg != nullptr) {
    if (!yarn_cfg_ok(rope_cfg)) return XMLA_ERR_INVALID_ARG;
    if (rope_cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
    tab = make_rope_table(rope_cfg);
  }
  const ProduceArgs a{(const __nv_bfloat16*)hidden, (const __nv_bfloat16*)W_kva,
                      (const __nv_bfloat16*)bias, T, (uint16_t*)pool, num_blocks, block_table,
                      max_blocks, batch, seq_ids, positions, status_dev,
                      rope_cfg != nullptr ? 1 : 0};
  const cudaError_t e = launch_pdl(kv_produce_kernel, dim3(kProdBlocks), dim3(kProdWarps * 32), 0,
                                   (cudaStream_t)stream, a, tab);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}
