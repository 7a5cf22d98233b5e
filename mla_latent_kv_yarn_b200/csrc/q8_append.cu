// Append of cache rows to the 8-bit paged latent cache.
//
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 三,
//      方案 A: a q8_0 KV cache ("--cache-type-k q8_0") halves the bf16 cache at
//      a small precision cost: 8-bit codes with one scale per block of 32 values.
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": a token's cache row is its 512-dim latent c_kv and its 64-dim
//      rope key.
//
// The row [c_kv | rotated k_pe] (576 values, bf16) is cut into 18 blocks of 32.
// Block exponent e: the smallest integer with 127 * 2^e >= the block's largest
// magnitude, clamped to [-14, 8]; codes round(x / 2^e) to nearest even,
// clamped to [-127, 127].  With the scale a power of two every stored value
// code * 2^e is exact in f16, the type the attention kernel consumes.
#include <cuda_bf16.h>

#include <cstdint>

#include "decode_chain.h"
#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

namespace {

constexpr int kQ8AppendWarps = 8;  // one cache row per warp

// Exponent of a block whose largest magnitude is amax (exact: frexp splits
// amax = m 2^k with m in [0.5, 1); 127 * 2^(k-7) covers it iff m <= 127/128).
__device__ __forceinline__ int q8_exponent(float amax) {
  if (!(amax > 0.f)) return kQ8EMin;
  int k;
  const float m = frexpf(amax, &k);
  const int e = m > 127.f / 128.f ? k - 6 : k - 7;
  return min(max(e, kQ8EMin), kQ8EMax);
}

}  // namespace

__global__ void __launch_bounds__(32 * kQ8AppendWarps)
    cache_append_q8_kernel(uint8_t* pool, int64_t num_blocks, const int32_t* block_table,
                           int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                           const int64_t* positions, const __nv_bfloat16* c_kv,
                           const __nv_bfloat16* k_pe, int32_t* status, int rotate,
                           const RopeTable tab, int64_t T) {
  __shared__ __align__(16) uint8_t rowbuf[kQ8AppendWarps][kQ8Row];
  __shared__ __align__(16) float rope_s[kQ8AppendWarps][kDRope];
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kQ8AppendWarps + warp;
  // the inputs may come from, and the rows' pages may still be read by, the
  // kernels launched before this one
  pdl_wait();
  if (t >= T) return;
  const int32_t s = seq_ids[t];
  const int64_t pos = positions[t];
  if (s < 0 || s >= batch || pos < 0 || pos >= (int64_t)max_blocks * kPage) {
    if (lane == 0) record_status(status, XMLA_ERR_DEVICE_OOB);
    return;
  }
  const int32_t blk = block_table[(int64_t)s * max_blocks + pos / kPage];
  if (blk < 0 || (int64_t)blk >= num_blocks) {
    if (lane == 0) record_status(status, XMLA_ERR_DEVICE_OOB);
    return;
  }
  // the rope key of the row, rotated (pair lane, lane + 32) and rounded to bf16
  {
    const float x1 = __bfloat162float(k_pe[t * kDRope + lane]);
    const float x2 = __bfloat162float(k_pe[t * kDRope + lane + 32]);
    float y1 = x1, y2 = x2;
    if (rotate) {
      double r1, r2;
      rope_pair((double)x1, (double)x2, pos, lane, tab, &r1, &r2);
      y1 = __bfloat162float(__double2bfloat16(r1));
      y2 = __bfloat162float(__double2bfloat16(r2));
    }
    rope_s[warp][lane] = y1;
    rope_s[warp][lane + 32] = y2;
  }
  __syncwarp();
  uint8_t* rb = rowbuf[warp];
  if (lane < kQ8Blocks) {
    float v[kQ8Block];
    if (lane < kDLatent / kQ8Block) {
      const uint4* src = reinterpret_cast<const uint4*>(c_kv + t * kDLatent + lane * kQ8Block);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = src[q];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * q + 2 * e] = __low2float(h[e]);
          v[8 * q + 2 * e + 1] = __high2float(h[e]);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < kQ8Block; ++k) v[k] = rope_s[warp][(lane - 16) * kQ8Block + k];
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < kQ8Block; ++k) amax = fmaxf(amax, fabsf(v[k]));
    const int e = q8_exponent(amax);
    uint32_t words[kQ8Block / 4];
#pragma unroll
    for (int q = 0; q < kQ8Block / 4; ++q) {
      uint32_t w = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // x * 2^-e is exact; rint to nearest even, then the code range
        const int c = min(127, max(-127, __float2int_rn(v[4 * q + k] * __int_as_float((127 - e) << 23))));
        w |= ((uint32_t)c & 0xffu) << (8 * k);
      }
      words[q] = w;
    }
    uint4* dst = reinterpret_cast<uint4*>(rb + lane * kQ8Block);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    rb[kDRow + lane] = (uint8_t)(int8_t)e;
  } else if (lane < kQ8Blocks + (kQ8Row - kDRow - kQ8Blocks)) {
    rb[kDRow + lane] = 0;  // the 14 pad bytes
  }
  __syncwarp();
  uint4* out = reinterpret_cast<uint4*>(pool + ((int64_t)blk * kPage + pos % kPage) * kQ8Row);
  const uint4* in = reinterpret_cast<const uint4*>(rb);
  for (int u = lane; u < kQ8Row / 16; u += 32) out[u] = in[u];
}

cudaError_t launch_cache_append_q8(uint8_t* pool, int64_t num_blocks, const int32_t* block_table,
                                   int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                                   const int64_t* positions, const __nv_bfloat16* c_kv,
                                   const __nv_bfloat16* k_pe, int32_t* status, int rotate,
                                   const RopeTable& tab, int64_t T, cudaStream_t st) {
  const int64_t blocks = (T + kQ8AppendWarps - 1) / kQ8AppendWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_pdl(cache_append_q8_kernel, dim3((unsigned)blocks), dim3(32 * kQ8AppendWarps), 0,
                    st, pool, num_blocks, block_table, max_blocks, batch, seq_ids, positions, c_kv,
                    k_pe, status, rotate, tab, T);
}

}  // namespace xmla
