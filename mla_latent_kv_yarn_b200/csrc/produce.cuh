// The producer of a decode step's cache rows: kv_a_proj_with_mqa of the new
// tokens' hidden states, RoPE of the rope key, append to the paged cache.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": kv_a_proj_with_mqa = Linear(hidden_size, kv_lora_rank +
//      qk_rope_head_dim) compresses each token into the 512-dim latent and the
//      64-dim rope key that the cache keeps.
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 一:
//      attention_bias false; rope_scaling yarn (the rotation, yarn.cuh).
// The model summary page "Xing4.0" (alphasignal.ai), architecture paragraph:
//      hidden size 3584.
//
// Work is dealt in blocks of 4 output columns (144 blocks): latent blocks take
// 4 consecutive latent columns, rope blocks take the pairs (i, i + 32) and
// (i + 1, i + 33) so that the rotation stays inside the block.  The warps of a
// block split the 3584-long dot products: every thread keeps its slices of the
// 4 weight rows in registers (loaded before the wait for the kernels launched
// before) and, token by token, multiplies them with its slice of the hidden
// state; warp sums meet in shared memory.  Each output is rounded to bf16 (as
// a bf16 Linear does), the rope key is rotated from that bf16 value (float64
// angle, one rounding), and the token's columns are written into its cache row.
#pragma once

#include <cstdint>

#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

constexpr int kHidden = 3584;
constexpr int kProdCols = 4;                         // output columns per block
constexpr int kProdTok = 8;                          // tokens reduced per pass
constexpr int kLatentBlocks = kDLatent / kProdCols;  // 128
constexpr int kRopeBlocks = kDRope / kProdCols;      // 16
constexpr int kProdBlocks = kLatentBlocks + kRopeBlocks;

// The step's new tokens and where their rows go.  hidden, positions, seq_ids
// and block_table are read only after the wait for the kernels launched before
// (no __restrict__: a preceding kernel may write them).
struct ProduceArgs {
  const __nv_bfloat16* hidden;  // [T, 3584]
  const __nv_bfloat16* W_kva;   // [576, 3584]
  const __nv_bfloat16* bias;    // [576] or null
  int64_t T;
  uint16_t* pool;  // [num_blocks, 64, 576] bf16 bits
  int64_t num_blocks;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t batch;
  const int32_t* seq_ids;    // [T]
  const int64_t* positions;  // [T]
  int32_t* status;
  int rotate;  // 0: store the raw rope key
};

// Output column of slot j (< 4) of block blk.
__device__ __forceinline__ int prod_column(int blk, int j) {
  if (blk < kLatentBlocks) return blk * kProdCols + j;
  const int r = blk - kLatentBlocks;  // rope block: pairs 2r, 2r + 1
  return kDLatent + 2 * r + (j & 1) + (j >> 1) * (kDRope / 2);
}

// Shared memory of one block, for kWarps warps.
template <int kWarps>
struct ProduceSmem {
  float part[kProdTok][kWarps][kProdCols];  // per-warp partial sums
  float y[kProdTok][kProdCols];             // bf16-rounded outputs
};

// Block blk of the producer, computed by the kWarps * 32 threads t of a CTA.
// sync(): barrier over those threads; wait(): the wait for the kernels
// launched before (called once, after the weight loads).
template <int kWarps, class Sync, class Wait>
__device__ __forceinline__ void produce_block(int blk, int t, const ProduceArgs& a,
                                              const RopeTable& tab, ProduceSmem<kWarps>& sm,
                                              Sync sync, Wait wait) {
  static_assert(kHidden % (kWarps * 8) == 0, "warps split the hidden dim in 16-byte vectors");
  constexpr int kWarpVec = kHidden / kWarps / 8;       // 16-byte vectors per warp and row
  constexpr int kLaneVec = (kWarpVec + 31) / 32;       // per lane (the last one partial)
  // tokens whose hidden slices are loaded together: 4 when the weight slices
  // leave room in the registers (8 warps), else 1
  constexpr int kBatch = kLaneVec <= 2 ? 4 : 1;
  const int lane = t & 31, warp = t >> 5;
  const int v0 = warp * kWarpVec + lane;  // this lane's vectors: v0 + 32 u, u < kLaneVec
  uint4 w[kProdCols][kLaneVec];
#pragma unroll
  for (int j = 0; j < kProdCols; ++j) {
    const uint4* row = reinterpret_cast<const uint4*>(a.W_kva + (int64_t)prod_column(blk, j) * kHidden);
#pragma unroll
    for (int u = 0; u < kLaneVec; ++u)
      w[j][u] = lane + 32 * u < kWarpVec ? row[v0 + 32 * u] : make_uint4(0u, 0u, 0u, 0u);
  }
  wait();

  for (int64_t t0 = 0; t0 < a.T; t0 += kProdTok) {
    const int nt = (int)min((int64_t)kProdTok, a.T - t0);
    // the hidden slices of kBatch tokens are requested together, then used
    for (int k0 = 0; k0 < nt; k0 += kBatch) {
      uint4 hb[kBatch][kLaneVec];
#pragma unroll
      for (int kk = 0; kk < kBatch; ++kk) {
        const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + (t0 + k0 + kk) * kHidden);
#pragma unroll
        for (int u = 0; u < kLaneVec; ++u)
          hb[kk][u] = k0 + kk < nt && lane + 32 * u < kWarpVec ? hrow[v0 + 32 * u]
                                                                : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kBatch; ++kk) {
        const int k = k0 + kk;
        if (k >= nt) break;  // nt is the same for every thread of the block
        const uint4* h = hb[kk];
        float acc[kProdCols];
#pragma unroll
        for (int j = 0; j < kProdCols; ++j) {
          acc[j] = 0.f;
#pragma unroll
          for (int u = 0; u < kLaneVec; ++u) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&h[u]);
            const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w[j][u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 hf = __bfloat1622float2(h2[e]);
              const float2 wf = __bfloat1622float2(w2[e]);
              acc[j] = fmaf(hf.x, wf.x, acc[j]);
              acc[j] = fmaf(hf.y, wf.y, acc[j]);
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        }
        if (lane < kProdCols) {
          float v = acc[0];
#pragma unroll
          for (int i = 1; i < kProdCols; ++i) v = lane == i ? acc[i] : v;
          sm.part[k][warp][lane] = v;
        }
      }
    }
    sync();
    // thread (token k, column slot j): sum the warps, add the bias, round to bf16
    if (t < nt * kProdCols) {
      const int k = t / kProdCols, j = t % kProdCols;
      float v = 0.f;
#pragma unroll
      for (int wp = 0; wp < kWarps; ++wp) v += sm.part[k][wp][j];
      if (a.bias != nullptr) v += __bfloat162float(a.bias[prod_column(blk, j)]);
      sm.y[k][j] = __bfloat162float(__float2bfloat16_rn(v));
    }
    sync();
    // thread (token k, p < 2): slots p and p + 2 -- two latent columns, or the
    // rope pair (i, i + 32) with i = 2r + p -- into the token's cache row
    if (t < nt * 2) {
      const int k = t / 2, pr = t % 2;
      const int64_t tok = t0 + k;
      const int32_t s = a.seq_ids[tok];
      const int64_t pos = a.positions[tok];
      int32_t cache_blk = -1;
      if (s >= 0 && s < a.batch && pos >= 0 && pos < (int64_t)a.max_blocks * kPage)
        cache_blk = a.block_table[(int64_t)s * a.max_blocks + pos / kPage];
      if (cache_blk < 0 || (int64_t)cache_blk >= a.num_blocks) {
        if (pr == 0) record_status(a.status, XMLA_ERR_DEVICE_OOB);
      } else {
        uint16_t* row = a.pool + ((int64_t)cache_blk * kPage + pos % kPage) * kDRow;
        float x = sm.y[k][pr], z = sm.y[k][pr + 2];
        if (blk >= kLatentBlocks && a.rotate) {
          double y1, y2;
          rope_pair((double)x, (double)z, pos, 2 * (blk - kLatentBlocks) + pr, tab, &y1, &y2);
          x = __bfloat162float(__double2bfloat16(y1));  // the one rounding of the rotation
          z = __bfloat162float(__double2bfloat16(y2));
        }
        const __nv_bfloat16 hx = __float2bfloat16_rn(x), hz = __float2bfloat16_rn(z);
        row[prod_column(blk, pr)] = *reinterpret_cast<const uint16_t*>(&hx);
        row[prod_column(blk, pr + 2)] = *reinterpret_cast<const uint16_t*>(&hz);
      }
    }
    sync();  // the shared sums are reused by the next tokens
  }
}

}  // namespace xmla
